"""The seeded generators produce the shapes and structure of the five workloads."""
import numpy as np

from mla_flash_attention_attn_b200 import workloads as W


def test_determinism_same_seed_same_bytes():
    a = W.make("v2lite_decode", n_kv=256)
    b = W.make("v2lite_decode", n_kv=256)
    assert np.array_equal(a.q.view(np.uint16), b.q.view(np.uint16))
    assert np.array_equal(a.kcache.view(np.uint16), b.kcache.view(np.uint16))


def test_tiny_decode_shapes():
    w = W.make("tiny_decode")
    assert w.q.shape == (1, 1, 16, 576) and w.q.dtype == np.float16
    assert w.kcache.shape == (1, 256, 576)
    assert np.all(w.mask == 0)
    assert abs(w.scale - 192 ** -0.5) < 1e-15


def test_v2lite_last_37_masked():
    w = W.make("v2lite_decode")
    m = w.mask[0, 0]
    assert m.shape == (4096,)
    assert np.all(np.isneginf(m[-37:])) and np.all(m[:-37] == 0)
    assert 0.45 < float(np.std(w.kcache.astype(np.float32))) < 0.55


def test_v3_lengths_and_padding():
    w = W.make("v3_batched_decode", n_kv=8192, len_lo=1000, len_hi=8192)
    assert w.q.shape == (8, 1, 128, 576)
    assert np.all((w.kv_len >= 1000) & (w.kv_len <= 8192))
    for b in range(8):
        L = w.kv_len[b]
        assert np.all(w.mask[b, 0, :L] == 0) and np.all(np.isneginf(w.mask[b, 0, L:]))
        # padding holds random values, not zeros
        if L < 8192:
            assert np.any(w.kcache[b, L:] != 0)


def test_v3_full_size_lengths_range():
    rng = np.random.Generator(np.random.PCG64(1003))
    lens = rng.integers(4096, 32768, size=8, endpoint=True)
    w_lens = W.v3_batched_decode.__defaults__  # defaults are the full sizes
    assert w_lens[0] == 1003 and w_lens[1] == 8 and w_lens[2] == 128
    assert np.all((lens >= 4096) & (lens <= 32768))


def test_prefill_causal_alignment():
    w = W.make("prefill_chunk", n_q=8, n_head=2, n_kv=40)
    past = 32
    for i in range(8):
        row = w.mask[0, i]
        assert np.all(row[: past + i + 1] == 0)
        assert np.all(np.isneginf(row[past + i + 1:]))


def test_sparse_block_pattern_full_size():
    w = W.make("sparse_q8_decode")
    keep = ~np.isneginf(w.mask[0, 0])
    assert w.kcache.shape == (1, 131072, 612) and w.kcache.dtype == np.uint8
    assert keep.sum() == 16384  # exactly 1/8 of the cells
    assert np.all(keep[-1024:])  # last 1024 always kept
    blocks = keep.reshape(-1, 64)
    assert np.all(blocks.all(axis=1) | (~blocks).all(axis=1))  # whole 64-cell blocks
    assert blocks.all(axis=1).sum() == 256


def test_q8_0_random_value_ranges():
    rng = np.random.Generator(np.random.PCG64(5))
    rows = W.q8_0_random(rng, (50,))
    blk = rows.reshape(50, 18, 34)
    d = blk[:, :, 0:2].copy().view(np.float16).astype(np.float32)
    q = blk[:, :, 2:].view(np.int8)
    assert np.all((d >= 0.5 / 127 - 1e-5) & (d <= 1.5 / 127 + 1e-5))
    assert q.min() >= -127 and q.max() <= 127


def test_bench_head_dim_512_drops_the_rope_columns_and_counts_1024_byte_rows():
    import types

    import bench

    a = types.SimpleNamespace(workload="v3_batched_decode", head_dim=512, wuv=False, mask_gather=False)
    w5 = bench.make_workload(a)
    w6 = W.make("v3_batched_decode")
    assert w5.q.shape[-1] == 512 and w5.kcache.shape[-1] == 512
    assert np.array_equal(w5.kcache, w6.kcache[..., :512]) and np.array_equal(w5.q, w6.q[..., :512])
    acc5, acc6 = bench.algorithmic(w5), bench.algorithmic(w6)
    assert acc5["kv_bytes"] * 1152 == acc6["kv_bytes"] * 1024
    assert acc5["flops"] * (576 + 512) == acc6["flops"] * (512 + 512)
    assert bench.workload_name(a) == "v3_batched_decode+dk512"
