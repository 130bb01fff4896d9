"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Tolerance (f16 paths): max-abs error <= 1e-2 and relative L2 error <= 2e-3 over
the compared outputs; compaction indices bit-exact. Outputs are pre-filled with
NaN and followed by a NaN canary region, so an unwritten or overrun cell shows.
"""
import numpy as np
import pytest

import oracle
from mla_flash_attention_attn_b200 import binding
from mla_flash_attention_attn_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3
CANARY = 4096


def torch_mod():
    import torch

    return torch


def assert_parity(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, what
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    nref = np.linalg.norm(ref)
    err = got - ref
    maxabs = float(np.max(np.abs(err))) if err.size else 0.0
    if nref == 0.0:
        assert maxabs == 0.0, f"{what}: expected exact zeros, max |err| {maxabs}"
        return
    rel = float(np.linalg.norm(err) / nref)
    assert maxabs <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {maxabs:.3g} rel-L2 {rel:.3g}"


def run_gpu(w, kv_len="auto", mask="auto", k_pad=0, **variants):
    """Run the workload through mla_fa_forward_ex; returns out [n_seq][n_q][n_head][512]."""
    torch = torch_mod()
    dev = torch.device("cuda")
    q = torch.from_numpy(w.q).to(dev)
    if k_pad:
        kbuf = torch.zeros((w.n_seq, w.n_kv + k_pad) + w.kcache.shape[2:], dtype=torch.float16,
                           device=dev)
        kbuf[:, : w.n_kv] = torch.from_numpy(w.kcache).to(dev)
        k = kbuf[:, : w.n_kv]
    else:
        k = torch.from_numpy(w.kcache).to(dev)
    m = None
    if mask == "auto" and w.mask is not None:
        m = torch.from_numpy(w.mask).to(dev)
    n_out = w.n_seq * w.n_q * w.n_head * 512
    big = torch.full((n_out + CANARY,), float("nan"), dtype=torch.float32, device=dev)
    out = big[:n_out].view(w.n_seq, w.n_q, w.n_head, 512)
    lens = w.kv_len if kv_len == "auto" else kv_len
    vt = {}
    for name in ("sinks", "alibi_slopes"):
        if variants.get(name) is not None:
            vt[name] = torch.from_numpy(np.asarray(variants[name], np.float32)).to(dev)
    binding.forward(q, k, w.kv_type, m, w.scale, out=out, kv_len=lens,
                    softcap=variants.get("softcap", 0.0),
                    mask_gather=variants.get("mask_gather", False), **vt)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    tail = big[n_out:]
    assert bool(torch.isnan(tail).all()), "write past the end of out"
    return out.cpu().numpy()


def oracle_rows(w, b, rows=None, use_mask=True):
    return oracle.attention(w.q[b], w.kcache[b], w.kv_type,
                            w.mask[b] if (use_mask and w.mask is not None) else None,
                            w.scale, rows=rows)


def check_all_rows(w, got, use_mask=True, what=""):
    for b in range(w.n_seq):
        ref = oracle_rows(w, b, use_mask=use_mask)
        assert_parity(got[b].reshape(-1, 512), ref, f"{what} seq {b}")


def test_tiny_decode_full_size():
    w = W.make("tiny_decode")
    check_all_rows(w, run_gpu(w), what="tiny_decode")


def test_v2lite_decode_full_size():
    w = W.make("v2lite_decode")
    check_all_rows(w, run_gpu(w), what="v2lite_decode")


@pytest.mark.parametrize("with_len", [True, False])
def test_v3_batched_reduced(with_len):
    w = W.make("v3_batched_decode", n_kv=2048, len_lo=100, len_hi=2048)
    got = run_gpu(w, kv_len="auto" if with_len else None)
    check_all_rows(w, got, what="v3 reduced")


def test_prefill_reduced_causal():
    w = W.make("prefill_chunk", n_q=8, n_head=128, n_kv=640)
    check_all_rows(w, run_gpu(w), what="prefill reduced")


@pytest.mark.parametrize("n_kv", [1, 2, 31, 63, 65, 127, 129, 255, 257, 1000])
def test_ragged_kv_lengths(n_kv):
    rng = np.random.default_rng(n_kv)
    w = W.make("tiny_decode", n_kv=n_kv)
    keep = rng.random(n_kv) < 0.8
    keep[rng.integers(0, n_kv)] = True
    w.mask[0, 0] = np.where(keep, rng.standard_normal(n_kv).astype(np.float16), -np.inf)
    check_all_rows(w, run_gpu(w), what=f"n_kv={n_kv}")


@pytest.mark.parametrize("n_head,n_q", [(1, 1), (7, 3), (16, 9), (64, 2), (100, 3), (128, 2)])
def test_head_counts_and_row_groups(n_head, n_q):
    rng = np.random.default_rng(n_head * 10 + n_q)
    n_kv = 300
    w = W.make("prefill_chunk", n_q=n_q, n_head=n_head, n_kv=n_kv)
    w.mask[0] = np.where(rng.random((n_q, n_kv)) < 0.7, np.float16(0), np.float16(-np.inf))
    w.mask[0, :, 0] = 0
    check_all_rows(w, run_gpu(w), what=f"H={n_head} n_q={n_q}")


def test_fully_masked_rows_give_zero():
    w = W.make("prefill_chunk", n_q=4, n_head=16, n_kv=200)
    w.mask[0, 1, :] = -np.inf
    w.mask[0, 3, :] = -np.inf
    got = run_gpu(w)
    assert np.all(got[0, 1] == 0) and np.all(got[0, 3] == 0)
    check_all_rows(w, got, what="fully masked")


def test_no_mask():
    w = W.make("tiny_decode", n_kv=333)
    check_all_rows(w, run_gpu(w, mask=None), use_mask=False, what="no mask")


def test_large_finite_mask_values_and_shift():
    w = W.make("tiny_decode", n_kv=400)
    rng = np.random.default_rng(3)
    w.mask[0, 0] = (rng.standard_normal(400) * 30).astype(np.float16)
    check_all_rows(w, run_gpu(w), what="large mask")


def test_rising_scores_rescale_every_few_steps():
    """One 128-row sequence of 2048 keys whose mask rises by 60 from the first key to the
    last: its rows' running maximum passes the rescale threshold every one or two 128-key
    steps. 74 one-key sequences beside it leave the plan unsplit (as many groups as SM
    pairs), so one unit takes all 16 steps and rescales O in TMEM while the P.V of the
    previous step may still be running."""
    n_seq, n_kv = 75, 2048
    w = W.make("v3_batched_decode", n_seq=n_seq, n_kv=n_kv, len_lo=1, len_hi=1)
    w.kv_len[0] = n_kv
    w.mask[0, 0] = np.linspace(0.0, 60.0, n_kv).astype(np.float16)
    got = run_gpu(w)
    for b in range(n_seq):
        # cells past a sequence's length are -inf in its mask and add nothing: the oracle
        # takes the valid prefix
        n = int(w.kv_len[b])
        ref = oracle.attention(w.q[b], w.kcache[b][:n], w.kv_type, w.mask[b][:, :n], w.scale)
        assert_parity(got[b].reshape(-1, 512), ref, f"rising scores seq {b}")


def test_zero_length_sequence_and_strided_cache():
    w = W.make("v3_batched_decode", n_seq=3, n_head=16, n_kv=700, len_lo=0, len_hi=700)
    w.kv_len[:] = [0, 1, 700]
    keep = np.arange(700)[None, :] < w.kv_len[:, None]
    w.mask[:, 0, :] = np.where(keep, np.float16(0), np.float16(-np.inf))
    got = run_gpu(w, k_pad=64)
    assert np.all(got[0] == 0)
    check_all_rows(w, got, what="kv_len 0/1/700")


def test_deterministic_repeat():
    w = W.make("v3_batched_decode", n_seq=2, n_kv=1500, len_lo=900, len_hi=1500)
    a = run_gpu(w)
    b = run_gpu(w)
    assert np.array_equal(a, b)


def test_split_plan_is_exercised():
    torch = torch_mod()
    w = W.make("v3_batched_decode", n_kv=2048, len_lo=1500, len_hi=2048)
    q = torch.from_numpy(w.q).cuda()
    k = torch.from_numpy(w.kcache).cuda()
    out = torch.empty(w.q.shape[:3] + (512,), dtype=torch.float32, device="cuda")
    args, keep = binding.make_args(q, k, 0, None, out, w.scale, kv_len=w.kv_len)
    units, splits = binding.mla_fa_query_plan(args)
    assert splits > 1 and units >= w.n_seq
    wp = W.make("prefill_chunk", n_q=64, n_head=128, n_kv=256)
    qp = torch.from_numpy(wp.q).cuda()
    kp = torch.from_numpy(wp.kcache).cuda()
    outp = torch.empty(wp.q.shape[:3] + (512,), dtype=torch.float32, device="cuda")
    args2, keep2 = binding.make_args(qp, kp, 0, None, outp, wp.scale)
    units2, splits2 = binding.mla_fa_query_plan(args2)
    assert splits2 == 1 and units2 == 64


def test_batch_larger_than_one_launch():
    # 130 sequences: the host splits the batch into launches of at most 128 sequences,
    # each with its own plan (and split partials + combine where a sequence splits)
    w = W.make("v3_batched_decode", n_seq=130, n_head=16, n_kv=600, len_lo=1, len_hi=600)
    check_all_rows(w, run_gpu(w), what="130 sequences")


def test_sparse_batch_larger_than_one_launch():
    # 130 single-group sequences with sparse masks, through the two sparse routes that
    # gather rows into the workspace (indexed by the sequence's place in the whole batch,
    # over two launches of the plan): the mask gather (an internal list per sequence) and
    # caller index lists from the compaction
    w = W.make("v3_batched_decode", seed=41, n_seq=130, n_head=16, n_kv=600, len_lo=1, len_hi=600)
    rng = np.random.default_rng(41)
    keep = (rng.random((130, 1, 600)) < 0.3) & (np.arange(600)[None, None, :] < w.kv_len[:, None, None])
    keep[:, 0, 0] = True
    w.mask = np.where(keep, rng.standard_normal((130, 1, 600)), -np.inf).astype(np.float16)
    check_all_rows(w, run_gpu(w, mask_gather=True), what="130 sequences, mask gather")
    w.sparse = True
    got, idx, cnt, status = run_sparse_gpu(w)
    assert status == 0
    for b in range(w.n_seq):
        lst = oracle.compact(w.mask[b, 0])
        assert cnt[b] == len(lst)
        ref = oracle.attention(w.q[b], w.kcache[b], w.kv_type, w.mask[b], w.scale, idx=lst)
        assert_parity(got[b].reshape(-1, 512), ref, f"130 sequences, index list {b}")


def test_many_splits_of_one_long_sequence():
    # one 16-head sequence of 20000 keys: 79 tiles over the 74 SM pairs, so its rows are
    # combined from 74 partials by the multi-group combine
    w = W.make("v3_batched_decode", n_seq=1, n_head=16, n_kv=20000, len_lo=20000, len_hi=20000)
    torch = torch_mod()
    q = torch.from_numpy(w.q).cuda()
    k = torch.from_numpy(w.kcache).cuda()
    out = torch.empty(w.q.shape[:3] + (512,), dtype=torch.float32, device="cuda")
    args, keep = binding.make_args(q, k, 0, None, out, w.scale, kv_len=w.kv_len)
    units, splits = binding.mla_fa_query_plan(args)
    assert splits >= 32, "the case must reach the multi-group combine"
    check_all_rows(w, run_gpu(w), what="one long sequence")


def test_simple_entry_point_matches_oracle():
    torch = torch_mod()
    w = W.make("v2lite_decode", n_kv=1111)
    q = torch.from_numpy(w.q[0]).cuda()
    k = torch.from_numpy(w.kcache[0]).cuda()
    m = torch.from_numpy(w.mask[0]).cuda()
    out = torch.full((1, 16, 512), float("nan"), dtype=torch.float32, device="cuda")
    binding.mla_fa_forward(q, k, 0, m, w.scale, out)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    assert_parity(out.cpu().numpy().reshape(-1, 512), oracle_rows(w, 0), "mla_fa_forward")


# ------------------------------------------------------------------ full sizes
def test_v3_batched_full_size_every_row():
    # all 8 x 128 rows of the benchmark's V3 batch, in the launch configuration bench.py
    # times (kv_len given, split plan of 74 units)
    w = W.make("v3_batched_decode")
    got = run_gpu(w)
    check_all_rows(w, got, what="v3 full")


def test_prefill_full_size_whole_groups():
    # whole 128-row groups (every head of a token: both CTAs' lanes of a unit) of the
    # first, a middle and the last query tokens, plus single rows elsewhere
    w = W.make("prefill_chunk")
    got = run_gpu(w)
    H = w.n_head
    toks = (0, 255, 511)
    rows = np.array([t * H + h for t in toks for h in range(H)] +
                    [t * H + h for t in (1, 128, 510) for h in (0, 63, 64, 127)], np.int32)
    ref = oracle_rows(w, 0, rows=rows)
    assert_parity(got[0].reshape(-1, 512)[rows], ref, "prefill full")


# ------------------------------------------------------------------ run-time error path
def test_bounded_wait_timeout_is_reported_and_device_stays_usable():
    w = W.make("tiny_decode", n_kv=64)
    binding.mla_debug_wait_timeout(1_000_000)  # 1 ms on a barrier nothing signals
    assert binding.mla_get_device_status() == -7
    assert binding.mla_get_device_status() == 0  # reading clears it
    check_all_rows(w, run_gpu(w), what="after timeout")


# ------------------------------------------------------------------ compaction
def compact_gpu(row_np, lib_ws=True):
    torch = torch_mod()
    n = row_np.shape[0]
    m = torch.from_numpy(row_np).cuda()
    idx = torch.full((n + CANARY,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    if lib_ws:
        binding.mla_compact_mask(m, idx, cnt)
    else:
        ws = torch.zeros(binding.mla_compact_workspace_size(1, n), dtype=torch.uint8, device="cuda")
        binding.mla_compact_mask_ex(m.view(1, n), idx[:n].view(1, n), cnt, ws)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    c = int(cnt.item())
    idx_h = idx.cpu().numpy()
    assert np.all(idx_h[c:] == -1), "write beyond the kept count"
    return idx_h[:c]


@pytest.mark.parametrize("n", [1, 7, 8, 9, 15, 16, 17, 2047, 2048, 2049, 5000, 16383, 16384, 16385,
                               40000, 65537, 100000, 262144, 262145, 600001])
@pytest.mark.parametrize("p_keep", [0.0, 0.1, 0.5, 1.0])
def test_compaction_bit_exact(n, p_keep):
    rng = np.random.default_rng(n + int(p_keep * 100))
    keep = rng.random(n) < p_keep
    row = np.where(keep, rng.standard_normal(n), -np.inf).astype(np.float16)
    row[rng.random(n) < 0.01] = np.float16(-65504.0)  # finite large negatives are kept
    assert np.array_equal(compact_gpu(row), oracle.compact(row))


def test_compaction_full_size_block_pattern_and_repeats():
    w = W.make("sparse_q8_decode")
    row = w.mask[0, 0]
    ref = oracle.compact(row)
    assert len(ref) == 16384
    for _ in range(3):  # repeated calls reuse the workspace (epoch-tagged flags)
        assert np.array_equal(compact_gpu(row), ref)
    assert np.array_equal(compact_gpu(row, lib_ws=False), ref)


def test_compaction_unaligned_row_start():
    torch = torch_mod()
    rng = np.random.default_rng(5)
    n = 3001
    base = np.where(rng.random(n + 1) < 0.4, np.float16(0), np.float16(-np.inf)).astype(np.float16)
    m = torch.from_numpy(base).cuda()[1:]  # 2-byte aligned only
    idx = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1,), dtype=torch.int32, device="cuda")
    binding.mla_compact_mask(m, idx, cnt)
    torch.cuda.synchronize()
    c = int(cnt.item())
    assert np.array_equal(idx.cpu().numpy()[:c], oracle.compact(base[1:]))


# ------------------------------------------------------------------ q8_0 cache and sparse indices
def q8_f16_rounded(rows_u8):
    """q8_0 rows -> f16 cache with each value d*q rounded once to f16 (the product of an
    f16 scale and an 8-bit integer is exact in float32, so this is RN_f16(d*q))."""
    n = rows_u8.shape[0]
    blk = rows_u8.reshape(n, 18, 34)
    d = blk[:, :, 0:2].copy().view(np.float16).astype(np.float32)  # [n][18][1]
    q = blk[:, :, 2:].view(np.int8).astype(np.float32)              # [n][18][32]
    return (d * q).astype(np.float16).reshape(n, 576)


def run_sparse_gpu(w, idx_rows=None, counts=None, use_gpu_compaction=True):
    """Compaction (GPU) then attention over the kept indices; returns (out, idx, count)."""
    torch = torch_mod()
    dev = torch.device("cuda")
    q = torch.from_numpy(w.q).to(dev)
    k = torch.from_numpy(w.kcache).to(dev)
    m = torch.from_numpy(w.mask).to(dev)
    idx = torch.full((w.n_seq, w.n_kv), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((w.n_seq,), dtype=torch.int32, device=dev)
    if use_gpu_compaction:
        ws = torch.zeros(binding.mla_compact_workspace_size(w.n_seq, w.n_kv), dtype=torch.uint8,
                         device=dev)
        binding.mla_compact_mask_ex(m[:, 0, :], idx, cnt, ws)
    else:
        for b in range(w.n_seq):
            idx[b, : len(idx_rows[b])] = torch.from_numpy(idx_rows[b]).to(dev)
        cnt.copy_(torch.tensor(counts, dtype=torch.int32))
    n_out = w.n_seq * w.n_q * w.n_head * 512
    big = torch.full((n_out + CANARY,), float("nan"), dtype=torch.float32, device=dev)
    out = big[:n_out].view(w.n_seq, w.n_q, w.n_head, 512)
    binding.forward(q, k, w.kv_type, m, w.scale, out=out, idx=idx, idx_count=cnt)
    torch.cuda.synchronize()
    status = binding.mla_get_device_status()
    assert bool(torch.isnan(big[n_out:]).all())
    return out.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy(), status


def test_q8_0_dense_matches_oracle_on_same_dequantised_values():
    w = W.make("sparse_q8_decode", n_kv=4096, n_head=128, tail_blocks=4)
    w.sparse = False
    got = run_gpu(w)
    kf16 = q8_f16_rounded(w.kcache[0])
    ref_same = oracle.attention(w.q[0], kf16, oracle.KV_F16, w.mask[0], w.scale)
    assert_parity(got[0].reshape(-1, 512), ref_same, "q8_0 vs oracle(f16-rounded d*q)")
    ref_exact = oracle_rows(w, 0)  # exact d*q in fp64
    assert_parity(got[0].reshape(-1, 512), ref_exact, "q8_0 vs oracle(exact d*q)")


@pytest.mark.parametrize("n_head", [16, 128])
def test_q8_0_ragged_no_mask(n_head):
    rng = np.random.default_rng(n_head)
    w = W.make("sparse_q8_decode", n_kv=1000, n_head=n_head, block=8, tail_blocks=2)
    w.sparse = False
    w.mask = None
    got = run_gpu(w, mask=None)
    ref = oracle.attention(w.q[0], q8_f16_rounded(w.kcache[0]), oracle.KV_F16, None, w.scale)
    assert_parity(got[0].reshape(-1, 512), ref, f"q8_0 H={n_head} no mask")


def test_sparse_f16_gather_equals_dense_masked():
    w = W.make("v2lite_decode", n_kv=3000, n_head=128, n_pad=0)
    rng = np.random.default_rng(9)
    keep = rng.random(3000) < 0.15
    keep[-7:] = True
    w.mask[0, 0] = np.where(keep, np.float16(0), np.float16(-np.inf))
    w.sparse = True
    got, idx, cnt, status = run_sparse_gpu(w)
    assert status == 0
    assert cnt[0] == keep.sum() and np.array_equal(idx[0, : cnt[0]], np.nonzero(keep)[0])
    ref = oracle_rows(w, 0)  # dense masked path
    assert_parity(got[0].reshape(-1, 512), ref, "sparse f16 gather")


def test_sparse_q8_reduced_chain():
    w = W.make("sparse_q8_decode", n_kv=16384, n_head=128, tail_blocks=4)
    got, idx, cnt, status = run_sparse_gpu(w)
    assert status == 0
    ref_idx = oracle.compact(w.mask[0, 0])
    assert cnt[0] == len(ref_idx) and np.array_equal(idx[0, : cnt[0]], ref_idx)
    kf16 = q8_f16_rounded(w.kcache[0])
    ref = oracle.attention(w.q[0], kf16, oracle.KV_F16, w.mask[0], w.scale, idx=ref_idx)
    assert_parity(got[0].reshape(-1, 512), ref, "sparse q8_0 chain")


def test_sparse_q8_full_size_every_row():
    w = W.make("sparse_q8_decode")
    got, idx, cnt, status = run_sparse_gpu(w)
    assert status == 0 and cnt[0] == 16384
    ref_idx = oracle.compact(w.mask[0, 0])
    assert np.array_equal(idx[0, : cnt[0]], ref_idx)
    ref = oracle.attention(w.q[0], w.kcache[0], oracle.KV_Q8_0, w.mask[0], w.scale, idx=ref_idx)
    assert_parity(got[0].reshape(-1, 512), ref, "sparse q8_0 full")


def test_sparse_count_zero_and_partial_lists():
    w = W.make("v3_batched_decode", n_seq=3, n_head=16, n_kv=900, len_lo=900, len_hi=900)
    w.mask[:] = 0
    rng = np.random.default_rng(4)
    lists = [np.array([], np.int32), np.sort(rng.choice(900, 50, replace=False)).astype(np.int32),
             np.arange(900, dtype=np.int32)]
    counts = [0, 50, 900]
    got, _, _, status = run_sparse_gpu(w, idx_rows=lists, counts=counts, use_gpu_compaction=False)
    assert status == 0
    assert np.all(got[0] == 0)
    for b in (1, 2):
        ref = oracle.attention(w.q[b], w.kcache[b], 0, w.mask[b], w.scale, idx=lists[b])
        assert_parity(got[b].reshape(-1, 512), ref, f"sparse list {b}")


@pytest.mark.parametrize("kv", ["f16", "q8_0"])
def test_sparse_out_of_range_index_is_reported_not_read(kv):
    if kv == "f16":
        w = W.make("tiny_decode", n_kv=300)
    else:
        w = W.make("sparse_q8_decode", n_kv=300, n_head=16, block=8, tail_blocks=1)
    w.mask[:] = 0
    # one index beyond n_kv, one negative: both dropped (zero row, -inf score)
    lst = np.array([3, 10, 299, 300 + 5, 17, -2, 250], np.int32)
    got, _, _, status = run_sparse_gpu(w, idx_rows=[lst], counts=[len(lst)], use_gpu_compaction=False)
    assert status == -9  # MLA_ERR_INDEX recorded; the bad rows are treated as dropped
    ok = np.array([3, 10, 299, 17, 250], np.int32)
    ref = oracle.attention(w.q[0], w.kcache[0], w.kv_type, w.mask[0], w.scale, idx=ok)
    assert_parity(got[0].reshape(-1, 512), ref, f"bad index dropped ({kv})")


@pytest.mark.parametrize("kv", ["f16", "q8_0"])
def test_index_list_paths_by_group_count(kv):
    # A sequence with a single 128-row group gathers its list's rows into a dense buffer
    # for the TMA-mode kernel; with several groups (3 query tokens x 128 heads) the list
    # is read by the gather modes inside the attention kernel. Both against the oracle,
    # and the kernels each path launches.
    torch = torch_mod()
    rng = np.random.default_rng(71 if kv == "f16" else 72)
    n_kv = 2600
    for n_q, n_head in ((1, 128), (3, 128)):
        if kv == "f16":
            w = W.make("prefill_chunk", seed=81, n_q=n_q, n_head=n_head, n_kv=n_kv)
        else:
            w = W.make("sparse_q8_decode", seed=82, n_kv=n_kv, n_head=n_head, block=8, tail_blocks=2)
            w.q = rng.standard_normal((1, n_q, n_head, 576)).astype(np.float16)
        w.mask = np.where(rng.random((1, n_q, n_kv)) < 0.9, rng.standard_normal((1, n_q, n_kv)),
                          -np.inf).astype(np.float16)
        lst = np.sort(rng.choice(n_kv, 700, replace=False)).astype(np.int32)
        dev = torch.device("cuda")
        q, k, m = (torch.from_numpy(x).to(dev) for x in (w.q, w.kcache, w.mask))
        idx = torch.full((1, n_kv), -1, dtype=torch.int32, device=dev)
        idx[0, : len(lst)] = torch.from_numpy(lst).to(dev)
        cnt = torch.tensor([len(lst)], dtype=torch.int32, device=dev)
        out = torch.full((1, n_q, n_head, 512), float("nan"), dtype=torch.float32, device=dev)
        ran = _launches(lambda: binding.forward(q, k, w.kv_type, m, w.scale, out=out, idx=idx, idx_count=cnt))
        assert binding.mla_get_device_status() == 0
        if n_q * n_head <= 128:
            assert ran.get("mla_gather_rows") == 1 and "mla_fwd_f16" in ran, ran
        else:
            assert "mla_gather_rows" not in ran, ran
            assert ("mla_fwd_q8_0" if kv == "q8_0" else "mla_fwd_gather_f16") in ran, ran
        kref = q8_f16_rounded(w.kcache[0]) if kv == "q8_0" else w.kcache[0]
        ref = oracle.attention(w.q[0], kref, oracle.KV_F16, w.mask[0], w.scale, idx=lst)
        assert_parity(out[0].reshape(-1, 512).cpu().numpy(), ref, f"index list {kv} n_q={n_q}")


@pytest.mark.parametrize("pad", [0, 3])
def test_q8_gathered_rows_at_the_cache_ends(pad):
    # The row gather copies each q8_0 row's 16-byte-aligned span (612-byte rows start 4
    # bytes apart modulo 16); a span that would reach past the end of the cache is read
    # word by word instead. Lists holding the first and last rows of every sequence, two
    # sequences, a contiguous cache and one with `pad` rows between sequences; the last
    # row of the cache starts 4 and 0 bytes past a 16-byte boundary in the two cases.
    torch = torch_mod()
    rng = np.random.default_rng(91 + pad)
    n_kv, n_seq, n_head = 1001, 2, 128
    k = W.q8_0_random(np.random.Generator(np.random.PCG64(92 + pad)), (n_seq, n_kv + pad))
    q = rng.standard_normal((n_seq, 1, n_head, 576)).astype(np.float16)
    mask = np.where(rng.random((n_seq, 1, n_kv)) < 0.95, rng.standard_normal((n_seq, 1, n_kv)),
                    -np.inf).astype(np.float16)
    lists = [np.unique(np.concatenate([[0, 1, 2, 3, n_kv - 2, n_kv - 1], rng.choice(n_kv, 240)])),
             np.array([0, n_kv - 1], dtype=np.int64)]
    dev = torch.device("cuda")
    kt = torch.from_numpy(k).to(dev)[:, :n_kv]  # sequences n_kv + pad rows apart
    qt, mt = torch.from_numpy(q).to(dev), torch.from_numpy(mask).to(dev)
    idx = torch.full((n_seq, n_kv), -1, dtype=torch.int32, device=dev)
    for b, lst in enumerate(lists):
        idx[b, : len(lst)] = torch.from_numpy(lst.astype(np.int32)).to(dev)
    cnt = torch.tensor([len(x) for x in lists], dtype=torch.int32, device=dev)
    out = torch.full((n_seq, 1, n_head, 512), float("nan"), dtype=torch.float32, device=dev)
    ran = _launches(lambda: binding.forward(qt, kt, binding.KV_Q8_0, mt, W.SCALE_192, out=out, idx=idx,
                                            idx_count=cnt))
    assert binding.mla_get_device_status() == 0
    assert ran.get("mla_gather_rows") == 1, ran
    last = (n_seq - 1) * (n_kv + pad) + n_kv - 1
    assert (612 * last) % 16 != 12  # the last row's span would pass the cache's end
    for b, lst in enumerate(lists):
        ref = oracle.attention(q[b], q8_f16_rounded(k[b, :n_kv]), oracle.KV_F16, mask[b], W.SCALE_192,
                               idx=lst.astype(np.int32))
        assert_parity(out[b].reshape(-1, 512).cpu().numpy(), ref, f"q8_0 gathered rows pad={pad} seq {b}")


# ---- fused value up-projection (out_proj = O . W_UV per head) ---------------------

# ---- mask gather: sparse attention straight from the mask (the compaction fused in) ----
# Dropping the cells whose mask is -inf leaves every row's softmax unchanged, so the
# reference is the oracle's dense masked attention.
def sparse_rows_mask(rng, n_q, n_kv, p_keep, shared_frac=0.0):
    """Per-token keep patterns: a shared random part plus each token's own cells."""
    shared = rng.random(n_kv) < p_keep * shared_frac
    own = rng.random((n_q, n_kv)) < p_keep * (1.0 - shared_frac)
    keep = own | shared[None]
    vals = rng.standard_normal((n_q, n_kv)).astype(np.float16)
    return np.where(keep, vals, np.float16(-np.inf)).astype(np.float16)


def test_mask_gather_f16_single_query():
    w = W.make("v2lite_decode", n_kv=3000, n_head=128, n_pad=0)
    rng = np.random.default_rng(21)
    keep = rng.random(3000) < 0.15
    keep[-7:] = True
    w.mask[0, 0] = np.where(keep, np.float16(0), np.float16(-np.inf))
    check_all_rows(w, run_gpu(w, mask_gather=True), what="mask gather f16")


@pytest.mark.parametrize("n_head,n_q", [(16, 8), (16, 19), (100, 3), (128, 3), (7, 5)])
def test_mask_gather_multi_query(n_head, n_q):
    # 128-row groups that span several tokens take the union of their masks; each row
    # still applies its own
    rng = np.random.default_rng(n_head * 100 + n_q)
    n_kv = 2500
    w = W.make("prefill_chunk", n_q=n_q, n_head=n_head, n_kv=n_kv)
    w.mask[0] = sparse_rows_mask(rng, n_q, n_kv, 0.2, shared_frac=0.5)
    w.mask[0, :, rng.integers(0, n_kv)] = 0
    check_all_rows(w, run_gpu(w, mask_gather=True), what=f"mask gather H={n_head} n_q={n_q}")


def test_mask_gather_ragged_batch_with_splits_and_empty_rows():
    w = W.make("v3_batched_decode", n_seq=5, n_head=16, n_kv=9000, len_lo=1, len_hi=9000)
    rng = np.random.default_rng(33)
    w.q = rng.standard_normal((5, 2, 16, 576)).astype(np.float16)
    w.kv_len = np.array([9000, 1, 0, 4097, 257], np.int32)
    w.mask = np.stack([sparse_rows_mask(rng, 2, 9000, 0.1) for _ in range(5)])
    w.mask[3] = np.float16(-np.inf)           # no kept cell in the whole sequence
    w.mask[4, 1] = np.float16(-np.inf)        # one token with no kept cell
    w.mask[1, :, 0] = 0
    got = run_gpu(w, mask_gather=True)
    assert np.all(got[2] == 0) and np.all(got[3] == 0) and np.all(got[4, 1] == 0)
    for b in range(w.n_seq):
        n = int(w.kv_len[b])
        ref = oracle.attention(w.q[b], w.kcache[b][:n], w.kv_type, w.mask[b][:, :n], w.scale) if n \
            else np.zeros((w.n_q * w.n_head, 512))
        assert_parity(got[b].reshape(-1, 512), ref, f"mask gather ragged seq {b}")


def test_mask_gather_every_cell_kept_equals_dense():
    w = W.make("v3_batched_decode", n_seq=2, n_head=128, n_kv=3000, len_lo=3000, len_hi=3000)
    dense = run_gpu(w)
    gath = run_gpu(w, mask_gather=True)
    assert_parity(gath.reshape(-1, 512), dense.reshape(-1, 512), "all kept vs dense")
    check_all_rows(w, gath, what="mask gather all kept")


def test_mask_gather_q8_0_reduced():
    w = W.make("sparse_q8_decode", n_kv=16384, n_head=128, tail_blocks=4)
    got = run_gpu(w, mask_gather=True)
    ref = oracle.attention(w.q[0], q8_f16_rounded(w.kcache[0]), oracle.KV_F16, w.mask[0], w.scale)
    assert_parity(got[0].reshape(-1, 512), ref, "mask gather q8_0")


def test_mask_gather_q8_0_full_size_every_row():
    w = W.make("sparse_q8_decode")
    got = run_gpu(w, mask_gather=True)
    ref = oracle.attention(w.q[0], w.kcache[0], oracle.KV_Q8_0, w.mask[0], w.scale)
    assert_parity(got[0].reshape(-1, 512), ref, "mask gather q8_0 full")


def test_mask_gather_q8_0_multi_query_ragged():
    rng = np.random.default_rng(44)
    w = W.make("sparse_q8_decode", n_kv=5000, n_head=16, block=8, tail_blocks=2)
    q = rng.standard_normal((1, 6, 16, 576)).astype(np.float16)
    w.q = q
    w.mask = sparse_rows_mask(rng, 6, 5000, 0.12, shared_frac=0.3)[None]
    got = run_gpu(w, mask_gather=True)
    ref = oracle.attention(w.q[0], q8_f16_rounded(w.kcache[0]), oracle.KV_F16, w.mask[0], w.scale)
    assert_parity(got[0].reshape(-1, 512), ref, "mask gather q8_0 multi-query")


def test_mask_gather_with_variants():
    w = W.make("prefill_chunk", n_q=4, n_head=16, n_kv=3000)
    rng = np.random.default_rng(55)
    w.mask[0] = sparse_rows_mask(rng, 4, 3000, 0.25)
    sinks = rng.standard_normal(16).astype(np.float32)
    got = run_gpu(w, mask_gather=True, sinks=sinks, softcap=30.0)
    ref = oracle.attention_variants(w.q[0], w.kcache[0], w.kv_type, w.mask[0], w.scale,
                                    softcap=30.0, sinks=sinks)
    assert_parity(got[0].reshape(-1, 512), ref, "mask gather + sinks + softcap")


def run_gpu_proj(w, wv, mask_gather=False):
    """mla_fa_forward_ex with wv set; returns out_proj [n_seq][n_q][n_head][128]."""
    torch = torch_mod()
    dev = torch.device("cuda")
    q = torch.from_numpy(w.q).to(dev)
    k = torch.from_numpy(w.kcache).to(dev)
    m = torch.from_numpy(w.mask).to(dev) if w.mask is not None else None
    n_out = w.n_seq * w.n_q * w.n_head * 128
    big = torch.full((n_out + CANARY,), float("nan"), dtype=torch.float32, device=dev)
    out_proj = big[:n_out].view(w.n_seq, w.n_q, w.n_head, 128)
    binding.forward_proj(q, k, w.kv_type, m, w.scale, torch.from_numpy(wv).to(dev),
                         out_proj=out_proj, kv_len=w.kv_len, mask_gather=mask_gather)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    assert bool(torch.isnan(big[n_out:]).all()), "write past the end of out_proj"
    return out_proj.cpu().numpy()


def check_proj(w, wv, got, what):
    rows = w.n_q * w.n_head
    heads = np.arange(rows) % w.n_head
    for b in range(w.n_seq):
        ref = oracle.project(oracle_rows(w, b), heads, wv)
        assert_parity(got[b].reshape(rows, 128), ref, f"{what} seq {b}")


@pytest.mark.parametrize("case", ["v3_split", "tiny_unsplit", "prefill_rows", "ragged_heads"])
def test_fused_projection_matches_oracle(case):
    if case == "v3_split":      # 8 sequences, split-KV partials
        w = W.make("v3_batched_decode", n_kv=2048, len_lo=100, len_hi=2048)
    elif case == "tiny_unsplit":  # one unit: the partial slot is forced
        w = W.make("tiny_decode", n_kv=300)
    elif case == "prefill_rows":  # 8 tokens x 128 heads: row batches span tokens
        w = W.make("prefill_chunk", n_q=8, n_head=128, n_kv=640)
    else:                          # 3 tokens x 5 heads: the last row batch is partial
        w = W.make("prefill_chunk", n_q=3, n_head=5, n_kv=300)
    wv = W.wv_random(n_head=w.n_head)
    got = run_gpu_proj(w, wv)
    check_proj(w, wv, got, case)


def test_fused_projection_with_mask_gather():
    w = W.make("prefill_chunk", n_q=3, n_head=128, n_kv=4000)
    rng = np.random.default_rng(66)
    w.mask[0] = sparse_rows_mask(rng, 3, 4000, 0.1)
    wv = W.wv_random(n_head=128)
    check_proj(w, wv, run_gpu_proj(w, wv, mask_gather=True), "projection + mask gather")


def test_fused_projection_with_an_empty_sequence():
    # a zero-length sequence projects a zero row (its lengths also set in the mask,
    # which the oracle follows)
    w = W.make("v3_batched_decode", n_seq=3, n_head=16, n_kv=700, len_lo=0, len_hi=700)
    w.kv_len[:] = [300, 0, 700]
    keep = np.arange(700)[None, :] < w.kv_len[:, None]
    w.mask[:, 0, :] = np.where(keep, np.float16(0), np.float16(-np.inf))
    wv = W.wv_random(n_head=16)
    got = run_gpu_proj(w, wv)
    assert np.all(got[1] == 0.0)
    check_proj(w, wv, got, "kv_len 300/0/700")


# ---- attention variants: logit softcap, ALiBi, sinks -----------------------------

def alibi_slopes(n_head):
    return np.array([2.0 ** (-8.0 * (h + 1) / n_head) for h in range(n_head)])


def check_variants(w, got, what, softcap=0.0, slopes=None, sinks=None, kcache=None, kv_type=None):
    for b in range(w.n_seq):
        ref = oracle.attention_variants(
            w.q[b], w.kcache[b] if kcache is None else kcache, w.kv_type if kv_type is None else kv_type,
            w.mask[b] if w.mask is not None else None, w.scale, softcap=softcap, slopes=slopes,
            pos0=int(w.kv_len[b]) - w.n_q, sinks=sinks)
        assert_parity(got[b].reshape(-1, 512), ref, f"{what} seq {b}")


def test_softcap_matches_oracle():
    w = W.make("tiny_decode", n_kv=300)
    got = run_gpu(w, softcap=5.0)
    check_variants(w, got, "softcap", softcap=5.0)


def test_alibi_matches_oracle_prefill_rows():
    w = W.make("prefill_chunk", n_q=8, n_head=128, n_kv=640)
    sl = alibi_slopes(128)
    got = run_gpu(w, alibi_slopes=sl)
    check_variants(w, got, "alibi", slopes=sl)


def test_alibi_long_sequence_precision():
    # biases up to 0.5 x 4095 relative to the last key
    w = W.make("v2lite_decode", n_kv=4096, n_head=16, n_pad=0)
    sl = alibi_slopes(16)
    got = run_gpu(w, alibi_slopes=sl)
    check_variants(w, got, "alibi long", slopes=sl)


def test_sinks_with_split_plan():
    w = W.make("v3_batched_decode", n_kv=2048, len_lo=100, len_hi=2048)
    sinks = np.random.default_rng(7).normal(0.0, 2.0, 128)
    got = run_gpu(w, sinks=sinks)
    check_variants(w, got, "sinks", sinks=sinks)


def test_sinks_unsplit_and_empty_sequence():
    w = W.make("v3_batched_decode", n_seq=3, n_head=16, n_kv=700, len_lo=0, len_hi=700)
    w.kv_len[:] = [300, 0, 700]
    keep = np.arange(700)[None, :] < w.kv_len[:, None]
    w.mask[:, 0, :] = np.where(keep, np.float16(0), np.float16(-np.inf))
    sinks = np.linspace(-3.0, 3.0, 16)
    got = run_gpu(w, sinks=sinks)
    assert np.all(got[1] == 0.0)
    check_variants(w, got, "sinks kv_len 300/0/700", sinks=sinks)


def test_all_variants_together():
    w = W.make("prefill_chunk", n_q=3, n_head=5, n_kv=300)
    sl = alibi_slopes(5)
    sinks = np.array([0.5, -1.0, 2.0, 0.0, 3.0])
    got = run_gpu(w, softcap=4.0, alibi_slopes=sl, sinks=sinks)
    check_variants(w, got, "all variants", softcap=4.0, slopes=sl, sinks=sinks)


def test_softcap_q8_0_dense():
    w = W.make("sparse_q8_decode", n_kv=2048, n_head=128, tail_blocks=4)
    w.sparse = False
    got = run_gpu(w, softcap=6.0)
    check_variants(w, got, "softcap q8_0", softcap=6.0, kcache=q8_f16_rounded(w.kcache[0]),
                   kv_type=oracle.KV_F16)


# ---- per-row log-sum-exp and the merge across calls (split-KV across devices) ----------
# Tolerance of the lse: 2e-3 absolute. A merge weighs a part by e^{lse}, so an lse error
# d changes that part's relative weight by about d; 2e-3 keeps merged rows inside the
# rel-L2 2e-3 budget of the attention output.
LSE_ATOL = 2e-3


def run_gpu_lse(w, idx=None, idx_count=None, mask_gather=False):
    torch = torch_mod()
    dev = torch.device("cuda")
    q = torch.from_numpy(w.q).to(dev)
    k = torch.from_numpy(w.kcache).to(dev)
    m = torch.from_numpy(w.mask).to(dev) if w.mask is not None else None
    rows = w.n_seq * w.n_q * w.n_head
    out = torch.full((w.n_seq, w.n_q, w.n_head, 512), float("nan"), device=dev)
    big = torch.full((rows + CANARY,), float("nan"), device=dev)
    lse = big[:rows].view(w.n_seq, w.n_q, w.n_head)
    binding.forward(q, k, w.kv_type, m, w.scale, out=out, kv_len=w.kv_len, idx=idx,
                    idx_count=idx_count, out_lse=lse, mask_gather=mask_gather)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    assert bool(torch.isnan(big[rows:]).all()), "write past the end of out_lse"
    return out.cpu().numpy(), lse.cpu().numpy()


def assert_lse(got, ref, what):
    got = np.asarray(got, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), f"{what}: -inf rows differ"
    fin = np.isfinite(ref)
    assert np.all(np.isfinite(got[fin])), f"{what}: non-finite lse"
    err = float(np.max(np.abs(got[fin] - ref[fin]))) if fin.any() else 0.0
    assert err <= LSE_ATOL, f"{what}: lse max-abs {err:.3g}"


@pytest.mark.parametrize("case", ["v3_split", "tiny_unsplit", "prefill_rows", "empty_and_masked"])
def test_out_lse_matches_oracle(case):
    if case == "v3_split":
        w = W.make("v3_batched_decode", n_kv=2048, len_lo=100, len_hi=2048)
    elif case == "tiny_unsplit":
        w = W.make("tiny_decode", n_kv=300)
    elif case == "prefill_rows":
        w = W.make("prefill_chunk", n_q=3, n_head=100, n_kv=700)
    else:
        w = W.make("v3_batched_decode", n_seq=3, n_head=16, n_kv=600, len_lo=600, len_hi=600)
        w.kv_len[:] = [600, 0, 350]
        w.mask[2] = np.float16(-np.inf)
    got, lse = run_gpu_lse(w)
    for b in range(w.n_seq):
        n = int(w.kv_len[b])
        if n == 0:
            assert np.all(got[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        o_ref, l_ref = oracle.attention_lse(w.q[b], w.kcache[b][:n], w.kv_type,
                                            None if w.mask is None else w.mask[b][:, :n], w.scale)
        assert_parity(got[b].reshape(-1, 512), o_ref, f"{case} out seq {b}")
        assert_lse(lse[b], l_ref, f"{case} lse seq {b}")


def test_out_lse_sparse_q8_and_mask_gather():
    torch = torch_mod()
    w = W.make("sparse_q8_decode", n_kv=16384, n_head=128, tail_blocks=4)
    ref_idx = oracle.compact(w.mask[0, 0])
    kf16 = q8_f16_rounded(w.kcache[0])
    o_ref, l_ref = oracle.attention_lse(w.q[0], kf16, oracle.KV_F16, w.mask[0], w.scale)
    idx = torch.full((1, w.n_kv), -1, dtype=torch.int32, device="cuda")
    idx[0, : len(ref_idx)] = torch.from_numpy(ref_idx).cuda()
    cnt = torch.tensor([len(ref_idx)], dtype=torch.int32, device="cuda")
    for what, kw in (("index list", dict(idx=idx, idx_count=cnt)), ("mask gather", dict(mask_gather=True))):
        got, lse = run_gpu_lse(w, **kw)
        assert_parity(got[0].reshape(-1, 512), o_ref, f"q8_0 {what} out")
        assert_lse(lse[0], l_ref, f"q8_0 {what} lse")


@pytest.mark.parametrize("world", [2, 3])
def test_split_kv_decode_emulated_on_one_gpu(world):
    # the ranks' calls of a split-KV decode, made one after another on one GPU: each
    # attends over its range of the cache with the lse, mla_fa_combine merges them
    torch = torch_mod()
    from mla_flash_attention_attn_b200 import split_kv

    # (the packed layout split_kv.decode gathers: each rank's O rows, then their lse)
    w = W.make("v3_batched_decode", n_kv=4096, len_lo=100, len_hi=4096)
    dev = torch.device("cuda")
    q = torch.from_numpy(w.q).to(dev)
    rows = w.n_seq * w.n_q * w.n_head
    parts = torch.empty((world, binding.packed_width(rows)), device=dev)
    for r, (lo, hi) in enumerate(split_kv.shard_bounds(w.n_kv, world)):
        k = torch.from_numpy(w.kcache[:, lo:hi].copy()).to(dev)
        m = torch.from_numpy(w.mask[:, :, lo:hi].copy()).to(dev)
        binding.forward(q, k, w.kv_type, m, w.scale,
                        out=parts[r, : rows * 512].view(w.n_seq, 1, w.n_head, 512),
                        kv_len=split_kv.shard_lengths(w.kv_len, lo, hi),
                        out_lse=parts[r, rows * 512:].view(w.n_seq, 1, w.n_head))
    lse_out = torch.empty((rows,), device=dev)
    out = binding.combine_packed(parts, rows, out_lse=lse_out)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    got = out.cpu().numpy().reshape(w.n_seq, -1, 512)
    lse = lse_out.cpu().numpy().reshape(w.n_seq, -1)
    for b in range(w.n_seq):
        n = int(w.kv_len[b])
        o_ref, l_ref = oracle.attention_lse(w.q[b], w.kcache[b][:n], w.kv_type, w.mask[b][:, :n], w.scale)
        assert_parity(got[b], o_ref, f"split-KV x{world} seq {b}")
        assert_lse(lse[b], l_ref, f"split-KV x{world} lse seq {b}")


@pytest.mark.parametrize("n_parts,rows", [(1, 5), (2, 1), (5, 1000), (33, 77)])
def test_combine_entry_point_matches_oracle(n_parts, rows):
    torch = torch_mod()
    rng = np.random.default_rng(n_parts * 1000 + rows)
    o = rng.standard_normal((n_parts, rows, 512)).astype(np.float32)
    lse = (rng.standard_normal((n_parts, rows)) * 20).astype(np.float32)
    lse[rng.random((n_parts, rows)) < 0.2] = -np.inf
    lse[:, 0] = -np.inf  # a row with no kept key in any part
    o_ref, l_ref = oracle.combine(o, lse)
    big = torch.full((rows * 512 + CANARY,), float("nan"), device="cuda")
    out = big[: rows * 512].view(rows, 512)
    lse_out = torch.empty((rows,), device="cuda")
    binding.combine(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(), out=out, out_lse=lse_out)
    torch.cuda.synchronize()
    assert bool(torch.isnan(big[rows * 512:]).all())
    got = out.cpu().numpy()
    assert np.all(got[0] == 0)
    # fp32 arithmetic on fp32 inputs: a few ulp of the largest term
    np.testing.assert_allclose(got, o_ref, rtol=1e-5, atol=2e-5)
    lg = lse_out.cpu().numpy()
    assert np.array_equal(np.isneginf(lg), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    np.testing.assert_allclose(lg[fin], l_ref[fin], rtol=0, atol=1e-4)


# ---- the DK = DV = 512 head shape (f16 cache, V = the whole row) -------------------------

def run_dk512(q, k, mask, scale, kv_len=None, idx=None, idx_count=None, **kw):
    torch = torch_mod()
    dev = torch.device("cuda")
    n_seq, n_q, n_head, _ = q.shape
    n_out = n_seq * n_q * n_head * 512
    big = torch.full((n_out + CANARY,), float("nan"), device=dev)
    out = big[:n_out].view(n_seq, n_q, n_head, 512)
    tq = torch.from_numpy(q).to(dev)
    tk = torch.from_numpy(k).to(dev)
    tm = None if mask is None else torch.from_numpy(mask).to(dev)
    binding.forward(tq, tk, 0, tm, scale, out=out, kv_len=kv_len, idx=idx, idx_count=idx_count, **kw)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    assert bool(torch.isnan(big[n_out:]).all()), "write past the end of out"
    return out.cpu().numpy()


@pytest.mark.parametrize("n_seq,n_q,n_head,n_kv", [(1, 1, 16, 300), (4, 1, 128, 3000), (1, 3, 100, 700),
                                                   (2, 2, 16, 1), (1, 1, 128, 257)])
def test_dk512_dense_matches_oracle(n_seq, n_q, n_head, n_kv):
    rng = np.random.default_rng(n_seq * 7 + n_q * 11 + n_head + n_kv)
    q = rng.standard_normal((n_seq, n_q, n_head, 512)).astype(np.float16)
    k = (0.5 * rng.standard_normal((n_seq, n_kv, 512))).astype(np.float16)
    mask = np.where(rng.random((n_seq, n_q, n_kv)) < 0.8, rng.standard_normal((n_seq, n_q, n_kv)),
                    -np.inf).astype(np.float16)
    mask[:, :, 0] = 0
    lens = [n_kv] + [max(1, n_kv - 37 * b) for b in range(1, n_seq)]
    got = run_dk512(q, k, mask, 0.04, kv_len=lens)
    for b in range(n_seq):
        n = lens[b]
        ref = oracle.attention(q[b], k[b, :n], oracle.KV_F16, mask[b, :, :n], 0.04)
        assert_parity(got[b].reshape(-1, 512), ref, f"dk512 seq {b}")


def test_dk512_index_list_equals_dense_masked():
    torch = torch_mod()
    rng = np.random.default_rng(61)
    n_kv = 5000
    q = rng.standard_normal((1, 1, 128, 512)).astype(np.float16)
    k = (0.5 * rng.standard_normal((1, n_kv, 512))).astype(np.float16)
    keep = rng.random(n_kv) < 0.12
    mask = np.where(keep, np.float16(0), np.float16(-np.inf)).astype(np.float16)[None, None]
    lst = np.nonzero(keep)[0].astype(np.int32)
    idx = torch.full((1, n_kv), -1, dtype=torch.int32, device="cuda")
    idx[0, : len(lst)] = torch.from_numpy(lst).cuda()
    cnt = torch.tensor([len(lst)], dtype=torch.int32, device="cuda")
    got = run_dk512(q, k, mask, 0.04, idx=idx, idx_count=cnt)
    ref = oracle.attention(q[0], k[0], oracle.KV_F16, mask[0], 0.04)
    assert_parity(got[0].reshape(-1, 512), ref, "dk512 index list")


def test_dk512_with_sinks_and_lse():
    torch = torch_mod()
    rng = np.random.default_rng(62)
    q = rng.standard_normal((2, 1, 16, 512)).astype(np.float16)
    k = (0.5 * rng.standard_normal((2, 2000, 512))).astype(np.float16)
    lse = torch.empty((2, 1, 16), device="cuda")
    got = run_dk512(q, k, None, 0.04, out_lse=lse)
    for b in range(2):
        o_ref, l_ref = oracle.attention_lse(q[b], k[b], oracle.KV_F16, None, 0.04)
        assert_parity(got[b].reshape(-1, 512), o_ref, f"dk512 lse out {b}")
        assert_lse(lse[b].cpu().numpy(), l_ref, f"dk512 lse {b}")
    sinks = rng.standard_normal(16).astype(np.float32)
    got = run_dk512(q, k, None, 0.04, sinks=torch.from_numpy(sinks).cuda())
    for b in range(2):
        # a sink is one more logit per head with no value: the row is the plain
        # attention scaled by its share e^{lse} / (e^{lse} + e^{sink})
        o_ref, l_ref = oracle.attention_lse(q[b], k[b], oracle.KV_F16, None, 0.04)
        share = 1.0 / (1.0 + np.exp(np.tile(sinks.astype(np.float64), 1) - l_ref))
        assert_parity(got[b].reshape(-1, 512), o_ref * share[:, None], f"dk512 sinks {b}")


# ------------------------------------------------------------------ tile ranges from the mask
def _launches(fn):
    binding.mla_profile_begin()
    fn()
    torch_mod().cuda.synchronize()
    return {k: v[0] for k, v in binding.mla_profile_end().items()}


def test_mask_derived_ranges_skip_leading_and_trailing_tiles():
    # a window of kept cells in the middle of each sequence, no host lengths: the scan
    # finds each group's first and last kept tile and the device plan spreads those tiles
    # over the SM pairs
    w = W.make("v3_batched_decode", seed=21, n_seq=3, n_kv=6000, len_lo=6000, len_hi=6000)
    windows = [(1000, 1777), (0, 300), (4100, 6000)]
    for b, (lo, hi) in enumerate(windows):
        w.mask[b, 0, :] = np.float16(-np.inf)
        w.mask[b, 0, lo:hi] = 0
    got = run_gpu(w, kv_len=None)
    check_all_rows(w, got, what="window")


def test_mask_derived_ranges_fully_masked_sequence_and_group():
    w = W.make("v3_batched_decode", seed=22, n_seq=2, n_head=100, n_kv=1500, len_lo=1500,
               len_hi=1500)
    w.q = np.ascontiguousarray(np.repeat(w.q, 3, axis=1))  # 3 tokens: groups span tokens
    w.mask = np.ascontiguousarray(np.repeat(w.mask, 3, axis=1))
    w.mask[0] = np.float16(-np.inf)        # a whole sequence masked
    w.mask[1, 1, :] = np.float16(-np.inf)  # one token of the other
    got = run_gpu(w, kv_len=None)
    assert np.all(got[0] == 0.0) and np.all(got[1, 1] == 0.0)
    check_all_rows(w, got, what="masked groups")


def test_mask_derived_ranges_are_the_path_taken():
    torch = torch_mod()
    w = W.make("v3_batched_decode", seed=23, n_seq=2, n_kv=3000, len_lo=1000, len_hi=3000)
    dev = torch.device("cuda")
    q, k, m = (torch.from_numpy(x).to(dev) for x in (w.q, w.kcache, w.mask))
    no_len = _launches(lambda: binding.forward(q, k, w.kv_type, m, w.scale))
    with_len = _launches(lambda: binding.forward(q, k, w.kv_type, m, w.scale, kv_len=w.kv_len))
    assert no_len.get("mla_scan") == 1 and no_len.get("mla_device_plan") == 1
    assert "mla_scan" not in with_len and "mla_device_plan" not in with_len
    assert binding.mla_get_device_status() == 0
