"""Split-KV decode across ranks, its orchestration on CPU with one, two and three gloo ranks.

The kernels need a GPU; here each rank's attention and the final merge are stand-ins
built on the oracle (with the same signatures as the library calls), so what runs is
the module's own logic: the cache ranges of the ranks, the per-sequence lengths inside
a range, the all-gather of (O, lse) in rank order, and the merge. The result must equal
the oracle's attention over the whole cache.
"""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_forward(q, k, kv_type, mask, scale, out=None, kv_len=None, out_lse=None):
    import torch

    import oracle

    for b in range(q.shape[0]):
        n = k.shape[1] if kv_len is None else int(kv_len[b])
        rows = q.shape[1] * q.shape[2]
        if n == 0:
            out[b].zero_()
            out_lse[b].fill_(-np.inf)
            continue
        m = None if mask is None else mask[b, :, :n].numpy()
        o, lse = oracle.attention_lse(q[b].numpy(), k[b, :n].numpy(), kv_type, m, scale)
        out[b].copy_(torch.from_numpy(o.reshape(out[b].shape)))
        out_lse[b].copy_(torch.from_numpy(lse.reshape(out_lse[b].shape)))


def _oracle_combine(parts, rows):
    import torch

    import oracle

    p = parts.numpy()
    o_all = p[:, : rows * 512].reshape(p.shape[0], rows, 512)
    lse_all = p[:, rows * 512:]
    o, _ = oracle.combine(o_all, lse_all)
    return torch.from_numpy(o).float()


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "OMP_NUM_THREADS": "2"})
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from mla_flash_attention_attn_b200 import split_kv
    from mla_flash_attention_attn_b200 import workloads as W

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    # 3 sequences of different lengths (one shorter than a rank's range, so some
    # ranks hold none of its cells), 2 query tokens x 4 heads, sparse f16 mask
    w = W.make("v3_batched_decode", n_seq=3, n_head=4, n_kv=700, len_lo=1, len_hi=700)
    rng = np.random.default_rng(7)
    q = rng.standard_normal((3, 2, 4, 576)).astype(np.float16)
    kv_len = [700, 150, 431]
    mask = np.where(rng.random((3, 2, 700)) < 0.6, rng.standard_normal((3, 2, 700)),
                    -np.inf).astype(np.float16)
    lo, hi = split_kv.shard_bounds(700, world)[rank]
    out = split_kv.decode(torch.from_numpy(q), torch.from_numpy(w.kcache[:, lo:hi].copy()), 0,
                          torch.from_numpy(mask[:, :, lo:hi].copy()), w.scale,
                          kv_len_shard=split_kv.shard_lengths(kv_len, lo, hi),
                          forward=_oracle_forward, combine=_oracle_combine)
    dist.destroy_process_group()
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), out.numpy())
    if rank == 0:
        import oracle

        ref = np.stack([oracle.attention(q[b], w.kcache[b, :kv_len[b]], 0,
                                         mask[b, :, :kv_len[b]], w.scale).reshape(2, 4, 512)
                        for b in range(3)])
        np.save(os.path.join(out_dir, "ref.npy"), ref)


@pytest.mark.parametrize("world", [1, 2, 3])
def test_split_kv_decode_over_gloo_ranks_equals_the_whole_cache(tmp_path, world):
    import torch.multiprocessing as mp

    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    ref = np.load(tmp_path / "ref.npy")
    for rank in range(world):
        got = np.load(tmp_path / f"rank{rank}.npy")
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)


def test_shard_bounds_and_lengths():
    sys.path.insert(0, ROOT)
    from mla_flash_attention_attn_b200 import split_kv

    assert split_kv.shard_bounds(10, 3) == [(0, 3), (3, 6), (6, 10)]
    assert split_kv.shard_bounds(4, 4) == [(0, 1), (1, 2), (2, 3), (3, 4)]
    with pytest.raises(ValueError):
        split_kv.shard_bounds(3, 4)
    assert split_kv.shard_lengths([10, 4, 0, 7], 3, 6) == [3, 1, 0, 3]
