"""GPU parity of the DK = 192 / DV = 128 head shape (a K and a V per KV head) against the
fp64 oracle `oracle.attention_heads`, through the C ABI (mla_fa_forward_ex with
head_dim = 192).

Tolerance as for the MLA shape: max-abs error <= 1e-2 and relative L2 error <= 2e-3.
Outputs are pre-filled with NaN and followed by a NaN canary region.
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


def assert_parity(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, what
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = got - ref
    nref = np.linalg.norm(ref)
    maxabs = float(np.max(np.abs(err))) if err.size else 0.0
    if nref == 0.0:
        assert maxabs == 0.0, f"{what}: expected zeros, max |err| {maxabs}"
        return
    rel = float(np.linalg.norm(err) / nref)
    assert maxabs <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {maxabs:.3g} rel-L2 {rel:.3g}"


def run(w, kv_len="auto", use_mask=True):
    import torch

    dev = torch.device("cuda")
    q = torch.from_numpy(w.q).to(dev)
    k = torch.from_numpy(w.k).to(dev)
    v = torch.from_numpy(w.v).to(dev)
    m = torch.from_numpy(w.mask).to(dev) if (use_mask and w.mask is not None) else None
    n_out = w.n_seq * w.n_q * w.n_head * 128
    big = torch.full((n_out + CANARY,), float("nan"), dtype=torch.float32, device=dev)
    out = big[:n_out].view(w.n_seq, w.n_q, w.n_head, 128)
    lens = [int(x) for x in w.kv_len] if kv_len == "auto" else kv_len
    binding.forward_heads(q, k, v, m, w.scale, out=out, kv_len=lens)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    assert bool(torch.isnan(big[n_out:]).all()), "write past the end of out"
    return out.cpu().numpy()


def check(w, got, lens=None, use_mask=True, what=""):
    for b in range(w.n_seq):
        L = w.n_kv if lens is None else int(lens[b])
        mask = w.mask[b, :, :L] if (use_mask and w.mask is not None) else None
        ref = oracle.attention_heads(w.q[b], w.k[b, :L], w.v[b, :L], mask, w.scale)
        assert_parity(got[b].reshape(-1, 128), ref, f"{what} seq {b}")


def plan_of(w):
    import torch

    dev = torch.device("cuda")
    q = torch.zeros(w.q.shape, dtype=torch.float16, device=dev)
    k = torch.zeros(w.k.shape, dtype=torch.float16, device=dev)
    v = torch.zeros(w.v.shape, dtype=torch.float16, device=dev)
    out = torch.zeros(w.q.shape[:3] + (128,), dtype=torch.float32, device=dev)
    args, keep = binding.make_heads_args(q, k, v, None, out, w.scale, [int(x) for x in w.kv_len])
    return binding.mla_fa_query_plan(args)


@pytest.mark.parametrize("n_q,n_head,n_kv_head,n_kv", [
    (37, 16, 16, 700),     # multi-head attention, ragged row groups and tiles
    (20, 32, 4, 513),      # grouped: 8 query heads per KV head, rows span tokens
    (3, 128, 1, 300),      # one shared KV head: 128 query heads, one 128-row group per token
    (1, 16, 16, 129),      # decode-sized, one key past a tile
])
def test_heads_prefill_causal(n_q, n_head, n_kv_head, n_kv):
    w = W.heads_prefill(n_q=n_q, n_head=n_head, n_kv_head=n_kv_head, n_kv=n_kv)
    check(w, run(w), what=f"heads {n_q}x{n_head}/{n_kv_head}")


def test_heads_no_mask_and_one_key():
    w = W.heads_prefill(n_q=5, n_head=8, n_kv_head=2, n_kv=1, causal=False)
    got = run(w, use_mask=False)
    check(w, got, use_mask=False, what="one key")
    # one key: every row is that key's V row of its KV head
    for h in range(8):
        assert np.allclose(got[0, :, h], w.v[0, 0, h // 4].astype(np.float64)[None, :], atol=1e-6)


def test_heads_ragged_batch_with_splits_and_an_empty_sequence():
    w = W.heads_prefill(n_seq=3, n_q=2, n_head=8, n_kv_head=8, n_kv=5000, causal=False)
    lens = [4999, 0, 1234]
    w.kv_len = np.array(lens, np.int32)
    units, splits = plan_of(w)
    assert splits > 1, "the case must exercise the split combine"
    got = run(w, kv_len=lens)
    assert np.all(got[1] == 0.0), "an empty sequence gives zeros"
    for b in (0, 2):
        L = lens[b]
        ref = oracle.attention_heads(w.q[b], w.k[b, :L], w.v[b, :L], w.mask[b, :, :L], w.scale)
        assert_parity(got[b].reshape(-1, 128), ref, f"ragged seq {b}")


def test_heads_single_long_sequence_many_splits():
    w = W.heads_prefill(n_seq=1, n_q=1, n_head=4, n_kv_head=4, n_kv=30000, causal=False)
    units, splits = plan_of(w)
    assert splits >= 16
    check(w, run(w), what="long sequence")


def test_heads_fully_masked_token_gives_zero():
    w = W.heads_prefill(n_q=6, n_head=16, n_kv_head=4, n_kv=400, causal=False)
    w.mask[0, 2, :] = np.float16(-np.inf)
    got = run(w)
    assert np.all(got[0, 2] == 0.0)
    check(w, got, what="masked token")


def test_heads_decode_batch():
    w = W.heads_decode(n_seq=8, len_lo=100, len_hi=3000)
    check(w, run(w), lens=w.kv_len, what="decode batch")


def test_heads_prefill_full_size_whole_groups():
    # the benchmark's 192 / 128 prefill workload; whole KV heads of three tokens
    w = W.heads_prefill()
    got = run(w)
    for t in (0, 255, 511):
        ref = oracle.attention_heads(w.q[0, t:t + 1], w.k[0], w.v[0], w.mask[0, t:t + 1], w.scale)
        assert_parity(got[0, t:t + 1].reshape(-1, 128), ref, f"prefill token {t}")
