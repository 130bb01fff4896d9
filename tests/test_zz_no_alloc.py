"""The forward entry point that allocates nothing.

Some callers cannot let a library call cudaMalloc: an engine that has reserved
nearly all device memory for its KV cache, a framework whose allocator must own
every byte, or a decode loop that cannot take the synchronisation cudaMalloc
may cause. mla_fa_forward_noalloc serves them by keeping its split-KV partials
in a static device array. These tests call it through the C ABI and check, on
two calls in a row with different inputs, that it gives what the allocating
entry point mla_fa_forward_ex gives and what the fp64 oracle gives, that the
other users of the array (the mask gather's cell lists and the fused
projection's partials) survive back-to-back calls of different shapes, that an
index list whose gathered rows would not fit the array is attended with the
in-kernel gather instead, and that a pass needing more scratch than the array
holds is refused before any launch.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import oracle
from mla_flash_attention_attn_b200 import binding
from mla_flash_attention_attn_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3


def _inputs(w, torch):
    dev = torch.device("cuda")
    q = torch.from_numpy(w.q).to(dev)
    k = torch.from_numpy(w.kcache).to(dev)
    m = torch.from_numpy(w.mask).to(dev)
    return q, k, m


def _compare(a, b, what):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    assert np.all(np.isfinite(a)), what
    err = a - b
    maxabs = float(np.abs(err).max())
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(b), 1e-30))
    assert maxabs <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {maxabs:.3g} rel-L2 {rel:.3g}"


def test_noalloc_matches_allocating_entry_point_on_two_calls():
    import torch

    binding.load()
    cases = [
        W.make("v3_batched_decode", n_kv=4096, len_lo=1000, len_hi=4096),
        W.make("v3_batched_decode", seed=77, n_seq=3, n_kv=3000, len_lo=200, len_hi=3000),
    ]
    for i, w in enumerate(cases):
        q, k, m = _inputs(w, torch)
        out_na = torch.full(w.q.shape[:3] + (512,), float("nan"), dtype=torch.float32,
                            device="cuda")
        args, keep = binding.make_args(q, k, w.kv_type, m, out_na, w.scale, kv_len=w.kv_len)
        units, splits = binding.mla_fa_query_plan(args)
        assert splits > 1, "the case must use split-KV scratch"
        need = binding.mla_fa_workspace_size(args)
        assert 0 < need <= binding.NOALLOC_SCRATCH_BYTES
        binding.mla_fa_forward_noalloc(args)
        ref = binding.forward(q, k, w.kv_type, m, w.scale, kv_len=w.kv_len)
        torch.cuda.synchronize()
        assert binding.mla_get_device_status() == 0
        got = out_na.cpu().numpy()
        _compare(got, ref.cpu().numpy(), f"call {i + 1}")
        for b in range(w.n_seq):
            exact = oracle.attention(w.q[b], w.kcache[b], w.kv_type, w.mask[b], w.scale)
            _compare(got[b].reshape(-1, 512), exact, f"call {i + 1} vs oracle, seq {b}")


def test_noalloc_mask_gather_and_projection_back_to_back():
    # Two more users of the shared array: the mask gather puts each unit's cell list
    # after the partials, and the fused projection makes every sequence write partials.
    # Back-to-back calls of different shapes leave stale contents behind; each call must
    # still read only what it wrote.
    import torch

    binding.load()
    dev = torch.device("cuda")
    # the mask gather on a sparse f16 mask (two sizes, so the lists move)
    for i, (n_kv, seed) in enumerate(((6000, 5), (2500, 6))):
        w = W.make("v2lite_decode", seed=seed, n_kv=n_kv, n_head=64, n_pad=0)
        rng = np.random.default_rng(seed)
        keep = rng.random(n_kv) < 0.2
        keep[-3:] = True
        w.mask[0, 0] = np.where(keep, np.float16(0), np.float16(-np.inf))
        q, k, m = _inputs(w, torch)
        out_na = torch.full(w.q.shape[:3] + (512,), float("nan"), dtype=torch.float32, device=dev)
        args, keep_alive = binding.make_args(q, k, w.kv_type, m, out_na, w.scale, mask_gather=True)
        assert binding.mla_fa_workspace_size(args) <= binding.NOALLOC_SCRATCH_BYTES
        binding.mla_fa_forward_noalloc(args)
        ref = binding.forward(q, k, w.kv_type, m, w.scale, mask_gather=True)
        torch.cuda.synchronize()
        assert binding.mla_get_device_status() == 0
        _compare(out_na.cpu().numpy(), ref.cpu().numpy(), f"mask gather call {i + 1}")
    # the fused projection (two batch shapes)
    for i, w in enumerate((W.make("v3_batched_decode", seed=8, n_seq=2, n_head=32, n_kv=2000,
                                  len_lo=900, len_hi=2000),
                           W.make("v3_batched_decode", seed=9, n_seq=3, n_head=16, n_kv=1500,
                                  len_lo=300, len_hi=1500))):
        q, k, m = _inputs(w, torch)
        wv = torch.from_numpy(W.wv_random(n_head=w.n_head)).to(dev)
        op_na = torch.full(w.q.shape[:3] + (128,), float("nan"), dtype=torch.float32, device=dev)
        args, keep_alive = binding.make_args(q, k, w.kv_type, m, None, w.scale, kv_len=w.kv_len,
                                             wv=wv, out_proj=op_na)
        assert binding.mla_fa_workspace_size(args) <= binding.NOALLOC_SCRATCH_BYTES
        binding.mla_fa_forward_noalloc(args)
        ref = binding.forward_proj(q, k, w.kv_type, m, w.scale, wv, kv_len=w.kv_len)
        torch.cuda.synchronize()
        assert binding.mla_get_device_status() == 0
        _compare(op_na.cpu().numpy(), ref.cpu().numpy(), f"projection call {i + 1}")


def test_noalloc_index_list_larger_than_its_scratch_takes_the_gather_modes():
    # The allocating entry point gathers an index list's rows into its workspace (here
    # 32768 rows of 1152 bytes, more than the scratch holds); the no-alloc entry point
    # then attends over the list with the in-kernel gather, which needs only the partials.
    import torch

    binding.load()
    dev = torch.device("cuda")
    w = W.make("sparse_q8_decode", n_kv=32768, n_head=128, tail_blocks=4)
    q, k, m = _inputs(w, torch)
    idx = torch.full((1, w.n_kv), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((1,), dtype=torch.int32, device=dev)
    cws = torch.zeros(binding.mla_compact_workspace_size(1, w.n_kv), dtype=torch.uint8, device=dev)
    binding.mla_compact_mask_ex(m[:, 0, :], idx, cnt, cws)
    out_na = torch.full(w.q.shape[:3] + (512,), float("nan"), dtype=torch.float32, device=dev)
    args, keep_alive = binding.make_args(q, k, w.kv_type, m, out_na, w.scale, idx=idx, idx_count=cnt)
    assert binding.mla_fa_workspace_size(args) > binding.NOALLOC_SCRATCH_BYTES
    binding.mla_fa_forward_noalloc(args)
    torch.cuda.synchronize()
    assert binding.mla_get_device_status() == 0
    ref_idx = oracle.compact(w.mask[0, 0])
    assert int(cnt[0]) == len(ref_idx)
    ref = oracle.attention(w.q[0], w.kcache[0], oracle.KV_Q8_0, w.mask[0], w.scale, idx=ref_idx)
    _compare(out_na[0].reshape(-1, 512).cpu().numpy(), ref, "no-alloc index list, gather modes")


def test_noalloc_refuses_a_pass_larger_than_its_scratch():
    import torch

    binding.load()
    lib = binding.load()
    # Find a batch that needs more partial slots than the scratch holds: with attention
    # sinks every sequence's 128-row groups write partials (a plain pass uses about one
    # slot per CTA pair, which always fits).
    dev = torch.device("cuda")
    found = None
    sinks = torch.zeros((128,), dtype=torch.float32, device=dev)
    for n_seq in (32, 64, 96, 128):
        q = torch.zeros((n_seq, 2, 128, 576), dtype=torch.float16, device=dev)
        k = torch.zeros((n_seq, 256, 576), dtype=torch.float16, device=dev)
        out = torch.zeros((n_seq, 2, 128, 512), dtype=torch.float32, device=dev)
        args, keep = binding.make_args(q, k, 0, None, out, 0.07, sinks=sinks)
        if binding.mla_fa_workspace_size(args) > binding.NOALLOC_SCRATCH_BYTES:
            found = (args, keep, q, k, out, sinks)
            break
        del q, k, out
    assert found is not None, "no batch exceeds the scratch size"
    args = found[0]
    rc = lib.mla_fa_forward_noalloc(ctypes.byref(args), None)
    assert rc == -5  # MLA_ERR_WORKSPACE, before any launch
