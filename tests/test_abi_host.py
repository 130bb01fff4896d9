"""C ABI checks that need no GPU: the library builds, loads, exports every symbol
include/mla_fa.h declares, and rejects bad arguments on the host before any
launch (no kernel runs here)."""
import ctypes

import numpy as np
import os
import shutil
import subprocess

import pytest

from mla_flash_attention_attn_b200 import binding, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def test_build_tracks_every_source_of_the_library():
    # the library is rebuilt when any file the translation unit includes is newer
    srcs = sorted(f for f in os.listdir(build.CSRC) if f.endswith((".cu", ".cuh", ".h")))
    assert build.DEPS == srcs
    assert "mla_gather.cuh" in srcs and "mla_heads.cuh" in srcs


def test_header_declares_the_boundary():
    names = binding.header_functions()
    for required in ("mla_fa_forward", "mla_fa_forward_ex", "mla_fa_workspace_size",
                     "mla_compact_mask", "mla_compact_mask_ex", "mla_get_device_status",
                     "mla_status_string", "mla_set_stream"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in binding.header_functions() if not hasattr(lib, n)]
    assert missing == []


def test_argument_struct_matches_the_header(tmp_path):
    # the ctypes mirror of mla_fa_args must agree with the C compiler on every field's
    # offset and on the size, or every field after a mismatch is read wrongly
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    fields = [f[0] for f in binding.mla_fa_args._fields_]
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include \"mla_fa.h\"\nint main(void) {\n"
                   + "".join(f'  printf("%zu\\n", offsetof(mla_fa_args, {f}));\n' for f in fields)
                   + '  printf("%zu\\n", sizeof(mla_fa_args));\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    want = [getattr(binding.mla_fa_args, f).offset for f in fields] + [ctypes.sizeof(binding.mla_fa_args)]
    assert got == want


def test_status_strings(lib):
    for code, name in binding.STATUS_NAMES.items():
        assert binding.mla_status_string(code).startswith(name)
    assert "unknown" in binding.mla_status_string(12345)
    assert lib.mla_version() >= 100


FAKE = 0x100000  # 16-byte aligned; never dereferenced: validation runs first


def base_args(**kw):
    a = binding.mla_fa_args()
    a.q = FAKE
    a.kcache = FAKE
    a.out = FAKE
    a.kcache_type = 0
    a.n_seq, a.n_q, a.n_head, a.n_kv = 1, 1, 16, 256
    a.scale = 0.07
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def call_ex(lib, a):
    return lib.mla_fa_forward_ex(ctypes.byref(a), None, 0, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), -1), (dict(kcache=None), -1), (dict(out=None), -1),
    (dict(kcache_type=7), -3),
    (dict(n_head=0), -2), (dict(n_head=129), -2), (dict(n_q=0), -2), (dict(n_kv=0), -2),
    (dict(n_seq=0), -2), (dict(scale=float("inf")), -2), (dict(scale=float("nan")), -2),
    (dict(q=FAKE + 8), -4), (dict(kcache=FAKE + 4), -4), (dict(out=FAKE + 2), -4),
    (dict(mask=FAKE + 1), -4), (dict(q_seq_stride=16 * 576 + 4, n_seq=2), -4),
    (dict(q_seq_stride=100, n_seq=2), -2), (dict(k_seq_stride=10, n_seq=2), -2),
    (dict(mask=FAKE, mask_row_stride=5), -2), (dict(out_seq_stride=-1), -2),
    (dict(idx=FAKE), -1),
    # fused value up-projection
    (dict(wv=FAKE, proj_dim=128), -1),                                  # no out_proj
    (dict(wv=FAKE, proj_dim=64, out_proj=FAKE), -8),                    # width not 128
    (dict(wv=FAKE + 2, proj_dim=128, out_proj=FAKE), -4),
    (dict(wv=FAKE, proj_dim=128, out_proj=FAKE + 4), -4),
    (dict(wv=FAKE, proj_dim=128, out_proj=FAKE, out_proj_seq_stride=100, n_seq=2), -2),
    (dict(wv=FAKE, proj_dim=128, out_proj=FAKE, out_proj_seq_stride=16 * 128 + 2, n_seq=2), -4),
    # the projection grid's y dimension: 4 CTAs per 8 (sequence, token) rows <= 65535
    (dict(wv=FAKE, proj_dim=128, out_proj=FAKE, n_seq=128, n_q=1050, n_head=1), -2),
    # attention variants
    (dict(softcap=-1.0), -2), (dict(softcap=float("nan")), -2), (dict(softcap=float("inf")), -2),
    (dict(alibi_slopes=FAKE, idx=FAKE, idx_count=FAKE), -8),
    (dict(sinks=FAKE + 2), -4), (dict(alibi_slopes=FAKE + 1), -4),
    # per-row lse: excludes sinks and the projection; 4-byte aligned
    (dict(out_lse=FAKE, sinks=FAKE), -8),
    (dict(out_lse=FAKE, wv=FAKE, proj_dim=128, out_proj=FAKE), -8),
    (dict(out_lse=FAKE + 2), -4),
    # head width: 576 or 512; 512 takes an f16 cache, no softcap, ALiBi or mask gather
    (dict(head_dim=256), -2), (dict(head_dim=513), -2),
    (dict(head_dim=512, kcache_type=1), -8), (dict(head_dim=512, softcap=5.0), -8),
    (dict(head_dim=512, alibi_slopes=FAKE), -8), (dict(head_dim=512, mask=FAKE, mask_gather=1), -8),
    (dict(head_dim=512, q_seq_stride=16 * 512 - 8, n_seq=2), -2),
    # mask gather: needs the mask, excludes an index list and ALiBi
    (dict(mask_gather=2, mask=FAKE), -2), (dict(mask_gather=1), -1),
    (dict(mask_gather=1, mask=FAKE, idx=FAKE, idx_count=FAKE), -8),
    (dict(mask_gather=1, mask=FAKE, alibi_slopes=FAKE), -8),
    # the DK = 192 / DV = 128 shape: needs v and a KV head count dividing n_head; dense f16
    # attention only; other widths take no v and no KV head count
    (dict(head_dim=192, n_kv_head=4), -1), (dict(head_dim=192, v=FAKE), -2),
    (dict(head_dim=192, v=FAKE, n_kv_head=3), -2), (dict(head_dim=192, v=FAKE, n_kv_head=32), -2),
    (dict(head_dim=192, v=FAKE + 8, n_kv_head=4), -4),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, kcache_type=1), -8),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, idx=FAKE, idx_count=FAKE), -8),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, sinks=FAKE), -8),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, out_lse=FAKE), -8),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, softcap=2.0), -8),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, mask=FAKE, mask_gather=1), -8),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, v_seq_stride=100, n_seq=2), -2),
    (dict(head_dim=192, v=FAKE, n_kv_head=4, out_seq_stride=16 * 128 - 4, n_seq=2), -2),
    (dict(v=FAKE), -2), (dict(n_kv_head=4), -2), (dict(head_dim=512, v=FAKE, n_kv_head=1), -2),
])
def test_argument_errors_are_returned_before_any_launch(lib, kw, expect):
    assert call_ex(lib, base_args(**kw)) == expect
    assert lib.mla_fa_workspace_size(ctypes.byref(base_args(**kw))) == 0


def test_projection_lets_out_be_null(lib):
    # out may be NULL when the projection is requested: without a GPU the valid call
    # stops at the device check, never at argument validation. The fake pointers must
    # never reach a kernel, so this runs only where no GPU exists.
    import torch

    if torch.cuda.is_available():
        pytest.skip("fake pointers: only meaningful without a GPU")
    a = base_args(out=None, wv=FAKE, proj_dim=128, out_proj=FAKE)
    assert call_ex(lib, a) in (-6, -8)


def test_kv_len_out_of_range_is_rejected(lib):
    lens = (ctypes.c_int32 * 2)(10, 300)
    a = base_args(n_seq=2, kv_len=ctypes.cast(lens, ctypes.c_void_p))
    assert call_ex(lib, a) == -2
    lens2 = (ctypes.c_int32 * 2)(-1, 3)
    a2 = base_args(n_seq=2, kv_len=ctypes.cast(lens2, ctypes.c_void_p))
    assert call_ex(lib, a2) == -2


def test_simple_entry_point_validates(lib):
    assert lib.mla_fa_forward(None, FAKE, 0, None, 1, 16, 256, 0.1, FAKE) == -1
    assert lib.mla_fa_forward(FAKE, FAKE, 2, None, 1, 16, 256, 0.1, FAKE) == -3
    assert lib.mla_fa_forward(FAKE, FAKE, 0, None, 1, 200, 256, 0.1, FAKE) == -2


def test_compaction_argument_errors(lib):
    assert lib.mla_compact_mask(None, 10, FAKE, FAKE, None) == -1
    assert lib.mla_compact_mask(FAKE, 0, FAKE, FAKE, None) == -2
    assert lib.mla_compact_mask_ex(FAKE + 1, 1, 10, 10, FAKE, 10, FAKE, FAKE, 4096, None) == -4
    assert lib.mla_compact_mask_ex(FAKE, 1, 10, 10, FAKE, 10, FAKE, None, 0, None) == -5
    assert lib.mla_compact_mask_ex(FAKE, 1, 5, 10, FAKE, 10, FAKE, FAKE, 4096, None) == -2
    # 256 bytes of row tickets, then 8 bytes of look-back state per 2048-cell tile
    assert lib.mla_compact_workspace_size(1, 131072) == 256 + 64 * 8
    assert lib.mla_compact_workspace_size(3, 2049) == 256 + 3 * 2 * 8
    assert lib.mla_compact_workspace_size(0, 10) == 0


def test_combine_argument_errors(lib):
    f = lib.mla_fa_combine
    assert f(None, FAKE, 2, 10, FAKE, None, None) == -1
    assert f(FAKE, None, 2, 10, FAKE, None, None) == -1
    assert f(FAKE, FAKE, 2, 10, None, None, None) == -1
    assert f(FAKE, FAKE, 0, 10, FAKE, None, None) == -2
    assert f(FAKE, FAKE, binding.COMBINE_MAX_PARTS + 1, 10, FAKE, None, None) == -2
    assert f(FAKE, FAKE, 2, 0, FAKE, None, None) == -2
    assert f(FAKE + 4, FAKE, 2, 10, FAKE, None, None) == -4
    assert f(FAKE, FAKE, 2, 10, FAKE + 8, None, None) == -4
    assert f(FAKE, FAKE + 2, 2, 10, FAKE, None, None) == -4
    assert f(FAKE, FAKE, 2, 10, FAKE, FAKE + 1, None) == -4


@pytest.mark.parametrize("args,expect", [
    ((None, 5 * 512, FAKE, 5, 2, 5, FAKE, None), -1),
    ((FAKE, 5 * 512 - 4, FAKE, 5, 2, 5, FAKE, None), -2),   # parts overlap
    ((FAKE, 5 * 512, FAKE, 4, 2, 5, FAKE, None), -2),
    ((FAKE, 5 * 512 + 2, FAKE, 5, 2, 5, FAKE, None), -4),   # O rows of a part misaligned
    ((FAKE, 5 * 513, FAKE, 5 * 513, 0, 5, FAKE, None), -2),
])
def test_strided_combine_argument_errors(lib, args, expect):
    o, os_, l, ls, n, rows, out, out_lse = args
    assert lib.mla_fa_combine_strided(o, os_, l, ls, n, rows, out, out_lse, None) == expect


def test_valid_arguments_reach_the_device_check(lib):
    # With no CUDA device visible a valid call stops at the device check. The fake
    # pointers must never reach a kernel, so this runs only where no GPU exists.
    import torch

    if torch.cuda.is_available():
        pytest.skip("fake pointers: only meaningful without a GPU")
    assert call_ex(lib, base_args()) in (-6, -8)


def test_binding_takes_the_head_width_from_q():
    # argument marshalling only (CPU tensors, no call into the library's kernels)
    import torch

    for dk in (576, 512):
        q = torch.zeros((2, 1, 4, dk), dtype=torch.float16)
        k = torch.zeros((2, 8, dk), dtype=torch.float16)
        out = torch.zeros((2, 1, 4, 512), dtype=torch.float32)
        a, _ = binding.marshal_args(q, k, 0, None, out, 0.1)
        assert a.head_dim == dk and a.q_seq_stride == 4 * dk and a.k_seq_stride == 8
    with pytest.raises(ValueError):
        binding.marshal_args(torch.zeros((1, 1, 4, 300), dtype=torch.float16),
                             torch.zeros((1, 8, 300), dtype=torch.float16), 0, None,
                             torch.zeros((1, 1, 4, 512)), 0.1)


def test_binding_refuses_host_tensors():
    # a host pointer handed to a kernel would be a bad device address
    import torch

    q = torch.zeros((1, 1, 4, 576), dtype=torch.float16)
    k = torch.zeros((1, 8, 576), dtype=torch.float16)
    out = torch.zeros((1, 1, 4, 512), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        binding.make_args(q, k, 0, None, out, 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        binding.combine(torch.zeros((2, 8, 512)), torch.zeros((2, 8)))


@pytest.mark.parametrize("bad", ["dtype", "shape", "strided", "device", "empty"])
def test_binding_tensor_checks(bad):
    # the per-tensor check that make_args and combine apply (run here on host tensors
    # against the host device; on a GPU the device is q's)
    import torch

    cpu = torch.device("cpu")
    good = torch.zeros((2, 3, 4, 512), dtype=torch.float32)
    binding._check_tensor(good, "out", torch.float32, (2, 3, 4, 512), cpu)
    t = {"dtype": good.half(),
         "shape": torch.zeros((2, 3, 4, 256), dtype=torch.float32),
         "strided": torch.zeros((2, 3, 8, 512), dtype=torch.float32)[:, :, ::2],
         "device": torch.zeros((2, 3, 4, 512), dtype=torch.float32, device="meta"),
         "empty": torch.zeros((2, 0, 4, 512), dtype=torch.float32)}[bad]
    with pytest.raises(ValueError):
        binding._check_tensor(t, "out", torch.float32, (2, None, 4, 512), cpu)


# ---- the split plan, on the host alone (mla_fa_plan_for_sms) -----------------------------
SLOT_BYTES = 128 * (512 * 2 + 4)  # one partial: 128 rows of f16 O / l and fp32 lse


def _plan(sm_count, n_seq, n_q, n_head, lens, **kw):
    lens_c = (ctypes.c_int32 * n_seq)(*lens)
    a = base_args(n_seq=n_seq, n_q=n_q, n_head=n_head, n_kv=max(lens),
                  kv_len=ctypes.cast(lens_c, ctypes.c_void_p), **kw)
    return binding.mla_fa_plan_for_sms(a, sm_count)


def test_plan_never_asks_for_more_units_than_sm_pairs():
    # the per-sequence split counts are rounded; their sum must still fit one wave of
    # CTA pairs, or the surplus units would run after the others
    rng = np.random.default_rng(5)
    for _ in range(200):
        n_seq = int(rng.integers(1, 30))
        lens = [int(x) for x in rng.integers(1, 60000, n_seq)]
        n_q = int(rng.integers(1, 3))
        sms = int(rng.choice([2, 16, 132, 148]))
        units, splits, ws = _plan(sms, n_seq, n_q, 128, lens)
        groups = (n_q * 128 + 127) // 128
        assert units >= n_seq * groups and splits >= 1
        if n_seq * groups < sms // 2:
            assert units <= sms // 2
        if splits == 1:
            assert ws == 0
        else:
            assert ws > 0 and ws % SLOT_BYTES == 0


def test_plan_of_a_batch_that_fills_the_gpu_has_no_splits():
    units, splits, ws = _plan(148, 100, 1, 128, [5000] * 100)
    assert (units, splits, ws) == (100, 1, 0)


def test_plan_partials_forced_by_sinks_and_lse():
    for kw in (dict(sinks=FAKE), dict(out_lse=FAKE)):
        units, splits, ws = _plan(148, 100, 1, 128, [300] * 100, **kw)
        assert (units, splits) == (100, 1) and ws == 100 * SLOT_BYTES


def test_plan_of_the_v3_decode_batch():
    # lengths of the V3 batched-decode workload (seed 1003): 540 tiles over 74 pairs
    lens = [12606, 9479, 20813, 11456, 12221, 18279, 28969, 23042]
    units, splits, ws = _plan(148, 8, 1, 128, lens)
    assert units == 74 and splits == 16 and ws == 74 * SLOT_BYTES


def test_plan_mask_gather_adds_the_cell_lists():
    units, splits, ws = _plan(148, 1, 1, 128, [131072], mask=FAKE)
    units_g, splits_g, ws_g = _plan(148, 1, 1, 128, [131072], mask=FAKE, mask_gather=1)
    assert (units_g, splits_g) == (units, splits)
    assert ws_g > ws  # the per-CTA lists of kept cells come after the partials


def test_plan_rejects_bad_sm_counts_and_arguments(lib):
    with pytest.raises(binding.MlaError):
        _plan(0, 1, 1, 16, [100])
    with pytest.raises(binding.MlaError):
        binding.mla_fa_plan_for_sms(base_args(n_head=0), 148)


def test_combine_binding_rejects_strided_parts():
    import torch

    o = torch.zeros((2, 8, 1024))[:, :, :512]  # a strided view
    with pytest.raises(ValueError):
        binding.combine(o, torch.zeros((2, 8)))


def test_plan_of_the_192_head_shape():
    # one CTA per (sequence, KV head, 128-row group, split); splits only while the unsplit
    # units leave SMs idle, never more units than SMs
    lens_c = (ctypes.c_int32 * 1)(30000)
    a = base_args(head_dim=192, v=FAKE, n_kv_head=4, n_head=4, n_kv=30000,
                  kv_len=ctypes.cast(lens_c, ctypes.c_void_p))
    units, splits, ws = binding.mla_fa_plan_for_sms(a, 148)
    assert units <= 148 and units == 4 * splits and splits >= 16
    assert ws == units * 128 * 129 * 4  # fp32 O rows and lse per slot
    b = base_args(head_dim=192, v=FAKE, n_kv_head=16, n_head=16, n_seq=10, n_q=1)
    units, splits, ws = binding.mla_fa_plan_for_sms(b, 148)
    assert (units, splits, ws) == (160, 1, 0)


def test_plan_of_mask_derived_ranges():
    # with a mask and no lengths (or with several query tokens) the tile ranges come from
    # the mask on the device: the launch has one unit per SM pair while there are fewer
    # groups than pairs (the device decides the splits: at most 16 per group with three
    # groups or more, else up to the pairs), else one unit per group
    a = base_args(n_seq=8, n_q=1, n_head=128, n_kv=32768, mask=FAKE)
    units, splits, ws = binding.mla_fa_plan_for_sms(a, 148)
    assert units == 74 and splits == 16 and ws > 74 * SLOT_BYTES
    units, splits, ws = binding.mla_fa_plan_for_sms(base_args(n_kv=32768, n_head=128, mask=FAKE), 148)
    assert units == 74 and splits == 74
    lens_c = (ctypes.c_int32 * 1)(16384)
    b = base_args(n_seq=1, n_q=512, n_head=128, n_kv=16384, mask=FAKE,
                  kv_len=ctypes.cast(lens_c, ctypes.c_void_p))
    units, splits, ws = binding.mla_fa_plan_for_sms(b, 148)
    assert (units, splits) == (512, 1) and 0 < ws < SLOT_BYTES  # descriptors only
    # lengths and one query token: the host plan, as before
    lens8 = (ctypes.c_int32 * 8)(*[12606, 9479, 20813, 11456, 12221, 18279, 28969, 23042])
    c = base_args(n_seq=8, n_q=1, n_head=128, n_kv=32768, mask=FAKE,
                  kv_len=ctypes.cast(lens8, ctypes.c_void_p))
    assert binding.mla_fa_plan_for_sms(c, 148) == (74, 16, 74 * SLOT_BYTES)
