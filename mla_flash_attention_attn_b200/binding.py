"""ctypes binding of libmla_fa.so (include/mla_fa.h), same names as the C ABI.

This module only marshals arguments: torch tensors are turned into device
pointers and sizes, and every step of the computation runs in the library's
CUDA kernels. There is no CPU path: if the library is missing or the device is
not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libmla_fa.so")
HEADER = os.path.join(ROOT, "include", "mla_fa.h")

DK = 576
DV = 512
Q8_ROW_BYTES = 612
KV_F16 = 0
KV_Q8_0 = 1

MLA_OK = 0
STATUS_NAMES = {
    0: "MLA_OK", -1: "MLA_ERR_NULL", -2: "MLA_ERR_SHAPE", -3: "MLA_ERR_TYPE",
    -4: "MLA_ERR_ALIGN", -5: "MLA_ERR_WORKSPACE", -6: "MLA_ERR_CUDA", -7: "MLA_ERR_TIMEOUT",
    -8: "MLA_ERR_UNSUPPORTED", -9: "MLA_ERR_INDEX",
}


class MlaError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class mla_fa_args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p),
        ("kcache", ctypes.c_void_p),
        ("kcache_type", ctypes.c_int),
        ("mask", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("n_seq", ctypes.c_int),
        ("n_q", ctypes.c_int),
        ("n_head", ctypes.c_int),
        ("n_kv", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("q_seq_stride", ctypes.c_int64),
        ("k_seq_stride", ctypes.c_int64),
        ("mask_seq_stride", ctypes.c_int64),
        ("mask_row_stride", ctypes.c_int64),
        ("out_seq_stride", ctypes.c_int64),
        ("kv_len", ctypes.c_void_p),
        ("idx", ctypes.c_void_p),
        ("idx_count", ctypes.c_void_p),
        ("idx_seq_stride", ctypes.c_int64),
        ("wv", ctypes.c_void_p),
        ("proj_dim", ctypes.c_int),
        ("out_proj", ctypes.c_void_p),
        ("out_proj_seq_stride", ctypes.c_int64),
        ("sinks", ctypes.c_void_p),
        ("alibi_slopes", ctypes.c_void_p),
        ("softcap", ctypes.c_float),
        ("mask_gather", ctypes.c_int),
        ("out_lse", ctypes.c_void_p),
        ("head_dim", ctypes.c_int),
        ("v", ctypes.c_void_p),
        ("v_seq_stride", ctypes.c_int64),
        ("n_kv_head", ctypes.c_int),
    ]


class mla_profile_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


_lib = None


def header_functions():
    """Names of the functions include/mla_fa.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(mla_\w+)\s*\(", text, flags=re.M)))


def load(path: str = LIB_PATH):
    """Load the library and declare the C signatures. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing: build it with `python -m mla_flash_attention_attn_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
    lib.mla_fa_forward.argtypes = [P, P, I, P, I, I, I, ctypes.c_float, P]
    lib.mla_fa_forward.restype = I
    lib.mla_set_stream.argtypes = [P]
    lib.mla_set_stream.restype = I
    lib.mla_fa_workspace_size.argtypes = [ctypes.POINTER(mla_fa_args)]
    lib.mla_fa_workspace_size.restype = Z
    lib.mla_fa_forward_ex.argtypes = [ctypes.POINTER(mla_fa_args), P, Z, P]
    lib.mla_fa_forward_ex.restype = I
    lib.mla_fa_query_plan.argtypes = [ctypes.POINTER(mla_fa_args), ctypes.POINTER(I),
                                      ctypes.POINTER(I)]
    lib.mla_fa_query_plan.restype = I
    lib.mla_compact_mask.argtypes = [P, I, P, P, P]
    lib.mla_compact_mask.restype = I
    lib.mla_compact_workspace_size.argtypes = [I, I]
    lib.mla_compact_workspace_size.restype = Z
    lib.mla_compact_mask_ex.argtypes = [P, I, ctypes.c_int64, I, P, ctypes.c_int64, P, P, Z, P]
    lib.mla_compact_mask_ex.restype = I
    lib.mla_get_device_status.argtypes = [P]
    lib.mla_get_device_status.restype = I
    lib.mla_debug_wait_timeout.argtypes = [U64, P]
    lib.mla_debug_wait_timeout.restype = I
    lib.mla_status_string.argtypes = [I]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_version.argtypes = []
    lib.mla_version.restype = I
    lib.mla_fa_forward_noalloc.argtypes = [ctypes.POINTER(mla_fa_args), P]
    lib.mla_fa_forward_noalloc.restype = I
    lib.mla_profile_begin.argtypes = []
    lib.mla_profile_begin.restype = I
    lib.mla_profile_end.argtypes = [ctypes.POINTER(mla_profile_entry), I, ctypes.POINTER(I)]
    lib.mla_profile_end.restype = I
    lib.mla_fa_plan_for_sms.argtypes = [ctypes.POINTER(mla_fa_args), I, ctypes.POINTER(I),
                                         ctypes.POINTER(I), ctypes.POINTER(Z)]
    lib.mla_fa_plan_for_sms.restype = I
    lib.mla_fa_combine.argtypes = [P, P, I, ctypes.c_int64, P, P, P]
    lib.mla_fa_combine.restype = I
    lib.mla_fa_combine_strided.argtypes = [P, ctypes.c_int64, P, ctypes.c_int64, I, ctypes.c_int64,
                                           P, P, P]
    lib.mla_fa_combine_strided.restype = I
    _lib = lib
    return lib


def _check(status, what):
    if status != MLA_OK:
        raise MlaError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _host_i32(arr):
    """Keep-alive ctypes int32 array for HOST arguments (kv_len)."""
    if arr is None:
        return None
    vals = [int(v) for v in arr]
    return (ctypes.c_int32 * len(vals))(*vals)


def _check_tensor(t, name, dtype, shape, device, row_contiguous=True):
    """Raise ValueError unless t is a tensor on `device` with this dtype and shape (None in
    `shape` matches any size) whose innermost dimension is dense and, with
    row_contiguous, whose every dimension below the first is dense as well (the C ABI
    takes one stride per sequence and none inside a sequence)."""
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if t.dim() != len(shape) or any(s is not None and t.shape[i] != s for i, s in enumerate(shape)):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
    if t.numel() == 0:
        raise ValueError(f"{name} is empty")
    if t.stride(-1) != 1:
        raise ValueError(f"{name} must be dense in its last dimension")
    if row_contiguous:
        expect = 1
        for i in range(t.dim() - 1, 0, -1):
            if t.shape[i] != 1 and t.stride(i) != expect:
                raise ValueError(f"{name} must be contiguous within its first dimension")
            expect *= t.shape[i]


def check_args(q, kcache, kv_type, mask, out, kv_len=None, idx=None, idx_count=None, wv=None,
               out_proj=None, sinks=None, alibi_slopes=None, out_lse=None):
    """The checks the C ABI cannot make, since it sees pointers and not buffers: every
    tensor is a CUDA tensor on q's device, with the dtype and size the header states for
    it. A host tensor, a wrong dtype or a short buffer would otherwise reach a kernel as a
    bad address. Raises ValueError."""
    import torch

    if q.dim() != 4:
        raise ValueError("q must be [n_seq][n_q][n_head][576 or 512]")
    if not q.is_cuda:
        raise ValueError("q must be a CUDA tensor")
    dev = q.device
    n_seq, n_q, n_head, dk = q.shape
    if dk not in (DK, DV):
        raise ValueError("q must end in 576 (or 512: the DK = DV = 512 head shape)")
    _check_tensor(q, "q", torch.float16, (n_seq, n_q, n_head, dk), dev)
    if int(kv_type) == KV_Q8_0:
        _check_tensor(kcache, "kcache", torch.uint8, (n_seq, None, Q8_ROW_BYTES), dev,
                      row_contiguous=False)
    else:
        _check_tensor(kcache, "kcache", torch.float16, (n_seq, None, dk), dev,
                      row_contiguous=False)
    if kcache.stride(1) != kcache.shape[2] or kcache.stride(0) % kcache.stride(1):
        raise ValueError("kcache rows must be dense and sequences a whole number of rows apart")
    n_kv = kcache.shape[1]
    if mask is not None:
        _check_tensor(mask, "mask", torch.float16, (n_seq, n_q, n_kv), dev, row_contiguous=False)
    if out is not None:
        _check_tensor(out, "out", torch.float32, (n_seq, n_q, n_head, DV), dev)
    if kv_len is not None and len(kv_len) != n_seq:
        raise ValueError("kv_len must hold one length per sequence")
    if idx is not None:
        if idx_count is None:
            raise ValueError("idx needs idx_count")
        _check_tensor(idx, "idx", torch.int32, (n_seq, None), dev, row_contiguous=False)
        _check_tensor(idx_count, "idx_count", torch.int32, (n_seq,), dev)
    if wv is not None:
        _check_tensor(wv, "wv", torch.float16, (n_head, DV, None), dev)
        if out_proj is None:
            raise ValueError("wv needs out_proj")
        _check_tensor(out_proj, "out_proj", torch.float32, (n_seq, n_q, n_head, wv.shape[2]), dev)
    for name, t in (("sinks", sinks), ("alibi_slopes", alibi_slopes)):
        if t is not None:
            _check_tensor(t, name, torch.float32, (n_head,), dev)
    if out_lse is not None:
        _check_tensor(out_lse, "out_lse", torch.float32, (n_seq, n_q, n_head), dev)


def make_args(q, kcache, kv_type, mask, out, scale, kv_len=None, idx=None, idx_count=None,
              wv=None, out_proj=None, sinks=None, alibi_slopes=None, softcap=0.0,
              mask_gather=False, out_lse=None):
    """Fill mla_fa_args from batched torch tensors, after check_args.

    q [n_seq][n_q][n_head][576] f16; kcache [n_seq][n_kv][576] f16 (or uint8 [..][612]);
    q [..][512] with kcache [..][512] f16 selects the DK = DV = 512 head shape;
    mask [n_seq][n_q][n_kv] f16 or None; out [n_seq][n_q][n_head][512] f32 (or None with
    wv); wv [n_head][512][128] f16 and out_proj [n_seq][n_q][n_head][128] f32 for the
    fused value up-projection; sinks / alibi_slopes fp32 [n_head] and softcap > 0 for
    the attention variants; mask_gather=True for sparse attention straight from the mask
    (the kernel compacts it, no index list); out_lse fp32 [n_seq][n_q][n_head] for each
    row's natural log-sum-exp. Returns (args, keepalive)."""
    check_args(q, kcache, kv_type, mask, out, kv_len=kv_len, idx=idx, idx_count=idx_count,
               wv=wv, out_proj=out_proj, sinks=sinks, alibi_slopes=alibi_slopes,
               out_lse=out_lse)
    return marshal_args(q, kcache, kv_type, mask, out, scale, kv_len, idx, idx_count, wv,
                        out_proj, sinks, alibi_slopes, softcap, mask_gather, out_lse)


def marshal_args(q, kcache, kv_type, mask, out, scale, kv_len=None, idx=None, idx_count=None,
                 wv=None, out_proj=None, sinks=None, alibi_slopes=None, softcap=0.0,
                 mask_gather=False, out_lse=None):
    """Pointers, sizes and strides of the tensors, with no checks (make_args checks first)."""
    n_seq, n_q, n_head, dk = q.shape
    if dk not in (DK, DV):
        raise ValueError("q must end in 576 (or 512: the DK = DV = 512 head shape)")
    a = mla_fa_args()
    a.q = q.data_ptr()
    a.kcache = kcache.data_ptr()
    a.kcache_type = int(kv_type)
    a.mask = None if mask is None else mask.data_ptr()
    a.out = None if out is None else out.data_ptr()
    a.n_seq, a.n_q, a.n_head, a.n_kv = n_seq, n_q, n_head, kcache.shape[1]
    a.scale = float(scale)
    a.q_seq_stride = q.stride(0)
    a.k_seq_stride = kcache.stride(0) // kcache.stride(1)
    if mask is not None:
        a.mask_seq_stride = mask.stride(0)
        a.mask_row_stride = mask.stride(1)
    a.out_seq_stride = 0 if out is None else out.stride(0)
    if wv is not None:
        a.wv = wv.data_ptr()
        a.proj_dim = int(wv.shape[2])
        a.out_proj = None if out_proj is None else out_proj.data_ptr()
        a.out_proj_seq_stride = 0 if out_proj is None else out_proj.stride(0)
    a.sinks = None if sinks is None else sinks.data_ptr()
    a.alibi_slopes = None if alibi_slopes is None else alibi_slopes.data_ptr()
    a.softcap = float(softcap)
    a.mask_gather = 1 if mask_gather else 0
    a.out_lse = None if out_lse is None else out_lse.data_ptr()
    a.head_dim = dk
    keep = _host_i32(kv_len)
    a.kv_len = None if keep is None else ctypes.cast(keep, ctypes.c_void_p)
    if idx is not None:
        a.idx = idx.data_ptr()
        a.idx_count = idx_count.data_ptr()
        a.idx_seq_stride = idx.stride(0)
    return a, keep


HEADS_DK = 192
HEADS_DV = 128


def make_heads_args(q, k, v, mask, out, scale, kv_len=None):
    """mla_fa_args for the DK = 192 / DV = 128 head shape (a K and a V per KV head):
    q [n_seq][n_q][n_head][192] f16, k [n_seq][n_kv][n_kv_head][192] f16,
    v [n_seq][n_kv][n_kv_head][128] f16, mask [n_seq][n_q][n_kv] f16 or None,
    out [n_seq][n_q][n_head][128] fp32. Checks the tensors first (device, dtype, size).
    Returns (args, keepalive)."""
    import torch

    if q.dim() != 4 or not q.is_cuda:
        raise ValueError("q must be a CUDA tensor [n_seq][n_q][n_head][192]")
    dev = q.device
    n_seq, n_q, n_head, _ = q.shape
    _check_tensor(q, "q", torch.float16, (n_seq, n_q, n_head, HEADS_DK), dev)
    if k.dim() != 4:
        raise ValueError("k must be [n_seq][n_kv][n_kv_head][192]")
    n_kv, n_kv_head = k.shape[1], k.shape[2]
    if n_kv_head < 1 or n_head % n_kv_head:
        raise ValueError("n_kv_head must divide n_head")
    for name, t, w in (("k", k, HEADS_DK), ("v", v, HEADS_DV)):
        _check_tensor(t, name, torch.float16, (n_seq, n_kv, n_kv_head, w), dev, row_contiguous=False)
        if t.stride(2) != w or t.stride(1) != n_kv_head * w or t.stride(0) % t.stride(1):
            raise ValueError(f"{name} rows must be dense and sequences a whole number of rows apart")
    if mask is not None:
        _check_tensor(mask, "mask", torch.float16, (n_seq, n_q, n_kv), dev, row_contiguous=False)
    _check_tensor(out, "out", torch.float32, (n_seq, n_q, n_head, HEADS_DV), dev)
    if kv_len is not None and len(kv_len) != n_seq:
        raise ValueError("kv_len must hold one length per sequence")
    a = mla_fa_args()
    a.q, a.kcache, a.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    a.kcache_type = KV_F16
    a.mask = None if mask is None else mask.data_ptr()
    a.out = out.data_ptr()
    a.n_seq, a.n_q, a.n_head, a.n_kv = n_seq, n_q, n_head, n_kv
    a.n_kv_head = n_kv_head
    a.scale = float(scale)
    a.head_dim = HEADS_DK
    a.q_seq_stride = q.stride(0)
    a.k_seq_stride = k.stride(0) // k.stride(1)
    a.v_seq_stride = v.stride(0) // v.stride(1)
    if mask is not None:
        a.mask_seq_stride = mask.stride(0)
        a.mask_row_stride = mask.stride(1)
    a.out_seq_stride = out.stride(0)
    keep = _host_i32(kv_len)
    a.kv_len = None if keep is None else ctypes.cast(keep, ctypes.c_void_p)
    return a, keep


def forward_heads(q, k, v, mask, scale, out=None, kv_len=None, workspace=None, stream=None):
    """The DK = 192 / DV = 128 head shape through mla_fa_forward_ex; allocates out and the
    workspace with torch if absent. Returns out [n_seq][n_q][n_head][128] fp32."""
    import torch

    if out is None:
        out = torch.empty(q.shape[:3] + (HEADS_DV,), dtype=torch.float32, device=q.device)
    args, keep = make_heads_args(q, k, v, mask, out, scale, kv_len)
    need = mla_fa_workspace_size(args)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    mla_fa_forward_ex(args, workspace if need else None, stream)
    del keep
    return out


def mla_fa_workspace_size(args) -> int:
    return int(load().mla_fa_workspace_size(ctypes.byref(args)))


def mla_fa_query_plan(args):
    units, splits = ctypes.c_int(0), ctypes.c_int(0)
    _check(load().mla_fa_query_plan(ctypes.byref(args), ctypes.byref(units), ctypes.byref(splits)),
           "mla_fa_query_plan")
    return units.value, splits.value


def mla_fa_plan_for_sms(args, sm_count):
    """Host-only plan for a GPU with sm_count SMs: (units, max_splits, workspace bytes)."""
    units, splits, ws = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_size_t(0)
    _check(load().mla_fa_plan_for_sms(ctypes.byref(args), int(sm_count), ctypes.byref(units),
                                      ctypes.byref(splits), ctypes.byref(ws)), "mla_fa_plan_for_sms")
    return units.value, splits.value, ws.value


def mla_fa_forward_ex(args, workspace=None, stream=None):
    ws_ptr = None if workspace is None else ctypes.c_void_p(workspace.data_ptr())
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().mla_fa_forward_ex(ctypes.byref(args), ws_ptr, ws_bytes, _stream_ptr(stream)),
           "mla_fa_forward_ex")


def mla_fa_forward(q, kcache, kv_type, mask, scale, out, stream=None):
    """Single-sequence call: q [n_q][n_head][576], kcache [n_kv][...], mask [n_q][n_kv]."""
    lib = load()
    _check(lib.mla_set_stream(_stream_ptr(stream)), "mla_set_stream")
    n_q, n_head, _ = q.shape
    _check(lib.mla_fa_forward(_ptr(q), _ptr(kcache), int(kv_type), _ptr(mask), n_q, n_head,
                              kcache.shape[0], float(scale), _ptr(out)), "mla_fa_forward")


def forward(q, kcache, kv_type, mask, scale, out=None, kv_len=None, idx=None, idx_count=None,
            workspace=None, stream=None, sinks=None, alibi_slopes=None, softcap=0.0,
            mask_gather=False, out_lse=None):
    """Batched forward through mla_fa_forward_ex; allocates out/workspace with torch if absent."""
    import torch

    if out is None:
        out = torch.empty(q.shape[:3] + (DV,), dtype=torch.float32, device=q.device)
    args, keep = make_args(q, kcache, kv_type, mask, out, scale, kv_len, idx, idx_count,
                           sinks=sinks, alibi_slopes=alibi_slopes, softcap=softcap,
                           mask_gather=mask_gather, out_lse=out_lse)
    need = mla_fa_workspace_size(args)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    mla_fa_forward_ex(args, workspace if need else None, stream)
    del keep
    return out


def forward_proj(q, kcache, kv_type, mask, scale, wv, out_proj=None, kv_len=None, idx=None,
                 idx_count=None, workspace=None, stream=None, mask_gather=False):
    """Forward with the fused value up-projection (wv [n_head][512][128] f16); returns
    out_proj [n_seq][n_q][n_head][128] f32. The 512-wide attention rows are not written."""
    import torch

    if out_proj is None:
        out_proj = torch.empty(q.shape[:3] + (int(wv.shape[2]),), dtype=torch.float32, device=q.device)
    args, keep = make_args(q, kcache, kv_type, mask, None, scale, kv_len, idx, idx_count, wv=wv,
                           out_proj=out_proj, mask_gather=mask_gather)
    need = mla_fa_workspace_size(args)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    mla_fa_forward_ex(args, workspace if need else None, stream)
    del keep
    return out_proj


COMBINE_MAX_PARTS = 1024  # MLA_COMBINE_MAX_PARTS


def combine(o_parts, lse_parts, out=None, out_lse=None, stream=None):
    """mla_fa_combine: merge partial results of the same rows over disjoint key sets.
    o_parts fp32 [n_parts][rows][512] (or [n_parts][..][512], rows = the product of the
    middle sizes), lse_parts fp32 [n_parts][rows] (natural log); returns out fp32
    [rows][512] (allocated if absent); out_lse fp32 [rows] is written if given."""
    import torch

    if not (o_parts.is_contiguous() and lse_parts.is_contiguous()):
        raise ValueError("o_parts and lse_parts must be contiguous")
    if not o_parts.is_cuda:
        raise ValueError("o_parts must be a CUDA tensor")
    dev = o_parts.device
    n_parts = o_parts.shape[0]
    if o_parts.dim() < 2 or o_parts.shape[-1] != DV or o_parts.numel() == 0:
        raise ValueError("o_parts must be [n_parts][...][512]")
    o = o_parts.view(n_parts, -1, DV)
    rows = o.shape[1]
    _check_tensor(o, "o_parts", torch.float32, (n_parts, rows, DV), dev)
    if lse_parts.numel() != n_parts * rows:
        raise ValueError(f"lse_parts must hold n_parts x rows = {n_parts * rows} values")
    lse = lse_parts.view(n_parts, rows)
    _check_tensor(lse, "lse_parts", torch.float32, (n_parts, rows), dev)
    if out is None:
        out = torch.empty((rows, DV), dtype=torch.float32, device=dev)
    if not out.is_contiguous() or out.numel() != rows * DV:
        raise ValueError(f"out must be contiguous with rows x 512 = {rows * DV} values")
    _check_tensor(out.view(rows, DV), "out", torch.float32, (rows, DV), dev)
    if out_lse is not None:
        if not out_lse.is_contiguous() or out_lse.numel() != rows:
            raise ValueError(f"out_lse must be contiguous with {rows} values")
        _check_tensor(out_lse.view(rows), "out_lse", torch.float32, (rows,), dev)
    _check(load().mla_fa_combine(_ptr(o), _ptr(lse), n_parts, rows, _ptr(out), _ptr(out_lse),
                                 _stream_ptr(stream)), "mla_fa_combine")
    return out


def packed_width(rows):
    """Floats of one packed part: rows x 512 of O, then the rows' lse."""
    return rows * DV + rows


def combine_packed(parts, rows, out=None, out_lse=None, stream=None):
    """mla_fa_combine_strided over packed parts: parts fp32 [n_parts][rows*512 + rows],
    each part its O rows then its rows' lse (natural log). Returns out fp32 [rows][512]."""
    import torch

    if not parts.is_cuda:
        raise ValueError("parts must be a CUDA tensor")
    width = packed_width(rows)
    if parts.dim() != 2 or parts.shape[1] != width:
        raise ValueError(f"parts must be [n_parts][{width}]")
    _check_tensor(parts, "parts", torch.float32, (parts.shape[0], width), parts.device)
    if out is None:
        out = torch.empty((rows, DV), dtype=torch.float32, device=parts.device)
    if not out.is_contiguous() or out.numel() != rows * DV:
        raise ValueError(f"out must be contiguous with rows x 512 = {rows * DV} values")
    _check_tensor(out.view(rows, DV), "out", torch.float32, (rows, DV), parts.device)
    if out_lse is not None:
        if not out_lse.is_contiguous() or out_lse.numel() != rows:
            raise ValueError(f"out_lse must be contiguous with {rows} values")
        _check_tensor(out_lse.view(rows), "out_lse", torch.float32, (rows,), parts.device)
    base = parts.data_ptr()
    _check(load().mla_fa_combine_strided(ctypes.c_void_p(base), width,
                                         ctypes.c_void_p(base + rows * DV * 4), width,
                                         parts.shape[0], rows, _ptr(out), _ptr(out_lse),
                                         _stream_ptr(stream)), "mla_fa_combine_strided")
    return out


def mla_compact_mask(mask_row, idx_out, count_out, stream=None):
    _check(load().mla_compact_mask(_ptr(mask_row), mask_row.numel(), _ptr(idx_out), _ptr(count_out),
                                   _stream_ptr(stream)), "mla_compact_mask")


def mla_compact_workspace_size(n_rows, n_kv) -> int:
    return int(load().mla_compact_workspace_size(int(n_rows), int(n_kv)))


def mla_compact_mask_ex(mask, idx_out, count_out, workspace, stream=None):
    """mask [n_rows][n_kv] f16, idx_out [n_rows][>= n_kv] int32, count_out [n_rows] int32."""
    n_rows, n_kv = mask.shape
    _check(load().mla_compact_mask_ex(_ptr(mask), n_rows, mask.stride(0), n_kv, _ptr(idx_out),
                                      idx_out.stride(0), _ptr(count_out), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream_ptr(stream)), "mla_compact_mask_ex")


def mla_get_device_status(stream=None) -> int:
    return int(load().mla_get_device_status(_stream_ptr(stream)))


def mla_debug_wait_timeout(timeout_ns, stream=None):
    _check(load().mla_debug_wait_timeout(int(timeout_ns), _stream_ptr(stream)),
           "mla_debug_wait_timeout")


def mla_status_string(status) -> str:
    return load().mla_status_string(int(status)).decode()


def mla_profile_begin():
    _check(load().mla_profile_begin(), "mla_profile_begin")


def mla_profile_end():
    """Stop profiling; returns {kernel name: (launches, total_ms)}."""
    buf = (mla_profile_entry * 16)()
    n = ctypes.c_int(0)
    _check(load().mla_profile_end(buf, 16, ctypes.byref(n)), "mla_profile_end")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(n.value)}


NOALLOC_SCRATCH_BYTES = 24 << 20


def mla_fa_forward_noalloc(args, stream=None):
    """Forward pass that allocates nothing (split-KV partials in the library's
    static scratch); raises MlaError(MLA_ERR_WORKSPACE) if the pass needs more."""
    _check(load().mla_fa_forward_noalloc(ctypes.byref(args), _stream_ptr(stream)),
           "mla_fa_forward_noalloc")
