"""fp64 CPU oracle for MLA attention over the compressed KV cache.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The CUDA library never loads it, and it shares no code with that
library: the two meet only through the seeded input generators.

The arithmetic lives in ``mla_oracle.c`` (plain C, fp64, OpenMP over query
rows). This module compiles it with gcc on first use and wraps it with ctypes.
What it computes and which page passage each part follows is written at the
top of ``mla_oracle.c``. Two definitions are plain numpy here, each with its
reading in its docstring: ``combine`` (the merge of partial results over
disjoint key sets) and ``attention_heads`` (a K and a V per KV head, the
DK = 192 / DV = 128 head shape).

Parity pins (checked by ``tests/test_oracle_pins.py`` against closed forms,
brute force and invariants, never against the oracle itself):
  attention (576- and 512-wide heads) / attention_lse / attention_online /
  attention_split / compact / dequant_q8_0 / project / attention_variants /
  combine / attention_heads.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

DK = 576
DV = 512
Q8_ROW_BYTES = 612
KV_F16 = 0
KV_Q8_0 = 1

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile mla_oracle.c into oracle/_build/liboracle.so (gcc, OpenMP)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".{os.getpid()}.tmp"
    cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L = ctypes.c_long
        I = ctypes.c_int
        D = ctypes.c_double
        lib.oracle_init.restype = None
        lib.oracle_max_threads.restype = I
        lib.oracle_set_threads.argtypes = [I]
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = D
        common = [P, P, I, P, P, L, I, I, L, D, P, L]
        lib.oracle_attention.argtypes = common + [P]
        lib.oracle_attention.restype = I
        lib.oracle_attention_lse.argtypes = common + [P, P]
        lib.oracle_attention_lse.restype = I
        lib.oracle_attention_dk.argtypes = [P, P, P, P, L, I, I, L, I, D, P, L, P, P]
        lib.oracle_attention_dk.restype = I
        lib.oracle_attention_online.argtypes = common + [L, P]
        lib.oracle_attention_online.restype = I
        lib.oracle_attention_split.argtypes = common + [P, I, P]
        lib.oracle_attention_split.restype = I
        lib.oracle_compact.argtypes = [P, L, P]
        lib.oracle_compact.restype = L
        lib.oracle_dequant_q8_0.argtypes = [P, L, P]
        lib.oracle_dequant_q8_0.restype = None
        lib.oracle_project.argtypes = [P, P, L, P, I, I, P]
        lib.oracle_project.restype = I
        D_ = ctypes.c_double
        lib.oracle_attention_variants.argtypes = [P, P, I, P, P, L, I, I, L, D_, D_, P, L, P, P]
        lib.oracle_attention_variants.restype = I
        lib.oracle_init()
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits16(a):
    """f16 array (or its uint16 bit view) as a C-contiguous uint16 array."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16/uint16, got {a.dtype}")
    return a


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def half_to_double(bits: int) -> float:
    return float(_load().oracle_half_to_double(int(bits)))


def _prep(q, kcache, kv_type, mask, idx, rows):
    q = _bits16(q)
    if q.ndim != 3 or q.shape[2] not in (DK, DV):
        raise ValueError("q must be [n_q][n_head][576] (or [..][512], f16 cache)")
    n_q, n_head, dk = q.shape
    if dk != DK and kv_type != KV_F16:
        raise ValueError("the 512-wide head shape takes an f16 cache")
    if kv_type == KV_F16:
        kc = _bits16(kcache)
        if kc.ndim != 2 or kc.shape[1] != dk:
            raise ValueError("f16 kcache must be [n_kv][dk], dk as q's")
    elif kv_type == KV_Q8_0:
        kc = np.ascontiguousarray(kcache, dtype=np.uint8)
        if kc.ndim != 2 or kc.shape[1] != Q8_ROW_BYTES:
            raise ValueError("q8_0 kcache must be [n_kv][612] bytes")
    else:
        raise ValueError("unknown kv_type")
    n_kv = kc.shape[0]
    m = None
    if mask is not None:
        m = _bits16(mask)
        if m.shape != (n_q, n_kv):
            raise ValueError("mask must be [n_q][n_kv]")
    ix = None if idx is None else np.ascontiguousarray(idx, dtype=np.int32)
    rw = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n_out = n_q * n_head if rw is None else len(rw)
    out = np.zeros((n_out, DV), dtype=np.float64)
    return q, kc, m, ix, rw, n_q, n_head, n_kv, out


def attention(q, kcache, kv_type=KV_F16, mask=None, scale=1.0, rows=None, idx=None):
    """Two-pass fp64 softmax(scale*Q.K^T + mask).V with V = K[:, :512].

    q: f16 [n_q][n_head][576]; kcache: f16 [n_kv][576] or q8_0 bytes [n_kv][612]
    (or q [..][512] with an f16 kcache [n_kv][512]: the DK = DV = 512 head shape);
    mask: f16 [n_q][n_kv] or None; idx: optional int32 kept rows (sparse);
    rows: optional row ids t*n_head+h to compute. Returns float64 [rows][512].
    """
    q, kc, m, ix, rw, n_q, n_head, n_kv, out = _prep(q, kcache, kv_type, mask, idx, rows)
    if q.shape[2] != DK:  # the DK = DV = 512 head shape
        rc = _load().oracle_attention_dk(_ptr(q), _ptr(kc), _ptr(m), _ptr(ix),
                                         0 if ix is None else len(ix), n_q, n_head, n_kv,
                                         q.shape[2], float(scale), _ptr(rw),
                                         0 if rw is None else len(rw), _ptr(out), None)
        if rc != 0:
            raise ValueError("oracle_attention_dk rejected its arguments")
        return out
    rc = _load().oracle_attention(_ptr(q), _ptr(kc), kv_type, _ptr(m), _ptr(ix),
                                  0 if ix is None else len(ix), n_q, n_head, n_kv, float(scale),
                                  _ptr(rw), 0 if rw is None else len(rw), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_attention rejected its arguments")
    return out


def attention_lse(q, kcache, kv_type=KV_F16, mask=None, scale=1.0, rows=None, idx=None):
    """attention() and, per row, the natural log-sum-exp of the scores,
    lse = log sum_j exp(scale*q.k_j + mask_j) (-inf for a row with nothing kept).
    Returns (float64 [rows][512], float64 [rows])."""
    q, kc, m, ix, rw, n_q, n_head, n_kv, out = _prep(q, kcache, kv_type, mask, idx, rows)
    lse = np.zeros(out.shape[0], dtype=np.float64)
    if q.shape[2] != DK:  # the DK = DV = 512 head shape
        rc = _load().oracle_attention_dk(_ptr(q), _ptr(kc), _ptr(m), _ptr(ix),
                                         0 if ix is None else len(ix), n_q, n_head, n_kv,
                                         q.shape[2], float(scale), _ptr(rw),
                                         0 if rw is None else len(rw), _ptr(out), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle_attention_dk rejected its arguments")
        return out, lse
    rc = _load().oracle_attention_lse(_ptr(q), _ptr(kc), kv_type, _ptr(m), _ptr(ix),
                                      0 if ix is None else len(ix), n_q, n_head, n_kv, float(scale),
                                      _ptr(rw), 0 if rw is None else len(rw), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention_lse rejected its arguments")
    return out, lse


def combine(o_parts, lse_parts):
    """Merge partial attention results of the same rows over disjoint key sets
    (split-KV across devices): with M = max_p lse_p and w_p = exp(lse_p - M),
    out = sum_p w_p o_p / sum_p w_p and lse = M + log(sum_p w_p). A row whose parts
    are all -inf gets out = 0 and lse = -inf. The merge follows from the softmax
    definition: o_p = sum_{j in part p} e^{s_j} v_j / e^{lse_p}. The pages give the
    running-max rescaling inside one pass (Vulkan FA for DeepSeek MLA article, section
    2.2); the merge across parts is the same rule applied to whole parts.
    o_parts float [P][rows][512], lse_parts float [P][rows]; returns float64
    ([rows][512], [rows])."""
    o = np.asarray(o_parts, dtype=np.float64)
    lse = np.asarray(lse_parts, dtype=np.float64)
    if o.ndim != 3 or lse.shape != o.shape[:2]:
        raise ValueError("o_parts [P][rows][512] and lse_parts [P][rows]")
    n_rows = o.shape[1]
    out = np.zeros((n_rows, o.shape[2]), dtype=np.float64)
    out_lse = np.full(n_rows, -np.inf)
    for r in range(n_rows):
        M = np.max(lse[:, r])
        if M == -np.inf:
            continue
        w = np.exp(lse[:, r] - M)
        out[r] = (w[:, None] * o[:, r, :]).sum(axis=0) / w.sum()
        out_lse[r] = M + np.log(w.sum())
    return out, out_lse


def attention_heads(q, k, v, mask=None, scale=1.0):
    """Attention with a K and a V per KV head, the layout of the DK = 192 / DV = 128 head
    shape (one of the head shapes the llama.cpp tag page lists for the Metal FA kernel,
    PR #29570): query head h reads KV head h // (n_head / n_kv_head), so n_kv_head =
    n_head is plain multi-head attention and n_kv_head = 1 shares one head, as the MLA
    cache does. Per query row, s_j = scale * q . k_j + mask_j, o = sum_j softmax(s)_j v_j;
    a row with nothing kept gives 0.

    q f16 [n_q][n_head][dk], k f16 [n_kv][n_kv_head][dk], v f16 [n_kv][n_kv_head][dv],
    mask f16 [n_q][n_kv] or None (shared by the heads of a token). fp64 throughout;
    returns float64 [n_q * n_head][dv], row t * n_head + h."""
    qd = np.asarray(q, dtype=np.float16).astype(np.float64)
    kd = np.asarray(k, dtype=np.float16).astype(np.float64)
    vd = np.asarray(v, dtype=np.float16).astype(np.float64)
    n_q, n_head, dk = qd.shape
    n_kv, n_kv_head, dk2 = kd.shape
    if dk2 != dk or vd.shape[:2] != (n_kv, n_kv_head) or n_head % n_kv_head:
        raise ValueError("q [n_q][H][dk], k [n][Hkv][dk], v [n][Hkv][dv], H a multiple of Hkv")
    group = n_head // n_kv_head
    md = None if mask is None else np.asarray(mask, dtype=np.float16).astype(np.float64)
    out = np.zeros((n_q, n_head, vd.shape[2]))
    for hk in range(n_kv_head):
        hs = slice(hk * group, (hk + 1) * group)
        s = scale * np.einsum("thc,nc->thn", qd[:, hs, :], kd[:, hk, :])  # [n_q][group][n_kv]
        if md is not None:
            s = s + md[:, None, :]
        m = s.max(axis=2, keepdims=True)
        kept = np.isfinite(m)
        p = np.where(kept, np.exp(s - np.where(kept, m, 0.0)), 0.0)
        den = p.sum(axis=2, keepdims=True)
        o = np.einsum("thn,nd->thd", p, vd[:, hk, :])
        out[:, hs, :] = np.where(den > 0, o / np.where(den > 0, den, 1.0), 0.0)
    return out.reshape(n_q * n_head, -1)


def attention_online(q, kcache, kv_type=KV_F16, mask=None, scale=1.0, tile=64, rows=None,
                     idx=None):
    """One-pass tiled online-softmax variant (running max m, running sum l)."""
    q, kc, m, ix, rw, n_q, n_head, n_kv, out = _prep(q, kcache, kv_type, mask, idx, rows)
    rc = _load().oracle_attention_online(_ptr(q), _ptr(kc), kv_type, _ptr(m), _ptr(ix),
                                         0 if ix is None else len(ix), n_q, n_head, n_kv,
                                         float(scale), _ptr(rw), 0 if rw is None else len(rw),
                                         int(tile), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_attention_online rejected its arguments")
    return out


def attention_split(q, kcache, kv_type=KV_F16, mask=None, scale=1.0, bounds=None, rows=None,
                    idx=None):
    """Split-KV variant: per-part (acc, m, l) merged by the log-sum-exp rule."""
    q, kc, m, ix, rw, n_q, n_head, n_kv, out = _prep(q, kcache, kv_type, mask, idx, rows)
    b = np.ascontiguousarray(bounds, dtype=np.int32)
    rc = _load().oracle_attention_split(_ptr(q), _ptr(kc), kv_type, _ptr(m), _ptr(ix),
                                        0 if ix is None else len(ix), n_q, n_head, n_kv,
                                        float(scale), _ptr(rw), 0 if rw is None else len(rw),
                                        _ptr(b), len(b) - 1, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_attention_split rejected its arguments")
    return out


def compact(mask_row):
    """Ascending int32 indices of the cells whose f16 bits are not -inf."""
    m = _bits16(mask_row).ravel()
    idx = np.empty(max(len(m), 1), dtype=np.int32)
    n = _load().oracle_compact(_ptr(m), len(m), _ptr(idx))
    return idx[:n].copy()


def dequant_q8_0(rows_bytes):
    """q8_0 rows [n][612] -> float64 [n][576], value = d * q per 32-block."""
    r = np.ascontiguousarray(rows_bytes, dtype=np.uint8)
    if r.ndim != 2 or r.shape[1] != Q8_ROW_BYTES:
        raise ValueError("q8_0 rows must be [n][612]")
    out = np.empty((r.shape[0], DK), dtype=np.float64)
    _load().oracle_dequant_q8_0(_ptr(r), r.shape[0], _ptr(out))
    return out


def attention_batched(q, kcache, kv_type=KV_F16, mask=None, scale=1.0, rows=None, idx=None,
                      counts=None):
    """Per-sequence loop for batched inputs.

    q [n_seq][n_q][n_head][576]; kcache [n_seq][n_kv][...]; mask [n_seq][n_q][n_kv] or None;
    rows: optional list (one array or None per sequence); idx/counts for sparse.
    Returns a list of float64 arrays, one per sequence.
    """
    outs = []
    for b in range(q.shape[0]):
        ib = None
        if idx is not None:
            ib = idx[b][: counts[b]] if counts is not None else idx[b]
        outs.append(attention(q[b], kcache[b], kv_type, None if mask is None else mask[b],
                              scale, None if rows is None else rows[b], ib))
    return outs


def project(o, heads, wv):
    """Value up-projection of attention rows: p[r][n] = sum_d o[r][d] * wv[heads[r]][d][n].

    o: float64 [n_rows][512] attention rows; heads: int [n_rows], the head of each row;
    wv: f16 [n_head][512][proj_dim]. Returns float64 [n_rows][proj_dim] (fp64 sums of
    exact products of the f16 weights)."""
    o = np.ascontiguousarray(o, dtype=np.float64)
    hd = np.ascontiguousarray(heads, dtype=np.int32)
    w = _bits16(wv)
    if o.ndim != 2 or o.shape[1] != DV or w.ndim != 3 or w.shape[1] != DV or len(hd) != o.shape[0]:
        raise ValueError("project: o [n][512], heads [n], wv [n_head][512][proj_dim]")
    n_head, _, proj_dim = w.shape
    out = np.zeros((o.shape[0], proj_dim), dtype=np.float64)
    rc = _load().oracle_project(_ptr(o), _ptr(hd), o.shape[0], _ptr(np.ascontiguousarray(w)),
                                n_head, proj_dim, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_project rejected its arguments")
    return out


def attention_variants(q, kcache, kv_type=KV_F16, mask=None, scale=1.0, idx=None, softcap=0.0,
                       slopes=None, pos0=0, sinks=None):
    """Attention with the optional variants: logit softcap (softcap > 0), ALiBi (slopes
    [n_head], bias slopes[h] * (j - (pos0 + t))) and attention sinks (sinks [n_head],
    one extra logit per head in the denominator). Returns float64 [n_q*n_head][512]."""
    q, kc, m, ix, _, n_q, n_head, n_kv, out = _prep(q, kcache, kv_type, mask, idx, None)
    sl = None if slopes is None else np.ascontiguousarray(slopes, dtype=np.float64)
    sk = None if sinks is None else np.ascontiguousarray(sinks, dtype=np.float64)
    if (sl is not None and sl.shape != (n_head,)) or (sk is not None and sk.shape != (n_head,)):
        raise ValueError("slopes and sinks are per head")
    rc = _load().oracle_attention_variants(_ptr(q), _ptr(kc), kv_type, _ptr(m), _ptr(ix),
                                           0 if ix is None else len(ix), n_q, n_head, n_kv,
                                           float(scale), float(softcap), _ptr(sl), int(pos0),
                                           _ptr(sk), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_attention_variants rejected its arguments")
    return out
