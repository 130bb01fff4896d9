"""Seeded synthetic inputs for the five MLA attention workloads.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it without sharing any of the method's code.

Layouts (host numpy arrays, C-contiguous):
  q       f16   [n_seq][n_q][n_head][576]   absorbed query: 512 latent + 64 rope
  kcache  f16   [n_seq][n_kv][576]          cache row: 512 latent then 64 rope
          uint8 [n_seq][n_kv][612]          q8_0 row: 18 x {f16 d, int8 q[32]}
  mask    f16   [n_seq][n_q][n_kv]          additive: 0 kept, -inf dropped
  kv_len  int32 [n_seq]                     cells before which the cache is valid

Every value is drawn in float32 from numpy's PCG64 with the workload's seed and
rounded to f16 once; the identical bytes feed the GPU and the oracle. The draw
order is fixed (lengths, Q, K, mask pattern) so a seed always gives the same
arrays. There is no public dataset behind these shapes: they are the cache
geometry of DeepSeek-V2-Lite / DeepSeek-V3 style models (one 576-wide cache head
shared by 16 or 128 query heads), with random values and no trained weights.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

DK = 576
DV = 512
Q8_BLOCK = 32
Q8_BLOCKS_PER_ROW = DK // Q8_BLOCK  # 18
Q8_BLOCK_BYTES = 2 + Q8_BLOCK       # f16 scale + 32 int8
Q8_ROW_BYTES = Q8_BLOCKS_PER_ROW * Q8_BLOCK_BYTES  # 612
KV_F16 = 0
KV_Q8_0 = 1
NEG_INF_F16_BITS = 0xFC00
SCALE_192 = 1.0 / math.sqrt(192.0)


@dataclasses.dataclass
class Workload:
    name: str
    q: np.ndarray
    kcache: np.ndarray
    kv_type: int
    mask: np.ndarray | None
    kv_len: np.ndarray
    scale: float
    seed: int
    # sparse workloads: the mask row is first compacted to an index list
    sparse: bool = False

    @property
    def n_seq(self):
        return self.q.shape[0]

    @property
    def n_q(self):
        return self.q.shape[1]

    @property
    def n_head(self):
        return self.q.shape[2]

    @property
    def n_kv(self):
        return self.kcache.shape[1]


def _normal_f16(rng, shape, std=1.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x.astype(np.float16)


def _mask_from_keep(keep):
    m = np.zeros(keep.shape, dtype=np.float16)
    m[~keep] = -np.inf
    return m


def q8_0_random(rng, shape_rows):
    """Random q8_0 rows: q ~ U{-127..127}, d = f16(U[0.5, 1.5] / 127) per block."""
    n = int(np.prod(shape_rows))
    qv = rng.integers(-127, 127, size=(n, Q8_BLOCKS_PER_ROW, Q8_BLOCK), endpoint=True,
                      dtype=np.int64).astype(np.int8)
    d = (rng.uniform(0.5, 1.5, size=(n, Q8_BLOCKS_PER_ROW)).astype(np.float32)
         / np.float32(127.0)).astype(np.float16)
    rows = np.empty((n, Q8_BLOCKS_PER_ROW, Q8_BLOCK_BYTES), dtype=np.uint8)
    rows[:, :, 0:2] = d.view(np.uint8).reshape(n, Q8_BLOCKS_PER_ROW, 2)
    rows[:, :, 2:] = qv.view(np.uint8)
    return rows.reshape(tuple(shape_rows) + (Q8_ROW_BYTES,))


def q8_0_pack(values_f16_bits_d, q_int8):
    """Assemble q8_0 rows from explicit scales (f16 [n][18]) and ints (int8 [n][18][32])."""
    n = q_int8.shape[0]
    rows = np.empty((n, Q8_BLOCKS_PER_ROW, Q8_BLOCK_BYTES), dtype=np.uint8)
    rows[:, :, 0:2] = np.ascontiguousarray(values_f16_bits_d, dtype=np.float16).view(
        np.uint8).reshape(n, Q8_BLOCKS_PER_ROW, 2)
    rows[:, :, 2:] = np.ascontiguousarray(q_int8, dtype=np.int8).view(np.uint8)
    return rows.reshape(n, Q8_ROW_BYTES)


# --------------------------------------------------------------------------------------
# The five workloads. Each builder takes size overrides so parity tests can run the same
# recipe at sizes the oracle finishes in seconds; the defaults are the full sizes.
# --------------------------------------------------------------------------------------

def tiny_decode(seed=1001, n_kv=256, n_head=16):
    """n_q=1, 16 heads, n_kv=256, Q,K ~ N(0,1), zero mask."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _normal_f16(rng, (1, 1, n_head, DK))
    k = _normal_f16(rng, (1, n_kv, DK))
    mask = np.zeros((1, 1, n_kv), dtype=np.float16)
    return Workload("tiny_decode", q, k, KV_F16, mask, np.array([n_kv], np.int32), SCALE_192,
                    seed)


def v2lite_decode(seed=1002, n_kv=4096, n_head=16, n_pad=37):
    """n_q=1, 16 heads, n_kv=4096, K ~ 0.5 N(0,1), Q ~ N(0,1), last 37 cells -inf."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _normal_f16(rng, (1, 1, n_head, DK))
    k = _normal_f16(rng, (1, n_kv, DK), std=0.5)
    keep = np.ones((1, 1, n_kv), dtype=bool)
    if n_pad:
        keep[..., n_kv - n_pad:] = False
    return Workload("v2lite_decode", q, k, KV_F16, _mask_from_keep(keep),
                    np.array([n_kv], np.int32), SCALE_192, seed)


def v3_batched_decode(seed=1003, n_seq=8, n_head=128, len_lo=4096, len_hi=32768, n_kv=None):
    """8 sequences x n_q=1, 128 heads, lengths ~ U{4096..32768}, padded cells -inf.

    The cache is padded to n_kv (default len_hi); the padding holds random values, not
    zeros, so that any leakage of a masked cell shows in the result."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = rng.integers(len_lo, len_hi, size=n_seq, endpoint=True).astype(np.int32)
    n_kv = int(len_hi if n_kv is None else n_kv)
    lens = np.minimum(lens, n_kv).astype(np.int32)
    q = _normal_f16(rng, (n_seq, 1, n_head, DK))
    k = _normal_f16(rng, (n_seq, n_kv, DK))
    keep = np.arange(n_kv)[None, None, :] < lens[:, None, None]
    return Workload("v3_batched_decode", q, k, KV_F16, _mask_from_keep(keep), lens, SCALE_192,
                    seed)


def prefill_chunk(seed=1004, n_q=512, n_head=128, n_kv=16384):
    """n_q new tokens at the end of an n_kv cache; query i sees key j iff
    j <= (n_kv - n_q) + i (causal)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _normal_f16(rng, (1, n_q, n_head, DK))
    k = _normal_f16(rng, (1, n_kv, DK))
    past = n_kv - n_q
    keep = np.arange(n_kv)[None, :] <= (past + np.arange(n_q))[:, None]
    return Workload("prefill_chunk", q, k, KV_F16, _mask_from_keep(keep[None]),
                    np.array([n_kv], np.int32), SCALE_192, seed)


def sparse_block_keep(rng, n_kv, block=64, keep_frac_den=8, tail_blocks=16):
    """Keep pattern: the last `tail_blocks` blocks of `block` cells always, plus random
    blocks drawn without replacement from the rest, so that exactly 1/keep_frac_den of
    the blocks are kept."""
    n_blocks = n_kv // block
    n_keep = n_blocks // keep_frac_den
    tail = min(tail_blocks, n_keep)
    head_pool = n_blocks - tail
    chosen = rng.choice(head_pool, size=n_keep - tail, replace=False)
    kept_blocks = np.concatenate([np.sort(chosen), np.arange(head_pool, n_blocks)])
    keep = np.zeros(n_kv, dtype=bool)
    for b_ in kept_blocks:
        keep[b_ * block:(b_ + 1) * block] = True
    return keep


def sparse_q8_decode(seed=1005, n_kv=131072, n_head=128, block=64, tail_blocks=16):
    """n_q=1, 128 heads, q8_0 cache of n_kv rows, mask keeps 1/8 of the 64-cell blocks
    (the last 16 blocks = 1024 cells always); compaction then attention."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _normal_f16(rng, (1, 1, n_head, DK))
    k = q8_0_random(rng, (1, n_kv))
    keep = sparse_block_keep(rng, n_kv, block=block, tail_blocks=tail_blocks)
    return Workload("sparse_q8_decode", q, k, KV_Q8_0, _mask_from_keep(keep[None, None]),
                    np.array([n_kv], np.int32), SCALE_192, seed, sparse=True)


@dataclasses.dataclass
class HeadsWorkload:
    """Inputs of the DK = 192 / DV = 128 head shape: a K and a V per KV head."""
    name: str
    q: np.ndarray       # f16 [n_seq][n_q][n_head][192]
    k: np.ndarray       # f16 [n_seq][n_kv][n_kv_head][192]
    v: np.ndarray       # f16 [n_seq][n_kv][n_kv_head][128]
    mask: np.ndarray | None
    kv_len: np.ndarray
    scale: float
    seed: int

    @property
    def n_seq(self):
        return self.q.shape[0]

    @property
    def n_q(self):
        return self.q.shape[1]

    @property
    def n_head(self):
        return self.q.shape[2]

    @property
    def n_kv(self):
        return self.k.shape[1]

    @property
    def n_kv_head(self):
        return self.k.shape[2]


def heads_prefill(seed=1007, n_seq=1, n_q=512, n_head=16, n_kv_head=16, n_kv=4096, causal=True,
                  lengths=None):
    """The non-absorbed MLA head (DK = 192: 128 nope + 64 rope, DV = 128) with the
    DeepSeek-V2-Lite head count: n_q new tokens at the end of each sequence, K and V per
    KV head (n_kv_head = n_head: multi-head attention), Q, K, V ~ N(0,1), causal f16 mask
    (query i of n_q sees key j iff j <= L - n_q + i), scale 1/sqrt(192). `lengths` (per
    sequence, <= n_kv) gives ragged sequences; cells past a length are -inf."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = np.full(n_seq, n_kv, np.int32) if lengths is None else np.asarray(lengths, np.int32)
    q = _normal_f16(rng, (n_seq, n_q, n_head, 192))
    k = _normal_f16(rng, (n_seq, n_kv, n_kv_head, 192))
    v = _normal_f16(rng, (n_seq, n_kv, n_kv_head, 128))
    j = np.arange(n_kv)[None, None, :]
    i = np.arange(n_q)[None, :, None]
    L = lens[:, None, None]
    keep = np.broadcast_to(j < L, (n_seq, n_q, n_kv))
    if causal:
        keep = keep & (j <= L - n_q + i)
    return HeadsWorkload("heads_prefill", q, k, v, _mask_from_keep(keep), lens, SCALE_192, seed)


def heads_decode(seed=1008, n_seq=8, n_head=16, n_kv_head=16, len_lo=1024, len_hi=8192, n_kv=None):
    """One query token per sequence over a ragged batch of K/V caches (lengths uniform in
    [len_lo, len_hi], padded cells -inf), the decode step of the same head shape."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = rng.integers(len_lo, len_hi, size=n_seq, endpoint=True).astype(np.int32)
    n_kv = int(len_hi if n_kv is None else n_kv)
    lens = np.minimum(lens, n_kv).astype(np.int32)
    q = _normal_f16(rng, (n_seq, 1, n_head, 192))
    k = _normal_f16(rng, (n_seq, n_kv, n_kv_head, 192))
    v = _normal_f16(rng, (n_seq, n_kv, n_kv_head, 128))
    keep = np.arange(n_kv)[None, None, :] < lens[:, None, None]
    return HeadsWorkload("heads_decode", q, k, v, _mask_from_keep(keep), lens, SCALE_192, seed)


BUILDERS = {
    "tiny_decode": tiny_decode,
    "v2lite_decode": v2lite_decode,
    "v3_batched_decode": v3_batched_decode,
    "prefill_chunk": prefill_chunk,
    "sparse_q8_decode": sparse_q8_decode,
}

def wv_random(seed=1006, n_head=128, proj_dim=128):
    """Synthetic value up-projection weights (no trained weights exist here): f16
    [n_head][512][proj_dim], normal with std 1/sqrt(512) so that a projected row has
    the scale of an attention row."""
    rng = np.random.default_rng(seed)
    return _normal_f16(rng, (n_head, 512, proj_dim), std=1.0 / np.sqrt(512.0))


# Full sizes, in the order the five workloads are listed in the benchmark definition.
WORKLOAD_ORDER = ["tiny_decode", "v2lite_decode", "v3_batched_decode", "prefill_chunk",
                  "sparse_q8_decode"]


def make(name, **overrides):
    return BUILDERS[name](**overrides)
