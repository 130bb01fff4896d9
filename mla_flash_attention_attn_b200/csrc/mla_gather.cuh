// Gather of an index list's cache rows into a dense f16 buffer, for the TMA-mode
// attention kernel (Vulkan FA for DeepSeek MLA article, section 2.2: the sparse pass
// attends only to the cells an index list keeps; llama.cpp b11413 release note: the
// list comes from the mask by compaction).
//
// A sequence attends to the cache rows idx[0..len) (len = min(idx_count, the length
// planned for it)). The attention kernel's gather modes fetch those rows one 32-value
// block at a time from a few producer warps per SM, so a step waits on chains of
// dependent loads. Here every SM gathers at once: a warp reads whole rows with
// coalesced loads, dequantises q8_0 blocks to f16 values d*q exactly as the attention
// kernel's producers do (f16 rows are copied), writes them to row `position` of the
// dense buffer, and writes each position's mask value of every query token. The
// attention kernel then streams the dense rows with TMA, in list order, with the
// gathered mask.
//
// An index outside [0, n_kv) gives a zero row and a -inf mask value (the cell drops
// out), and records MLA_ERR_INDEX, as in the gather modes. The rows from len up to the
// next 128-row boundary are zeroed: a pipeline step reads them, and a finite row under
// a -inf score adds nothing (uninitialised workspace could hold NaN).
#pragma once
#include <cstdint>

#include "mla_common.cuh"
#include "mla_fwd.cuh"

namespace mla {

struct GatherParams {
  const int32_t* idx;        // [seq][idx_seq_stride] cell indices
  const int32_t* idx_count;  // [seq] list lengths
  int64_t idx_seq_stride;
  const uint8_t* kcache;     // cache row (b, j) at (b * k_seq_stride + j) * row_bytes
  int64_t k_seq_stride;      // rows
  int64_t kcache_bytes;      // bytes of kcache that may be read: up to the end of row (n_seq - 1, n_kv - 1)
  int n_kv;
  const uint16_t* mask;      // f16 bits [seq][n_q][cells], or nullptr (all cells 0)
  int64_t mask_seq_stride;   // elements
  int64_t mask_row_stride;   // elements
  int n_q;
  uint16_t* rows;            // f16 [seq][cap][head width]: the gathered rows
  uint16_t* gmask;           // f16 [seq][n_q][gmask_stride]: their mask values
  int64_t cap;               // rows per sequence in `rows`
  int64_t gmask_stride;      // >= cap
  uint64_t timeout_ns;       // bound of each wait for the copy engine
};

// Grid (blocks, sequences of the launch); 256 threads. A warp takes kRows positions at a
// time and reads their indices. q8_0 rows (612 bytes, 4-byte aligned) come into the
// warp's shared-memory stage by the copy engine: one bulk copy per row of the 624-byte,
// 16-byte-aligned span that holds it, all on one barrier of the warp (a copy takes none
// of the SM's load slots, so many rows are in flight at once); a row whose span would
// reach past either end of the cache is read word by word instead. The warp then
// dequantises each row from the stage in 16-byte chunks of f16 values, stored
// coalesced. f16 rows are read with
// coalesced 16-byte loads and written out as read. kMode: kModeQ8 (612-byte q8_0 rows)
// or kModeGatherF16 (f16 rows of 64 * kNC values); kNC: 64-column chunks of the head
// width.
template <int kMode, int kNC>
__global__ void __launch_bounds__(256)
    mla_gather_rows_kernel(const __grid_constant__ Plan plan, const __grid_constant__ GatherParams g) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the lists are written by the kernel before
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr bool kQ8 = kMode == kModeQ8;
  constexpr int kWidth = 64 * kNC;                      // f16 values of a gathered row
  constexpr int kRowBytes = kQ8 ? kQ8RowBytes : 2 * kWidth;
  constexpr int kRows = kQ8 ? 4 : 2;                    // positions in flight per warp
  constexpr int kQ8Words = kQ8RowBytes / 4;             // 153 (rows are 4-byte aligned)
  constexpr int kSlotBytes = (kQ8RowBytes + 12 + 15) / 16 * 16;  // 624: the span of a row
  constexpr int kSlotWords = kSlotBytes / 4;
  constexpr int kF16Vec = kWidth / 8;                   // 16-byte chunks of an f16 row
  constexpr int kF16PerLane = (kF16Vec + 31) / 32;
  constexpr int kChunks = kWidth / 8;                   // 16-byte chunks of a gathered row (72)
  static_assert(kSlotBytes % 16 == 0 && kSlotWords >= 3 + kQ8Words, "a row's span fits its slot");
  __shared__ __align__(128) uint32_t stage[kQ8 ? 8 * kRows * kSlotWords : 4];
  __shared__ uint64_t wbar[8];  // one barrier per warp: its rows' copies have landed
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (kQ8) {
    if (lane == 0) {
      mbar_init(&wbar[warp], 1);
      fence_mbar_init();
    }
    __syncwarp();
  }
  const int b = blockIdx.y;
  const int b_abs = plan.seq_offset + b;
  const int len = min(max(__ldg(g.idx_count + b_abs), 0), plan.kv_len[b]);
  const int pad_end = (int)min(g.cap, ((int64_t)len + 127) / 128 * 128);
  const int32_t* idx_row = g.idx + (int64_t)b_abs * g.idx_seq_stride;
  const uint8_t* cache_seq = g.kcache + (int64_t)b_abs * g.k_seq_stride * kRowBytes;
  uint16_t* out_seq = g.rows + (int64_t)b_abs * g.cap * kWidth;
  const int n_warps = gridDim.x * 8;
  uint32_t phase = 0;
  bool failed = false;
  for (int r0 = (blockIdx.x * 8 + warp) * kRows; r0 < pad_end; r0 += n_warps * kRows) {
    // cache row of each position: >= 0, or -1 (past the list: a zero row) or -2 (an
    // invalid index: a zero row and a -inf mask value)
    int key[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int pos = r0 + u;
      int k = -1;
      if (pos < len) {
        k = __ldg(idx_row + pos);
        if (k < 0 || k >= g.n_kv) {
          if (lane == 0) record_status(kStatusIndex);
          k = -2;
        }
      }
      key[u] = k;
    }
    // the positions' mask values (lane t: query token t, the first 32 tokens), loaded
    // while the rows are in flight
    uint16_t mv0[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      mv0[u] = 0xFC00u;  // -inf: an invalid index drops out
      if (key[u] >= 0 && lane < g.n_q)
        mv0[u] = g.mask != nullptr
                     ? __ldg(g.mask + (int64_t)b_abs * g.mask_seq_stride + (int64_t)lane * g.mask_row_stride + key[u])
                     : (uint16_t)0;
    }
    if constexpr (kQ8) {
      uint32_t* sw = stage + warp * kRows * kSlotWords;
      // row u's span starts off[u] words before the row
      int off[kRows];
      bool by_copy[kRows];
      const uint8_t* span[kRows];
      uint32_t bytes = 0;
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const uint8_t* src = cache_seq + (int64_t)max(key[u], 0) * kRowBytes;
        span[u] = reinterpret_cast<const uint8_t*>(reinterpret_cast<uintptr_t>(src) & ~static_cast<uintptr_t>(15));
        off[u] = (int)((reinterpret_cast<uintptr_t>(src) & 15) >> 2);
        by_copy[u] = key[u] >= 0 && span[u] >= g.kcache && span[u] + kSlotBytes <= g.kcache + g.kcache_bytes;
        if (by_copy[u]) bytes += kSlotBytes;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&wbar[warp], bytes);  // completes at once when no row is copied
#pragma unroll
        for (int u = 0; u < kRows; ++u)
          if (by_copy[u]) bulk_load(sw + u * kSlotWords, span[u], kSlotBytes, &wbar[warp]);
      }
      // a row at either end of the cache: word loads, to the place its span would give
#pragma unroll
      for (int u = 0; u < kRows; ++u)
        if (key[u] >= 0 && !by_copy[u]) {
          const uint32_t* src = reinterpret_cast<const uint32_t*>(cache_seq + (int64_t)key[u] * kRowBytes);
          for (int w = lane; w < kQ8Words; w += 32) sw[u * kSlotWords + off[u] + w] = __ldg(src + w);
        }
      if (!__all_sync(0xffffffffu, mbar_wait(&wbar[warp], phase, g.timeout_ns))) {
        // the copies may still land: stop here and let the end of the kernel wait for them
        if (lane == 0) record_status(kStatusTimeout);
        failed = true;
        break;
      }
      phase ^= 1;
      __syncwarp();
      // The f16 row is written in 16-byte chunks, chunk c = values 8c..8c+7 (a quarter of
      // block c / 4), lane l taking chunks l, l + 32, l + 64: each store instruction covers
      // 512 contiguous bytes of the row. A chunk's value d * q is formed as in the
      // attention kernel's producers: the int8 q goes into the mantissa of 1024 + (q + 128),
      // 1152 is taken off and the f16 product with d is rounded once.
      const __half2 bias = __float2half2_rn(1152.f);
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int pos = r0 + u;
        if (pos >= pad_end) continue;
        const uint32_t* sr = sw + u * kSlotWords;  // the row starts at byte 4 off[u]
        uint4* dst = reinterpret_cast<uint4*>(out_seq + (int64_t)pos * kWidth);
#pragma unroll
        for (int j = 0; j < (kChunks + 31) / 32; ++j) {
          const int c = lane + 32 * j;
          if (c >= kChunks) continue;
          uint32_t h[4] = {0u, 0u, 0u, 0u};  // zeros for an invalid index and past the list
          if (key[u] >= 0) {
            const int b0 = 4 * off[u] + 34 * (c >> 2);  // the block's first byte (its scale d)
            const uint32_t dw = sr[b0 >> 2];
            const __half2 d2 = __half2half2(__ushort_as_half((unsigned short)((b0 & 2) ? (dw >> 16) : (dw & 0xFFFFu))));
            const int b1 = b0 + 2 + 8 * (c & 3);          // the chunk's 8 int8 values
            const uint32_t sh = (b1 & 2) ? 16u : 0u;
            const uint32_t a0 = sr[b1 >> 2], a1 = sr[(b1 >> 2) + 1];
            const uint32_t a2 = sh ? sr[(b1 >> 2) + 2] : 0u;  // inside the row when the values straddle it
            const uint32_t x[2] = {__funnelshift_r(a0, a1, sh) ^ 0x80808080u, __funnelshift_r(a1, a2, sh) ^ 0x80808080u};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t wd = __byte_perm(x[k >> 1], 0x64646464u, (k & 1) ? 0x4342 : 0x4140);
              __half2 v = *reinterpret_cast<const __half2*>(&wd);
              v = __hmul2(__hsub2(v, bias), d2);
              h[k] = *reinterpret_cast<uint32_t*>(&v);
            }
          }
          dst[c] = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
      // the stage is read (generic proxy) before the next copies overwrite it (async proxy)
      fence_proxy_async_smem();
      __syncwarp();
    } else {
      uint4 v[kRows][kF16PerLane];
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const uint4* src = reinterpret_cast<const uint4*>(cache_seq + (int64_t)max(key[u], 0) * kRowBytes);
#pragma unroll
        for (int j = 0; j < kF16PerLane; ++j) {
          const int c = lane + 32 * j;
          v[u][j] = (key[u] >= 0 && c < kF16Vec) ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int pos = r0 + u;
        if (pos >= pad_end) continue;
        uint4* dst = reinterpret_cast<uint4*>(out_seq + (int64_t)pos * kWidth);
#pragma unroll
        for (int j = 0; j < kF16PerLane; ++j)
          if (lane + 32 * j < kF16Vec) dst[lane + 32 * j] = v[u][j];
      }
    }
    // the positions' mask values, one query token per lane (tokens past the first 32 are
    // read here)
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int pos = r0 + u;
      if (pos >= len) continue;
      for (int t = lane; t < g.n_q; t += 32) {
        uint16_t mv = mv0[u];
        if (t >= 32) {
          mv = 0xFC00u;
          if (key[u] >= 0)
            mv = g.mask != nullptr
                     ? __ldg(g.mask + (int64_t)b_abs * g.mask_seq_stride + (int64_t)t * g.mask_row_stride + key[u])
                     : (uint16_t)0;
        }
        g.gmask[((int64_t)b_abs * g.n_q + t) * g.gmask_stride + pos] = mv;
      }
    }
  }
  if (failed) sleep_at_least_ns(100000);  // copies in flight land before the CTA's shared memory goes
}

}  // namespace mla
