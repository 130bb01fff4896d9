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
  int n_kv;
  const uint16_t* mask;      // f16 bits [seq][n_q][cells], or nullptr (all cells 0)
  int64_t mask_seq_stride;   // elements
  int64_t mask_row_stride;   // elements
  int n_q;
  uint16_t* rows;            // f16 [seq][cap][head width]: the gathered rows
  uint16_t* gmask;           // f16 [seq][n_q][gmask_stride]: their mask values
  int64_t cap;               // rows per sequence in `rows`
  int64_t gmask_stride;      // >= cap
};

// Grid (blocks, sequences of the launch); 256 threads. A warp takes kRows positions at a
// time: it reads their indices, then their rows with coalesced loads (lane l takes the
// row's words l, l+32, ...), all in flight together. f16 rows are written out as read;
// q8_0 rows go through the warp's shared-memory stage, from which 18 lanes each
// dequantise one 32-value block per row. kMode: kModeQ8 (612-byte q8_0 rows) or
// kModeGatherF16 (f16 rows of 64 * kNC values); kNC: 64-column chunks of the head width.
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
  constexpr int kQ8PerLane = (kQ8Words + 31) / 32;
  constexpr int kF16Vec = kWidth / 8;                   // 16-byte chunks of an f16 row
  constexpr int kF16PerLane = (kF16Vec + 31) / 32;
  constexpr int kBlocks = kQ8RowBytes / 34;             // q8_0 blocks of a row (18)
  __shared__ uint32_t stage[kQ8 ? 8 * kRows * kQ8Words : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int b_abs = plan.seq_offset + b;
  const int len = min(max(__ldg(g.idx_count + b_abs), 0), plan.kv_len[b]);
  const int pad_end = (int)min(g.cap, ((int64_t)len + 127) / 128 * 128);
  const int32_t* idx_row = g.idx + (int64_t)b_abs * g.idx_seq_stride;
  const uint8_t* cache_seq = g.kcache + (int64_t)b_abs * g.k_seq_stride * kRowBytes;
  uint16_t* out_seq = g.rows + (int64_t)b_abs * g.cap * kWidth;
  const int n_warps = gridDim.x * 8;
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
    if constexpr (kQ8) {
      uint32_t wv[kRows][kQ8PerLane];
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(cache_seq + (int64_t)max(key[u], 0) * kRowBytes);
#pragma unroll
        for (int j = 0; j < kQ8PerLane; ++j) {
          const int w = lane + 32 * j;
          wv[u][j] = (key[u] >= 0 && w < kQ8Words) ? __ldg(src + w) : 0u;
        }
      }
      uint32_t* sw = stage + warp * kRows * kQ8Words;
#pragma unroll
      for (int u = 0; u < kRows; ++u)
#pragma unroll
        for (int j = 0; j < kQ8PerLane; ++j)
          if (lane + 32 * j < kQ8Words) sw[u * kQ8Words + lane + 32 * j] = wv[u][j];
      __syncwarp();
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int pos = r0 + u;
        if (lane < kBlocks && pos < pad_end) {
          // block `lane` starts at byte 34 lane of the row: word 17 lane / 2, 2 bytes in
          // for an odd block; its 9 words stay inside the staged row
          RawBlock<kModeQ8> rb;
          rb.valid = key[u] >= 0;
          rb.odd = (lane & 1) != 0;
          const uint32_t* src = sw + u * kQ8Words + ((17 * lane) >> 1);
#pragma unroll
          for (int i = 0; i < 9; ++i) rb.w[i] = src[i];
          uint32_t h[16];
          block_values<kModeQ8>(rb, h);  // zeros for an invalid index and past the list
          uint4* dst = reinterpret_cast<uint4*>(out_seq + (int64_t)pos * kWidth + 32 * lane);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
      }
      __syncwarp();  // the stage is read before the next positions overwrite it
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
    // the positions' mask values, one query token per lane
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int pos = r0 + u;
      if (pos >= len) continue;
      for (int t = lane; t < g.n_q; t += 32) {
        uint16_t mv = 0xFC00u;  // -inf: an invalid index drops out
        if (key[u] >= 0)
          mv = g.mask != nullptr
                   ? __ldg(g.mask + (int64_t)b_abs * g.mask_seq_stride + (int64_t)t * g.mask_row_stride + key[u])
                   : (uint16_t)0;
        g.gmask[((int64_t)b_abs * g.n_q + t) * g.gmask_stride + pos] = mv;
      }
    }
  }
}

}  // namespace mla
