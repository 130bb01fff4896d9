// Gather of an index list's cache rows into a dense f16 buffer, for the TMA-mode
// attention kernel (Vulkan FA for DeepSeek MLA article, section 2.2: the sparse pass
// attends only to the cells an index list keeps; llama.cpp b11413 release note: the
// list comes from the mask by compaction).
//
// A sequence attends to the cache rows idx[0..len) (len = min(idx_count, the length
// planned for it)). The attention kernel's gather modes fetch those rows one 32-value
// block at a time from a few producer warps per SM, so a step waits on chains of
// dependent loads. Here every SM gathers at once: item (position, block) reads one
// block of the row at idx[position] (q8_0: 34 bytes, dequantised to 32 f16 values d*q
// exactly as the attention kernel's producers do; f16: 64 bytes) and writes it to row
// `position` of the dense buffer, and the first block of a position also writes the
// position's mask value of every query token. The attention kernel then streams the
// dense rows with TMA, in list order, with the gathered mask.
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

// Grid (blocks, sequences of the launch); 256 threads; each thread takes kBatch items per
// round, their loads issued together. kMode: kModeQ8 (612-byte q8_0 rows) or kModeGatherF16
// (f16 rows of 64 * kNC values); kNC: 64-column chunks of the head width.
template <int kMode, int kNC>
__global__ void __launch_bounds__(256)
    mla_gather_rows_kernel(const __grid_constant__ Plan plan, const __grid_constant__ GatherParams g) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the index lists are written by the kernel before
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int kBlocks = 2 * kNC;                       // 32-value blocks of a row
  constexpr int kRowBytes = kMode == kModeQ8 ? kQ8RowBytes : 128 * kNC;
  constexpr int kWidth = 64 * kNC;                       // f16 values of a gathered row
  constexpr int kBatch = 4;
  const int b = blockIdx.y;
  const int b_abs = plan.seq_offset + b;
  const int len = min(max(__ldg(g.idx_count + b_abs), 0), plan.kv_len[b]);
  const int64_t pad_end = min(g.cap, ((int64_t)len + 127) / 128 * 128);
  const int64_t n_items = (int64_t)len * kBlocks;
  const int64_t n_all = pad_end * kBlocks;
  const int32_t* idx_row = g.idx + (int64_t)b_abs * g.idx_seq_stride;
  const int64_t seq_row0 = (int64_t)b_abs * g.k_seq_stride;
  uint16_t* out_seq = g.rows + (int64_t)b_abs * g.cap * kWidth;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n_all; i0 += kBatch * stride) {
    RawBlock<kMode> rb[kBatch];
    int key[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t it = i0 + u * stride;
      key[u] = -1;
      rb[u].valid = false;
      rb[u].odd = false;
      if (it < n_items) {
        const int pos = (int)(it / kBlocks);
        const int k = __ldg(idx_row + pos);
        if (k >= 0 && k < g.n_kv) {
          key[u] = k;
          rb[u].valid = true;
          load_block<kMode, kRowBytes>(g.kcache, seq_row0 + k, (int)(it - (int64_t)pos * kBlocks), rb[u]);
        } else {
          record_status(kStatusIndex);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t it = i0 + u * stride;
      if (it >= n_all) continue;
      const int64_t pos = it / kBlocks;
      const int blk = (int)(it - pos * kBlocks);
      uint32_t h[16];
      block_values<kMode>(rb[u], h);  // zeros for an invalid index and past len
      uint4* dst = reinterpret_cast<uint4*>(out_seq + pos * kWidth + 32 * blk);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
      if (blk == 0 && it < n_items) {
        for (int t = 0; t < g.n_q; ++t) {
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
}

}  // namespace mla
