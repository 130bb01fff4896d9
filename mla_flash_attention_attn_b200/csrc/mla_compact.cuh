// Single-pass compaction of an f16 mask row into the ascending list of kept
// cell indices (llama.cpp b11413 release note, "single-scan sparse FA index
// compaction": contiguous segments, a count per segment, one scan over the
// counts giving each segment its output offset; the list stays ascending).
//
// Mapping: a thread's segment is 8 consecutive cells (one 16-byte load); a CTA covers
// 256 segments = 2048 cells, so a row of 131072 cells is read by 64 CTAs on as many SMs
// (8 CTAs of 16384 cells left the row's latency on a few SMs). The scan over segment
// counts is done in one pass: warp shuffle scan, then a scan of the 8 warp totals, then
// a decoupled look-back across CTAs (one warp reads 32 predecessor flags per round trip,
// so the last tile of such a row needs two). CTAs take their tile in ticket order
// (atomicAdd), so every tile a CTA waits on belongs to a CTA that is already
// running; each wait is bounded and reports MLA_ERR_TIMEOUT instead of hanging.
// Look-back flags carry a per-call epoch, so stale flags from an earlier call
// read as "not ready" and the flag array needs no clearing between calls.
#pragma once
#include <cuda_fp16.h>

#include "mla_common.cuh"
#include "mla_fwd.cuh"

namespace mla {

namespace compact {
constexpr int kThreads = 256;
constexpr int kCellsPerThread = 8;
constexpr int kTileCells = kThreads * kCellsPerThread;  // 2048
constexpr uint32_t kStateAggregate = 1;
constexpr uint32_t kStateInclusive = 2;
constexpr uint16_t kNegInfBits = 0xFC00;
}  // namespace compact

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// One tile of one row: keep bits of the tile's cells from keep_of(cell0, n) (bit k:
// cell cell0 + k kept, n cells of the segment in range), then the scan, the look-back
// and the ascending writes. Workspace per row: one ticket counter (int) and n_tiles
// look-back flags (u64 = tag<<32 | value, tag = epoch*4 + state).
template <class KeepOf>
__device__ __forceinline__ void compact_row_tile(int row, int n_tiles, int n_cells, KeepOf keep_of,
                                                 int32_t* __restrict__ idx_out, int64_t idx_row_stride,
                                                 int32_t* __restrict__ count_out, int* __restrict__ tickets,
                                                 unsigned long long* __restrict__ flags, uint32_t epoch,
                                                 uint64_t timeout_ns) {
  using namespace compact;
  __shared__ int s_tile;
  __shared__ int s_warp_tot[kThreads / 32];
  __shared__ int s_excl;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_tile = atomicAdd(&tickets[row], 1);
  // the kernel that follows may start its setup now; it waits for this grid to
  // complete before it reads the index lists
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __syncthreads();
  const int tile = s_tile;
  const int64_t cell0 = (int64_t)tile * kTileCells + (int64_t)tid * kCellsPerThread;

  // keep bits of this thread's cells
  static_assert(kCellsPerThread == 8, "one 16-byte load per segment");
  const int64_t left = (int64_t)n_cells - cell0;
  const int n_in = left <= 0 ? 0 : (left < kCellsPerThread ? (int)left : kCellsPerThread);
  const uint32_t keep = n_in > 0 ? keep_of(cell0, n_in) : 0u;
  const int cnt = __popc(keep);

  // warp inclusive scan of the segment counts
  int inc = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += y;
  }
  if (lane == 31) s_warp_tot[warp] = inc;
  __syncthreads();

  unsigned long long* rflags = flags + (int64_t)row * n_tiles;
  if (warp == 0) {
    int wt = lane < kThreads / 32 ? s_warp_tot[lane] : 0;
    int winc = wt;
#pragma unroll
    for (int d = 1; d < kThreads / 32; d <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, winc, d);
      if (lane >= d) winc += y;
    }
    if (lane < kThreads / 32) s_warp_tot[lane] = winc - wt;  // exclusive offsets of warps
    const int agg = __shfl_sync(0xffffffffu, winc, kThreads / 32 - 1);
    const uint32_t tag_agg = epoch * 4u + kStateAggregate;
    const uint32_t tag_inc = epoch * 4u + kStateInclusive;
    int excl = 0;
    if (tile == 0) {
      if (lane == 0) st_release_u64(&rflags[0], ((unsigned long long)tag_inc << 32) | (uint32_t)agg);
    } else {
      if (lane == 0) st_release_u64(&rflags[tile], ((unsigned long long)tag_agg << 32) | (uint32_t)agg);
      // Warp-wide look-back: lane l inspects tile (top - l); a window of 32
      // predecessors costs one round trip. Sum aggregates down to the nearest
      // inclusive prefix; tiles before 0 count as an inclusive prefix of 0.
      int top = tile - 1;
      bool timed_out = false;
      uint64_t t0 = 0;
      while (true) {
        const int j = top - lane;
        uint32_t state = kStateInclusive, val = 0;
        if (j >= 0) {
          const unsigned long long f = ld_acquire_u64(&rflags[j]);
          const uint32_t tag = (uint32_t)(f >> 32);
          state = tag == tag_inc ? kStateInclusive : (tag == tag_agg ? kStateAggregate : 0u);
          val = (uint32_t)f;
        }
        const uint32_t inc_mask = __ballot_sync(0xffffffffu, state == kStateInclusive);
        const uint32_t wait_mask = __ballot_sync(0xffffffffu, state == 0u);
        const int first_inc = inc_mask ? __ffs(inc_mask) - 1 : 32;
        const uint32_t upto = first_inc >= 31 ? 0xffffffffu : ((2u << first_inc) - 1u);
        if (wait_mask & upto) {  // a needed predecessor has not published yet
          if (t0 == 0) t0 = globaltimer_ns();
          if (globaltimer_ns() - t0 > timeout_ns) {
            timed_out = true;
            break;
          }
          continue;
        }
        int part = (lane <= first_inc) ? (int)val : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        excl += part;
        if (first_inc < 32) break;
        top -= 32;
        t0 = 0;
      }
      if (timed_out && lane == 0) record_status(kStatusTimeout);
      if (lane == 0)
        st_release_u64(&rflags[tile], ((unsigned long long)tag_inc << 32) | (uint32_t)(excl + agg));
    }
    if (lane == 0) {
      s_excl = excl;
      if (tile == n_tiles - 1) {
        count_out[row] = excl + agg;
        tickets[row] = 0;  // every CTA of this row has drawn its ticket
      }
    }
  }
  __syncthreads();

  // ascending writes: tile offset + warp offset + offset within the warp
  int pos = s_excl + s_warp_tot[warp] + (inc - cnt);
  int32_t* orow = idx_out + (int64_t)row * idx_row_stride;
  for (int k = 0; k < kCellsPerThread; ++k)
    if (keep & (1u << k)) orow[pos++] = (int32_t)(cell0 + k);
}

// Keep bits of n cells from cell0 of an f16 mask row: one 16-byte load when the 8 cells
// are whole and aligned, else cell by cell.
__device__ __forceinline__ uint32_t keep_bits(const uint16_t* mrow, int64_t cell0, int n) {
  using namespace compact;
  uint32_t keep = 0;
  if (n == kCellsPerThread && ((reinterpret_cast<uintptr_t>(mrow + cell0) & 15) == 0)) {
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(mrow + cell0));
    const uint32_t w[4] = {v0.x, v0.y, v0.z, v0.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      keep |= (uint32_t)((w[h] & 0xFFFFu) != kNegInfBits) << (2 * h);
      keep |= (uint32_t)((w[h] >> 16) != kNegInfBits) << (2 * h + 1);
    }
  } else {
    for (int k = 0; k < n; ++k)
      if (__ldg(mrow + cell0 + k) != kNegInfBits) keep |= 1u << k;
  }
  return keep;
}

// Grid: (tiles_per_row, n_rows): the kept cells of each mask row.
__global__ void __launch_bounds__(compact::kThreads)
    mla_compact_kernel(const uint16_t* __restrict__ mask, int64_t mask_row_stride, int n_kv,
                       int32_t* __restrict__ idx_out, int64_t idx_row_stride,
                       int32_t* __restrict__ count_out, int* __restrict__ tickets,
                       unsigned long long* __restrict__ flags, uint32_t epoch,
                       uint64_t timeout_ns) {
  const int row = blockIdx.y;
  const uint16_t* mrow = mask + (int64_t)row * mask_row_stride;
  compact_row_tile(
      row, gridDim.x, n_kv, [&](int64_t cell0, int n) { return keep_bits(mrow, cell0, n); }, idx_out,
      idx_row_stride, count_out, tickets, flags, epoch, timeout_ns);
}

// Grid: (tiles of the longest sequence, sequences of the launch): the cells of sequence
// b's first plan.kv_len[b] that any of its n_q query tokens keeps (the union of the
// token rows' masks), as one list per sequence. A programmatic dependent of the kernel
// before it.
__global__ void __launch_bounds__(compact::kThreads)
    mla_compact_union_kernel(const __grid_constant__ Plan plan, const uint16_t* __restrict__ mask,
                             int64_t mask_seq_stride, int64_t mask_row_stride,
                             int32_t* __restrict__ idx_out, int64_t idx_row_stride,
                             int32_t* __restrict__ count_out, int* __restrict__ tickets,
                             unsigned long long* __restrict__ flags, uint32_t epoch,
                             uint64_t timeout_ns) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.y;
  const uint16_t* mseq = mask + (int64_t)(plan.seq_offset + b) * mask_seq_stride;
  const int n_q = plan.n_q;
  compact_row_tile(
      b, gridDim.x, plan.kv_len[b],
      [&](int64_t cell0, int n) {
        uint32_t keep = 0;
        for (int t = 0; t < n_q; ++t) keep |= keep_bits(mseq + (int64_t)t * mask_row_stride, cell0, n);
        return keep;
      },
      idx_out + (int64_t)plan.seq_offset * idx_row_stride, idx_row_stride, count_out + plan.seq_offset,
      tickets, flags, epoch, timeout_ns);
}

}  // namespace mla
