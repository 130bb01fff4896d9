// Flash attention with a K and a V per KV head: the DK = 192 / DV = 128 head shape (one of
// the head shapes the llama.cpp tag page lists for the Metal FA kernel, PR #29570), read as
// the non-absorbed MLA head. Query head h reads KV head h / group (group = n_head /
// n_kv_head; group = 1 is multi-head attention), and per query row
//   S = scale * q . k_j + mask_j,   o = sum_j softmax(S)_j v_j
// tile by tile with a running max and sum (Vulkan FA for DeepSeek MLA article, sections
// 2.1-2.2), the scores never leaving the SM.
//
// One CTA per work unit = (sequence, KV head, 128 rows, KV split). The rows of a KV head
// are its group's (token, head) pairs, row rho = t * group + hg for query head
// kvh * group + hg, so the query heads of a group share every K and V tile it loads.
// Hardware mapping (one SM, tcgen05 cta_group::1, M = 128):
//  * Q: the unit's 128 rows x 192 columns, staged in shared memory by the softmax warps
//    (three 64-column chunks, 128-byte swizzle), resident for the whole unit.
//  * Q.K^T: N = 128 keys per tile, 3 chunks x 4 MMAs of K = 16; K chunks {128 keys x 64
//    columns} arrive by TMA through a ring of stages.
//  * P.V: N = 128 value columns, K = 16 keys per MMA; A (P) from TMEM, B (V) from V stages
//    {64 keys x 128 columns} loaded by TMA from the V tensor.
//  * TMEM (cta_group::1, M = 128: lane = row): S 128 columns, P 64 columns (f16 pairs), O
//    128 columns. Each lane holds its whole row.
//  * Two softmax warpgroups share each tile: warpgroup w takes keys [64w, 64w+64) of
//    every row (S columns, P columns, and O columns [64w, 64w+64) for the rescale and the
//    epilogue); the two swap their row maxima through shared memory, so both raise the
//    reference max at the same tiles, and their row sums add up at the end.
//  * The softmax frees S as soon as the scores are in registers, so Q.K^T of the next
//    tile overlaps it; P is written once P.V of the previous tile has completed.
// Every wait is bounded (params.timeout_ns); a timeout records MLA_ERR_TIMEOUT and the
// thread stops issuing, as in the MLA kernel.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>

#include "mla_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {

namespace heads {

constexpr int kHeadDK = 192;
constexpr int kHeadDV = 128;
constexpr int kRows = 128;            // M: rows of a unit
constexpr int kTile = 128;            // N of Q.K^T: keys per tile
constexpr int kChunks = kHeadDK / 64;     // 64-column chunks of a K row
constexpr int kKStages = 4;
constexpr int kVStages = 4;
constexpr int kChunkBytes = 16384;    // 128 rows (or keys) x 64 columns f16
constexpr int kVStageBytes = 16384;   // 64 keys x 128 value columns f16
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kChunks * kChunkBytes;
constexpr int kOffV = kOffK + kKStages * kChunkBytes;
constexpr int kOffBar = kOffV + kVStages * kVStageBytes;
constexpr int kBarBytes = 8 * (2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 1);
constexpr int kOffTmemSlot = kOffBar + kBarBytes;
constexpr int kOffXmax = kOffTmemSlot + 16;                 // float[2 tile parities][2 warpgroups][128]
constexpr int kOffXl = kOffXmax + 2 * 2 * kRows * 4;        // float[2 warpgroups][128]
constexpr int kSmemBytes = kOffXl + 2 * kRows * 4;
constexpr int kSmemAlloc = kSmemBytes + 1024;
constexpr int kThreads = 384;        // roles in warps 0-3, two softmax warpgroups
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemP = 128;
constexpr uint32_t kTmemO = 256;
constexpr float kRescaleThreshold = 5.5451774f;  // 8 ln 2
constexpr int kPlanMaxSeq = 128;
static_assert(kSmemAlloc <= 232448, "shared memory beyond the 227 KB per-CTA limit");
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0, "128-byte swizzle needs 1 KB alignment");

constexpr uint32_t kIdescQK = idesc_f16_f32(128, kTile, 0, 0);  // A, B K-major
constexpr uint32_t kIdescPV = idesc_f16_f32(128, kHeadDV, 0, 1);    // A (P, TMEM), B (V) MN-major

struct Bars {
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t v_full[kVStages];
  uint64_t v_empty[kVStages];
  uint64_t s_full;
  uint64_t s_free;      // 8 softmax warps
  uint64_t p_full[2];   // 8 softmax warps
  uint64_t o_done[2];
  uint64_t q_full;      // 4 softmax warps: Q staged in shared memory
};
static_assert(sizeof(Bars) == kBarBytes, "barrier block size");

// How one launch divides its sequences: a unit is (sequence, KV head, 128-row group, split).
struct Plan {
  int n_seq, seq_offset;
  int n_q, n_head, n_kv_head, group;  // group = n_head / n_kv_head
  int rows;                           // rows of one KV head: n_q * group
  int groups;                         // 128-row groups of one KV head
  int n_kv;
  int total_units;
  int unit_base[kPlanMaxSeq + 1];     // first unit of each sequence
  int n_split[kPlanMaxSeq];
  int kv_len[kPlanMaxSeq];
  int ws_base[kPlanMaxSeq];           // first partial slot (-1: direct output)
};

struct Params {
  const uint16_t* q;       // f16
  const uint16_t* mask;    // f16 bits or nullptr
  float* out;              // fp32
  float* ws_o;             // fp32 [slot][128 rows][128] split partials (O_s / l_s)
  float* ws_lse;           // fp32 [slot][128] log2-sum-exp of each partial
  int64_t q_seq_stride, mask_seq_stride, mask_row_stride, out_seq_stride;  // elements
  float scale;
  int mask_vec_ok;
  uint64_t timeout_ns;
};

// unit -> (sequence in launch, KV head, group, split)
__device__ __forceinline__ void decode(const Plan& plan, int unit, int& b, int& kvh, int& g, int& s) {
  int lo = 0, hi = plan.n_seq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (plan.unit_base[mid] <= unit) lo = mid; else hi = mid - 1;
  }
  b = lo;
  int local = unit - plan.unit_base[b];
  const int ns = plan.n_split[b];
  s = local % ns;
  local /= ns;
  g = local % plan.groups;
  kvh = local / plan.groups;
}

}  // namespace heads

__global__ void __launch_bounds__(heads::kThreads, 1)
    mla_heads_fwd_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ heads::Plan plan, const __grid_constant__ heads::Params p) {
  using namespace heads;
  extern __shared__ uint8_t smem_raw[];
  if (dynamic_smem_bytes() < (uint32_t)kSmemAlloc) {
    if (threadIdx.x == 0) record_status(kStatusLaunch);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;
  Bars& bars = *reinterpret_cast<Bars*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmemSlot);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t to = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars.k_full[i], 1);
      mbar_init(&bars.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bars.v_full[i], 1);
      mbar_init(&bars.v_empty[i], 1);
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.s_free, 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.p_full[i], 8);
      mbar_init(&bars.o_done[i], 1);
    }
    mbar_init(&bars.q_full, 4);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) tmem_alloc_1sm(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");

  int b, kvh, g, s;
  decode(plan, blockIdx.x, b, kvh, g, s);
  const int b_abs = plan.seq_offset + b;
  const int n_split = plan.n_split[b];
  const int len = plan.kv_len[b];
  const int n_tiles_total = (len + kTile - 1) / kTile;
  const int tile_begin = (int)((int64_t)s * n_tiles_total / n_split);
  const int tile_end = (int)((int64_t)(s + 1) * n_tiles_total / n_split);
  const int n_tiles = tile_end - tile_begin;
  const int key_end = min(len, tile_end * kTile);
  bool failed = false;

  if (warp == 0) {
    // ================= K producer: 3 chunks of 64 columns per 128-key tile
    if (n_tiles > 0 && elect_one()) {
      int stage = 0;
      uint32_t ph = 0;
      for (int i = 0; i < n_tiles && !failed; ++i)
        for (int c = 0; c < kChunks; ++c) {
          if (!mbar_wait(&bars.k_empty[stage], ph ^ 1, to)) {
            failed = true;
            record_status(kStatusTimeout);
            break;
          }
          mbar_arrive_expect_tx(&bars.k_full[stage], kChunkBytes);
          tma_load_4d(sK + stage * kChunkBytes, &tm_k, &bars.k_full[stage], 64 * c, kvh,
                      (tile_begin + i) * kTile, b_abs);
          if (++stage == kKStages) { stage = 0; ph ^= 1; }
        }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ================= V producer: 2 stages of 64 keys x 128 value columns per tile
    if (n_tiles > 0 && elect_one()) {
      int stage = 0;
      uint32_t ph = 0;
      for (int i = 0; i < n_tiles && !failed; ++i)
        for (int h = 0; h < kTile / 64; ++h) {
          if (!mbar_wait(&bars.v_empty[stage], ph ^ 1, to)) {
            failed = true;
            record_status(kStatusTimeout);
            break;
          }
          mbar_arrive_expect_tx(&bars.v_full[stage], kVStageBytes);
          // one box {64 columns, 64 keys, 2 column blocks}: lands as [block][key][64]
          tma_load_5d(sV + stage * kVStageBytes, &tm_v, &bars.v_full[stage], 0,
                      (tile_begin + i) * kTile + 64 * h, 0, kvh, b_abs);
          if (++stage == kVStages) { stage = 0; ph ^= 1; }
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================= Q.K^T issuer
    if (n_tiles > 0 && elect_one()) {
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      int kst = 0;
      uint32_t kph = 0;
      if (!mbar_wait(&bars.q_full, 0, to)) {
        failed = true;
        record_status(kStatusTimeout);
      }
      for (int t = 0; t < n_tiles && !failed; ++t) {
        if (t >= 1 && !mbar_wait(&bars.s_free, (t - 1) & 1, to)) {
          failed = true;
          record_status(kStatusTimeout);
          break;
        }
        for (int c = 0; c < kChunks; ++c) {
          if (!mbar_wait(&bars.k_full[kst], kph, to)) {
            failed = true;
            record_status(kStatusTimeout);
            break;
          }
          tc_fence_after();
          const uint64_t a0 = dq + (uint32_t)(c * (kChunkBytes >> 4));
          const uint64_t b0 = dk + (uint32_t)(kst * (kChunkBytes >> 4));
          mma_f16_ss_1sm(tmem + kTmemS, a0, b0, kIdescQK, c ? 1u : 0u);
          mma_f16_ss_1sm(tmem + kTmemS, a0 + 2, b0 + 2, kIdescQK, 1u);
          mma_f16_ss_1sm(tmem + kTmemS, a0 + 4, b0 + 4, kIdescQK, 1u);
          mma_f16_ss_1sm(tmem + kTmemS, a0 + 6, b0 + 6, kIdescQK, 1u);
          mma_commit_1sm(&bars.k_empty[kst]);
          if (++kst == kKStages) { kst = 0; kph ^= 1; }
        }
        if (failed) break;
        mma_commit_1sm(&bars.s_full);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ================= P.V issuer: A (P) from TMEM, 16 keys per MMA = 8 columns of P
    if (n_tiles > 0 && elect_one()) {
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), 8192, 1024);
      int vst = 0;
      uint32_t vph = 0;
      for (int t = 0; t < n_tiles && !failed; ++t) {
        if (!mbar_wait(&bars.p_full[t & 1], (t >> 1) & 1, to)) {
          failed = true;
          record_status(kStatusTimeout);
          break;
        }
        for (int h = 0; h < kTile / 64; ++h) {
          if (!mbar_wait(&bars.v_full[vst], vph, to)) {
            failed = true;
            record_status(kStatusTimeout);
            break;
          }
          tc_fence_after();
          const uint32_t a0 = tmem + kTmemP + 32u * (uint32_t)h;
          const uint64_t b0 = dv + (uint32_t)(vst * (kVStageBytes >> 4));
          mma_f16_ts_1sm(tmem + kTmemO, a0, b0, kIdescPV, (t > 0 || h > 0) ? 1u : 0u);
          mma_f16_ts_1sm(tmem + kTmemO, a0 + 8, b0 + 128, kIdescPV, 1u);
          mma_f16_ts_1sm(tmem + kTmemO, a0 + 16, b0 + 256, kIdescPV, 1u);
          mma_f16_ts_1sm(tmem + kTmemO, a0 + 24, b0 + 384, kIdescPV, 1u);
          mma_commit_1sm(&bars.v_empty[vst]);
          if (++vst == kVStages) { vst = 0; vph ^= 1; }
        }
        if (failed) break;
        mma_commit_1sm(&bars.o_done[t & 1]);
      }
    }
    __syncwarp();
  } else {
    // ================= softmax / correction / epilogue warpgroups: thread = TMEM lane = row;
    // warpgroup kw takes keys [64 kw, 64 kw + 64) of each tile
    const int kw = warp >= 8 ? 1 : 0;
    const int r = (threadIdx.x - 128) & 127;
    float* xmax = reinterpret_cast<float*>(smem + kOffXmax);
    float* xl = reinterpret_cast<float*>(smem + kOffXl);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int rho = g * kRows + r;                  // row within the KV head
    const bool row_valid = rho < plan.rows;
    const int tok = row_valid ? rho / plan.group : 0;
    const int head = kvh * plan.group + (row_valid ? rho % plan.group : 0);
    const uint16_t* mrow = (p.mask != nullptr && row_valid)
                               ? p.mask + (int64_t)b_abs * p.mask_seq_stride + (int64_t)tok * p.mask_row_stride
                               : nullptr;
    auto wait_local = [&](uint64_t* bar, uint32_t parity) {
      bool ok = failed ? true : mbar_wait(bar, parity, to);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && !failed) {
        failed = true;
        if (lane == 0) record_status(kStatusTimeout);
      }
    };
    if (n_tiles > 0 && kw == 0) {
      // this row of Q into the three swizzled chunks (rows past the unit's rows: zeros)
      const uint4* qsrc = reinterpret_cast<const uint4*>(
          p.q + (int64_t)b_abs * p.q_seq_stride + ((int64_t)tok * plan.n_head + head) * kHeadDK);
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 v = row_valid ? __ldg(qsrc + 8 * c + j) : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(sQ + c * kChunkBytes + r * 128 + ((j ^ (r & 7)) << 4)) = v;
        }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.q_full);
    }
    float m_ref = -INFINITY;
    float l_sum = 0.f;
    const bool vec_ok = mrow == nullptr || p.mask_vec_ok;
    constexpr int kKeys = kTile / 2;  // keys of a tile per warpgroup
    // The mask of a tile (each row its own token's) is loaded into registers during the
    // previous tile, once that tile's mask is used, and brought into L2 kMaskAhead tiles ahead,
    // so that its latency stays off the softmax's path (half tiles inside the mask row
    // take this path; a ragged half tile goes key by key).
    constexpr int kMaskAhead = 4;
    auto half_key0 = [&](int t) { return (tile_begin + t) * kTile + kKeys * kw; };
    auto vec_half = [&](int t) { return vec_ok && half_key0(t) + kKeys <= key_end; };
    auto prefetch_mask = [&](int t) {
      if (mrow != nullptr && half_key0(t) + kKeys <= plan.n_kv) {
        prefetch_l2(mrow + half_key0(t));
        prefetch_l2(reinterpret_cast<const uint8_t*>(mrow + half_key0(t)) + 2 * kKeys - 2);  // its last cell
      }
    };
    uint4 mvec[kKeys / 8];
    auto load_mask = [&](int t) {
#pragma unroll
      for (int c = 0; c < kKeys / 8; ++c)
        mvec[c] = mrow ? __ldg(reinterpret_cast<const uint4*>(mrow + half_key0(t)) + c) : make_uint4(0u, 0u, 0u, 0u);
    };
    for (int t = 0; t < kMaskAhead && t < n_tiles; ++t) prefetch_mask(t);
    bool vec_next = n_tiles > 0 && vec_half(0);
    if (vec_next) load_mask(0);
    for (int i = 0; i < n_tiles; ++i) {
      const int key0 = half_key0(i);  // this warpgroup's first key
      const bool vec_mask = vec_next;
      wait_local(&bars.s_full, i & 1);
      tc_fence_after();
      uint32_t sr[kKeys];
#pragma unroll
      for (int q = 0; q < kKeys / 32; ++q)
        tmem_ld32(tmem + lane_base + kTmemS + kKeys * kw + 32 * q,
                  *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * q));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free);
      float x[kKeys];
      if (vec_mask) {
        // whole half tile: the mask loaded during the previous tile (zeros without a mask)
#pragma unroll
        for (int c = 0; c < kKeys / 8; ++c) {
          const uint4 mv = mvec[c];
          const uint32_t w[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[h]));
            x[8 * c + 2 * h] = fmaf(__uint_as_float(sr[8 * c + 2 * h]), p.scale, f.x);
            x[8 * c + 2 * h + 1] = fmaf(__uint_as_float(sr[8 * c + 2 * h + 1]), p.scale, f.y);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < kKeys; ++j) {
          const int key = key0 + j;
          float mv = 0.f;
          if (mrow != nullptr && key < key_end) mv = __half2float(__ushort_as_half(__ldg(mrow + key)));
          x[j] = key < key_end ? fmaf(__uint_as_float(sr[j]), p.scale, mv) : -INFINITY;
        }
      }
      // next tile's mask, as soon as this tile's is used: the load has the rest of the
      // tile to land
      vec_next = i + 1 < n_tiles && vec_half(i + 1);
      if (vec_next) load_mask(i + 1);
      if (i + kMaskAhead < n_tiles) prefetch_mask(i + kMaskAhead);
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) m8[u] = x[u];
#pragma unroll
      for (int j = 8; j < kKeys; ++j) m8[j & 7] = fmaxf(m8[j & 7], x[j]);
      float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      // the row's max over the whole tile: swap halves with the other warpgroup (a slot
      // per tile parity: the other warpgroup may write the next tile's before this one
      // reads)
      xmax[((i & 1) * 2 + kw) * kRows + r] = mt;
      named_bar_sync(1, 256);
      mt = fmaxf(mt, xmax[((i & 1) * 2 + (kw ^ 1)) * kRows + r]);
      const bool need = mt > m_ref + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx((m_ref - mt) * kLog2e);  // 0 when m_ref = -inf
        m_ref = mt;
      }
      const float nb = (m_ref == -INFINITY) ? 0.f : -m_ref * kLog2e;
      uint32_t pk[kKeys / 2];
      float ls8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ls8[u] = 0.f;
#pragma unroll
      for (int j = 0; j < kKeys / 2; ++j) {
        const float e0 = ex2_approx(fmaf(x[2 * j], kLog2e, nb));
        const float e1 = ex2_approx(fmaf(x[2 * j + 1], kLog2e, nb));
        __half2 h2 = __floats2half2_rn(e0, e1);
        pk[j] = *reinterpret_cast<uint32_t*>(&h2);
        ls8[j & 7] += e0 + e1;
      }
      l_sum = l_sum * alpha +
              (((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7])));
      // P (and O) are free once P.V of the previous tile has completed
      if (i > 0) wait_local(&bars.o_done[(i - 1) & 1], ((i - 1) >> 1) & 1);
      tc_fence_after();
      tmem_st32(tmem + lane_base + kTmemP + (kKeys / 2) * kw, *reinterpret_cast<uint32_t(*)[32]>(pk));
      if (__any_sync(0xffffffffu, need && i > 0)) {
        // this warpgroup's half of the row's O columns
#pragma unroll 1
        for (int cc = 2 * kw; cc < 2 * kw + 2; ++cc) {
          uint32_t v[32];
          const uint32_t a = tmem + lane_base + kTmemO + cc * 32;
          tmem_ld32(a, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
          tmem_st32(a, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[i & 1]);
    }
    // ---- epilogue: O / l to the output row, or a split partial and its lse; each
    // warpgroup writes its half of the row's columns
    if (n_tiles > 0) wait_local(&bars.o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    tc_fence_after();
    xl[kw * kRows + r] = l_sum;
    named_bar_sync(1, 256);
    const float l_tot = xl[r] + xl[kRows + r];
    const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
    const int slot = plan.ws_base[b] >= 0 ? plan.ws_base[b] + (kvh * plan.groups + g) * n_split + s : -1;
    float4* dst = nullptr;
    if (row_valid)
      dst = slot >= 0 ? reinterpret_cast<float4*>(p.ws_o + ((int64_t)slot * kRows + r) * kHeadDV)
                      : reinterpret_cast<float4*>(p.out + (int64_t)b_abs * p.out_seq_stride +
                                                  ((int64_t)tok * plan.n_head + head) * kHeadDV);
#pragma unroll 1
    for (int cc = 2 * kw; cc < 2 * kw + 2; ++cc) {
      uint32_t v[32];
      if (n_tiles > 0) {
        tmem_ld32(tmem + lane_base + kTmemO + cc * 32, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      }
      if (dst != nullptr) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[8 * cc + j] = make_float4(__uint_as_float(v[4 * j]) * inv_l, __uint_as_float(v[4 * j + 1]) * inv_l,
                                        __uint_as_float(v[4 * j + 2]) * inv_l, __uint_as_float(v[4 * j + 3]) * inv_l);
      }
    }
    if (kw == 0 && slot >= 0 && row_valid)
      p.ws_lse[(int64_t)slot * kRows + r] = l_tot > 0.f ? m_ref * kLog2e + __log2f(l_tot) : -INFINITY;
  }

  if (failed) sleep_at_least_ns(100000);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_1sm(tmem, kTmemCols);
  }
}

// LSE combine of the split partials of the 192 / 128 head shape: one warp per row, lane l
// owning value columns 4l..4l+3; O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M).
// Launched as a programmatic dependent of the forward kernel.
__global__ void __launch_bounds__(128)
    mla_heads_combine_kernel(const __grid_constant__ heads::Plan plan, const float* __restrict__ ws_o,
                             const float* __restrict__ ws_lse, float* __restrict__ out,
                             int64_t out_seq_stride) {
  using namespace heads;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.y;
  const int rid = blockIdx.x * 4 + (threadIdx.x >> 5);  // row of this sequence: kvh * rows + rho
  const int lane = threadIdx.x & 31;
  if (plan.ws_base[b] < 0 || rid >= plan.n_kv_head * plan.rows) return;
  const int kvh = rid / plan.rows, rho = rid % plan.rows;
  const int g = rho / kRows, r = rho % kRows;
  const int ns = plan.n_split[b];
  const int slot0 = plan.ws_base[b] + (kvh * plan.groups + g) * ns;
  float mx = -INFINITY;
  for (int sp = 0; sp < ns; ++sp) mx = fmaxf(mx, __ldg(ws_lse + (int64_t)(slot0 + sp) * kRows + r));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -INFINITY) {
    float wsum = 0.f;
    for (int sp = 0; sp < ns; ++sp) {
      const float l = __ldg(ws_lse + (int64_t)(slot0 + sp) * kRows + r);
      const float w = l == -INFINITY ? 0.f : ex2_approx(l - mx);
      const float4 x = __ldg(reinterpret_cast<const float4*>(ws_o + ((int64_t)(slot0 + sp) * kRows + r) * kHeadDV) + lane);
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
      wsum += w;
    }
    const float inv = 1.f / wsum;
    acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
  }
  const int tok = rho / plan.group, head = kvh * plan.group + rho % plan.group;
  reinterpret_cast<float4*>(out + (int64_t)(plan.seq_offset + b) * out_seq_stride +
                            ((int64_t)tok * plan.n_head + head) * kHeadDV)[lane] = acc;
}

}  // namespace mla
