// MLA flash attention forward on sm_100a: one 2-CTA cluster per work unit.
//
// Per unit (sequence b, 128-row group g, KV split s) the pair computes, for
// its 128 query rows (row = token*n_head + head) and its range of key tiles,
//   S = scale * Q K^T + mask      (Q: 128 x 576, K tile: 128 keys x 576)
//   online softmax with running max m and running sum l per row
//   O += P V                      (V = first 512 columns of the same K rows)
// tile by tile, with S, P and O never leaving the SM pair (Vulkan FA for
// DeepSeek MLA article, sections 2.1-2.2; V taken from the K row per the
// ik_llama.cpp -mla guide, section "-mla四檔語義").
//
// Hardware mapping (cta_group::2, M = 128 rows, 64 rows in each CTA):
//  * Each CTA keeps its 64 Q rows in shared memory (9 chunks of 64 columns,
//    128-byte swizzle) for the whole unit.
//  * Q.K^T: N = 128 keys; CTA c loads keys [64c, 64c+64) of each tile, so the
//    pair reads every K byte once. In TMEM, lane r holds keys 0..63 of row r
//    and lane r+64 keys 64..127 (64 columns per S buffer, two buffers).
//  * P.V: N = 256 value columns per MMA, two MMAs per 16 keys; CTA c loads
//    value columns [256j+128c, +128) of the tile's rows. O lives in TMEM
//    (256 columns per CTA: lane r holds 128 of row r's values per MMA half).
//  * K and V chunks (8 KB each) stream through one ring of shared-memory
//    stages filled by TMA; the MMA thread releases a stage with tcgen05.commit.
//  * Softmax warpgroup: thread = TMEM lane; the two lanes of a row exchange
//    their tile maximum through shared memory. The reference max is raised
//    only when a tile's max exceeds it by more than 2^8, so O is rescaled in
//    TMEM rarely; P (f16, <= 256) goes to shared memory as the A operand.
//
// Every mbarrier wait is bounded (MlaFwdParams::timeout_ns). On a timeout the
// thread records MLA_ERR_TIMEOUT in the device status word and "fails
// through": it stops waiting but keeps the same control flow, so every warp
// still reaches every named/cluster barrier and the kernel ends.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>

#include "mla_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {

__device__ int g_status;  // first run-time error of this device (0 = none)

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

struct MlaFwdParams {
  const uint16_t* mask;      // f16 bits, or nullptr
  float* out;                // fp32 [seq][rows][512]
  float* ws_o;               // fp32 [slot][128][512] split partials
  float* ws_lse;             // fp32 [slot][128] log2-sum-exp of each partial
  int64_t mask_seq_stride;   // elements
  int64_t mask_row_stride;   // elements
  int64_t out_seq_stride;    // elements
  float scale_log2;          // scale * log2(e)
  int mask_vec_ok;           // mask rows allow 16-byte loads
  uint64_t timeout_ns;
  // cache rows read by the gather / dequant producer (modes other than TMA)
  const uint8_t* kcache;     // row (b, j) at (b*k_seq_stride + j) * row_bytes
  int64_t k_seq_stride;      // rows
  int n_kv;
  // sparse: sequence b attends to rows idx[b*idx_seq_stride + i], i < idx_count[b]
  const int32_t* idx;
  const int32_t* idx_count;
  int64_t idx_seq_stride;
};

// How K/V tiles reach shared memory.
enum FwdMode {
  kModeTma = 0,       // f16 cache, contiguous keys: TMA tensor loads
  kModeGatherF16 = 1, // f16 cache, rows chosen by an index list: warp-group loads
  kModeQ8 = 2         // q8_0 cache (dense or indexed): warp-group loads + dequant to f16
};

namespace fwd {

constexpr int kStages = 12;
constexpr int kChunkBytes = 8192;                 // one ring stage
constexpr int kQBytes = 9 * kChunkBytes;          // 64 rows x 576 f16
constexpr int kPBufBytes = 2 * kChunkBytes;       // 64 rows x 128 keys f16
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kQBytes;
constexpr int kOffP = kOffRing + kStages * kChunkBytes;
constexpr int kOffBar = kOffP + 2 * kPBufBytes;
constexpr int kNumBars = 2 * kStages + 1 + 2 + 2 + 2;
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kOffXmax = ((kOffTmemSlot + 4 + 15) / 16) * 16;  // float[2][128]
constexpr int kOffXl = kOffXmax + 2 * 128 * 4;                  // float[128]
constexpr int kSmemBytes = kOffXl + 128 * 4;
constexpr int kSmemAlloc = kSmemBytes + 1024;                   // 1024-byte alignment slack
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 128;                                // O columns start
constexpr float kRescaleThreshold = 8.0f;                       // log2 units

constexpr uint32_t kIdescQK = idesc_f16_f32(128, 128, 0, 0);    // K-major A and B
constexpr uint32_t kIdescPV = idesc_f16_f32(128, 256, 0, 1);    // B (V) MN-major

struct Bars {
  uint64_t ring_full[kStages];   // leader: both CTAs' TMA bytes for a stage
  uint64_t ring_empty[kStages];  // both: the MMAs reading a stage are done
  uint64_t q_full;               // leader: Q of both CTAs loaded
  uint64_t s_full[2];            // both: S buffer written by Q.K^T
  uint64_t p_full[2];            // leader: P written (8 warp arrivals, both CTAs)
  uint64_t o_done[2];            // both: P.V of a tile (parity-indexed) complete
};

}  // namespace fwd

// Unit index -> (sequence in launch, group, split). Binary search over unit_base.
__device__ __forceinline__ void decode_unit(const Plan& plan, int unit, int& b, int& g, int& s) {
  int lo = 0, hi = plan.n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (plan.unit_base[mid] <= unit) lo = mid; else hi = mid - 1;
  }
  b = lo;
  int local = unit - plan.unit_base[b];
  int ns = plan.n_split[b];
  g = local / ns;
  s = local - g * ns;
}

template <int kMode>
struct FwdCfg {
  static constexpr bool kManual = kMode != kModeTma;
  static constexpr int kThreads = kManual ? 384 : 256;  // + 4 producer warps when manual
  static constexpr int kRowBytes = kMode == kModeQ8 ? kQ8RowBytes : 2 * kDK;
};

// q8_0 block (f16 d, then 32 int8) -> 32 f16 values d*q (one rounding each), as
// 16 half2 words. An int8 q is biased to u = q + 128 and placed in the low
// mantissa bits of 1024.0 (0x6400), giving exactly 1024 + u; subtracting 1152
// leaves q exactly, and one f16 multiply by d rounds d*q once.
__device__ __forceinline__ void dequant_q8_block(const uint8_t* blk, uint32_t (&h)[16]) {
  const uint16_t dbits = __ldg(reinterpret_cast<const unsigned short*>(blk));
  const __half2 d2 = __half2half2(__ushort_as_half(dbits));
  const __half2 bias = __float2half2_rn(1152.f);
  const unsigned short* qw = reinterpret_cast<const unsigned short*>(blk + 2);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t u = (uint32_t)__ldg(qw + k) ^ 0x8080u;
    const uint32_t w = __byte_perm(u, 0x64646464u, 0x4140);
    __half2 v = *reinterpret_cast<const __half2*>(&w);
    v = __hmul2(__hsub2(v, bias), d2);
    h[k] = *reinterpret_cast<uint32_t*>(&v);
  }
}

template <int kMode>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(FwdCfg<kMode>::kThreads, 1)
    mla_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Plan plan,
                   const __grid_constant__ MlaFwdParams p) {
  using namespace fwd;
  constexpr bool kManual = FwdCfg<kMode>::kManual;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sRing = smem + kOffRing;
  uint8_t* sP = smem + kOffP;
  Bars& bars = *reinterpret_cast<Bars*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmemSlot);
  float* xmax = reinterpret_cast<float*>(smem + kOffXmax);
  float* xl = reinterpret_cast<float*>(smem + kOffXl);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint64_t to = p.timeout_ns;

  // ---- work unit
  int b, g, s;
  decode_unit(plan, blockIdx.x >> 1, b, g, s);
  const int b_abs = plan.seq_offset + b;
  const int n_split = plan.n_split[b];
  const bool sparse = p.idx != nullptr;
  const int len = sparse ? min(max(__ldg(p.idx_count + b_abs), 0), plan.kv_len[b]) : plan.kv_len[b];
  const int n_tiles_total = (len + kTileKeys - 1) / kTileKeys;
  const int tile_begin = (int)((int64_t)s * n_tiles_total / n_split);
  const int tile_end = (int)((int64_t)(s + 1) * n_tiles_total / n_split);
  const int n_tiles = tile_end - tile_begin;
  const int key_end = min(len, tile_end * kTileKeys);
  const int row0 = g * kRowsPerGroup;

  // ---- setup: barriers, TMEM
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars.ring_full[i], kManual ? 8 : 1);
      mbar_init(&bars.ring_empty[i], 1);
    }
    mbar_init(&bars.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 8);
      mbar_init(&bars.o_done[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    if (!kManual) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
  }
  if (warp == 1) tmem_alloc_2sm(tmem_slot, kTmemCols);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if constexpr (kManual) {
    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
  }
  if (warp == 0) {
    // ================= producer: TMA loads of Q, then (TMA mode) K and V chunks
    if (n_tiles > 0 && elect_one()) {
      const uint32_t q_full_l = mapa_shared(smem_u32(&bars.q_full), 0);
      if (rank == 0) mbar_arrive_expect_tx(&bars.q_full, 2 * kQBytes);
      for (int c = 0; c < 9; ++c)
        tma_load_3d_2sm(sQ + c * kChunkBytes, &tm_q, q_full_l, 64 * c,
                        row0 + kRowsPerCta * (int)rank, b_abs);
    }
    if (!kManual && n_tiles > 0 && elect_one()) {
      int stage = 0;
      uint32_t ephase = 0;
      auto acquire = [&]() {
        if (!failed && !mbar_wait(&bars.ring_empty[stage], ephase ^ 1, to)) {
          failed = true;
          record_status(kStatusTimeout);
        }
        if (rank == 0) mbar_arrive_expect_tx(&bars.ring_full[stage], 2 * kChunkBytes);
      };
      auto full_l = [&]() { return mapa_shared(smem_u32(&bars.ring_full[stage]), 0); };
      auto advance = [&]() {
        if (++stage == kStages) { stage = 0; ephase ^= 1; }
      };
      auto issue_k = [&](int i) {
        const int key0 = (tile_begin + i) * kTileKeys + 64 * (int)rank;
        for (int c = 0; c < 9; ++c) {
          acquire();
          tma_load_3d_2sm(sRing + stage * kChunkBytes, &tm_k, full_l(), 64 * c, key0, b_abs);
          advance();
        }
      };
      auto issue_v = [&](int j) {
        const int key0 = (tile_begin + j) * kTileKeys;
        for (int kb = 0; kb < 4; ++kb)
          for (int nb = 0; nb < 2; ++nb) {
            acquire();
            const int col = 256 * nb + 128 * (int)rank;
            uint32_t fl = full_l();
            tma_load_3d_2sm(sRing + stage * kChunkBytes, &tm_v, fl, col, key0 + 32 * kb, b_abs);
            tma_load_3d_2sm(sRing + stage * kChunkBytes + 4096, &tm_v, fl, col + 64,
                            key0 + 32 * kb, b_abs);
            advance();
          }
      };
      issue_k(0);
      for (int i = 1; i < n_tiles; ++i) {
        issue_k(i);
        issue_v(i - 1);
      }
      issue_v(n_tiles - 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================= MMA issuer (leader CTA, one thread)
    if (rank == 0 && n_tiles > 0 && elect_one()) {
      auto wait_or_fail = [&](uint64_t* bar, uint32_t parity, bool cluster_scope) {
        if (failed) return;
        bool ok = cluster_scope ? mbar_wait_cluster(bar, parity, to) : mbar_wait(bar, parity, to);
        if (!ok) {
          failed = true;
          record_status(kStatusTimeout);
        }
      };
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t ring_addr = smem_u32(sRing);
      const uint32_t p_addr = smem_u32(sP);
      wait_or_fail(&bars.q_full, 0, false);
      tc_fence_after();
      int stage = 0;
      uint32_t fphase = 0;
      auto advance = [&]() {
        if (++stage == kStages) { stage = 0; fphase ^= 1; }
      };
      auto pv = [&](int j) {
        wait_or_fail(&bars.p_full[j & 1], (j >> 1) & 1, true);
        tc_fence_after();
        for (int kb = 0; kb < 4; ++kb)
          for (int nb = 0; nb < 2; ++nb) {
            wait_or_fail(&bars.ring_full[stage], fphase, kManual);
            tc_fence_after();
            for (int k2 = 0; k2 < 2; ++k2) {
              const int kk = 2 * kb + k2;
              uint64_t ad = smem_desc_sw128(
                  p_addr + (j & 1) * kPBufBytes + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024);
              uint64_t bd = smem_desc_sw128(ring_addr + stage * kChunkBytes + k2 * 2048, 4096, 1024);
              mma_f16_ss_2sm(tmem + kTmemO + nb * 128, ad, bd, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_2sm_mc(&bars.ring_empty[stage], 0x3);
            advance();
          }
        mma_commit_2sm_mc(&bars.o_done[j & 1], 0x3);
      };
      for (int i = 0; i < n_tiles; ++i) {
        const uint32_t d_s = tmem + (i & 1) * 64;
        for (int c = 0; c < 9; ++c) {
          wait_or_fail(&bars.ring_full[stage], fphase, kManual);
          tc_fence_after();
          for (int kk = 0; kk < 4; ++kk) {
            uint64_t ad = smem_desc_sw128(q_addr + c * kChunkBytes + kk * 32, 16, 1024);
            uint64_t bd = smem_desc_sw128(ring_addr + stage * kChunkBytes + kk * 32, 16, 1024);
            mma_f16_ss_2sm(d_s, ad, bd, kIdescQK, (c | kk) ? 1u : 0u);
          }
          mma_commit_2sm_mc(&bars.ring_empty[stage], 0x3);
          advance();
        }
        mma_commit_2sm_mc(&bars.s_full[i & 1], 0x3);
        if (i > 0) pv(i - 1);
      }
      pv(n_tiles - 1);
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ================= gather / dequant producer (manual modes): 4 warps, 128 threads
    if constexpr (kManual) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 128;");
      const int pt = threadIdx.x - 256;
      const int64_t seq_row0 = (int64_t)b_abs * p.k_seq_stride;
      const int32_t* idx_row = sparse ? p.idx + (int64_t)b_abs * p.idx_seq_stride : nullptr;
      // cache row of key position `pos` in this unit's selection, or -1 (zero fill)
      auto resolve = [&](int pos) -> int {
        if (pos >= len) return -1;
        if (!sparse) return pos < p.n_kv ? pos : -1;
        const int key = __ldg(idx_row + pos);
        if (key < 0 || key >= p.n_kv) {
          record_status(kStatusIndex);
          return -1;
        }
        return key;
      };
      // 32 consecutive values of a cache row, as f16, into 4 swizzled 16-byte chunks
      auto fill32 = [&](uint8_t* row_dst, int row_in_atom, int key, int col32, int chunk0) {
        uint32_t h[16];
        if (key < 0) {
#pragma unroll
          for (int k = 0; k < 16; ++k) h[k] = 0u;
        } else if constexpr (kMode == kModeQ8) {
          const uint8_t* rowp = p.kcache + (seq_row0 + key) * kQ8RowBytes;
          dequant_q8_block(rowp + col32 * 34, h);
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(
              p.kcache + (seq_row0 + key) * (2 * kDK) + col32 * 64);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 v = __ldg(src + k);
            h[4 * k] = v.x; h[4 * k + 1] = v.y; h[4 * k + 2] = v.z; h[4 * k + 3] = v.w;
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(row_dst + (((chunk0 + k) ^ (row_in_atom & 7)) << 4)) =
              make_uint4(h[4 * k], h[4 * k + 1], h[4 * k + 2], h[4 * k + 3]);
      };
      int stage = 0;
      uint32_t ephase = 0;
      auto acquire = [&]() {
        bool ok = failed ? true : mbar_wait(&bars.ring_empty[stage], ephase ^ 1, to);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && !failed) {
          failed = true;
          if (lane == 0) record_status(kStatusTimeout);
        }
      };
      auto publish = [&]() {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bars.ring_full[stage]), 0));
        if (++stage == kStages) { stage = 0; ephase ^= 1; }
      };
      // K chunk: 64 keys (this CTA's half of the tile) x 64 columns = 2 blocks of 32
      auto issue_k = [&](int i) {
        const int kl = pt >> 1, half = pt & 1;
        const int key = resolve((tile_begin + i) * kTileKeys + 64 * (int)rank + kl);
        for (int c = 0; c < 9; ++c) {
          acquire();
          fill32(sRing + stage * kChunkBytes + kl * 128, kl, key, 2 * c + half, 4 * half);
          publish();
        }
      };
      // V chunk: 32 keys x this CTA's 128 value columns (two 64-column boxes)
      auto issue_v = [&](int j) {
        const int kl = pt >> 2, q4 = pt & 3;
        const int box = q4 >> 1, half = q4 & 1;
        const int kbase = (tile_begin + j) * kTileKeys;
        for (int kb = 0; kb < 4; ++kb) {
          const int key = resolve(kbase + 32 * kb + kl);
          for (int nb = 0; nb < 2; ++nb) {
            acquire();
            const int col32 = 8 * nb + 4 * (int)rank + q4;
            fill32(sRing + stage * kChunkBytes + box * 4096 + kl * 128, kl, key, col32, 4 * half);
            publish();
          }
        }
      };
      if (n_tiles > 0) {
        issue_k(0);
        for (int i = 1; i < n_tiles; ++i) {
          issue_k(i);
          issue_v(i - 1);
        }
        issue_v(n_tiles - 1);
      }
    }
  } else if (warp >= 4) {
    // ================= softmax / correction / epilogue warpgroup
    if constexpr (kManual) asm volatile("setmaxnreg.inc.sync.aligned.u32 256;");
    const int L = threadIdx.x - 128;          // TMEM lane
    const int r = L & 63;                     // row within this CTA
    const int kh = L >> 6;                    // which 64 keys of a tile this lane holds
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int row = row0 + kRowsPerCta * (int)rank + r;  // row within the sequence
    const bool row_valid = row < plan.rows;
    const int tok = row / plan.n_head;
    const uint16_t* mrow = (p.mask != nullptr && row_valid)
                               ? p.mask + (int64_t)b_abs * p.mask_seq_stride +
                                     (int64_t)tok * p.mask_row_stride
                               : nullptr;
    const uint32_t p_full_l0 = mapa_shared(smem_u32(&bars.p_full[0]), 0);
    const uint32_t p_full_l1 = mapa_shared(smem_u32(&bars.p_full[1]), 0);
    auto wait_local = [&](uint64_t* bar, uint32_t parity) {
      bool ok = failed ? true : mbar_wait(bar, parity, to);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && !failed) {
        failed = true;
        if (lane == 0) record_status(kStatusTimeout);
      }
    };

    float m_ref = -INFINITY;  // reference max (log2 units) used for exponentiation
    float l_part = 0.f;       // this lane's half of the row sum, relative to m_ref

    for (int i = 0; i < n_tiles; ++i) {
      const int sb = i & 1;
      const int key0 = (tile_begin + i) * kTileKeys + 64 * kh;
      wait_local(&bars.s_full[sb], (i >> 1) & 1);
      tc_fence_after();
      uint32_t sr[64];
      {
        uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t (&c)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld32(tmem + lane_base + sb * 64, a);
        tmem_ld32(tmem + lane_base + sb * 64 + 32, c);
        tmem_wait_ld();
      }
      // scores in log2 units; cells beyond the unit's keys are dropped
      float x[64];
      const bool full_range = key0 + 64 <= key_end;
      if (kManual && sparse) {
        const int32_t* ix = p.idx + (int64_t)b_abs * p.idx_seq_stride;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int pos = key0 + j;
          float mv = 0.f;
          bool ok = pos < key_end;
          if (ok) {
            const int cell = __ldg(ix + pos);
            ok = cell >= 0 && cell < p.n_kv;
            if (ok && mrow != nullptr) mv = __half2float(__ushort_as_half(__ldg(mrow + cell)));
          }
          x[j] = ok ? fmaf(__uint_as_float(sr[j]), p.scale_log2, mv * kLog2e) : -INFINITY;
        }
      } else if (mrow != nullptr && full_range && p.mask_vec_ok) {
        const uint4* mv = reinterpret_cast<const uint4*>(mrow + key0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v = __ldg(mv + c);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[h]));
            x[8 * c + 2 * h] = fmaf(__uint_as_float(sr[8 * c + 2 * h]), p.scale_log2, f.x * kLog2e);
            x[8 * c + 2 * h + 1] =
                fmaf(__uint_as_float(sr[8 * c + 2 * h + 1]), p.scale_log2, f.y * kLog2e);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int key = key0 + j;
          float mv = 0.f;
          if (mrow != nullptr && key < key_end)
            mv = __half2float(__ushort_as_half(__ldg(mrow + key)));
          x[j] = key < key_end ? fmaf(__uint_as_float(sr[j]), p.scale_log2, mv * kLog2e) : -INFINITY;
        }
      }
      float mt = x[0];
#pragma unroll
      for (int j = 1; j < 64; ++j) mt = fmaxf(mt, x[j]);
      xmax[sb * 128 + L] = mt;
      named_bar_sync(1, 128);
      mt = fmaxf(mt, xmax[sb * 128 + (L ^ 64)]);

      const bool need = mt > m_ref + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_ref - mt);  // 0 when m_ref = -inf
        m_ref = mt;
      }
      const float mref_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t pk[32];
      float lsum = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        __half2 h2 = __floats2half2_rn(ex2_approx(x[2 * j] - mref_use),
                                       ex2_approx(x[2 * j + 1] - mref_use));
        pk[j] = *reinterpret_cast<uint32_t*>(&h2);
        float2 f2 = __half22float2(h2);
        lsum += f2.x + f2.y;
      }
      l_part = l_part * alpha + lsum;

      // P buffer sb is free once P.V of tile i-2 has completed
      if (i >= 2) wait_local(&bars.o_done[sb], ((i - 2) >> 1) & 1);
      {
        uint8_t* base = sP + sb * kPBufBytes + kh * kChunkBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          *reinterpret_cast<uint4*>(base + ((c ^ (r & 7)) << 4)) = v;
        }
      }
      // rescale O (only when some row of this warp raised its reference max)
      if (__any_sync(0xffffffffu, need && i > 0)) {
        wait_local(&bars.o_done[(i - 1) & 1], ((i - 1) >> 1) & 1);
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t v[32];
          const uint32_t a = tmem + lane_base + kTmemO + cc * 32;
          tmem_ld32(a, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
          tmem_st32(a, v);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(sb ? p_full_l1 : p_full_l0);
    }

    // ---- epilogue
    if (n_tiles > 0) wait_local(&bars.o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1);
    tc_fence_after();
    xl[L] = l_part;
    named_bar_sync(1, 128);
    const float l_tot = l_part + xl[L ^ 64];
    const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
    const int ws_slot = plan.ws_base[b] >= 0 ? plan.ws_base[b] + g * n_split + s : -1;
    float* dst = nullptr;
    if (ws_slot < 0)
      dst = p.out + (int64_t)b_abs * p.out_seq_stride + (int64_t)row * kDV;
    else
      dst = p.ws_o + ((int64_t)ws_slot * kRowsPerGroup + kRowsPerCta * rank + r) * kDV;
    for (int nb = 0; nb < 2; ++nb)
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        if (n_tiles > 0) {
          tmem_ld32(tmem + lane_base + kTmemO + nb * 128 + cc * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        }
        if (row_valid) {
          float4* o4 = reinterpret_cast<float4*>(dst + 256 * nb + 128 * kh + 32 * cc);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            o4[q4] = make_float4(__uint_as_float(v[4 * q4]) * inv_l,
                                 __uint_as_float(v[4 * q4 + 1]) * inv_l,
                                 __uint_as_float(v[4 * q4 + 2]) * inv_l,
                                 __uint_as_float(v[4 * q4 + 3]) * inv_l);
        }
      }
    if (ws_slot >= 0 && kh == 0 && row_valid)
      p.ws_lse[(int64_t)ws_slot * kRowsPerGroup + kRowsPerCta * rank + r] =
          l_tot > 0.f ? m_ref + __log2f(l_tot) : -INFINITY;
  }

  // ---- teardown
  if (failed) nanosleep_ns(100000);  // let copies issued before the failure land
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

// LSE combine of split-KV partials (one warp per query row):
//   O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M),  M = max_s lse_s,
// where O_s is split s normalised by its own sum and lse_s = log2 of that sum
// relative to the split's max; splits with no kept cell have lse_s = -inf.
__global__ void __launch_bounds__(128) mla_combine_kernel(const __grid_constant__ Plan plan,
                                                          const float* __restrict__ ws_o,
                                                          const float* __restrict__ ws_lse,
                                                          float* __restrict__ out,
                                                          int64_t out_seq_stride) {
  const int b = blockIdx.y;
  const int ns = plan.n_split[b];
  if (plan.ws_base[b] < 0) return;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= plan.rows) return;
  const int lane = threadIdx.x & 31;
  const int g = row / kRowsPerGroup;
  const int rin = row % kRowsPerGroup;
  const int slot0 = plan.ws_base[b] + g * ns;
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, ws_lse[(int64_t)(slot0 + s) * kRowsPerGroup + rin]);
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -INFINITY) {
    float wsum = 0.f;
    for (int s = 0; s < ns; ++s) {
      const float lse = ws_lse[(int64_t)(slot0 + s) * kRowsPerGroup + rin];
      if (lse == -INFINITY) continue;
      const float w = ex2_approx(lse - mx);
      wsum += w;
      const float4* src =
          reinterpret_cast<const float4*>(ws_o + ((int64_t)(slot0 + s) * kRowsPerGroup + rin) * kDV);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = __ldg(src + lane + 32 * k);
        acc[k].x = fmaf(w, v.x, acc[k].x);
        acc[k].y = fmaf(w, v.y, acc[k].y);
        acc[k].z = fmaf(w, v.z, acc[k].z);
        acc[k].w = fmaf(w, v.w, acc[k].w);
      }
    }
    const float inv = 1.f / wsum;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[k].x *= inv; acc[k].y *= inv; acc[k].z *= inv; acc[k].w *= inv;
    }
  }
  float4* dst = reinterpret_cast<float4*>(out + (int64_t)(plan.seq_offset + b) * out_seq_stride +
                                          (int64_t)row * kDV);
#pragma unroll
  for (int k = 0; k < 4; ++k) dst[lane + 32 * k] = acc[k];
}

// Waits on a barrier that nothing ever signals, with a bounded wait, and records
// the timeout: exercises the run-time error path without faulting anything.
__global__ void mla_wait_timeout_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns)) record_status(kStatusTimeout);
}

}  // namespace mla
