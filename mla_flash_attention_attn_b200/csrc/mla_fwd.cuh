// MLA flash attention forward on sm_100a: one 2-CTA cluster per work unit.
//
// Per unit (sequence b, 128-row group g, KV split s) the pair computes, for
// its 128 query rows (row = token*n_head + head) and its range of keys,
//   S = scale * Q K^T + mask      (Q: 128 x 576, a step of kTK keys x 576)
//   online softmax with running max m and running sum l per row
//   O += P V                      (V = first 512 columns of the same K rows)
// step by step, with S, P and O never leaving the SM pair (Vulkan FA for
// DeepSeek MLA article, sections 2.1-2.2; V taken from the K row per the
// ik_llama.cpp -mla guide, section "-mla四檔語義").
//
// Hardware mapping (cta_group::2, M = 128 rows, 64 rows in each CTA):
//  * Each CTA keeps its 64 Q rows in shared memory (9 chunks of 64 columns,
//    128-byte swizzle) for the whole unit; they arrive with the first step's K.
//  * Q.K^T: N = kTK keys (a step of 128 or 256, fwd::Geo); CTA c loads keys
//    [c kTK/2, (c+1) kTK/2) of each step, so the pair reads every K byte once. In
//    TMEM, lane r holds the first kTK/2 keys of row r and lane r+64 the others.
//  * P.V: N = 256 value columns per MMA (one value half), K = 16 keys; CTA c
//    loads value columns [256j+128c, +128) of the step's rows. A (P) is read from
//    TMEM and O accumulates in TMEM (256 columns per CTA: lane r holds 128 of row
//    r's values per value half).
//  * TMEM: S buffers, P buffers (f16 pairs of all keys of the step in both lanes
//    of a row), O (256 columns). With 128-key steps two S and two P buffers let
//    Q.K^T of the next step run while the softmax reads S and the softmax write P
//    while P.V of the previous step reads the other P; with 256-key steps there is
//    one of each, and the softmax frees S as soon as the scores are in registers.
//  * K stages (kTK/2 keys x 64 columns) and V stages (16 KB: 64 keys x 128 value
//    columns) stream through two rings of shared-memory stages; every stage is
//    4 MMAs and one tcgen05.commit releases it.
//  * Two threads issue MMAs: one for Q.K^T, one for P.V. An issuing thread
//    cannot run ahead of the tensor pipe, so the cycles it spends waiting on a
//    barrier would idle the pipe; with two issuers one's wait is covered by the
//    other's MMAs.
//  * Softmax warpgroup: thread = TMEM lane; the two lanes of a row exchange
//    their step maximum and their P halves through shared memory. The reference
//    max is raised only when a step's max exceeds it by more than 2^8, so O is
//    rescaled in TMEM rarely.
//  * Epilogue: O / l is staged in shared memory and written by TMA stores.
//
// Every mbarrier wait is bounded (MlaFwdParams::timeout_ns). On a timeout the
// thread records MLA_ERR_TIMEOUT in the device status word and "fails
// through": it stops waiting but keeps the same control flow, so every warp
// still reaches every named/cluster barrier and the kernel ends.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>

#include "mla_common.cuh"
#include "mla_plan.cuh"
#include "sm100_ptx.cuh"

namespace mla {

__device__ int g_status;  // first run-time error of this device (0 = none)

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

struct MlaFwdParams {
  const uint16_t* mask;      // f16 bits, or nullptr
  float* out;                // fp32 [seq][rows][512]
  uint16_t* ws_o;            // f16 [slot][128][512] split partials (O_s / l_s)
  float* ws_lse;             // fp32 [slot][128] log2-sum-exp of each partial
  int64_t mask_seq_stride;   // elements
  int64_t mask_row_stride;   // elements
  int64_t out_seq_stride;    // elements
  float scale;               // softmax scale (natural units)
  int mask_vec_ok;           // mask rows allow 16-byte loads
  uint64_t timeout_ns;
  // cache rows read by the gather / dequant producer (modes other than TMA)
  const uint8_t* kcache;     // row (b, j) at (b*k_seq_stride + j) * row_bytes
  int64_t k_seq_stride;      // rows
  int n_kv;
  // query rows read by the manual producers: row r of sequence b at q + b*q_seq_stride + r*576
  const uint16_t* q;
  int64_t q_seq_stride;      // elements
  // sparse: sequence b attends to rows idx[b*idx_seq_stride + i], i < idx_count[b]; in
  // TMA mode with idx == nullptr, idx_count (when set) bounds the rows of sequence b
  // (rows gathered from an index list)
  const int32_t* idx;
  const int32_t* idx_count;
  int64_t idx_seq_stride;
  // variants (0 / nullptr = off): logit softcap, ALiBi slopes per head
  float softcap;
  const float* slopes;
  // mask gather (no index list): unit u, CTA rank r lists its kept cells at
  // gather_list + (2u + r) * gather_stride
  int mask_gather;
  int32_t* gather_list;
  int64_t gather_stride;
  // device plan (tile ranges found from the mask on the device): unit u's descriptor;
  // nullptr: the host plan
  const DevUnit* units;
};

// How K/V tiles reach shared memory.
enum FwdMode {
  kModeTma = 0,       // f16 cache, contiguous keys: TMA tensor loads
  kModeGatherF16 = 1, // f16 cache, rows chosen by an index list: warp-group loads
  kModeQ8 = 2         // q8_0 cache (dense or indexed): warp-group loads + dequant to f16
};

namespace fwd {

constexpr int kChunkBytes = 8192;                 // 64 rows x 64 f16 (one swizzle tile)
constexpr int kQBytes = 9 * kChunkBytes;          // this CTA's 64 query rows x 576, resident
constexpr int kVStageBytes = 2 * kChunkBytes;     // V stage: 64 keys x 128 value columns
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 5.5451774f;   // 8 ln 2 (natural units)

// Layout of the pipeline for steps of kTK keys (one Q.K^T MMA has N = kTK; CTA c
// loads keys [c kTK/2, (c+1) kTK/2) of a step):
//  * kTK = 256: one S buffer and one P buffer of 128 TMEM columns; the K ring holds 4
//    stages of 128 keys x 64 columns (16 KB).
//  * kTK = 128: two S buffers and two P buffers of 64 columns (step i uses buffer
//    i % 2), so that Q.K^T of step i+1 runs while the softmax reads S(i), and the
//    softmax writes P(i) while P.V(i-1) still reads P(i-1); the K ring holds 10 stages
//    of 64 keys x 64 columns (8 KB), more than a step's 9 chunks.
// TMEM columns: S buffers from 0, P buffers from 128 (f16 pairs of all kTK keys of the
// step, in both lanes of a row), O from 256 (256 fp32 columns: 128 values of each value
// half per lane).
template <int kTK>
struct Geo {
  static_assert(kTK == 128 || kTK == 256, "steps of 128 or 256 keys");
  static constexpr int kBufs = kTK == 128 ? 2 : 1;        // S buffers and P buffers
  static constexpr int kKStages = kTK == 128 ? 10 : 4;    // ring of Q.K^T operand stages
  static constexpr int kVStages = 3;                      // ring of P.V operand stages (L2-resident V)
  static constexpr int kKStageBytes = kTK * 64;           // kTK/2 keys x 64 columns, f16
  static constexpr int kXWords = kTK / 4;                 // f16 pairs a lane swaps per step
  static constexpr int kXBytes = 128 * kXWords * 4;       // P exchange buffer
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKStageBytes;
  static constexpr int kOffX = kOffV + kVStages * kVStageBytes;
  static constexpr int kOffBar = kOffX + kXBytes;
  static constexpr int kBarBytes = 8 * (2 * kKStages + 2 * kVStages + 2 * kBufs + 2 + 2 + 1);
  static constexpr int kOffTmemSlot = kOffBar + kBarBytes;
  static constexpr int kOffXmax = ((kOffTmemSlot + 4 + 15) / 16) * 16;  // float[2][128]
  static constexpr int kOffXl = kOffXmax + 2 * 128 * 4;                  // float[128]
  static constexpr int kSmemBytes = kOffXl + 128 * 4;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;                   // 1024-byte alignment slack
  static constexpr uint32_t kSCols = kTK / 2;   // TMEM columns of one S or one P buffer
  static constexpr uint32_t kTmemS = 0;
  static constexpr uint32_t kTmemP = 128;
  static constexpr uint32_t kTmemO = 256;
  static constexpr uint32_t kIdescQK = idesc_f16_f32(128, kTK, 0, 0);  // K-major A and B
  static constexpr uint32_t kIdescPV = idesc_f16_f32(128, 256, 0, 1);  // A (P, TMEM) K-major, B (V) MN-major

  static_assert(kSmemAlloc <= 232448, "shared memory beyond the 227 KB per-CTA limit");
  static_assert(kBufs * kSCols <= kTmemP && kTmemP + kBufs * kSCols <= kTmemO && kTmemO + 256 <= kTmemCols,
                "S, P and O exceed the TMEM allocation");
  static_assert(kOffQ % 1024 == 0 && kOffK % 1024 == 0 && kOffV % 1024 == 0,
                "128-byte swizzle needs 1 KB alignment");
  static_assert(kOffBar >= 128 * 1024, "the epilogue stages O in the first 128 KB");
};

template <int kKS, int kVS, int kB>
struct BarsT {
  uint64_t k_full[kKS];          // leader: both CTAs' K chunk bytes landed
  uint64_t k_empty[kKS];         // both: the Q.K^T MMAs reading a stage are done
  uint64_t v_full[kVS];          // leader: both CTAs' V chunk bytes landed
  uint64_t v_empty[kVS];         // both: the P.V MMAs reading a V stage are done
  uint64_t s_full[kB];           // both: S buffer written by Q.K^T
  uint64_t s_free[kB];           // leader: S buffer read out by the softmax (8 warp arrivals)
  uint64_t p_full[2];            // leader: P written to TMEM (8 warp arrivals, both CTAs)
  uint64_t o_done[2];            // both: P.V of a step (parity-indexed) complete
  uint64_t q_full;               // leader, gather modes: both CTAs' Q rows landed (TMA)
};
template <int kTK>
using BarsOf = BarsT<Geo<kTK>::kKStages, Geo<kTK>::kVStages, Geo<kTK>::kBufs>;
static_assert(sizeof(BarsOf<256>) == Geo<256>::kBarBytes && sizeof(BarsOf<128>) == Geo<128>::kBarBytes,
              "barrier block size");

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
};

// q8_0 block (f16 d, then 32 int8) -> 32 f16 values d*q (one rounding each), as
// 16 half2 words. An int8 q is biased to u = q + 128 and placed in the low
// mantissa bits of 1024.0 (0x6400), giving exactly 1024 + u; subtracting 1152
// leaves q exactly, and one f16 multiply by d rounds d*q once.
//
// A block is 34 bytes at 2-byte alignment (rows are 612 bytes): it is read as the
// 9 aligned 32-bit words that cover it. An even block starts 4-byte aligned and is
// never the last block of its row; an odd block starts 2 bytes into its first
// word; either way the 36 bytes read stay inside the row.
template <int kMode>
struct RawBlock {
  uint32_t w[kMode == kModeQ8 ? 9 : 16];  // f16: the 32 values; q8_0: 9 words cover the block
  bool odd;        // q8_0: the block starts 2 bytes into w[0]
  bool valid;      // false: zero fill
};

// kRowBytes: bytes of an f16 cache row (2 x its head width)
template <int kMode, int kRowBytes>
__device__ __forceinline__ void load_block(const uint8_t* kcache, int64_t row, int col32,
                                           RawBlock<kMode>& rb) {
  if constexpr (kMode == kModeQ8) {
    const uint8_t* blk = kcache + row * kQ8RowBytes + col32 * 34;
    const uintptr_t a = reinterpret_cast<uintptr_t>(blk);
    const uint32_t* w4 = reinterpret_cast<const uint32_t*>(a & ~static_cast<uintptr_t>(3));
#pragma unroll
    for (int i = 0; i < 9; ++i) rb.w[i] = __ldg(w4 + i);
    rb.odd = (a & 2) != 0;
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(kcache + row * kRowBytes + col32 * 64);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 v = __ldg(src + k);
      rb.w[4 * k] = v.x; rb.w[4 * k + 1] = v.y; rb.w[4 * k + 2] = v.z; rb.w[4 * k + 3] = v.w;
    }
  }
}

template <int kMode>
__device__ __forceinline__ void block_values(const RawBlock<kMode>& rb, uint32_t (&h)[16]) {
  if (!rb.valid) {
#pragma unroll
    for (int k = 0; k < 16; ++k) h[k] = 0u;
    return;
  }
  if constexpr (kMode == kModeQ8) {
    // the block's own 32-bit words B[j] = block bytes 4j..4j+3 (j = 0..8): an odd block
    // starts 2 bytes into rb.w[0], so each is a funnel shift of two loaded words
    const uint32_t sh = rb.odd ? 16u : 0u;
    uint32_t x[9];
#pragma unroll
    for (int j = 0; j < 9; ++j) {
      const uint32_t hi = j < 8 ? rb.w[j + 1] : 0u;  // bytes past the block are unused
      x[j] = __funnelshift_r(rb.w[j], hi, sh) ^ 0x80808080u;  // int8 q -> q + 128
    }
    const __half2 d2 = __half2half2(__ushort_as_half((unsigned short)((x[0] ^ 0x80808080u) & 0xFFFFu)));
    const __half2 bias = __float2half2_rn(1152.f);
    // int8 pair k sits in block bytes 2+2k, 3+2k: the high half of B[k/2] for even k,
    // the low half of B[k/2+1] for odd k; each byte goes into 0x64 to make 1024 + u
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t wd = (k & 1) ? __byte_perm(x[(k >> 1) + 1], 0x64646464u, 0x4140)
                                  : __byte_perm(x[k >> 1], 0x64646464u, 0x4342);
      __half2 v = *reinterpret_cast<const __half2*>(&wd);
      v = __hmul2(__hsub2(v, bias), d2);
      h[k] = *reinterpret_cast<uint32_t*>(&v);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) h[k] = rb.w[k];
  }
}

// kVariant: the instance that applies the logit softcap and ALiBi; kGather: the instance
// that compacts the mask itself (gather modes only). The host launches them only when a
// call asks for them, so the common path carries none of that code. kNC: 64-column
// chunks of the head width, 9 (576: 512 latent + 64 RoPE) or 8 (the DK = DV = 512
// shape, f16 cache, V the whole row). kTK: keys of a pipeline step (128 or 256; the
// gather modes take 256).
template <int kMode, bool kVariant, bool kGather, int kNC, int kTK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(FwdCfg<kMode>::kThreads, 1)
    mla_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ Plan plan,
                   const __grid_constant__ MlaFwdParams p) {
  using namespace fwd;
  using G = Geo<kTK>;
  constexpr bool kManual = FwdCfg<kMode>::kManual;
  static_assert(kNC == 9 || (kNC == 8 && kMode != kModeQ8), "head width 576, or 512 with an f16 cache");
  static_assert(kTK == 256 || !kManual, "the gather modes' producers fill 256-key steps");
  constexpr int kKStages = G::kKStages;
  constexpr int kKStageBytes = G::kKStageBytes;
  constexpr int kVStages = G::kVStages;
  constexpr int kXRounds = 1;                   // P exchange rounds per step
  constexpr int kXWords = G::kXWords;
  constexpr int kBufs = G::kBufs;
  constexpr uint32_t kSCols = G::kSCols;
  constexpr uint32_t kTmemS = G::kTmemS, kTmemP = G::kTmemP, kTmemO = G::kTmemO;
  constexpr uint32_t kIdescQK = G::kIdescQK, kIdescPV = G::kIdescPV;
  using Bars = BarsOf<kTK>;
  // bytes of a cache row: q8_0 rows are 612 bytes; f16 rows 2 x the head width
  constexpr int kRowBytes = kMode == kModeQ8 ? kQ8RowBytes : 128 * kNC;
  extern __shared__ uint8_t smem_raw[];
  // a launch with too little dynamic shared memory reports and returns (every CTA takes
  // this branch, so no cluster barrier is left waiting)
  if (dynamic_smem_bytes() < (uint32_t)G::kSmemAlloc) {
    if (threadIdx.x == 0) record_status(kStatusLaunch);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + G::kOffQ;
  uint8_t* sK = smem + G::kOffK;
  uint8_t* sV = smem + G::kOffV;
  uint4* sX = reinterpret_cast<uint4*>(smem + G::kOffX);
  Bars& bars = *reinterpret_cast<Bars*>(smem + G::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + G::kOffTmemSlot);
  float* xmax = reinterpret_cast<float*>(smem + G::kOffXmax);
  float* xl = reinterpret_cast<float*>(smem + G::kOffXl);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint64_t to = p.timeout_ns;

  // ---- setup: barriers, TMEM (nothing here reads global memory: the kernel may run
  // as a programmatic dependent of the kernel that writes its inputs)
  if (threadIdx.x == 0) {
    // manual modes: 2 producer warps per ring in each CTA arrive on the leader
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars.k_full[i], kManual ? 4 : 1);
      mbar_init(&bars.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bars.v_full[i], kManual ? 4 : 1);
      mbar_init(&bars.v_empty[i], 1);
    }
    for (int i = 0; i < kBufs; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], 8);
    }
    mbar_init(&bars.q_full, 1);
    for (int i = 0; i < 2; ++i) {
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
  // inputs written by the previous kernel of the stream (the compaction, say) are
  // visible from here on; a launch without the programmatic attribute returns at once
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- work unit: from the host plan, or from the device plan's descriptor (an idle
  // descriptor leaves the unit without tiles and without output)
  int b, g, s, n_split;
  bool idle = false;
  DevUnit du = {0, 0, 0, 1, 0, 0, -1, 0};
  if (p.units != nullptr) {
    du = p.units[blockIdx.x >> 1];
    idle = du.b < 0;
    b = idle ? 0 : du.b;
    g = du.g;
    s = du.s;
    n_split = du.n_split;
  } else {
    decode_unit(plan, blockIdx.x >> 1, b, g, s);
    n_split = plan.n_split[b];
  }
  const int b_abs = plan.seq_offset + b;
  const int row0 = g * kRowsPerGroup;
  constexpr bool gather = kManual && kGather;
  const bool sparse = p.idx != nullptr || gather;
  // positions of the unit: an index list (its tiles of the sequence's list), or, with
  // the mask gather, every kept cell of the chunks dealt to its split (below)
  int len, tile_begin, n_tiles, key_end;
  // the unit's index list, recomputed where it is read (cheaper than a live register)
  auto list_ptr = [&]() -> const int32_t* {
    return gather ? p.gather_list + (int64_t)(2 * (blockIdx.x >> 1) + rank) * p.gather_stride
                  : p.idx + (int64_t)b_abs * p.idx_seq_stride;
  };
  if (gather) {
    // The sequence's first kv_len cells, in chunks of 8, are dealt round-robin to its
    // splits (chunk j to split j mod n_split), so that a run of kept cells (a recent
    // window, say) is shared out instead of landing on one split. Each split compacts
    // its chunks here into an ascending list of the cells that some row of this group
    // keeps (mask != -inf): a thread takes one chunk, a block scan gives its offset.
    // Both CTAs of the pair build the same list.
    const int cells = plan.kv_len[b];
    const int n_chunks = (cells + 7) >> 3;
    const int t_lo = row0 / plan.n_head;
    const int t_hi = min(plan.rows - 1, row0 + kRowsPerGroup - 1) / plan.n_head;
    int32_t* out_list = p.gather_list + (int64_t)(2 * (blockIdx.x >> 1) + rank) * p.gather_stride;
    int* scan = reinterpret_cast<int*>(xmax);  // warp totals of one pass
    const uint16_t* mseq = p.mask + (int64_t)b_abs * p.mask_seq_stride;
    constexpr int kT = FwdCfg<kMode>::kThreads;
    int base = 0;
    for (int i0 = 0; (int64_t)s + (int64_t)n_split * i0 < n_chunks; i0 += kT) {
      const int64_t j = (int64_t)s + (int64_t)n_split * (i0 + (int)threadIdx.x);
      const int cell0 = (int)(8 * j);
      uint32_t keep = 0;
      if (j < n_chunks) {
        const int n_in = min(8, cells - cell0);
        for (int t = t_lo; t <= t_hi; ++t) {
          const uint16_t* mr = mseq + (int64_t)t * p.mask_row_stride + cell0;
          if (p.mask_vec_ok && n_in == 8) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(mr));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if ((w[k] & 0xFFFFu) != 0xFC00u) keep |= 1u << (2 * k);
              if ((w[k] >> 16) != 0xFC00u) keep |= 2u << (2 * k);
            }
          } else {
            for (int k = 0; k < n_in; ++k)
              if (__ldg(mr + k) != 0xFC00u) keep |= 1u << k;
          }
        }
      }
      const int cnt = __popc(keep);
      int inc = cnt;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += y;
      }
      if (lane == 31) scan[warp] = inc;
      __syncthreads();
      int woff = 0, total = 0;
      for (int w = 0; w < kT / 32; ++w) {
        const int tw = scan[w];
        if (w < warp) woff += tw;
        total += tw;
      }
      int pos = base + woff + inc - cnt;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (keep & (1u << k)) out_list[pos++] = cell0 + k;
      base += total;
      __syncthreads();  // the warp totals are read before the next pass overwrites them
    }
    __syncthreads();  // the list is complete and visible to every thread of this CTA
    len = base;
    tile_begin = 0;
    n_tiles = (len + kTK - 1) / kTK;
    key_end = len;
  } else {
    // an index list (or, in TMA mode, the rows gathered from one) ends at its count
    len = (sparse || p.idx_count != nullptr) ? min(max(__ldg(p.idx_count + b_abs), 0), plan.kv_len[b])
                                             : plan.kv_len[b];
    if (p.units != nullptr) {
      // tiles the mask leaves something in (dense mode; the range is within the length)
      tile_begin = du.tile_begin;
      n_tiles = idle ? 0 : du.n_tiles;
      key_end = min(len, (tile_begin + n_tiles) * kTK);
    } else {
      const int n_tiles_total = (len + kTK - 1) / kTK;
      tile_begin = (int)((int64_t)s * n_tiles_total / n_split);
      const int tile_end = (int)((int64_t)(s + 1) * n_tiles_total / n_split);
      n_tiles = tile_end - tile_begin;
      key_end = min(len, tile_end * kTK);
    }
  }
  // the plan's tiles are the pipeline's steps of kTK keys (the host plans in steps of
  // the instance it launches), over [key_start, key_end)
  const int key_start = tile_begin * kTK;
  const int n_steps = n_tiles;
  bool failed = false;

  if constexpr (kManual) {
    // registers per thread: warps 0-3 (TMA, MMA issuers) 96, producers 152, softmax
    // 256; 4 warps x 32 x (96 + 152 + 256) = 64512 = the 384 x 168 launched
    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 96;");
  }
  if (warp == 0) {
    // ================= producer (TMA mode): K chunks; the first step's stages also
    // bring the matching chunk of this CTA's 64 query rows, which stay resident
    if (!kManual && n_steps > 0 && elect_one()) {
      // this CTA's kTK/2 keys of each step, 9 chunks of 64 columns, as far ahead as the
      // ring allows (only Q.K^T consumption frees stages)
      int stage = 0;
      uint32_t ephase = 0;
      for (int i = 0; i < n_steps && !failed; ++i) {
        const int key0 = key_start + i * kTK + (kTK / 2) * (int)rank;
        for (int c = 0; c < kNC; ++c) {
          if (!mbar_wait(&bars.k_empty[stage], ephase ^ 1, to)) {
            // stop issuing: a stage may still be in use, and the copies already in
            // flight (at most one ring) land before the teardown
            failed = true;
            record_status(kStatusTimeout);
            break;
          }
          if (rank == 0)
            mbar_arrive_expect_tx(&bars.k_full[stage], 2 * (kKStageBytes + (i == 0 ? kChunkBytes : 0)));
          const uint32_t fl = mapa_shared(smem_u32(&bars.k_full[stage]), 0);
          tma_load_3d_2sm(sK + stage * kKStageBytes, &tm_k, fl, 64 * c, key0, b_abs);
          if (i == 0)
            tma_load_3d_2sm(sQ + c * kChunkBytes, &tm_q, fl, 64 * c, row0 + kRowsPerCta * (int)rank,
                            b_abs);
          if (++stage == kKStages) { stage = 0; ephase ^= 1; }
        }
      }
    }
    // gather modes: this CTA's Q rows by TMA (the producers gather K and V)
    if (kManual && n_steps > 0 && elect_one()) {
      if (rank == 0) mbar_arrive_expect_tx(&bars.q_full, 2 * kNC * kChunkBytes);
      const uint32_t fq = mapa_shared(smem_u32(&bars.q_full), 0);
      for (int c = 0; c < kNC; ++c)
        tma_load_3d_2sm(sQ + c * kChunkBytes, &tm_q, fq, 64 * c, row0 + kRowsPerCta * (int)rank, b_abs);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ================= V producer (TMA mode): value columns of each tile, own ring
    if (!kManual && n_steps > 0 && elect_one()) {
      int stage = 0;
      uint32_t ephase = 0;
      for (int j = 0; j < n_steps && !failed; ++j) {
        const int key0 = key_start + j * kTK;
        for (int kg = 0; kg < kTK / 64 && !failed; ++kg)
          for (int nb = 0; nb < 2; ++nb) {
            if (!mbar_wait(&bars.v_empty[stage], ephase ^ 1, to)) {
              failed = true;  // stop issuing (see the K producer)
              record_status(kStatusTimeout);
              break;
            }
            if (rank == 0) mbar_arrive_expect_tx(&bars.v_full[stage], 2 * kVStageBytes);
            // one 16 KB box: 64 keys x 2 column blocks of 64 (this CTA's 128 value columns
            // of value half nb), landing as [column block][key][64 columns]
            const uint32_t fl = mapa_shared(smem_u32(&bars.v_full[stage]), 0);
            tma_load_4d_2sm(sV + stage * kVStageBytes, &tm_v, fl, 0, key0 + 64 * kg,
                            4 * nb + 2 * (int)rank, b_abs);
            if (++stage == kVStages) { stage = 0; ephase ^= 1; }
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================= Q.K^T issuer (leader CTA, one thread). Two threads issue MMAs:
    // an issuing thread cannot run ahead of the tensor pipe, so the time it spends
    // waiting on a barrier would leave the pipe idle; with Q.K^T and P.V on separate
    // threads one thread's wait is covered by the other's MMAs. A commit tracks the
    // MMAs of the thread that issues it.
    if (rank == 0 && n_steps > 0 && elect_one()) {
      // Descriptor bases; an operand at byte offset `off` within a region is the base
      // plus off/16 (the start address field is the low 14 bits, no carry possible
      // below 256 KB).
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      constexpr uint32_t kStageUnits = kKStageBytes >> 4;  // stage stride
      constexpr uint32_t kQUnits = kChunkBytes >> 4;       // Q chunk stride
      int kst = 0;
      uint32_t kph = 0;
      // Q chunk c is resident once the first step's stage c has landed (TMA mode) or
      // once q_full completes (gather modes)
      if (kManual && !mbar_wait(&bars.q_full, 0, to)) {
        failed = true;
        record_status(kStatusTimeout);
      }
      // On a timeout the issuer stops (no further MMAs or commits); the waits that
      // depend on its commits then time out in turn and the kernel winds down.
      for (int t = 0; t < n_steps && !failed; ++t) {
        // S buffer t % kBufs is free once the softmax has read the scores of step t - kBufs
        const int sb = t % kBufs;
        if (t >= kBufs && !mbar_wait_cluster(&bars.s_free[sb], ((t - kBufs) / kBufs) & 1, to)) {
          failed = true;
          record_status(kStatusTimeout);
          break;
        }
        const uint32_t d_s = tmem + kTmemS + sb * kSCols;
        for (int c = 0; c < kNC; ++c) {
          const bool ok = kManual ? mbar_wait_cluster(&bars.k_full[kst], kph, to)
                                  : mbar_wait(&bars.k_full[kst], kph, to);
          if (!ok) {
            failed = true;
            record_status(kStatusTimeout);
            break;
          }
          tc_fence_after();
          const uint64_t b0 = dk + (uint32_t)(kst * kStageUnits);
          const uint64_t a0 = dq + (uint32_t)(c * kQUnits);
          mma_f16_ss_2sm(d_s, a0, b0, kIdescQK, c ? 1u : 0u);
          mma_f16_ss_2sm(d_s, a0 + 2, b0 + 2, kIdescQK, 1u);
          mma_f16_ss_2sm(d_s, a0 + 4, b0 + 4, kIdescQK, 1u);
          mma_f16_ss_2sm(d_s, a0 + 6, b0 + 6, kIdescQK, 1u);
          mma_commit_2sm_mc(&bars.k_empty[kst], 0x3);
          if (++kst == kKStages) { kst = 0; kph ^= 1; }
        }
        if (failed) break;
        mma_commit_2sm_mc(&bars.s_full[sb], 0x3);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ================= P.V issuer (leader CTA, one thread): per step, wait for P, then
    // consume the V stages (64 keys x one 256-column half each) in the producer's order.
    // A (P) is read from TMEM: 16 keys per MMA are 8 columns of the P buffer.
    if (rank == 0 && n_steps > 0 && elect_one()) {
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), 8192, 1024);
      constexpr uint32_t kVUnits = kVStageBytes >> 4;   // V stage stride
      int vst = 0;
      uint32_t vph = 0;
      for (int t = 0; t < n_steps && !failed; ++t) {  // stops on a timeout, as above
        if (!mbar_wait_cluster(&bars.p_full[t & 1], (t >> 1) & 1, to)) {
          failed = true;
          record_status(kStatusTimeout);
          break;
        }
        const uint32_t p_buf = tmem + kTmemP + (t % kBufs) * kSCols;
        for (int kg = 0; kg < kTK / 64 && !failed; ++kg)
          for (int nb = 0; nb < 2; ++nb) {
            const bool ok = kManual ? mbar_wait_cluster(&bars.v_full[vst], vph, to)
                                    : mbar_wait(&bars.v_full[vst], vph, to);
            if (!ok) {
              failed = true;
              record_status(kStatusTimeout);
              break;
            }
            tc_fence_after();
            const uint32_t a0 = p_buf + (uint32_t)(kg * 32);
            const uint64_t b0 = dv + (uint32_t)(vst * kVUnits);
            const uint32_t d = tmem + kTmemO + nb * 128;
            mma_f16_ts_2sm(d, a0, b0, kIdescPV, (t > 0 || kg > 0) ? 1u : 0u);
            mma_f16_ts_2sm(d, a0 + 8, b0 + 128, kIdescPV, 1u);
            mma_f16_ts_2sm(d, a0 + 16, b0 + 256, kIdescPV, 1u);
            mma_f16_ts_2sm(d, a0 + 24, b0 + 384, kIdescPV, 1u);
            mma_commit_2sm_mc(&bars.v_empty[vst], 0x3);
            if (++vst == kVStages) { vst = 0; vph ^= 1; }
          }
        if (failed) break;
        mma_commit_2sm_mc(&bars.o_done[t & 1], 0x3);
      }
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ================= gather / dequant producers (manual modes): warps 8-9 fill the
    // K ring, warps 10-11 the V ring (64 threads per ring)
    if constexpr (kManual) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 152;");
      const bool k_side = warp < 10;
      const int pt = (threadIdx.x - 256) & 63;
      const int64_t seq_row0 = (int64_t)b_abs * p.k_seq_stride;
      const int32_t* idx_row = sparse ? list_ptr() : nullptr;
      // cache row of key position `pos` in this unit's selection, or -1 (zero fill)
      auto resolve = [&](int pos) -> int {
        if (pos >= len) return -1;
        if (!sparse) return pos < p.n_kv ? pos : -1;
        const int key = idx_row[pos];  // plain load: the gather list is written in this kernel
        if (key < 0 || key >= p.n_kv) {
          record_status(kStatusIndex);
          return -1;
        }
        return key;
      };
      // 32 consecutive values of a cache row: read, then convert to f16 and store as 4
      // swizzled 16-byte chunks of the row.
      // Blocks per batch: the next batch's loads are in flight while this one is
      // converted and stored (two batches fit the producers' 152 registers)
      constexpr int kLoadBatch = 2;
      auto load32 = [&](int key, int col32, RawBlock<kMode>& rb) {
        rb.valid = key >= 0;
        rb.odd = false;
        if (rb.valid) load_block<kMode, kRowBytes>(p.kcache, seq_row0 + key, col32, rb);
      };
      auto store32 = [&](uint8_t* row_dst, int row_in_atom, int chunk0, const RawBlock<kMode>& rb) {
        uint32_t h[16];
        block_values<kMode>(rb, h);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(row_dst + (((chunk0 + k) ^ (row_in_atom & 7)) << 4)) =
              make_uint4(h[4 * k], h[4 * k + 1], h[4 * k + 2], h[4 * k + 3]);
      };
      const int n_stages = k_side ? kKStages : kVStages;
      uint64_t* full = k_side ? bars.k_full : bars.v_full;
      uint64_t* empty = k_side ? bars.k_empty : bars.v_empty;
      uint8_t* ring = k_side ? sK : sV;
      int stage = 0;
      uint32_t ephase = 0;
      auto acquire = [&]() {
        bool ok = failed ? true : mbar_wait(&empty[stage], ephase ^ 1, to);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && !failed) {
          failed = true;
          if (lane == 0) record_status(kStatusTimeout);
        }
      };
      auto publish = [&]() {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&full[stage]), 0));
        if (++stage == n_stages) { stage = 0; ephase ^= 1; }
      };
      if (k_side) {
        // K chunk items: 128 keys (this CTA's half of the tile) x 2 blocks of 32 columns;
        // thread pt takes keys pt/2 + 32q (q = 0..3) and block half pt%2. The loads of a
        // batch of kLoadBatch blocks go out before the previous batch is converted and
        // stored, so a chunk's load latency overlaps the previous chunk's work.
        constexpr int kBpc = 4 / kLoadBatch;  // batches per stage
        for (int i = 0; i < n_steps; ++i) {
          const int kbase = key_start + i * kTK + (kTK / 2) * (int)rank;
          const int half = pt & 1;
          int keys[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) keys[q] = resolve(kbase + 32 * q + (pt >> 1));
          // Bring this CTA's rows of the tile into L2 now: the 9 stages below then read
          // them at L2 latency. The two threads of a key split the row's 128-byte lines
          // (every prefetched address lies inside the row).
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (keys[q] < 0) continue;
            const uint8_t* rowp = p.kcache + (seq_row0 + keys[q]) * kRowBytes;
            for (int off = 128 * half; off < kRowBytes; off += 256) prefetch_l2(rowp + off);
            if (half == 1) prefetch_l2(rowp + kRowBytes - 1);
          }
          RawBlock<kMode> cur[kLoadBatch];
#pragma unroll
          for (int q = 0; q < kLoadBatch; ++q) load32(keys[q], half, cur[q]);
          for (int c = 0; c < kNC; ++c) {
            uint8_t* st = nullptr;
#pragma unroll
            for (int bq = 0; bq < kBpc; ++bq) {
              const bool last = bq + 1 == kBpc;
              const int nc = last ? c + 1 : c;          // stage of the next batch
              const int nq0 = last ? 0 : (bq + 1) * kLoadBatch;
              RawBlock<kMode> nxt[kLoadBatch];
#pragma unroll
              for (int q = 0; q < kLoadBatch; ++q) {
                if (nc < kNC) load32(keys[nq0 + q], 2 * nc + half, nxt[q]);
                else { nxt[q].valid = false; nxt[q].odd = false; }
              }
              if (bq == 0) {
                acquire();
                st = ring + stage * kKStageBytes;
              }
#pragma unroll
              for (int q = 0; q < kLoadBatch; ++q) {
                const int kl = 32 * (bq * kLoadBatch + q) + (pt >> 1);
                store32(st + kl * 128, kl, 4 * half, cur[q]);
              }
#pragma unroll
              for (int q = 0; q < kLoadBatch; ++q) cur[q] = nxt[q];
            }
            publish();
          }
        }
      } else {
        // V stage items: 64 keys x this CTA's 128 value columns of one value half (4
        // blocks of 32 in two 64-column boxes); thread pt takes keys pt/4 + 16q and
        // 32-column block pt%4. As on the K side, each batch's loads go out before the
        // previous batch is stored, and the keys of the next 64-key group are resolved
        // one group ahead.
        const int q4 = pt & 3, box = q4 >> 1, half = q4 & 1;
        constexpr int kBpc = 4 / kLoadBatch;  // batches per stage
        for (int j = 0; j < n_steps; ++j) {
          const int kbase = key_start + j * kTK;
          int kc[4], kn[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) kc[q] = resolve(kbase + (pt >> 2) + 16 * q);
          RawBlock<kMode> cur[kLoadBatch];
#pragma unroll
          for (int q = 0; q < kLoadBatch; ++q) load32(kc[q], 4 * (int)rank + q4, cur[q]);
          for (int kg = 0; kg < kTK / 64; ++kg) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              kn[q] = kg + 1 < kTK / 64 ? resolve(kbase + 64 * (kg + 1) + (pt >> 2) + 16 * q) : -1;
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              uint8_t* st = nullptr;
#pragma unroll
              for (int bq = 0; bq < kBpc; ++bq) {
                // next batch: the same stage, else the other value half, else the next group
                const bool last = bq + 1 == kBpc;
                const bool next_group = last && nb == 1;
                const int nnb = last ? nb ^ 1 : nb;
                const int nq0 = last ? 0 : (bq + 1) * kLoadBatch;
                RawBlock<kMode> nxt[kLoadBatch];
#pragma unroll
                for (int q = 0; q < kLoadBatch; ++q) {
                  const int key = next_group ? kn[nq0 + q] : kc[nq0 + q];
                  if (!next_group || kg + 1 < kTK / 64) load32(key, 8 * nnb + 4 * (int)rank + q4, nxt[q]);
                  else { nxt[q].valid = false; nxt[q].odd = false; }
                }
                if (bq == 0) {
                  acquire();
                  st = ring + stage * kVStageBytes + box * 8192;
                }
#pragma unroll
                for (int q = 0; q < kLoadBatch; ++q) {
                  const int kl = (pt >> 2) + 16 * (bq * kLoadBatch + q);
                  store32(st + kl * 128, kl, 4 * half, cur[q]);
                }
#pragma unroll
                for (int q = 0; q < kLoadBatch; ++q) cur[q] = nxt[q];
              }
              publish();
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) kc[q] = kn[q];
          }
        }
      }
    }
  } else if (warp >= 4) {
    // ================= softmax / correction / epilogue warpgroup
    if constexpr (kManual) asm volatile("setmaxnreg.inc.sync.aligned.u32 256;");
    const int L = threadIdx.x - 128;          // TMEM lane
    const int r = L & 63;                     // row within this CTA
    const int kh = L >> 6;                    // which half of a step's keys this lane holds
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int row = row0 + kRowsPerCta * (int)rank + r;  // row within the sequence
    const bool row_valid = row < plan.rows && !idle;
    const int tok = row / plan.n_head;
    const uint16_t* mrow = (p.mask != nullptr && row_valid)
                               ? p.mask + (int64_t)b_abs * p.mask_seq_stride +
                                     (int64_t)tok * p.mask_row_stride
                               : nullptr;
    const uint32_t s_free_l0 = mapa_shared(smem_u32(&bars.s_free[0]), 0);
    const uint32_t s_free_l1 = mapa_shared(smem_u32(&bars.s_free[kBufs - 1]), 0);
    // variants: the ALiBi bias is slope * (key - position of the query), the query
    // tokens being the last n_q positions of the sequence (with sinks the softmax is no
    // longer shift invariant, so this position is the defined one)
    const float slope =
        (kVariant && p.slopes != nullptr && row_valid) ? __ldg(p.slopes + row % plan.n_head) : 0.f;
    const int alibi_ref = len - plan.n_q + tok;
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

    float m_ref = -INFINITY;  // reference max (natural units) used for exponentiation
    float l_part = 0.f;       // this lane's half of the row sum, relative to m_ref

    constexpr int kHalf = kTK / 2;  // keys of one lane in a step
    // The mask loads of a step are issued while the previous step is still being
    // processed (after its exponentials), so their latency is hidden. Full tiles take
    // this vector path (zeros without a mask); a ragged last tile goes key by key.
    uint4 mvec[kHalf / 8];
    // Sparse (index list): every tile takes this path; mvec then holds, as f16 pairs,
    // the mask value of each position's kept cell (0 without a mask) or -inf for a
    // position past the list or an invalid cell. The index loads of a group of 64
    // positions are issued together, then its mask gathers.
    // A row past the sequence's rows is computed but never stored: it takes the vector
    // path with a zero mask, so that its lanes follow the same path as their warp's
    // valid rows.
    // A ragged tile (the unit's keys end inside it) takes the vector path too while its
    // mask loads stay inside the mask row, and then drops the cells past the unit's last
    // key; otherwise it goes key by key.
    auto mask_vec_ok = [&](int t) {
      if ((kManual && sparse) || !row_valid) return true;
      const int k0 = key_start + t * kTK + kHalf * kh;
      if (mrow == nullptr) return true;  // no mask: zeros
      return p.mask_vec_ok && (k0 + kHalf <= key_end || k0 + kHalf <= p.n_kv);
    };
    auto load_mask = [&](int t) {
      const int k0 = key_start + t * kTK + kHalf * kh;
      if (!row_valid) {
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) mvec[c] = make_uint4(0u, 0u, 0u, 0u);
      } else if (kManual && sparse) {
        const int32_t* ix = list_ptr();
        uint32_t* mw = reinterpret_cast<uint32_t*>(mvec);
        static_assert(!kManual || kHalf == 128, "index-list steps of 256 keys");
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          int cl[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const int pos = k0 + 64 * g + j;
            cl[j] = pos < key_end ? ix[pos] : -1;
          }
          unsigned short hv[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const bool ok = cl[j] >= 0 && cl[j] < p.n_kv;
            unsigned short h = ok ? (unsigned short)0 : (unsigned short)0xFC00u;  // 0 or -inf
            if (ok && mrow != nullptr) h = __ldg(mrow + cl[j]);
            hv[j] = h;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) mw[32 * g + j] = (uint32_t)hv[2 * j] | ((uint32_t)hv[2 * j + 1] << 16);
        }
      } else if (mrow == nullptr) {
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) mvec[c] = make_uint4(0u, 0u, 0u, 0u);
      } else {
        const uint4* mv = reinterpret_cast<const uint4*>(mrow + k0);
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) mvec[c] = __ldg(mv + c);
      }
    };
    // The mask cells of a step are a fresh DRAM read (a decode reads each once), and their
    // load for step i+1 is issued during step i: too late to hide the latency of a loaded
    // DRAM. Each lane's slice is therefore brought into L2 kMaskAhead steps ahead (dense
    // steps whose slice lies inside the mask row).
    constexpr int kMaskAhead = 4;
    auto prefetch_mask = [&](int t) {
      if ((kManual && sparse) || mrow == nullptr) return;
      const int k0 = key_start + t * kTK + kHalf * kh;
      if (k0 + kHalf > p.n_kv) return;
#pragma unroll
      for (int c = 0; c < kHalf * 2; c += 128) prefetch_l2(reinterpret_cast<const uint8_t*>(mrow + k0) + c);
    };
    for (int t = 0; t < kMaskAhead && t < n_steps; ++t) prefetch_mask(t);
    bool vec_next = n_steps > 0 && mask_vec_ok(0);
    if (vec_next) load_mask(0);

    for (int i = 0; i < n_steps; ++i) {
      const int sb = i & 1;          // max-exchange slot and p_full barrier
      const int buf = i % kBufs;     // S and P buffers of this step
      const int key0 = key_start + i * kTK + kHalf * kh;
      const bool vec_mask = vec_next;
      wait_local(&bars.s_full[buf], (i / kBufs) & 1);
      tc_fence_after();
      // scores x = scale * s + mask (natural units); cells beyond the unit's keys are
      // dropped. kHalf values per lane, read from TMEM with kHalf / 32 loads and one wait.
      uint32_t sr[kHalf];
#pragma unroll
      for (int q = 0; q < kHalf / 32; ++q)
        tmem_ld32(tmem + lane_base + kTmemS + buf * kSCols + 32 * q,
                  *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * q));
      tmem_wait_ld();
      // the scores are in registers: Q.K^T may overwrite this S buffer (the loads are
      // complete, so a relaxed arrive suffices)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(buf ? s_free_l1 : s_free_l0);
      float x[kHalf];
      if constexpr (kVariant) {
        // softcapped (or plainly scaled) score, then the mask, then the ALiBi bias
        const float cap = p.softcap;
        const float sc = cap > 0.f ? p.scale / cap : 0.f;
        const uint32_t* mw = reinterpret_cast<const uint32_t*>(mvec);
#pragma unroll
        for (int j = 0; j < kHalf; ++j) {
          const int key = key0 + j;
          float sv = __uint_as_float(sr[j]);
          sv = cap > 0.f ? cap * tanhf(sv * sc) : sv * p.scale;
          float mv;
          if (vec_mask) {
            const uint32_t w = mw[j >> 1];
            mv = __half2float(__ushort_as_half((unsigned short)((j & 1) ? (w >> 16) : (w & 0xFFFFu))));
          } else {
            mv = (mrow != nullptr && key < key_end) ? __half2float(__ushort_as_half(__ldg(mrow + key))) : 0.f;
          }
          const float xv = fmaf(slope, (float)(key - alibi_ref), sv + mv);
          x[j] = key < key_end ? xv : -INFINITY;
        }
      } else {
        if (vec_mask) {
#pragma unroll
          for (int c = 0; c < kHalf / 8; ++c) {
            const uint4 v = mvec[c];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[h]));
              const int j = 8 * c + 2 * h;
              x[j] = fmaf(__uint_as_float(sr[j]), p.scale, f.x);
              x[j + 1] = fmaf(__uint_as_float(sr[j + 1]), p.scale, f.y);
            }
          }
          if (key0 + kHalf > key_end) {  // ragged tile: cells past the unit's keys drop out
#pragma unroll
            for (int j = 0; j < kHalf; ++j)
              if (key0 + j >= key_end) x[j] = -INFINITY;
          }
        } else {
#pragma unroll
          for (int j = 0; j < kHalf; ++j) {
            const int key = key0 + j;
            float mv = 0.f;
            if (mrow != nullptr && key < key_end)
              mv = __half2float(__ushort_as_half(__ldg(mrow + key)));
            x[j] = key < key_end ? fmaf(__uint_as_float(sr[j]), p.scale, mv) : -INFINITY;
          }
        }
      }
      // row max over this lane's kHalf keys (8 independent chains), then over the pair
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) m8[u] = x[u];
#pragma unroll
      for (int j = 8; j < kHalf; ++j) m8[j & 7] = fmaxf(m8[j & 7], x[j]);
      float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      xmax[sb * 128 + L] = mt;
      named_bar_sync(1, 128);
      mt = fmaxf(mt, xmax[sb * 128 + (L ^ 64)]);

      const bool need = mt > m_ref + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx((m_ref - mt) * kLog2e);  // 0 when m_ref = -inf
        m_ref = mt;
      }
      // p = 2^(x log2 e - m_ref log2 e), rounded to f16 for the P.V MMA; the row sum
      // adds the unrounded values (8 independent chains)
      const float nb = (m_ref == -INFINITY) ? 0.f : -m_ref * kLog2e;
      uint32_t pk[kHalf / 2];
      float ls8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ls8[u] = 0.f;
#pragma unroll
      for (int j = 0; j < kHalf / 2; ++j) {
        const float e0 = ex2_approx(fmaf(x[2 * j], kLog2e, nb));
        const float e1 = ex2_approx(fmaf(x[2 * j + 1], kLog2e, nb));
        __half2 h2 = __floats2half2_rn(e0, e1);
        pk[j] = *reinterpret_cast<uint32_t*>(&h2);
        ls8[j & 7] += e0 + e1;
      }
      const float lsum = ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
      l_part = l_part * alpha + lsum;
      // next step's mask: its loads overlap the rest of this step (the scores are dead)
      vec_next = i + 1 < n_steps && mask_vec_ok(i + 1);
      if (vec_next) load_mask(i + 1);
      if (i + kMaskAhead < n_steps) prefetch_mask(i + kMaskAhead);

      // P goes to TMEM as the A operand of P.V. That MMA reads A for the value columns
      // of the first N half from lanes 0-63 and for the second half from lanes 64-127,
      // so each of a row's two lanes needs all kTK keys: the lanes of a row swap their
      // kHalf keys through shared memory (the previous step's reads of the exchange
      // buffer finished before the max exchange barrier above).
      {
        // keys 0..kHalf-1 of the step in the buffer's first kHalf/2 columns, the other
        // kHalf keys in the next kHalf/2; kXRounds rounds of kXWords f16 pairs
        const uint32_t a = tmem + lane_base + kTmemP + buf * kSCols;
        const uint32_t a_own = a + (kHalf / 2) * kh, a_peer = a + (kHalf / 2) * (kh ^ 1);
#pragma unroll
        for (int rd = 0; rd < kXRounds; ++rd) {
          const int w0 = rd * kXWords;
          if (rd > 0) named_bar_sync(1, 128);  // the partner has read the previous round
#pragma unroll
          for (int gq = 0; gq < kXWords / 4; ++gq)
            sX[gq * 128 + L] = make_uint4(pk[w0 + 4 * gq], pk[w0 + 4 * gq + 1], pk[w0 + 4 * gq + 2],
                                          pk[w0 + 4 * gq + 3]);
          named_bar_sync(1, 128);
          uint32_t pw[kXWords];
#pragma unroll
          for (int gq = 0; gq < kXWords / 4; ++gq) {
            const uint4 v = sX[gq * 128 + (L ^ 64)];
            pw[4 * gq] = v.x; pw[4 * gq + 1] = v.y; pw[4 * gq + 2] = v.z; pw[4 * gq + 3] = v.w;
          }
          if (rd == 0) {
            // this P buffer is free once P.V of step i - kBufs has completed (with one
            // buffer that also leaves O free)
            if (i >= kBufs) wait_local(&bars.o_done[(i - kBufs) & 1], ((i - kBufs) >> 1) & 1);
            tc_fence_after();
          }
#pragma unroll
          for (int u = 0; u < kXWords / 32; ++u)
            tmem_st32(a_own + w0 + 32 * u, *reinterpret_cast<uint32_t(*)[32]>(pk + w0 + 32 * u));
#pragma unroll
          for (int u = 0; u < kXWords / 32; ++u)
            tmem_st32(a_peer + w0 + 32 * u, *reinterpret_cast<uint32_t(*)[32]>(pw + 32 * u));
        }
        tmem_wait_st();
      }
      // rescale O (only when some row of this warp raised its reference max), once
      // P.V(i-1) has completed (P.V(i) waits for this step's P)
      if (__any_sync(0xffffffffu, need && i > 0)) {
        if (kBufs > 1) {
          wait_local(&bars.o_done[(i - 1) & 1], ((i - 1) >> 1) & 1);
          tc_fence_after();
        }
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
      // P is in TMEM and complete (tcgen05.wait::st above): a relaxed arrive hands it over
      // without waiting for this thread's mask loads of the next tile, which a release
      // would (that wait cost 1-4 us per tile)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(sb ? p_full_l1 : p_full_l0);
    }

    // ---- epilogue
    if (n_steps > 0) wait_local(&bars.o_done[(n_steps - 1) & 1], ((n_steps - 1) >> 1) & 1);
    // a dependent (combine) launch may start scheduling; it waits for this grid's end
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    tc_fence_after();
    xl[L] = l_part;
    named_bar_sync(1, 128);
    const float l_tot = l_part + xl[L ^ 64];
    const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
    const int ws_slot = p.units != nullptr ? du.slot
                        : (plan.ws_base[b] >= 0 ? plan.ws_base[b] + g * n_split + s : -1);
    // O / l goes out through shared memory: each warp stages its 32 rows as eight
    // 32 x 32 fp32 boxes, or for a split partial four 32 x 64 f16 boxes (128-byte rows,
    // 16-byte chunks XOR-swizzled by row, the layout of a 128-byte-swizzle tensor map),
    // and one lane stores them with TMA.
    // Every MMA has finished (last o_done), so the operand rings are free; the 4
    // warps use the first 128 KB. Rows beyond the tensor are clipped by the store.
    // A warp whose 32 rows all lie past the sequence's rows has nothing to store.
    if (__any_sync(0xffffffffu, row_valid)) {
      const int wq = warp - 4;  // row half (wq & 1) of key half kh = wq >> 1
      uint8_t* wbox = smem + wq * 8 * 4096;
      const bool part = ws_slot >= 0;  // f16 partial (tm_w) or the fp32 output (tm_o)
      const CUtensorMap* tm = part ? &tm_w : &tm_o;
      const int y = (ws_slot >= 0 ? ws_slot * kRowsPerGroup : row0) + kRowsPerCta * (int)rank +
                    32 * (wq & 1);
      const int z = ws_slot >= 0 ? 0 : b_abs;
      // groups of kEpi 32-column TMEM loads under one wait (fewer in the manual modes,
      // whose register budget is smaller); each group's boxes are stored while the next
      // group is read
      constexpr int kEpi = kManual ? 2 : 4;
#pragma unroll 1
      for (int g0 = 0; g0 < 8; g0 += kEpi) {
        uint32_t v[kEpi][32];
        if (n_steps > 0) {
#pragma unroll
          for (int u = 0; u < kEpi; ++u) tmem_ld32(tmem + lane_base + kTmemO + 32 * (g0 + u), v[u]);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int u = 0; u < kEpi; ++u)
#pragma unroll
            for (int j = 0; j < 32; ++j) v[u][j] = 0u;
        }
        if (part) {
          // TMEM groups i, i+1 (i even) are 64 adjacent value columns: one f16 box
#pragma unroll
          for (int u = 0; u < kEpi; u += 2) {
            uint8_t* rowp = wbox + ((g0 + u) >> 1) * 4096 + lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t* x = &v[u + (c >> 2)][8 * (c & 3)];
              uint32_t h[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const __half2 hh = __floats2half2_rn(__uint_as_float(x[2 * k]) * inv_l,
                                                     __uint_as_float(x[2 * k + 1]) * inv_l);
                h[k] = *reinterpret_cast<const uint32_t*>(&hh);
              }
              *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < kEpi; ++u) {
            uint8_t* rowp = wbox + (g0 + u) * 4096 + lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<float4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                  make_float4(__uint_as_float(v[u][4 * c]) * inv_l, __uint_as_float(v[u][4 * c + 1]) * inv_l,
                              __uint_as_float(v[u][4 * c + 2]) * inv_l,
                              __uint_as_float(v[u][4 * c + 3]) * inv_l);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // TMEM columns 32i..32i+31 are value columns 256 (i / 4) + 128 kh + 32 (i % 4)
          if (part) {
            for (int u = 0; u < kEpi; u += 2) {
              const int i = g0 + u;
              tma_store_3d(tm, wbox + (i >> 1) * 4096, 256 * (i >> 2) + 128 * kh + 32 * (i & 3), y, z);
            }
          } else {
            for (int u = 0; u < kEpi; ++u) {
              const int i = g0 + u;
              tma_store_3d(tm, wbox + i * 4096, 256 * (i >> 2) + 128 * kh + 32 * (i & 3), y, z);
            }
          }
          bulk_commit_group();
        }
      }
      if (lane == 0) bulk_wait_group_read0();
      __syncwarp();
    }
    if (ws_slot >= 0 && kh == 0 && row_valid)
      p.ws_lse[(int64_t)ws_slot * kRowsPerGroup + kRowsPerCta * rank + r] =
          l_tot > 0.f ? m_ref * kLog2e + __log2f(l_tot) : -INFINITY;
  }

  // ---- teardown
  // A thread that gave up stops issuing at once; the copies and MMAs it issued before
  // (at most one ring of stages) land well within 100 us, before the cluster barrier
  // lets either CTA exit or free TMEM.
  if (failed) sleep_at_least_ns(100000);
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

// Four consecutive f16 partial values (one 8-byte load) as floats.
__device__ __forceinline__ float4 part4(uint2 r) {
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&r.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&r.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// LSE combine of split-KV partials (one CTA of 128 threads per query row, thread t
// owning value columns 4t..4t+3):
//   O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M),  M = max_s lse_s,
// where O_s is split s normalised by its own sum and lse_s = log2 of that sum
// relative to the split's max; splits with no kept cell have lse_s = -inf.
// Lane s of every warp holds lse_s (the host uses this kernel up to 16 splits). The
// loads of the first 16 partial rows are issued together with the lse loads, before
// the weights are known, so a row with at most 16 splits costs one round trip to
// memory. Launched as a programmatic dependent of the forward kernel:
// griddepcontrol.wait returns once the forward grid has completed and its partials
// are visible.
__global__ void __launch_bounds__(128) mla_combine_kernel(const __grid_constant__ Plan plan,
                                                          const uint16_t* __restrict__ ws_o,
                                                          const float* __restrict__ ws_lse,
                                                          float* __restrict__ out,
                                                          int64_t out_seq_stride,
                                                          const float* __restrict__ sinks,
                                                          float* __restrict__ out_lse,
                                                          const int2* __restrict__ gsplit) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.y;
  const int row = blockIdx.x;
  if (row >= plan.rows) return;
  const int g = row / kRowsPerGroup;
  // the group's first partial slot and splits: the host plan's, or the device plan's table
  int slot0, ns;
  if (gsplit != nullptr) {
    const int2 gs = gsplit[b * plan.groups + g];
    slot0 = gs.x;
    ns = min(gs.y, 32);
  } else {
    slot0 = plan.ws_base[b] >= 0 ? plan.ws_base[b] + g * plan.n_split[b] : -1;
    ns = min(plan.n_split[b], 32);
  }
  if (slot0 < 0) return;  // written by the attention kernel itself
  const int lane = threadIdx.x & 31;
  const int rin = row % kRowsPerGroup;
  const float* lse_col = ws_lse + (int64_t)slot0 * kRowsPerGroup + rin;
  constexpr int64_t kSplitStride4 = (int64_t)kRowsPerGroup * kDV / 4;  // 4-value groups per slot
  const uint2* src0 =
      reinterpret_cast<const uint2*>(ws_o + ((int64_t)slot0 * kRowsPerGroup + rin) * kDV) + threadIdx.x;
  const float lse_l = lane < ns ? __ldg(lse_col + (int64_t)lane * kRowsPerGroup) : -INFINITY;
  constexpr int kFirst = 16;
  uint2 v[kFirst];
#pragma unroll
  for (int u = 0; u < kFirst; ++u) v[u] = u < ns ? __ldg(src0 + u * kSplitStride4) : make_uint2(0u, 0u);
  float mx = lse_l;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  // an attention sink is one more split with lse = sink (log2 units) and no value
  const float snk = sinks != nullptr ? __ldg(sinks + row % plan.n_head) * kLog2e : -INFINITY;
  mx = fmaxf(mx, snk);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (mx != -INFINITY) {
    const float wl = lse_l == -INFINITY ? 0.f : ex2_approx(lse_l - mx);
    wsum = wl;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    if (snk != -INFINITY) wsum += ex2_approx(snk - mx);
#pragma unroll
    for (int u = 0; u < kFirst; ++u) {
      const float w = __shfl_sync(0xffffffffu, wl, u);  // 0 past ns
      const float4 x = part4(v[u]);
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
    }
    for (int s = kFirst; s < ns; ++s) {
      const float w = __shfl_sync(0xffffffffu, wl, s);
      const float4 x = part4(__ldg(src0 + s * kSplitStride4));
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
    }
    const float inv = 1.f / wsum;
    acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
  }
  float4* dst = reinterpret_cast<float4*>(out + (int64_t)(plan.seq_offset + b) * out_seq_stride +
                                          (int64_t)row * kDV);
  dst[threadIdx.x] = acc;
  // the row's natural log-sum-exp (mx and wsum are in log2 units)
  if (out_lse != nullptr && threadIdx.x == 0)
    out_lse[(int64_t)(plan.seq_offset + b) * plan.rows + row] =
        mx == -INFINITY ? -INFINITY : (mx + log2f(wsum)) * kLn2;
}

// The same combine for rows with many splits: one CTA of 4 warps per (query row,
// quarter of the value columns), lane l owning columns 128 q + 4l .. +3 of quarter q.
// Every warp holds the lse of the first 96 splits (lane l: splits l, l+32, l+64) and
// derives the weights itself; warp w sums the splits s = w (mod 4). The lse loads and
// the loads of up to kCombPer partial rows per warp are issued together, so a row with
// at most 96 splits costs one round trip to memory; the warps' sums meet in shared
// memory. Launched as a programmatic dependent of the forward kernel.
constexpr int kCombPer = 24;  // partial rows per warp held in registers

__global__ void __launch_bounds__(128)
    mla_combine_wide_kernel(const __grid_constant__ Plan plan, const uint16_t* __restrict__ ws_o,
                            const float* __restrict__ ws_lse, float* __restrict__ out,
                            int64_t out_seq_stride, const float* __restrict__ sinks,
                            float* __restrict__ out_lse, const int2* __restrict__ gsplit) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float4 red[4][32];
  const int b = blockIdx.z;
  const int row = blockIdx.x;
  const int qtr = blockIdx.y;
  if (row >= plan.rows) return;  // the whole CTA leaves
  const int g = row / kRowsPerGroup;
  // the group's first partial slot and splits: the host plan's, or the device plan's table
  int ns, slot0;
  if (gsplit != nullptr) {
    const int2 gs = gsplit[b * plan.groups + g];
    slot0 = gs.x;
    ns = gs.y;
  } else {
    ns = plan.n_split[b];
    slot0 = plan.ws_base[b] >= 0 ? plan.ws_base[b] + g * ns : -1;
  }
  if (slot0 < 0) return;  // written by the attention kernel itself
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int rin = row % kRowsPerGroup;
  const float* lse_col = ws_lse + (int64_t)slot0 * kRowsPerGroup + rin;
  constexpr int64_t kSplitStride4 = (int64_t)kRowsPerGroup * kDV / 4;  // 4-value groups per slot
  const uint2* src0 = reinterpret_cast<const uint2*>(ws_o + ((int64_t)slot0 * kRowsPerGroup + rin) * kDV) +
                      qtr * 32 + lane;
  float lse[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int sp = lane + 32 * k;
    lse[k] = sp < ns ? __ldg(lse_col + (int64_t)sp * kRowsPerGroup) : -INFINITY;
  }
  uint2 v[kCombPer];
#pragma unroll
  for (int j = 0; j < kCombPer; ++j) {
    const int sp = warp + 4 * j;
    v[j] = sp < ns ? __ldg(src0 + sp * kSplitStride4) : make_uint2(0u, 0u);
  }
  float mx = fmaxf(fmaxf(lse[0], lse[1]), lse[2]);
  for (int sp = lane + 96; sp < ns; sp += 32) mx = fmaxf(mx, __ldg(lse_col + (int64_t)sp * kRowsPerGroup));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  // an attention sink is one more split with lse = sink (log2 units) and no value
  const float snk = sinks != nullptr ? __ldg(sinks + row % plan.n_head) * kLog2e : -INFINITY;
  mx = fmaxf(mx, snk);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (mx != -INFINITY) {  // the same for every warp
    float w[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) w[k] = lse[k] == -INFINITY ? 0.f : ex2_approx(lse[k] - mx);
    wsum = (w[0] + w[1]) + w[2];
    for (int sp = lane + 96; sp < ns; sp += 32) {
      const float l = __ldg(lse_col + (int64_t)sp * kRowsPerGroup);
      wsum += l == -INFINITY ? 0.f : ex2_approx(l - mx);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    if (snk != -INFINITY) wsum += ex2_approx(snk - mx);
#pragma unroll
    for (int j = 0; j < kCombPer; ++j) {
      const int sp = warp + 4 * j;  // the same in every lane
      const float wk = sp < 32 ? w[0] : (sp < 64 ? w[1] : w[2]);
      const float ww = __shfl_sync(0xffffffffu, wk, sp & 31);
      if (sp < ns && sp < 96) {
        const float4 x = part4(v[j]);
        acc.x = fmaf(ww, x.x, acc.x);
        acc.y = fmaf(ww, x.y, acc.y);
        acc.z = fmaf(ww, x.z, acc.z);
        acc.w = fmaf(ww, x.w, acc.w);
      }
    }
    // splits past 96 (this warp's share), one at a time
    for (int sp = warp + 96; sp < ns; sp += 4) {
      const float l = __ldg(lse_col + (int64_t)sp * kRowsPerGroup);
      const float ww = l == -INFINITY ? 0.f : ex2_approx(l - mx);
      const float4 x = part4(__ldg(src0 + sp * kSplitStride4));
      acc.x = fmaf(ww, x.x, acc.x);
      acc.y = fmaf(ww, x.y, acc.y);
      acc.z = fmaf(ww, x.z, acc.z);
      acc.w = fmaf(ww, x.w, acc.w);
    }
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float4 t = red[0][lane];
#pragma unroll
    for (int q = 1; q < 4; ++q) {
      const float4 o = red[q][lane];
      t.x += o.x; t.y += o.y; t.z += o.z; t.w += o.w;
    }
    if (mx != -INFINITY) {
      const float inv = 1.f / wsum;
      t.x *= inv; t.y *= inv; t.z *= inv; t.w *= inv;
    }
    float4* dst = reinterpret_cast<float4*>(out + (int64_t)(plan.seq_offset + b) * out_seq_stride +
                                            (int64_t)row * kDV) + qtr * 32 + lane;
    *dst = t;
    // the row's natural log-sum-exp (mx and wsum are in log2 units)
    if (out_lse != nullptr && qtr == 0 && lane == 0)
      out_lse[(int64_t)(plan.seq_offset + b) * plan.rows + row] =
          mx == -INFINITY ? -INFINITY : (mx + log2f(wsum)) * kLn2;
  }
}

// Merge of n_parts partial results of the same rows over disjoint key sets
// (mla_fa_combine): the log-sum-exp combine across calls, with natural-log lse.
// One CTA of 128 threads per row (grid-stride over the rows), thread i owning value
// columns 4i..4i+3; every thread reads the parts' lse (the same addresses across the
// CTA), then sums the weighted parts. Part p's rows start o_stride (and lse_stride)
// floats after part p - 1's, so the parts may sit in one packed buffer per part.
__global__ void __launch_bounds__(128)
    mla_merge_kernel(const float* __restrict__ o_parts, int64_t o_stride, const float* __restrict__ lse_parts,
                     int64_t lse_stride, int n_parts, int64_t rows, float* __restrict__ out,
                     float* __restrict__ out_lse) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    float mx = -INFINITY;
    for (int p = 0; p < n_parts; ++p) mx = fmaxf(mx, __ldg(lse_parts + (int64_t)p * lse_stride + r));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (mx != -INFINITY) {
#pragma unroll 4
      for (int p = 0; p < n_parts; ++p) {
        const float l = __ldg(lse_parts + (int64_t)p * lse_stride + r);
        const float w = l == -INFINITY ? 0.f : ex2_approx((l - mx) * kLog2e);
        if (w == 0.f) continue;  // the same in every thread of the CTA
        const float4 x =
            __ldg(reinterpret_cast<const float4*>(o_parts + (int64_t)p * o_stride + r * kDV) + threadIdx.x);
        acc.x = fmaf(w, x.x, acc.x);
        acc.y = fmaf(w, x.y, acc.y);
        acc.z = fmaf(w, x.z, acc.z);
        acc.w = fmaf(w, x.w, acc.w);
        wsum += w;
      }
      const float inv = 1.f / wsum;
      acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
    }
    reinterpret_cast<float4*>(out + r * kDV)[threadIdx.x] = acc;
    if (out_lse != nullptr && threadIdx.x == 0) out_lse[r] = mx == -INFINITY ? -INFINITY : mx + logf(wsum);
  }
}

// LSE combine fused with the value up-projection W_UV of each head (ik_llama.cpp -mla
// guide, section on tensor derivation: wkv_b is split per head into wk_b and wv_b,
// "128 x 512 x 128"; Vulkan FA article, section 6.1: fold the projection matrices into
// the attention kernel):
//   out_proj[b][t][h][n] = sum_{d<512} O[b][t][h][d] * wv[h][d][n],   n < 128,
// where O is the combined, normalised attention row (as mla_combine_kernel computes it).
// A cluster of 4 CTAs per (head h, batch of kProjRows (b, t) rows of this launch); CTA q
// of the cluster takes latent columns [128q, 128q+128). Its 32 KB slice of W_h is one
// contiguous bulk copy into shared memory, issued first. The combine is separable by
// column, so CTA q reads only its quarter of the partial rows: warp w combines row w of
// the batch (lane l: columns 4l..4l+3 of the quarter), with the lse of up to 96 splits
// and the first 16 partial rows loaded together. Then thread (warp w, lane l) multiplies
// the quarter's 128 latent columns of row l / 4 into output columns 16 w + 4 (l % 4) .. +3
// (each warp its own 16 output columns, so no sum across warps), and the 4 CTAs' sums
// meet over distributed shared memory (CTA q adds up rows 2q, 2q+1). Launched as a
// programmatic dependent of the forward kernel; the weight slice, which the forward
// does not write, is requested before the wait for the forward's partials.
constexpr int kProjRows = 8;
constexpr int kProjDim = 128;
constexpr int kProjWBytes = 128 * kProjDim * 2;                       // W slice: 32 KB
constexpr int kProjORow = 132;                                        // padded o_s row
constexpr int kProjSmem = kProjWBytes + kProjRows * kProjORow * 4 +   // W, o_s
                          kProjRows * kProjDim * 4 + 16;              // CTA sum, barrier

__global__ void __cluster_dims__(1, 4, 1) __launch_bounds__(256, 2)
    mla_combine_proj_kernel(const __grid_constant__ Plan plan, const uint16_t* __restrict__ ws_o,
                            const float* __restrict__ ws_lse, const uint16_t* __restrict__ wv,
                            float* __restrict__ out_proj, int64_t op_seq_stride,
                            const float* __restrict__ sinks) {
  extern __shared__ __align__(128) uint8_t proj_smem[];
  // a launch with too little dynamic shared memory reports and returns (every CTA takes
  // this branch, so no cluster barrier is left waiting)
  if (dynamic_smem_bytes() < (uint32_t)kProjSmem) {
    if (threadIdx.x == 0) record_status(kStatusLaunch);
    return;
  }
  const uint16_t* w_s = reinterpret_cast<const uint16_t*>(proj_smem);               // [128 d][128 n]
  float (*o_s)[kProjORow] = reinterpret_cast<float (*)[kProjORow]>(proj_smem + kProjWBytes);
  float (*part)[kProjDim] =
      reinterpret_cast<float (*)[kProjDim]>(proj_smem + kProjWBytes + kProjRows * kProjORow * 4);
  uint64_t* wbar = reinterpret_cast<uint64_t*>(proj_smem + kProjWBytes + kProjRows * kProjORow * 4 +
                                               kProjRows * kProjDim * 4);
  const int h = blockIdx.x;
  const uint32_t qtr = cluster_ctarank();
  const int j0 = (int)(blockIdx.y >> 2) * kProjRows;
  const int nrows = plan.n_seq * plan.n_q;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int64_t kSplitStride4 = (int64_t)kRowsPerGroup * kDV / 4;
  // this CTA's slice of W_h first: it is an input of the call, not written by the
  // forward kernel, so it is requested before the wait for the forward's partials
  if (threadIdx.x == 0) {
    mbar_init(wbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(wbar, kProjWBytes);
    bulk_load(proj_smem, wv + ((int64_t)h * kDV + 128 * qtr) * kProjDim, kProjWBytes, wbar);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {
    // ---- combine columns 128 qtr + 4 lane .. +3 of row j0 + warp
    const int j = j0 + warp;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < nrows) {
      const int b = j / plan.n_q, t = j - (j / plan.n_q) * plan.n_q;
      const int row = t * plan.n_head + h;
      const int ns = plan.n_split[b];
      const int slot0 = plan.ws_base[b] + (row / kRowsPerGroup) * ns;
      const int rin = row % kRowsPerGroup;
      const float* lse_col = ws_lse + (int64_t)slot0 * kRowsPerGroup + rin;
      const uint2* src0 = reinterpret_cast<const uint2*>(ws_o + ((int64_t)slot0 * kRowsPerGroup + rin) * kDV) +
                          32 * qtr + lane;
      float lse[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int sp = lane + 32 * k;
        lse[k] = sp < ns ? __ldg(lse_col + (int64_t)sp * kRowsPerGroup) : -INFINITY;
      }
      uint2 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        v[u] = u < ns ? __ldg(src0 + (int64_t)u * kSplitStride4) : make_uint2(0u, 0u);
      float mx = fmaxf(fmaxf(lse[0], lse[1]), lse[2]);
      for (int sp = lane + 96; sp < ns; sp += 32) mx = fmaxf(mx, __ldg(lse_col + (int64_t)sp * kRowsPerGroup));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      // an attention sink is one more split with lse = sink (log2 units) and no value
      const float snk = sinks != nullptr ? __ldg(sinks + h) * kLog2e : -INFINITY;
      mx = fmaxf(mx, snk);
      if (mx != -INFINITY) {
        float wk[3];
#pragma unroll
        for (int k = 0; k < 3; ++k) wk[k] = lse[k] == -INFINITY ? 0.f : ex2_approx(lse[k] - mx);
        float wsum = (wk[0] + wk[1]) + wk[2];
        for (int sp = lane + 96; sp < ns; sp += 32) {
          const float l = __ldg(lse_col + (int64_t)sp * kRowsPerGroup);
          wsum += l == -INFINITY ? 0.f : ex2_approx(l - mx);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
        if (snk != -INFINITY) wsum += ex2_approx(snk - mx);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float w = __shfl_sync(0xffffffffu, wk[0], u);  // 0 past ns
          const float4 x = part4(v[u]);
          acc.x = fmaf(w, x.x, acc.x);
          acc.y = fmaf(w, x.y, acc.y);
          acc.z = fmaf(w, x.z, acc.z);
          acc.w = fmaf(w, x.w, acc.w);
        }
        for (int sp = 16; sp < ns; ++sp) {
          float w;  // split sp's weight, the same in every lane
          if (sp < 96) {
            const float x = sp < 32 ? wk[0] : (sp < 64 ? wk[1] : wk[2]);
            w = __shfl_sync(0xffffffffu, x, sp & 31);
          } else {
            const float l = __ldg(lse_col + (int64_t)sp * kRowsPerGroup);
            w = l == -INFINITY ? 0.f : ex2_approx(l - mx);
          }
          const float4 x = part4(__ldg(src0 + (int64_t)sp * kSplitStride4));
          acc.x = fmaf(w, x.x, acc.x);
          acc.y = fmaf(w, x.y, acc.y);
          acc.z = fmaf(w, x.z, acc.z);
          acc.w = fmaf(w, x.w, acc.w);
        }
        const float inv = 1.f / wsum;
        acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
      }
    }
    *reinterpret_cast<float4*>(&o_s[warp][4 * lane]) = acc;
  }
  __syncthreads();  // o_s complete; the barrier init is visible to every thread
  if (!mbar_wait(wbar, 0, 2000000000ull)) record_status(kStatusTimeout);
  // ---- project this quarter: row l / 4, output columns 16 warp + 4 (l % 4) .. +3, over
  //      the quarter's 128 latent columns (o_s rows are padded: the 8 rows of a warp's
  //      loads fall in different banks; the W loads of a warp are 4 distinct words)
  {
    const int pr = lane >> 2, pc = 16 * warp + 4 * (lane & 3);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
    for (int d = 0; d < 128; ++d) {
      const uint2 w2 = *reinterpret_cast<const uint2*>(w_s + d * kProjDim + pc);
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w2.x));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&w2.y));
      const float o = o_s[pr][d];
      a0 = fmaf(o, f0.x, a0);
      a1 = fmaf(o, f0.y, a1);
      a2 = fmaf(o, f1.x, a2);
      a3 = fmaf(o, f1.y, a3);
    }
    *reinterpret_cast<float4*>(&part[pr][pc]) = make_float4(a0, a1, a2, a3);
  }
  // ---- the cluster's 4 quarters: CTA qtr adds up rows 2 qtr, 2 qtr + 1
  cluster_sync();
  {
    const int r = 2 * (int)qtr + (threadIdx.x >> 7), n = threadIdx.x & 127;
    const uint32_t local = smem_u32(&part[r][n]);
    float sum = 0.f;
#pragma unroll
    for (uint32_t c = 0; c < 4; ++c) sum += ld_shared_cluster_f32(mapa_shared(local, c));
    const int j = j0 + r;
    if (j < nrows) {
      const int b = j / plan.n_q, t = j - (j / plan.n_q) * plan.n_q;
      out_proj[(int64_t)(plan.seq_offset + b) * op_seq_stride + (int64_t)(t * plan.n_head + h) * kProjDim + n] = sum;
    }
  }
  // the peers have read this CTA's sums before it exits (their loads have returned by
  // the time they arrive: an execution barrier suffices)
  cluster_sync_relaxed();
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
