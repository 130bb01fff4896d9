// Host side of libmla_fa.so: argument checks, the split-KV launch plan, TMA
// tensor maps and the kernel launches behind the C ABI in include/mla_fa.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <utility>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/mla_fa.h"
#include "mla_common.cuh"
#include "mla_compact.cuh"
#include "mla_fwd.cuh"
#include "mla_gather.cuh"
#include "mla_heads.cuh"

namespace {

using mla::Plan;

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait
constexpr int kMinKeysPerSplit = 256;  // a KV split holds at least this many keys (one 256-key tile)

thread_local cudaStream_t t_stream = nullptr;

struct DeviceState {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  bool fwd_attr_set = false;
  bool heads_attr_set = false;
  void* fwd_ws = nullptr;  // workspace of mla_fa_forward
  size_t fwd_ws_bytes = 0;
  void* cmp_ws = nullptr;  // workspace of mla_compact_mask
  size_t cmp_ws_bytes = 0;
  uint32_t cmp_epoch = 1;
};

std::mutex g_mutex;
std::vector<DeviceState> g_dev;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

PFN_cuCtxGetCurrent_v4000 g_ctx_get_current = nullptr;
PFN_cuCtxGetDevice_v2000 g_ctx_get_device = nullptr;

void* driver_fn(const char* name) {
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return fn;
}

// The library links its own copy of the CUDA runtime. The device the caller
// works on (e.g. the one torch made current on this thread) is taken from the
// driver's current context, so both runtimes agree on the device.
int sync_device_with_context(int* dev) {
  if (g_ctx_get_current == nullptr) {
    g_ctx_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(driver_fn("cuCtxGetCurrent"));
    g_ctx_get_device = reinterpret_cast<PFN_cuCtxGetDevice_v2000>(driver_fn("cuCtxGetDevice"));
  }
  CUcontext ctx = nullptr;
  CUdevice cdev = 0;
  if (g_ctx_get_current && g_ctx_get_device && g_ctx_get_current(&ctx) == CUDA_SUCCESS &&
      ctx != nullptr && g_ctx_get_device(&cdev) == CUDA_SUCCESS) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MLA_ERR_CUDA;
    if (cur != (int)cdev && cudaSetDevice((int)cdev) != cudaSuccess) return MLA_ERR_CUDA;
    *dev = (int)cdev;
    return MLA_OK;
  }
  return cudaGetDevice(dev) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int current_device(DeviceState** st) {
  int dev = 0;
  if (sync_device_with_context(&dev) != MLA_OK) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mutex);
  if ((int)g_dev.size() <= dev) g_dev.resize(dev + 1);
  DeviceState& s = g_dev[dev];
  if (!s.probed) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MLA_ERR_CUDA;
    s.supported = (prop.major == 10 && prop.minor == 0);
    s.sm_count = prop.multiProcessorCount;
    s.probed = true;
  }
  if (!s.supported) return MLA_ERR_UNSUPPORTED;
  if (g_encode == nullptr) {
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(driver_fn("cuTensorMapEncodeTiled"));
    if (g_encode == nullptr) return MLA_ERR_CUDA;
  }
  *st = &s;
  return MLA_OK;
}

// ---------------------------------------------------------------- profiling
enum KernelId {
  kKernFwdF16 = 0,
  kKernFwdGather = 1,
  kKernFwdQ8 = 2,
  kKernCombine = 3,
  kKernCompact = 4,
  kKernWaitTest = 5,
  kKernMerge = 6,
  kKernHeads = 7,
  kKernHeadsCombine = 8,
  kKernScan = 9,
  kKernDevPlan = 10,
  kKernGatherRows = 11,
  kNumKernels
};
const char* const kKernelNames[kNumKernels] = {"mla_fwd_f16", "mla_fwd_gather_f16", "mla_fwd_q8_0",
                                               "mla_combine", "mla_compact", "mla_wait_timeout",
                                               "mla_merge", "mla_fwd_heads", "mla_combine_heads",
                                               "mla_scan", "mla_device_plan", "mla_gather_rows"};
struct ProfRecord {
  cudaEvent_t start, stop;
  int kernel;
};
std::mutex g_prof_mutex;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets one launch with events when profiling is on.
struct ProfScope {
  cudaEvent_t stop = nullptr;
  int kernel;
  cudaStream_t stream;
  ProfScope(int k, cudaStream_t s) : kernel(k), stream(s) {
    std::lock_guard<std::mutex> lk(g_prof_mutex);
    if (!g_prof_on) return;
    cudaEvent_t start = prof_event();
    stop = prof_event();
    cudaEventRecord(start, stream);
    g_prof_records.push_back({start, stop, k});
  }
  ~ProfScope() {
    if (stop) cudaEventRecord(stop, stream);
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct Resolved {
  mla_fa_args a;
  int rows;
  int64_t q_ss, k_ss, m_ss, m_rs, o_ss, idx_ss, op_ss;
  bool proj;  // fused value up-projection: every sequence writes split partials
  bool sinks; // attention sinks: every sequence writes split partials (the combine adds them)
  bool lse;   // per-row log-sum-exp output: every sequence writes partials (the combine writes it)
  int dk;     // head width: MLA_DK, MLA_DV for the DK = DV = 512 shape, MLA_HEADS_DK
  int64_t v_ss;  // DK = 192 shape: rows between sequences of v
  bool no_gathered_rows = false;  // sparse calls keep the gather modes (a scratch too small for the rows)
};

int validate(const mla_fa_args* a, Resolved* r) {
  if (a == nullptr) return MLA_ERR_NULL;
  const bool proj = a->wv != nullptr;
  if (a->q == nullptr || a->kcache == nullptr || (a->out == nullptr && !proj)) return MLA_ERR_NULL;
  if (proj && a->out_proj == nullptr) return MLA_ERR_NULL;
  if (proj && a->proj_dim != MLA_PROJ_DIM) return MLA_ERR_UNSUPPORTED;
  if (!(a->softcap >= 0.f) || std::isinf(a->softcap)) return MLA_ERR_SHAPE;  // NaN, <0, inf
  if (a->alibi_slopes != nullptr && a->idx != nullptr) return MLA_ERR_UNSUPPORTED;
  if (a->mask_gather != 0 && a->mask_gather != 1) return MLA_ERR_SHAPE;
  if (a->mask_gather && a->mask == nullptr) return MLA_ERR_NULL;
  if (a->mask_gather && (a->idx != nullptr || a->alibi_slopes != nullptr)) return MLA_ERR_UNSUPPORTED;
  if (a->out_lse != nullptr && (a->sinks != nullptr || proj)) return MLA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(a->sinks) & 3) || (reinterpret_cast<uintptr_t>(a->alibi_slopes) & 3) ||
      (reinterpret_cast<uintptr_t>(a->out_lse) & 3))
    return MLA_ERR_ALIGN;
  if (a->kcache_type != MLA_KV_F16 && a->kcache_type != MLA_KV_Q8_0) return MLA_ERR_TYPE;
  // head width: 576, or 512 (f16 cache; dense or index-list attention, no softcap,
  // ALiBi or mask gather), or 192 (a K and a V per KV head; dense, f16)
  const int dk = a->head_dim == 0 ? MLA_DK : a->head_dim;
  if (dk != MLA_DK && dk != MLA_DV && dk != MLA_HEADS_DK) return MLA_ERR_SHAPE;
  if (dk != MLA_HEADS_DK && (a->v != nullptr || a->n_kv_head != 0 || a->v_seq_stride != 0))
    return MLA_ERR_SHAPE;
  if (dk == MLA_HEADS_DK) {
    if (a->v == nullptr) return MLA_ERR_NULL;
    if (a->n_kv_head < 1 || a->n_head < 1 || a->n_head % a->n_kv_head != 0) return MLA_ERR_SHAPE;
    if (a->kcache_type != MLA_KV_F16 || a->idx != nullptr || a->mask_gather != 0 || proj ||
        a->sinks != nullptr || a->alibi_slopes != nullptr || a->softcap > 0.f || a->out_lse != nullptr)
      return MLA_ERR_UNSUPPORTED;
    if (a->v_seq_stride < 0) return MLA_ERR_SHAPE;
    if (!aligned16(a->v)) return MLA_ERR_ALIGN;
  }
  if (dk == MLA_DV && (a->kcache_type != MLA_KV_F16 || a->softcap > 0.f || a->alibi_slopes != nullptr ||
                       a->mask_gather != 0))
    return MLA_ERR_UNSUPPORTED;
  if (a->n_seq < 1 || a->n_q < 1 || a->n_head < 1 || a->n_head > MLA_MAX_HEADS || a->n_kv < 1)
    return MLA_ERR_SHAPE;
  if (!std::isfinite(a->scale)) return MLA_ERR_SHAPE;
  const int64_t rows = (int64_t)a->n_q * a->n_head;
  if (rows > (1 << 24)) return MLA_ERR_SHAPE;
  // the projection's grid has 4 CTAs per 8 (sequence, token) rows of a launch in its y
  // dimension (at most 65535)
  if (proj && (int64_t)4 *
                  (((int64_t)std::min(a->n_seq, mla::kPlanMaxSeq) * a->n_q + mla::kProjRows - 1) /
                   mla::kProjRows) > 65535)
    return MLA_ERR_SHAPE;
  if (a->idx != nullptr && a->idx_count == nullptr) return MLA_ERR_NULL;
  r->a = *a;
  r->rows = (int)rows;
  r->dk = dk;
  r->q_ss = a->q_seq_stride ? a->q_seq_stride : rows * dk;
  r->k_ss = a->k_seq_stride ? a->k_seq_stride : a->n_kv;
  r->v_ss = a->v_seq_stride ? a->v_seq_stride : a->n_kv;
  if (r->v_ss < a->n_kv) return MLA_ERR_SHAPE;
  r->m_rs = a->mask_row_stride ? a->mask_row_stride : a->n_kv;
  r->m_ss = a->mask_seq_stride ? a->mask_seq_stride : (int64_t)a->n_q * r->m_rs;
  const int dv = dk == MLA_HEADS_DK ? MLA_HEADS_DV : MLA_DV;
  r->o_ss = a->out_seq_stride ? a->out_seq_stride : rows * dv;
  r->idx_ss = a->idx_seq_stride ? a->idx_seq_stride : a->n_kv;
  r->proj = proj;
  r->sinks = a->sinks != nullptr;
  r->lse = a->out_lse != nullptr;
  r->op_ss = proj ? (a->out_proj_seq_stride ? a->out_proj_seq_stride : rows * MLA_PROJ_DIM) : 0;
  if (proj && (a->out_proj_seq_stride < 0 || r->op_ss < rows * MLA_PROJ_DIM)) return MLA_ERR_SHAPE;
  if (proj && (!aligned16(a->wv) || !aligned16(a->out_proj) || (r->op_ss % 4) != 0))
    return MLA_ERR_ALIGN;
  if (r->q_ss < rows * dk || r->k_ss < a->n_kv || r->m_rs < a->n_kv ||
      r->m_ss < (int64_t)(a->n_q - 1) * r->m_rs + a->n_kv || r->o_ss < rows * dv ||
      r->idx_ss < 0)
    return MLA_ERR_SHAPE;
  if (a->q_seq_stride < 0 || a->k_seq_stride < 0 || a->mask_seq_stride < 0 ||
      a->mask_row_stride < 0 || a->out_seq_stride < 0 || a->idx_seq_stride < 0)
    return MLA_ERR_SHAPE;
  if (!aligned16(a->q) || !aligned16(a->kcache) || (a->out != nullptr && !aligned16(a->out)))
    return MLA_ERR_ALIGN;
  if ((r->q_ss % 8) != 0 || (r->o_ss % 4) != 0) return MLA_ERR_ALIGN;
  if (a->mask != nullptr && (reinterpret_cast<uintptr_t>(a->mask) & 1)) return MLA_ERR_ALIGN;
  if (a->kv_len != nullptr)
    for (int b = 0; b < a->n_seq; ++b)
      if (a->kv_len[b] < 0 || a->kv_len[b] > a->n_kv) return MLA_ERR_SHAPE;
  if (a->idx != nullptr && ((reinterpret_cast<uintptr_t>(a->idx) & 3) ||
                            (reinterpret_cast<uintptr_t>(a->idx_count) & 3)))
    return MLA_ERR_ALIGN;
  return MLA_OK;
}

// Split plan for sequences [s0, s0+n). Returns the partial slots it needs.
// Keys per pipeline step of the attention kernel, which is also the plan's tile. The TMA
// mode (dense f16 cache) takes steps of 128 keys when a sequence's keys are read by a
// single 128-row group: the cache then streams from DRAM once, and 128-key steps
// double-buffer S and P in TMEM, so that the K stream and Q.K^T run on while the softmax
// and P.V work on the previous step. With several groups per sequence (a prefill chunk)
// the keys come back from L2 and the MMAs bound the kernel: steps of 256 keys issue half
// as many MMAs and softmax rounds per key. The gather and q8_0 modes take 256.
// Sparse calls of a single 128-row group (a decode): an index list (the caller's, or
// with the mask gather one built here from the mask by mla_compact_union_kernel) has its
// rows gathered into a dense f16 buffer in the workspace (mla_gather_rows_kernel, every
// SM at once), and the TMA-mode kernel streams that buffer. With more groups per
// sequence each group would re-read the list's rows, so those calls keep the gather
// modes.
bool gathered_rows(const Resolved& r) {
  return (r.a.idx != nullptr || r.a.mask_gather) && r.rows <= mla::kRowsPerGroup && r.dk != MLA_HEADS_DK &&
         !r.no_gathered_rows;
}
// The list is built here (mask gather) rather than passed in.
bool internal_list(const Resolved& r) { return gathered_rows(r) && r.a.mask_gather; }

// Rows per sequence in the gathered buffer: the most any sequence's list can use.
int64_t gathered_cap(const Resolved& r) {
  int64_t m = 0;
  for (int b = 0; b < r.a.n_seq; ++b) m = std::max<int64_t>(m, r.a.kv_len ? r.a.kv_len[b] : r.a.n_kv);
  if (r.a.idx != nullptr) m = std::min<int64_t>(m, r.idx_ss);
  return std::max<int64_t>(1, m);
}
int64_t gathered_mask_stride(const Resolved& r) { return (gathered_cap(r) + 63) / 64 * 64; }
size_t align256(size_t x) { return (x + 255) / 256 * 256; }
// Layout of the gathered region (offsets from its start): rows, mask values, and for an
// internal list the list, its counts, and the compaction's tickets and look-back flags
// (one launch's sequences at a time, cleared before each launch).
struct GatheredLayout {
  size_t mask, list, count, tickets, flags, bytes;
  int tiles;  // compaction tiles of the longest list
};
GatheredLayout gathered_layout(const Resolved& r) {
  GatheredLayout l = {};
  if (!gathered_rows(r)) return l;
  const int64_t cap = gathered_cap(r);
  l.mask = align256((size_t)r.a.n_seq * cap * r.dk * 2);
  l.list = l.mask + align256((size_t)r.a.n_seq * r.a.n_q * gathered_mask_stride(r) * 2);
  l.bytes = l.list;
  if (internal_list(r)) {
    l.tiles = (int)((cap + mla::compact::kTileCells - 1) / mla::compact::kTileCells);
    l.count = l.list + align256((size_t)r.a.n_seq * cap * 4);
    l.tickets = l.count + align256((size_t)r.a.n_seq * 4);
    l.flags = l.tickets + align256((size_t)mla::kPlanMaxSeq * 4);
    l.bytes = l.flags + align256((size_t)mla::kPlanMaxSeq * l.tiles * 8);
  }
  return l;
}
// Bytes of the gathered region (every sequence of the call).
size_t gathered_bytes(const Resolved& r) { return gathered_layout(r).bytes; }

int kernel_step(const Resolved& r) {
  const mla_fa_args& a = r.a;
  const bool tma = gathered_rows(r) || (a.kcache_type != MLA_KV_Q8_0 && a.idx == nullptr && !a.mask_gather);
  return tma && r.rows <= mla::kRowsPerGroup ? 128 : 256;
}

int build_plan(const Resolved& r, int s0, int n, int sm_count, Plan* plan) {
  std::memset(plan, 0, sizeof(Plan));
  const mla_fa_args& a = r.a;
  plan->tile_keys = kernel_step(r);
  plan->n_seq = n;
  plan->seq_offset = s0;
  plan->rows = r.rows;
  plan->groups = (r.rows + mla::kRowsPerGroup - 1) / mla::kRowsPerGroup;
  plan->n_head = a.n_head;
  plan->n_q = a.n_q;
  plan->n_kv = a.n_kv;
  const int pairs = std::max(1, sm_count / 2);
  int64_t sum_tiles = 0;
  std::vector<int> tiles(n);
  for (int b = 0; b < n; ++b) {
    // sparse: the kept count is only known on the device; plan for the most it can be
    int len = a.kv_len ? a.kv_len[s0 + b] : a.n_kv;
    if (a.idx != nullptr) len = (int)std::min<int64_t>(len, r.idx_ss);
    plan->kv_len[b] = len;
    tiles[b] = (len + plan->tile_keys - 1) / plan->tile_keys;
    sum_tiles += tiles[b];
  }
  const int64_t total_groups = (int64_t)n * plan->groups;
  std::vector<int> nsplit(n, 1);
  if (total_groups < pairs && sum_tiles > 0) {
    int64_t want_units = 0;
    for (int b = 0; b < n; ++b) {
      const double want = (double)pairs * tiles[b] / ((double)sum_tiles * plan->groups);
      int ns = (int)std::floor(want + 0.5);
      ns = std::min(ns, std::max(1, tiles[b] / (kMinKeysPerSplit / plan->tile_keys)));
      nsplit[b] = std::max(ns, 1);
      want_units += (int64_t)plan->groups * nsplit[b];
    }
    // Rounding can ask for more units than there are SM pairs, and the surplus would
    // run as a second wave. Take splits back one at a time from the sequence whose
    // units grow least (in tiles per unit) by losing one.
    while (want_units > pairs) {
      int best = -1;
      int64_t best_load = 0;
      for (int b = 0; b < n; ++b) {
        if (nsplit[b] <= 1) continue;
        const int64_t load = (tiles[b] + nsplit[b] - 2) / (nsplit[b] - 1);  // ceil(t / (ns - 1))
        if (best < 0 || load < best_load) {
          best = b;
          best_load = load;
        }
      }
      if (best < 0) break;
      --nsplit[best];
      want_units -= plan->groups;
    }
  }
  int units = 0, slots = 0;
  for (int b = 0; b < n; ++b) {
    const int ns = nsplit[b];
    plan->n_split[b] = ns;
    plan->unit_base[b] = units;
    units += plan->groups * ns;
    if (ns > 1 || r.proj || r.sinks || r.lse) {
      plan->ws_base[b] = slots;
      slots += plan->groups * ns;
    } else {
      plan->ws_base[b] = -1;
    }
  }
  plan->unit_base[n] = units;
  plan->total_units = units;
  return slots;
}

// One split partial: 128 rows of O_s / l_s in f16, and their 128 fp32 log-sum-exps.
size_t slot_bytes() { return (size_t)mla::kRowsPerGroup * (mla::kDV * 2 + sizeof(float)); }

// Mask gather: entries of one CTA's cell list (8 per chunk of the most chunks a
// split is dealt, rounded up to 64) and the bytes of all lists of a launch.
int64_t gather_stride(const Plan& plan) {
  int64_t m = 0;
  for (int b = 0; b < plan.n_seq; ++b) {
    const int64_t chunks = ((int64_t)plan.kv_len[b] + 7) / 8;
    m = std::max<int64_t>(m, 8 * ((chunks + plan.n_split[b] - 1) / plan.n_split[b]));
  }
  return std::max<int64_t>(64, (m + 63) / 64 * 64);
}
size_t gather_bytes(const Resolved& r, const Plan& plan, int slots) {
  if (!r.a.mask_gather || gathered_rows(r)) return 0;
  const size_t head = (size_t)slots * slot_bytes();
  const size_t start = (head + 255) / 256 * 256;
  return start - head + (size_t)2 * plan.total_units * gather_stride(plan) * sizeof(int32_t);
}

// ------------------------------------------------ the DK = 192 / DV = 128 head shape
// Split plan for sequences [s0, s0+n): a unit is (sequence, KV head, 128-row group,
// split), one CTA each. When the unsplit units do not fill the SMs, each sequence gets
// splits in proportion to its tiles (all of its KV heads and groups the same number),
// never more units than SMs. Returns the partial slots it needs.
int build_heads_plan(const Resolved& r, int s0, int n, int sm_count, mla::heads::Plan* plan) {
  using namespace mla::heads;
  std::memset(plan, 0, sizeof(*plan));
  const mla_fa_args& a = r.a;
  plan->n_seq = n;
  plan->seq_offset = s0;
  plan->n_q = a.n_q;
  plan->n_head = a.n_head;
  plan->n_kv_head = a.n_kv_head;
  plan->group = a.n_head / a.n_kv_head;
  plan->rows = a.n_q * plan->group;
  plan->groups = (plan->rows + kRows - 1) / kRows;
  plan->n_kv = a.n_kv;
  const int per_seq = a.n_kv_head * plan->groups;  // unsplit units of one sequence
  const int sms = std::max(1, sm_count);
  int64_t sum_tiles = 0;
  std::vector<int> tiles(n);
  for (int b = 0; b < n; ++b) {
    plan->kv_len[b] = a.kv_len ? a.kv_len[s0 + b] : a.n_kv;
    tiles[b] = (plan->kv_len[b] + kTile - 1) / kTile;
    sum_tiles += tiles[b];
  }
  // When the unsplit units do not fill the SMs, splits go one at a time to the sequence
  // whose units are longest (in tiles), within one, two or three waves of units; the
  // wave count kept is the one with the shortest estimate: the larger of the longest
  // unit and the average work per SM, plus each wave's fixed cost (set-up, first loads,
  // epilogue: about kWaveCostTiles tiles). A decode batch of ragged lengths with many
  // KV heads per sequence (16 units per split) otherwise leaves its longest sequences
  // unsplit, each on one SM.
  constexpr double kWaveCostTiles = 3.0;
  std::vector<int> nsplit(n, 1);
  if ((int64_t)n * per_seq < sms && sum_tiles > 0) {
    double best_est = 0.0;
    std::vector<int> ns(n);
    for (int waves = 1; waves <= 3; ++waves) {
      std::fill(ns.begin(), ns.end(), 1);
      int64_t units = (int64_t)n * per_seq;
      auto load = [&](int b) { return (double)tiles[b] / ns[b]; };
      while (units + per_seq <= (int64_t)waves * sms) {
        int arg = -1;
        for (int b = 0; b < n; ++b)
          if (ns[b] < tiles[b] && (arg < 0 || load(b) > load(arg))) arg = b;
        if (arg < 0) break;
        ++ns[arg];
        units += per_seq;
      }
      double max_load = 0.0;
      for (int b = 0; b < n; ++b) max_load = std::max(max_load, load(b));
      const double avg = (double)sum_tiles * per_seq / sms;
      const double est = std::max(max_load, avg) + kWaveCostTiles * (double)((units + sms - 1) / sms);
      if (waves == 1 || est < best_est) {
        best_est = est;
        nsplit = ns;
      }
    }
  }
  int units = 0, slots = 0;
  for (int b = 0; b < n; ++b) {
    plan->n_split[b] = nsplit[b];
    plan->unit_base[b] = units;
    units += per_seq * nsplit[b];
    if (nsplit[b] > 1) {
      plan->ws_base[b] = slots;
      slots += per_seq * nsplit[b];
    } else {
      plan->ws_base[b] = -1;
    }
  }
  plan->unit_base[n] = units;
  plan->total_units = units;
  return slots;
}

size_t heads_slot_bytes() {
  return (size_t)mla::heads::kRows * (mla::heads::kHeadDV + 1) * sizeof(float);
}

size_t heads_workspace_for(const Resolved& r, int sm_count, int* max_units, int* max_splits) {
  size_t need = 0;
  int mu = 0, ms = 0;
  mla::heads::Plan plan;
  for (int s0 = 0; s0 < r.a.n_seq; s0 += mla::heads::kPlanMaxSeq) {
    const int n = std::min(mla::heads::kPlanMaxSeq, r.a.n_seq - s0);
    const int slots = build_heads_plan(r, s0, n, sm_count, &plan);
    need = std::max(need, (size_t)slots * heads_slot_bytes());
    mu = std::max(mu, plan.total_units);
    for (int b = 0; b < n; ++b) ms = std::max(ms, plan.n_split[b]);
  }
  if (max_units) *max_units = mu;
  if (max_splits) *max_splits = ms;
  return need;
}

int run_heads(const Resolved& r, DeviceState* st, void* ws, size_t ws_bytes, cudaStream_t stream) {
  using namespace mla::heads;
  const mla_fa_args& a = r.a;
  const size_t need = heads_workspace_for(r, st->sm_count, nullptr, nullptr);
  if (need > 0 && (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)))
    return MLA_ERR_WORKSPACE;
  // K: {192 columns, KV heads, keys, sequences}, box {64, 1, 128 keys, 1} -> [key][64]
  const uint64_t krow = (uint64_t)a.n_kv_head * kHeadDK * 2;
  CUtensorMap tm_k, tm_v;
  {
    cuuint64_t dims[4] = {(cuuint64_t)kHeadDK, (cuuint64_t)a.n_kv_head, (cuuint64_t)a.n_kv, (cuuint64_t)a.n_seq};
    cuuint64_t strides[3] = {(cuuint64_t)kHeadDK * 2, krow, (cuuint64_t)r.k_ss * krow};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kTile, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    if (g_encode(&tm_k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(a.kcache), dims, strides,
                 box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  // V: {64 columns, keys, 2 column blocks, KV heads, sequences}, box {64, 64 keys, 2, 1, 1}
  // -> [block][key][64], the MN-major B operand of P.V
  {
    const uint64_t vrow = (uint64_t)a.n_kv_head * kHeadDV * 2;
    cuuint64_t dims[5] = {64, (cuuint64_t)a.n_kv, 2, (cuuint64_t)a.n_kv_head, (cuuint64_t)a.n_seq};
    cuuint64_t strides[4] = {vrow, 128, (cuuint64_t)kHeadDV * 2, (cuuint64_t)r.v_ss * vrow};
    cuuint32_t box[5] = {64, 64, 2, 1, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    if (g_encode(&tm_v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void*>(a.v), dims, strides, box,
                 es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  if (!st->heads_attr_set) {
    if (cudaFuncSetAttribute(mla::mla_heads_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemAlloc) != cudaSuccess)
      return MLA_ERR_CUDA;
    st->heads_attr_set = true;
  }
  mla::heads::Params p;
  p.q = static_cast<const uint16_t*>(a.q);
  p.mask = static_cast<const uint16_t*>(a.mask);
  p.out = a.out;
  p.q_seq_stride = r.q_ss;
  p.mask_seq_stride = r.m_ss;
  p.mask_row_stride = r.m_rs;
  p.out_seq_stride = r.o_ss;
  p.scale = a.scale;
  p.mask_vec_ok = (a.mask != nullptr && aligned16(a.mask) && (r.m_ss % 8) == 0 && (r.m_rs % 8) == 0);
  p.timeout_ns = kDefaultTimeoutNs;
  mla::heads::Plan plan;
  for (int s0 = 0; s0 < a.n_seq; s0 += kPlanMaxSeq) {
    const int n = std::min(kPlanMaxSeq, a.n_seq - s0);
    const int slots = build_heads_plan(r, s0, n, st->sm_count, &plan);
    p.ws_o = static_cast<float*>(ws);
    p.ws_lse = slots ? reinterpret_cast<float*>(static_cast<char*>(ws) +
                                                (size_t)slots * kRows * kHeadDV * sizeof(float))
                     : nullptr;
    if (plan.total_units == 0) continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.total_units);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    {
      ProfScope prof(kKernHeads, stream);
      e = cudaLaunchKernelEx(&cfg, mla::mla_heads_fwd_kernel, tm_k, tm_v, plan, p);
    }
    if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    if (slots > 0) {
      cudaLaunchConfig_t ccfg = cfg;
      ccfg.gridDim = dim3((a.n_kv_head * plan.rows + 3) / 4, n);
      ccfg.blockDim = dim3(128);
      ccfg.dynamicSmemBytes = 0;
      {
        ProfScope prof(kKernHeadsCombine, stream);
        e = cudaLaunchKernelEx(&ccfg, mla::mla_heads_combine_kernel, plan, (const float*)p.ws_o,
                               (const float*)p.ws_lse, a.out, (int64_t)r.o_ss);
      }
      if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
  }
  return MLA_OK;
}

// ------------------------------------------------ the device plan (tile ranges from the mask)
// Used by dense f16 calls with a mask that either give no lengths or have several query
// tokens (a causal prefill chunk ends each token's keys at a different tile): the mask
// decides each group's tiles. Calls with lengths and one query token keep the host plan.
bool use_device_plan(const Resolved& r) {
  const mla_fa_args& a = r.a;
  return a.mask != nullptr && (a.kv_len == nullptr || a.n_q > 1) && a.kcache_type == MLA_KV_F16 &&
         a.idx == nullptr && !a.mask_gather && !r.proj && !r.sinks && !r.lse;
}

struct DevLayout {
  int n_groups, grid_units, slots;
  size_t off_ranges, off_units, off_gsplit, bytes;
};

// Workspace of one launch of the device plan: partial slots (at most one per SM pair, and
// only when there are fewer groups than pairs), then the ranges, unit descriptors and the
// per-group split table.
DevLayout dev_layout(int n_seq, int groups, int sm_count) {
  DevLayout l;
  const int pairs = std::max(1, sm_count / 2);
  l.n_groups = n_seq * groups;
  const bool split = l.n_groups < pairs && l.n_groups <= mla::kDevPlanMaxGroups;
  l.grid_units = l.n_groups >= pairs ? l.n_groups : pairs;
  l.slots = split ? pairs : 0;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  l.off_ranges = up((size_t)l.slots * slot_bytes());
  l.off_units = up(l.off_ranges + (size_t)l.n_groups * sizeof(int2));
  l.off_gsplit = up(l.off_units + (size_t)l.grid_units * sizeof(mla::DevUnit));
  l.bytes = l.off_gsplit + (size_t)l.n_groups * sizeof(int2);
  return l;
}

// Splits one group may take in the device plan: with three groups or more at most 16, so
// the combine reads a row's partials in one round trip (an even share is at most a third
// of the SM pairs); with fewer groups as many as the SM pairs, for the wide combine.
int dev_max_split(const DevLayout& l) { return l.n_groups >= 3 ? 16 : std::max(1, l.slots); }

size_t workspace_for(const Resolved& r, int sm_count, int* max_units, int* max_splits) {
  if (r.dk == MLA_HEADS_DK) return heads_workspace_for(r, sm_count, max_units, max_splits);
  if (use_device_plan(r)) {
    // the split counts are decided on the device: report the launch shape and the most
    // splits a group can take
    size_t need = 0;
    int mu = 0, ms = 1;
    const int groups = (r.rows + mla::kRowsPerGroup - 1) / mla::kRowsPerGroup;
    for (int s0 = 0; s0 < r.a.n_seq; s0 += mla::kPlanMaxSeq) {
      const int n = std::min(mla::kPlanMaxSeq, r.a.n_seq - s0);
      const DevLayout l = dev_layout(n, groups, sm_count);
      need = std::max(need, l.bytes);
      mu = std::max(mu, l.grid_units);
      if (l.slots > 0) ms = std::max(ms, dev_max_split(l));
    }
    if (max_units) *max_units = mu;
    if (max_splits) *max_splits = ms;
    return need;
  }
  size_t need = 0;
  int mu = 0, ms = 0;
  Plan plan;
  for (int s0 = 0; s0 < r.a.n_seq; s0 += mla::kPlanMaxSeq) {
    const int n = std::min(mla::kPlanMaxSeq, r.a.n_seq - s0);
    const int slots = build_plan(r, s0, n, sm_count, &plan);
    need = std::max(need, (size_t)slots * slot_bytes() + gather_bytes(r, plan, slots));
    mu = std::max(mu, plan.total_units);
    for (int b = 0; b < n; ++b) ms = std::max(ms, plan.n_split[b]);
  }
  if (max_units) *max_units = mu;
  if (max_splits) *max_splits = ms;
  // gathered rows: after the partials (the same offset for every launch of the call)
  if (gathered_rows(r)) need = (need + 255) / 256 * 256 + gathered_bytes(r);
  return need;
}

// Offset of the gathered rows in the workspace (256-aligned, after every launch's partials).
size_t gathered_offset(const Resolved& r, int sm_count) {
  size_t need = 0;
  Plan plan;
  for (int s0 = 0; s0 < r.a.n_seq; s0 += mla::kPlanMaxSeq) {
    const int n = std::min(mla::kPlanMaxSeq, r.a.n_seq - s0);
    const int slots = build_plan(r, s0, n, sm_count, &plan);
    need = std::max(need, (size_t)slots * slot_bytes() + gather_bytes(r, plan, slots));
  }
  return (need + 255) / 256 * 256;
}

int make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
             uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult res = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// fp32 [d2][d1][512] output view for the kernel's TMA stores: boxes of 32 rows x 32
// columns, 128-byte swizzle (the layout the kernel stages in shared memory).
int make_out_map(CUtensorMap* m, void* base, uint64_t d1, uint64_t d2, uint64_t stride2_bytes) {
  cuuint64_t dims[3] = {(cuuint64_t)MLA_DV, d1, d2};
  cuuint64_t strides[2] = {(cuuint64_t)MLA_DV * 4, stride2_bytes};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult res = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// f16 [rows][512] view of the split partials for the kernel's TMA stores: boxes of 32
// rows x 64 columns (128-byte rows), 128-byte swizzle.
int make_part_map(CUtensorMap* m, void* base, uint64_t rows) {
  cuuint64_t dims[3] = {(cuuint64_t)MLA_DV, rows, 1};
  cuuint64_t strides[2] = {(cuuint64_t)MLA_DV * 2, (cuuint64_t)rows * MLA_DV * 2};
  cuuint32_t box[3] = {64, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult res = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// One instance of the attention kernel, with its block size and shared memory (cfg has
// the rest).
template <int kMode, bool kVariant, bool kGather, int kNC = 9, int kTK = 256>
cudaError_t launch_fwd(cudaLaunchConfig_t cfg, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                       const CUtensorMap& tm_v, const CUtensorMap& tm_o, const CUtensorMap& tm_w,
                       const mla::Plan& plan, const mla::MlaFwdParams& p) {
  cfg.blockDim = dim3(mla::FwdCfg<kMode>::kThreads);
  cfg.dynamicSmemBytes = mla::fwd::Geo<kTK>::kSmemAlloc;
  return cudaLaunchKernelEx(&cfg, mla::mla_fwd_kernel<kMode, kVariant, kGather, kNC, kTK>, tm_q, tm_k,
                            tm_v, tm_o, tm_w, plan, p);
}


int run_forward(const Resolved& r, DeviceState* st, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (r.dk == MLA_HEADS_DK) return run_heads(r, st, ws, ws_bytes, stream);
  const mla_fa_args& a = r.a;
  const size_t need = workspace_for(r, st->sm_count, nullptr, nullptr);
  if (need > 0 && (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)))
    return MLA_ERR_WORKSPACE;
  // index lists of a single group: the rows are gathered into the workspace first, and
  // the TMA mode streams them (gathered_rows)
  const bool gat = gathered_rows(r);
  const int mode = gat ? mla::kModeTma
                   : a.kcache_type == MLA_KV_Q8_0 ? mla::kModeQ8
                   : (a.idx != nullptr || a.mask_gather ? mla::kModeGatherF16 : mla::kModeTma);
  const int64_t g_cap = gat ? gathered_cap(r) : 0;
  const int64_t g_mstride = gat ? gathered_mask_stride(r) : 0;
  uint16_t* g_rows = nullptr;
  uint16_t* g_mask = nullptr;
  const GatheredLayout gl = gathered_layout(r);
  char* g_base = nullptr;
  if (gat) {
    g_base = static_cast<char*>(ws) + gathered_offset(r, st->sm_count);
    g_rows = reinterpret_cast<uint16_t*>(g_base);
    g_mask = reinterpret_cast<uint16_t*>(g_base + gl.mask);
  }
  // the list the rows are gathered from: the caller's, or the one built here
  const int32_t* list = a.idx;
  const int32_t* list_count = a.idx_count;
  int64_t list_stride = r.idx_ss;
  if (internal_list(r)) {
    list = reinterpret_cast<const int32_t*>(g_base + gl.list);
    list_count = reinterpret_cast<const int32_t*>(g_base + gl.count);
    list_stride = g_cap;
  }
  // the cells the TMA mode streams: the cache, or the gathered rows
  const void* k_base = gat ? static_cast<const void*>(g_rows) : a.kcache;
  const uint64_t k_rows = gat ? (uint64_t)g_cap : (uint64_t)a.n_kv;
  CUtensorMap tm_q, tm_k, tm_v;
  const uint64_t row_bytes = (uint64_t)r.dk * 2;
  const uint64_t k_seq_bytes = gat ? (uint64_t)g_cap * row_bytes : (uint64_t)r.k_ss * row_bytes;
  int rc = make_map(&tm_q, a.q, r.dk, r.rows, a.n_seq, row_bytes, (uint64_t)r.q_ss * 2, 64, 64);
  if (rc == MLA_OK && mode == mla::kModeTma) {
    rc = make_map(&tm_k, k_base, r.dk, k_rows, a.n_seq, row_bytes, k_seq_bytes, 64,
                  (uint32_t)kernel_step(r) / 2);
    if (rc == MLA_OK) {
      // value view: {64 columns, keys, 8 column blocks, sequences}; a box of
      // {64, 64, 2, 1} lands as [column block][key][64 columns]
      cuuint64_t dims[4] = {64, (cuuint64_t)k_rows, 8, (cuuint64_t)a.n_seq};
      cuuint64_t strides[3] = {row_bytes, 128, k_seq_bytes};
      cuuint32_t box[4] = {64, 64, 2, 1};
      cuuint32_t es[4] = {1, 1, 1, 1};
      CUresult res = g_encode(&tm_v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(k_base),
                              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      rc = res == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
    }
  } else {
    tm_k = tm_q;  // unused by the gather / dequant modes
    tm_v = tm_q;
  }
  CUtensorMap tm_o;
  // with the projection every sequence writes partials and the kernel never stores
  // to out (which may be NULL): the output map then views the workspace (the first
  // 64 fp32 rows, inside the first slot)
  if (rc == MLA_OK) {
    if (r.proj)
      rc = make_out_map(&tm_o, ws, (uint64_t)mla::kRowsPerGroup / 2, 1,
                        (uint64_t)mla::kRowsPerGroup / 2 * MLA_DV * 4);
    else
      rc = make_out_map(&tm_o, a.out, (uint64_t)r.rows, (uint64_t)a.n_seq, (uint64_t)r.o_ss * 4);
  }
  if (rc != MLA_OK) return rc;
  if (!st->fwd_attr_set) {
    constexpr int kSmem256 = mla::fwd::Geo<256>::kSmemAlloc, kSmem128 = mla::fwd::Geo<128>::kSmemAlloc;
    const std::pair<const void*, int> fwd_kernels[] = {
        {(const void*)mla::mla_fwd_kernel<mla::kModeTma, false, false, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeTma, true, false, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeTma, false, false, 9, 128>, kSmem128},
        {(const void*)mla::mla_fwd_kernel<mla::kModeTma, true, false, 9, 128>, kSmem128},
        {(const void*)mla::mla_fwd_kernel<mla::kModeGatherF16, false, false, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeGatherF16, true, false, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeGatherF16, false, true, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeGatherF16, true, true, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeQ8, false, false, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeQ8, true, false, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeQ8, false, true, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeQ8, true, true, 9, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeTma, false, false, 8, 256>, kSmem256},
        {(const void*)mla::mla_fwd_kernel<mla::kModeTma, false, false, 8, 128>, kSmem128},
        {(const void*)mla::mla_fwd_kernel<mla::kModeGatherF16, false, false, 8, 256>, kSmem256}};
    bool ok = true;
    for (const auto& k : fwd_kernels)
      ok = ok && cudaFuncSetAttribute(k.first, cudaFuncAttributeMaxDynamicSharedMemorySize, k.second) ==
                     cudaSuccess;
    if (!ok ||
        cudaFuncSetAttribute(mla::mla_combine_proj_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             mla::kProjSmem) != cudaSuccess)
      return MLA_ERR_CUDA;
    st->fwd_attr_set = true;
  }
  mla::MlaFwdParams p;
  p.mask = static_cast<const uint16_t*>(a.mask);
  p.out = a.out;
  p.mask_seq_stride = r.m_ss;
  p.mask_row_stride = r.m_rs;
  p.out_seq_stride = r.o_ss;
  p.scale = a.scale;
  p.mask_vec_ok = (a.mask != nullptr && aligned16(a.mask) && (r.m_ss % 8) == 0 && (r.m_rs % 8) == 0);
  p.timeout_ns = kDefaultTimeoutNs;
  p.kcache = static_cast<const uint8_t*>(a.kcache);
  p.q = static_cast<const uint16_t*>(a.q);
  p.q_seq_stride = r.q_ss;
  p.k_seq_stride = r.k_ss;
  p.n_kv = a.n_kv;
  p.idx = a.idx;
  p.idx_count = a.idx_count;
  if (gat) {
    // the kernel streams the gathered rows, with their gathered mask values, up to each
    // list's count
    p.idx = nullptr;
    p.idx_count = list_count;
    p.mask = g_mask;
    p.mask_seq_stride = (int64_t)a.n_q * g_mstride;
    p.mask_row_stride = g_mstride;
    p.mask_vec_ok = 1;
    p.n_kv = (int)g_mstride;
  }
  p.idx_seq_stride = r.idx_ss;
  p.softcap = a.softcap;
  p.slopes = a.alibi_slopes;
  Plan plan;
  for (int s0 = 0; s0 < a.n_seq; s0 += mla::kPlanMaxSeq) {
    const int n = std::min(mla::kPlanMaxSeq, a.n_seq - s0);
    const bool dev = use_device_plan(r);
    int slots = build_plan(r, s0, n, st->sm_count, &plan);
    DevLayout dl = {};
    p.units = nullptr;
    int2* d_gsplit = nullptr;
    if (dev) {
      // the grid and the partial slots are sized for the device plan, which the scan and
      // plan kernels fill in before the attention kernel reads them
      dl = dev_layout(n, plan.groups, st->sm_count);
      slots = dl.slots;
      plan.total_units = dl.grid_units;
      int2* d_ranges = reinterpret_cast<int2*>(static_cast<char*>(ws) + dl.off_ranges);
      p.units = reinterpret_cast<const mla::DevUnit*>(static_cast<char*>(ws) + dl.off_units);
      d_gsplit = reinterpret_cast<int2*>(static_cast<char*>(ws) + dl.off_gsplit);
      cudaLaunchConfig_t scfg = {};
      scfg.gridDim = dim3(dl.n_groups);
      scfg.blockDim = dim3(256);
      scfg.stream = stream;
      cudaLaunchAttribute sattr[1];
      sattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      sattr[0].val.programmaticStreamSerializationAllowed = 1;
      scfg.attrs = sattr;
      scfg.numAttrs = 1;
      cudaError_t se;
      {
        ProfScope prof(kKernScan, stream);
        se = cudaLaunchKernelEx(&scfg, mla::mla_scan_kernel, plan, static_cast<const uint16_t*>(a.mask),
                                (int64_t)r.m_ss, (int64_t)r.m_rs, p.mask_vec_ok, d_ranges);
      }
      if (se != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
      scfg.gridDim = dim3(1);
      {
        ProfScope prof(kKernDevPlan, stream);
        se = cudaLaunchKernelEx(&scfg, mla::mla_device_plan_kernel, plan, (const int2*)d_ranges,
                                std::max(1, st->sm_count / 2), dev_max_split(dl), dl.grid_units,
                                const_cast<mla::DevUnit*>(p.units), d_gsplit);
      }
      if (se != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
    p.ws_o = static_cast<uint16_t*>(ws);
    p.ws_lse = slots ? reinterpret_cast<float*>(static_cast<char*>(ws) +
                                                (size_t)slots * mla::kRowsPerGroup * mla::kDV * 2)
                     : nullptr;
    p.mask_gather = gat ? 0 : a.mask_gather;
    p.gather_list = nullptr;
    p.gather_stride = 0;
    if (p.mask_gather) {
      const size_t head = (size_t)slots * slot_bytes();
      p.gather_list = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + (head + 255) / 256 * 256);
      p.gather_stride = gather_stride(plan);
    }
    CUtensorMap tm_w = tm_o;  // unused when no sequence of this launch is split
    if (slots > 0) {
      rc = make_part_map(&tm_w, ws, (uint64_t)slots * mla::kRowsPerGroup);
      if (rc != MLA_OK) return rc;
    }
    if (internal_list(r)) {
      // the list of each sequence: the cells its query tokens keep (mask gather)
      int* tickets = reinterpret_cast<int*>(g_base + gl.tickets);
      auto* flags = reinterpret_cast<unsigned long long*>(g_base + gl.flags);
      if (cudaMemsetAsync(g_base + gl.tickets, 0, gl.bytes - gl.tickets, stream) != cudaSuccess)
        return MLA_ERR_CUDA;
      uint32_t epoch;
      {
        std::lock_guard<std::mutex> lk(g_mutex);
        epoch = st->cmp_epoch;
        st->cmp_epoch = (st->cmp_epoch + 1) & 0x3FFFFFFFu;
        if (st->cmp_epoch == 0) st->cmp_epoch = 1;
      }
      cudaLaunchConfig_t ccfg = {};
      ccfg.gridDim = dim3(gl.tiles, n);
      ccfg.blockDim = dim3(mla::compact::kThreads);
      ccfg.stream = stream;
      cudaLaunchAttribute cattr[1];
      cattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      cattr[0].val.programmaticStreamSerializationAllowed = 1;
      ccfg.attrs = cattr;
      ccfg.numAttrs = 1;
      cudaError_t ce;
      {
        ProfScope prof(kKernCompact, stream);
        ce = cudaLaunchKernelEx(&ccfg, mla::mla_compact_union_kernel, plan, static_cast<const uint16_t*>(a.mask),
                                (int64_t)r.m_ss, (int64_t)r.m_rs, const_cast<int32_t*>(list), list_stride,
                                const_cast<int32_t*>(list_count), tickets, flags, epoch, kDefaultTimeoutNs);
      }
      if (ce != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
    if (gat) {
      // the lists' rows (and mask values) into the dense buffer, every SM at once; a
      // programmatic dependent of the kernel that wrote the lists
      mla::GatherParams gp;
      gp.idx = list;
      gp.idx_count = list_count;
      gp.idx_seq_stride = list_stride;
      gp.kcache = static_cast<const uint8_t*>(a.kcache);
      gp.k_seq_stride = r.k_ss;
      const int64_t cache_row = a.kcache_type == MLA_KV_Q8_0 ? (int64_t)mla::kQ8RowBytes : (int64_t)r.dk * 2;
      gp.kcache_bytes = ((int64_t)(a.n_seq - 1) * r.k_ss + a.n_kv) * cache_row;
      gp.n_kv = a.n_kv;
      gp.mask = static_cast<const uint16_t*>(a.mask);
      gp.mask_seq_stride = r.m_ss;
      gp.mask_row_stride = r.m_rs;
      gp.n_q = a.n_q;
      gp.rows = g_rows;
      gp.gmask = g_mask;
      gp.cap = g_cap;
      gp.gmask_stride = g_mstride;
      gp.timeout_ns = kDefaultTimeoutNs;
      const int64_t rows_per_cta = a.kcache_type == MLA_KV_Q8_0 ? 32 : 16;  // 8 warps x positions in flight
      const int per_seq = std::max(1, (st->sm_count * 4 + n - 1) / n);
      cudaLaunchConfig_t gcfg = {};
      gcfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>((g_cap + rows_per_cta - 1) / rows_per_cta, per_seq)), n);
      gcfg.blockDim = dim3(256);
      gcfg.stream = stream;
      cudaLaunchAttribute gattr[1];
      gattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      gattr[0].val.programmaticStreamSerializationAllowed = 1;
      gcfg.attrs = gattr;
      gcfg.numAttrs = 1;
      cudaError_t ge;
      {
        ProfScope prof(kKernGatherRows, stream);
        if (a.kcache_type == MLA_KV_Q8_0)
          ge = cudaLaunchKernelEx(&gcfg, mla::mla_gather_rows_kernel<mla::kModeQ8, 9>, plan, gp);
        else if (r.dk == MLA_DK)
          ge = cudaLaunchKernelEx(&gcfg, mla::mla_gather_rows_kernel<mla::kModeGatherF16, 9>, plan, gp);
        else
          ge = cudaLaunchKernelEx(&gcfg, mla::mla_gather_rows_kernel<mla::kModeGatherF16, 8>, plan, gp);
      }
      if (ge != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
    // launched as a programmatic dependent of the stream's previous kernel: its setup
    // overlaps that kernel's tail, and griddepcontrol.wait in the kernel precedes
    // every read of its inputs
    cudaLaunchConfig_t fcfg = {};
    fcfg.gridDim = dim3(2 * plan.total_units);
    fcfg.stream = stream;
    cudaLaunchAttribute fattr[1];
    fattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    fattr[0].val.programmaticStreamSerializationAllowed = 1;
    fcfg.attrs = fattr;
    fcfg.numAttrs = 1;
    // the softcap / ALiBi instance and the mask-gather instance only when the call
    // asks for them
    const bool variant = a.softcap > 0.f || a.alibi_slopes != nullptr;
    const bool gather = a.mask_gather != 0;
    cudaError_t fe;
    {
      ProfScope prof(mode == mla::kModeTma ? kKernFwdF16
                     : mode == mla::kModeGatherF16 ? kKernFwdGather : kKernFwdQ8, stream);
      const bool step128 = mode == mla::kModeTma && plan.tile_keys == 128;
      if (r.dk != MLA_DK)  // the DK = DV = 512 shape: dense or index-list, f16 cache
        fe = mode == mla::kModeTma
                 ? (step128 ? launch_fwd<mla::kModeTma, false, false, 8, 128>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p)
                            : launch_fwd<mla::kModeTma, false, false, 8>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p))
                 : launch_fwd<mla::kModeGatherF16, false, false, 8>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p);
      else if (mode == mla::kModeTma && step128)
        fe = variant ? launch_fwd<mla::kModeTma, true, false, 9, 128>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p)
                     : launch_fwd<mla::kModeTma, false, false, 9, 128>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p);
      else if (mode == mla::kModeTma)
        fe = variant ? launch_fwd<mla::kModeTma, true, false>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p)
                     : launch_fwd<mla::kModeTma, false, false>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p);
      else if (mode == mla::kModeGatherF16)
        fe = gather ? (variant ? launch_fwd<mla::kModeGatherF16, true, true>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p)
                               : launch_fwd<mla::kModeGatherF16, false, true>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p))
                    : (variant ? launch_fwd<mla::kModeGatherF16, true, false>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p)
                               : launch_fwd<mla::kModeGatherF16, false, false>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p));
      else
        fe = gather ? (variant ? launch_fwd<mla::kModeQ8, true, true>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p)
                               : launch_fwd<mla::kModeQ8, false, true>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p))
                    : (variant ? launch_fwd<mla::kModeQ8, true, false>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p)
                               : launch_fwd<mla::kModeQ8, false, false>(fcfg, tm_q, tm_k, tm_v, tm_o, tm_w, plan, p));
    }
    if (fe != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    if (slots > 0) {
      // launched as a programmatic dependent of the forward kernel so that its launch
      // overlaps the forward's last CTAs. Up to 16 splits: one 128-thread CTA per row
      // (one round trip); more: one CTA per (row, quarter of the value columns)
      int ns_max = 1;
      for (int b = 0; b < n; ++b) ns_max = std::max(ns_max, plan.n_split[b]);
      // the device plan's splits are known only on the device: at most dev_max_split
      const bool wide = dev ? dev_max_split(dl) > 16 : ns_max > 16;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = wide ? dim3(r.rows, 4, n) : dim3(r.rows, n);
      cfg.blockDim = dim3(128);
      cfg.dynamicSmemBytes = 0;
      if (r.proj) {
        // fused projection: a cluster of 4 CTAs (the quarters of the latent columns) per
        // (head, batch of 8 (sequence, token) rows)
        const int nrows = n * a.n_q;
        cfg.gridDim = dim3(a.n_head, 4 * ((nrows + mla::kProjRows - 1) / mla::kProjRows));
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = mla::kProjSmem;
      }
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cudaError_t ce;
      {
        ProfScope prof(kKernCombine, stream);
        if (r.proj)
          ce = cudaLaunchKernelEx(&cfg, mla::mla_combine_proj_kernel, plan, (const uint16_t*)p.ws_o,
                                  (const float*)p.ws_lse, static_cast<const uint16_t*>(a.wv),
                                  a.out_proj, (int64_t)r.op_ss, a.sinks);
        else if (wide)
          ce = cudaLaunchKernelEx(&cfg, mla::mla_combine_wide_kernel, plan, (const uint16_t*)p.ws_o,
                                  (const float*)p.ws_lse, a.out, (int64_t)r.o_ss, a.sinks, a.out_lse,
                                  (const int2*)d_gsplit);
        else
          ce = cudaLaunchKernelEx(&cfg, mla::mla_combine_kernel, plan, (const uint16_t*)p.ws_o,
                                  (const float*)p.ws_lse, a.out, (int64_t)r.o_ss, a.sinks, a.out_lse,
                                  (const int2*)d_gsplit);
      }
      if (ce != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
  }
  return MLA_OK;
}

int ensure_ws(void** ptr, size_t* have, size_t need) {
  if (*have >= need) return MLA_OK;
  if (*ptr) cudaFree(*ptr);
  *ptr = nullptr;
  *have = 0;
  if (cudaMalloc(ptr, need) != cudaSuccess) return MLA_ERR_CUDA;
  *have = need;
  return MLA_OK;
}

// Scratch of mla_fa_forward_noalloc: the workspace of one call (the split-KV
// partials: f16 O rows, then fp32 lse; with the in-kernel mask gather, the units' cell
// lists after them; for a single-group sparse call whose rows fit, the gathered rows,
// their mask values and the internal list), in static device memory so that the call
// allocates nothing.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
std::vector<void*> g_noalloc_ptr;  // per device: device address of g_noalloc_scratch

// Device address of the scratch array on device `dev` (which must be current).
// Looked up once per device; host code cannot use the symbol itself as a pointer.
int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mutex);
  if ((int)g_noalloc_ptr.size() <= dev) g_noalloc_ptr.resize(dev + 1, nullptr);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return MLA_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" {

int mla_version(void) { return 100; }

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_NULL: return "MLA_ERR_NULL: a required pointer is NULL";
    case MLA_ERR_SHAPE: return "MLA_ERR_SHAPE: a size or stride is out of range";
    case MLA_ERR_TYPE: return "MLA_ERR_TYPE: unknown kcache_type";
    case MLA_ERR_ALIGN: return "MLA_ERR_ALIGN: a pointer or stride breaks 16-byte alignment";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace missing or too small";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA runtime call failed";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a kernel's bounded wait ran out";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: valid but unsupported here";
    case MLA_ERR_INDEX: return "MLA_ERR_INDEX: a sparse index is outside [0, n_kv)";
    default: return "unknown mla status";
  }
}

int mla_set_stream(void* cuda_stream) {
  t_stream = static_cast<cudaStream_t>(cuda_stream);
  return MLA_OK;
}

size_t mla_fa_workspace_size(const mla_fa_args* a) {
  Resolved r;
  if (validate(a, &r) != MLA_OK) return 0;
  DeviceState* st = nullptr;
  if (current_device(&st) != MLA_OK) return 0;
  return workspace_for(r, st->sm_count, nullptr, nullptr);
}

int mla_fa_query_plan(const mla_fa_args* a, int* units, int* max_splits) {
  Resolved r;
  int rc = validate(a, &r);
  if (rc != MLA_OK) return rc;
  DeviceState* st = nullptr;
  rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  workspace_for(r, st->sm_count, units, max_splits);
  return MLA_OK;
}

int mla_fa_plan_for_sms(const mla_fa_args* a, int sm_count, int* units, int* max_splits,
                        size_t* workspace_bytes) {
  if (sm_count < 1) return MLA_ERR_SHAPE;
  Resolved r;
  int rc = validate(a, &r);
  if (rc != MLA_OK) return rc;
  int u = 0, m = 0;
  const size_t need = workspace_for(r, sm_count, &u, &m);
  if (units) *units = u;
  if (max_splits) *max_splits = m;
  if (workspace_bytes) *workspace_bytes = need;
  return MLA_OK;
}

int mla_fa_forward_ex(const mla_fa_args* a, void* workspace, size_t ws_bytes, void* stream) {
  Resolved r;
  int rc = validate(a, &r);
  if (rc != MLA_OK) return rc;
  DeviceState* st = nullptr;
  rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  return run_forward(r, st, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

int mla_fa_forward_noalloc(const mla_fa_args* a, void* stream) {
  Resolved r;
  int rc = validate(a, &r);
  if (rc != MLA_OK) return rc;
  DeviceState* st = nullptr;
  rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  // a sparse pass whose gathered rows do not fit the scratch takes the gather modes,
  // which need only the partials
  if (workspace_for(r, st->sm_count, nullptr, nullptr) > (size_t)MLA_NOALLOC_SCRATCH_BYTES)
    r.no_gathered_rows = true;
  if (workspace_for(r, st->sm_count, nullptr, nullptr) > (size_t)MLA_NOALLOC_SCRATCH_BYTES)
    return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  rc = noalloc_scratch(dev, &scratch);
  if (rc != MLA_OK) return rc;
  return run_forward(r, st, scratch, MLA_NOALLOC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
}

int mla_fa_forward(const void* q, const void* kcache, int kcache_type, const void* mask, int n_q,
                   int n_head, int n_kv, float scale, float* out) {
  mla_fa_args a;
  std::memset(&a, 0, sizeof(a));
  a.q = q;
  a.kcache = kcache;
  a.kcache_type = kcache_type;
  a.mask = mask;
  a.out = out;
  a.n_seq = 1;
  a.n_q = n_q;
  a.n_head = n_head;
  a.n_kv = n_kv;
  a.scale = scale;
  Resolved r;
  int rc = validate(&a, &r);
  if (rc != MLA_OK) return rc;
  DeviceState* st = nullptr;
  rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  const size_t need = workspace_for(r, st->sm_count, nullptr, nullptr);
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    rc = ensure_ws(&st->fwd_ws, &st->fwd_ws_bytes, need);
  }
  if (rc != MLA_OK) return rc;
  return run_forward(r, st, st->fwd_ws, st->fwd_ws_bytes, t_stream);
}

size_t mla_compact_workspace_size(int n_rows, int n_kv) {
  if (n_rows < 1 || n_kv < 1) return 0;
  const int64_t tiles = (n_kv + mla::compact::kTileCells - 1) / mla::compact::kTileCells;
  const size_t tickets = (((size_t)n_rows * 4) + 255) / 256 * 256;
  return tickets + (size_t)n_rows * tiles * 8;
}

int mla_compact_mask_ex(const void* mask, int n_rows, int64_t mask_row_stride, int n_kv,
                        int32_t* idx_out, int64_t idx_row_stride, int32_t* count_out,
                        void* workspace, size_t ws_bytes, void* stream) {
  if (mask == nullptr || idx_out == nullptr || count_out == nullptr) return MLA_ERR_NULL;
  if (n_rows < 1 || n_kv < 1) return MLA_ERR_SHAPE;
  if (mask_row_stride == 0) mask_row_stride = n_kv;
  if (idx_row_stride == 0) idx_row_stride = n_kv;
  if (mask_row_stride < n_kv || idx_row_stride < n_kv) return MLA_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(mask) & 1) || (reinterpret_cast<uintptr_t>(idx_out) & 3) ||
      (reinterpret_cast<uintptr_t>(count_out) & 3))
    return MLA_ERR_ALIGN;
  const size_t need = mla_compact_workspace_size(n_rows, n_kv);
  if (workspace == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return MLA_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  int rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  uint32_t epoch;
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    epoch = st->cmp_epoch;
    st->cmp_epoch = (st->cmp_epoch + 1) & 0x3FFFFFFFu;
    if (st->cmp_epoch == 0) st->cmp_epoch = 1;
  }
  const int tiles = (n_kv + mla::compact::kTileCells - 1) / mla::compact::kTileCells;
  const size_t tickets_bytes = (((size_t)n_rows * 4) + 255) / 256 * 256;
  int* tickets = static_cast<int*>(workspace);
  auto* flags = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) + tickets_bytes);
  dim3 grid(tiles, n_rows);
  {
    ProfScope prof(kKernCompact, static_cast<cudaStream_t>(stream));
    mla::mla_compact_kernel<<<grid, mla::compact::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(mask), mask_row_stride, n_kv, idx_out, idx_row_stride,
        count_out, tickets, flags, epoch, kDefaultTimeoutNs);
  }
  if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

int mla_fa_combine_strided(const float* o_parts, int64_t o_part_stride, const float* lse_parts,
                           int64_t lse_part_stride, int n_parts, int64_t rows, float* out,
                           float* out_lse, void* stream) {
  if (o_parts == nullptr || lse_parts == nullptr || out == nullptr) return MLA_ERR_NULL;
  if (n_parts < 1 || n_parts > MLA_COMBINE_MAX_PARTS || rows < 1) return MLA_ERR_SHAPE;
  if (o_part_stride < rows * MLA_DV || lse_part_stride < rows) return MLA_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(o_parts) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (reinterpret_cast<uintptr_t>(lse_parts) & 3) || (reinterpret_cast<uintptr_t>(out_lse) & 3) ||
      (o_part_stride % 4) != 0)
    return MLA_ERR_ALIGN;
  DeviceState* st = nullptr;
  int rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  const unsigned grid = (unsigned)std::min<int64_t>(rows, (int64_t)1 << 30);
  {
    ProfScope prof(kKernMerge, static_cast<cudaStream_t>(stream));
    mla::mla_merge_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(
        o_parts, o_part_stride, lse_parts, lse_part_stride, n_parts, rows, out, out_lse);
  }
  if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

int mla_fa_combine(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows,
                   float* out, float* out_lse, void* stream) {
  return mla_fa_combine_strided(o_parts, rows * MLA_DV, lse_parts, rows, n_parts, rows, out, out_lse,
                                stream);
}

int mla_compact_mask(const void* mask_row, int n_kv, int32_t* idx_out, int32_t* count_out,
                     void* stream) {
  if (mask_row == nullptr || idx_out == nullptr || count_out == nullptr) return MLA_ERR_NULL;
  if (n_kv < 1) return MLA_ERR_SHAPE;
  DeviceState* st = nullptr;
  int rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  const size_t need = mla_compact_workspace_size(1, n_kv);
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    const bool fresh = st->cmp_ws_bytes < need;
    rc = ensure_ws(&st->cmp_ws, &st->cmp_ws_bytes, need);
    if (rc == MLA_OK && fresh &&
        cudaMemset(st->cmp_ws, 0, st->cmp_ws_bytes) != cudaSuccess)
      rc = MLA_ERR_CUDA;
  }
  if (rc != MLA_OK) return rc;
  return mla_compact_mask_ex(mask_row, 1, n_kv, n_kv, idx_out, n_kv, count_out, st->cmp_ws,
                             st->cmp_ws_bytes, stream ? stream : t_stream);
}

int mla_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, mla::g_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(mla::g_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  }
  return v;
}

int mla_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  DeviceState* st = nullptr;
  int rc = current_device(&st);
  if (rc != MLA_OK) return rc;
  {
    ProfScope prof(kKernWaitTest, static_cast<cudaStream_t>(stream));
    mla::mla_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_prof_mutex);
  for (auto& rec : g_prof_records) {
    g_prof_pool.push_back(rec.start);
    g_prof_pool.push_back(rec.stop);
  }
  g_prof_records.clear();
  g_prof_on = true;
  return MLA_OK;
}

int mla_profile_end(mla_profile_entry* entries, int max_entries, int* n_entries) {
  std::lock_guard<std::mutex> lk(g_prof_mutex);
  g_prof_on = false;
  int launches[kNumKernels] = {0};
  double ms[kNumKernels] = {0.0};
  int rc = MLA_OK;
  for (auto& rec : g_prof_records) {
    float t = 0.f;
    if (cudaEventSynchronize(rec.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, rec.start, rec.stop) != cudaSuccess)
      rc = MLA_ERR_CUDA;
    launches[rec.kernel] += 1;
    ms[rec.kernel] += t;
    g_prof_pool.push_back(rec.start);
    g_prof_pool.push_back(rec.stop);
  }
  g_prof_records.clear();
  int n = 0;
  for (int k = 0; k < kNumKernels; ++k) {
    if (launches[k] == 0) continue;
    if (entries != nullptr && n < max_entries) {
      std::memset(&entries[n], 0, sizeof(mla_profile_entry));
      std::strncpy(entries[n].name, kKernelNames[k], sizeof(entries[n].name) - 1);
      entries[n].launches = launches[k];
      entries[n].total_ms = ms[k];
    }
    ++n;
  }
  if (n_entries) *n_entries = std::min(n, max_entries);
  return rc;
}

}  // extern "C"
