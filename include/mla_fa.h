/*
 * mla_fa.h -- C ABI of libmla_fa.so: fused flash attention for Multi-head
 * Latent Attention (MLA) over the compressed KV cache, on NVIDIA B200 (sm_100a).
 *
 * What the library computes (one query row = one (token t, head h) pair):
 *
 *     S[j]   = scale * dot(q[t,h,0:576], k[j,0:576]) + mask[t,j]
 *     P      = softmax over j of S
 *     out[t,h,0:512] = sum_j P[j] * k[j,0:512]
 *
 * Sources (web pages on MLA flash attention):
 *  - Cache row = kv_lora_rank (512) latent followed by the n_embd_head_qk_rope
 *    (64) RoPE key, 576 values, one row per token, shared by all query heads:
 *    ik_llama.cpp "-mla" guide, section "MLA 是什麼".
 *  - With flash attention there is only a K cache; V is derived from it. Here
 *    V = the first 512 columns of the same row: ik_llama.cpp "-mla" guide,
 *    section "-mla四檔語義". Q arrives already absorbed (576 wide); the
 *    up/down projections are outside this library.
 *  - Block-wise online softmax with a running max m and running sum l, so the
 *    score matrix never reaches device memory: Vulkan FA for DeepSeek MLA
 *    article, sections 2.1-2.2.
 *  - f16 additive mask: baguaai flash-attention tag page (PR #23764 item).
 *  - Quantised q8_0 K cache (-ctk q8_0): ik_llama.cpp "-mla" guide, section
 *    on recommended command lines; sparse FA over a quantised cache and the
 *    single-scan mask-index compaction: llama.cpp b11413 release note.
 *
 * Conventions for every entry point:
 *  - All pointers to tensors are DEVICE pointers owned by the caller, except
 *    where an argument says HOST. The library never frees caller memory.
 *  - Every call checks its arguments on the host before any launch and
 *    returns a mla_status; nothing aborts, throws or prints.
 *  - Launches go to the given CUDA stream (cudaStream_t passed as void*;
 *    NULL = the legacy default stream). No call synchronises the stream except
 *    mla_get_device_status.
 *  - Errors a kernel meets at run time (a bounded wait that ran out) are
 *    recorded in a per-device status word read by mla_get_device_status.
 */
#ifndef MLA_FA_H
#define MLA_FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_DK 576            /* cache row / query width: 512 latent + 64 rope */
#define MLA_DV 512            /* value width: the first 512 columns of a row   */
#define MLA_Q8_0_BLOCK 32     /* q8_0: 32 int8 per block                        */
#define MLA_Q8_0_ROW_BYTES 612 /* q8_0: 18 blocks x {f16 d; int8 q[32]}         */
#define MLA_MAX_HEADS 128
#define MLA_PROJ_DIM 128      /* output width of the fused value up-projection   */
#define MLA_HEADS_DK 192      /* head shape with a K and a V per KV head: K width */
#define MLA_HEADS_DV 128      /*   ... and V width                                 */

typedef enum {
  MLA_KV_F16 = 0,  /* row = 576 f16 (1152 bytes) */
  MLA_KV_Q8_0 = 1  /* row = 18 blocks of {f16 d; int8 q[32]} (612 bytes), value = d*q */
} mla_kv_type;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_NULL = -1,        /* a required pointer is NULL                      */
  MLA_ERR_SHAPE = -2,       /* a size or stride is out of range                */
  MLA_ERR_TYPE = -3,        /* unknown kcache_type                             */
  MLA_ERR_ALIGN = -4,       /* a pointer or stride breaks 16-byte alignment    */
  MLA_ERR_WORKSPACE = -5,   /* workspace missing or smaller than required      */
  MLA_ERR_CUDA = -6,        /* a CUDA runtime call failed; as a device status:
                               a kernel launched with less dynamic shared memory
                               than it needs (it returned without working)      */
  MLA_ERR_TIMEOUT = -7,     /* a kernel's bounded wait ran out (device status) */
  MLA_ERR_UNSUPPORTED = -8, /* valid but unsupported (e.g. no sm_100 device)   */
  MLA_ERR_INDEX = -9        /* a sparse index outside [0, n_kv) (device status) */
} mla_status;

/* Full argument set of the batched / sparse forward pass.
 *
 * q       f16, element (b, t, h, c) at q[b*q_seq_stride + (t*n_head + h)*dk + c], dk the
 *         head width (576, or 512 with head_dim = 512)
 * kcache  row (b, j) at byte offset (b*k_seq_stride + j) * row_bytes, where
 *         row_bytes = 2*dk (MLA_KV_F16: 1152, or 1024) or 612 (MLA_KV_Q8_0); the
 *         bytes from kcache to the end of row (n_seq - 1, n_kv - 1) must be one
 *         readable buffer (a gather of listed q8_0 rows copies each row's 16-byte
 *         aligned span, up to 12 bytes next to the row, inside that range)
 * mask    f16 or NULL, element (b, t, j) at mask[b*mask_seq_stride + t*mask_row_stride + j];
 *         0 keeps a cell, -inf drops it, any finite value is added to the score;
 *         shared by all heads of a token
 * out     fp32, element (b, t, h, d) at out[b*out_seq_stride + (t*n_head + h)*512 + d]
 * kv_len  HOST int32[n_seq] or NULL: cells j >= kv_len[b] are dropped; NULL means
 *         n_kv for every sequence. With an f16 cache and no idx, whole 256-key tiles
 *         are loaded: rows from kv_len[b] up to the next multiple of 256 (and below
 *         n_kv) are read and weighted by exactly 0, so they must hold finite values
 *         (a NaN or Inf there would reach the output)
 * idx     DEVICE int32 or NULL (sparse): sequence b attends only to cache rows
 *         idx[b*idx_seq_stride + i] for i < idx_count[b], each in [0, n_kv) and,
 *         as mla_compact_mask writes them, ascending; the mask (if any) is still
 *         indexed by the original cell j = idx[...]
 * idx_count DEVICE int32[n_seq]; required with idx. Read on the device: no host sync.
 * wv      DEVICE f16 or NULL: the value up-projection W_UV of each head, element
 *         (h, d, n) at wv[(h*512 + d)*proj_dim + n] (wv_b of the ik_llama.cpp -mla guide,
 *         section on tensor derivation: per head 512 latent columns -> 128). When set,
 *         the call writes out_proj instead of out (out may then be NULL):
 *           out_proj(b, t, h, n) = sum_{d<512} O(b, t, h, d) * wv(h, d, n)
 *         with O the attention row that out would hold; 16-byte aligned
 * proj_dim output width of the projection; must be MLA_PROJ_DIM (128) when wv is set
 * out_proj DEVICE fp32, element (b, t, h, n) at
 *         out_proj[b*out_proj_seq_stride + (t*n_head + h)*proj_dim + n]; 16-byte aligned
 * sinks   DEVICE fp32 [n_head] or NULL: attention sinks, one extra logit per head in
 *         the softmax denominator with no value:
 *           o = sum_j e^{s_j} v_j / (e^{sinks[h]} + sum_j e^{s_j})
 * alibi_slopes DEVICE fp32 [n_head] or NULL: ALiBi, s_j += alibi_slopes[h] * (j - p_t)
 *         with j the key's cache position and p_t = kv_len[b] - n_q + t the query's
 *         position (the n_q query tokens are the last positions of the sequence).
 *         Not supported with idx (MLA_ERR_UNSUPPORTED)
 * softcap > 0: logit softcap, the scaled score becomes softcap * tanh(score / softcap)
 *         before the mask is added; 0 = off
 * (the variants are named for the Metal FA kernel of the llama.cpp tag page, PR
 * #29570; these formulas are this library's reading of them)
 * mask_gather 1: sparse attention straight from the mask, without an index list
 *         (for any n_q): only the cache rows that some query row of a 128-row group
 *         keeps (mask != -inf) are attended, and each row still applies its own mask.
 *         When a sequence has a single 128-row group (n_q * n_head <= 128), its list
 *         of such cells is built in the workspace (the union of its tokens' masks,
 *         one compaction) and attended as an index list (below); with more groups the
 *         cells, in chunks of 8, are dealt round-robin to a sequence's KV splits and
 *         every work unit compacts its chunks inside the attention kernel. Requires
 *         mask, excludes idx and alibi_slopes. The workspace then also holds the cell
 *         lists
 * out_lse DEVICE fp32 [n_seq][n_q][n_head] or NULL: each row's natural log-sum-exp of
 *         its scores, lse = log sum_j exp(scale q.k_j + mask_j) (-inf for a row with
 *         nothing kept), next to out. With it, partial results of the same rows over
 *         disjoint key ranges (a cache split across devices, say) merge exactly with
 *         mla_fa_combine. Every sequence then writes partials. Excludes sinks and wv
 *         (MLA_ERR_UNSUPPORTED); 4-byte aligned
 * head_dim 0 or MLA_DK (576): the latent + RoPE row above. MLA_DV (512): the DK = DV =
 *         512 head shape (one of the head shapes the llama.cpp tag page lists for the
 *         Metal FA kernel, PR #29570): q and the cache rows are 512 wide and V is the
 *         whole row. f16 cache only (else MLA_ERR_UNSUPPORTED); dense or index-list
 *         attention, with sinks, out_lse and wv as above; softcap, ALiBi and mask_gather
 *         MLA_ERR_UNSUPPORTED. MLA_HEADS_DK (192): the DK = 192 / DV = 128 head shape of
 *         the same list, read as attention with a K and a V per KV head (below).
 *         Other values MLA_ERR_SHAPE
 *
 * The DK = 192 / DV = 128 shape (head_dim = MLA_HEADS_DK): n_kv_head KV heads, query
 * head h reads KV head h / (n_head / n_kv_head) (n_kv_head = n_head: multi-head
 * attention; fewer: grouped heads sharing a K and a V); per query row
 *     S[j] = scale * dot(q[t,h,0:192], k[j,kvh,0:192]) + mask[t,j]
 *     out[t,h,0:128] = sum_j softmax(S)[j] * v[j,kvh,0:128]
 * q       f16, element (b, t, h, c) at q[b*q_seq_stride + (t*n_head + h)*192 + c]
 * kcache  f16 K, element (b, j, kvh, c) at kcache[(b*k_seq_stride + j)*n_kv_head*192 + kvh*192 + c]
 * v       f16 V, element (b, j, kvh, d) at v[(b*v_seq_stride + j)*n_kv_head*128 + kvh*128 + d]
 * out     fp32, element (b, t, h, d) at out[b*out_seq_stride + (t*n_head + h)*128 + d]
 * mask and kv_len as above (the mask shared by the heads of a token). f16 only; idx,
 * mask_gather, wv, sinks, ALiBi, softcap and out_lse MLA_ERR_UNSUPPORTED. q, kcache, v
 * and out 16-byte aligned. Other head widths take v = NULL and n_kv_head = 0.
 * v_seq_stride rows between sequences of v (0 = n_kv); n_kv_head must divide n_head.
 * A stride of 0 means "dense" (the natural value for the given sizes).
 */
typedef struct mla_fa_args {
  const void* q;
  const void* kcache;
  int kcache_type;
  const void* mask;
  float* out;
  int n_seq;
  int n_q;
  int n_head;
  int n_kv;
  float scale;
  int64_t q_seq_stride;     /* elements; 0 = n_q*n_head*dk                     */
  int64_t k_seq_stride;     /* rows;     0 = n_kv                              */
  int64_t mask_seq_stride;  /* elements; 0 = n_q*mask_row_stride               */
  int64_t mask_row_stride;  /* elements; 0 = n_kv                              */
  int64_t out_seq_stride;   /* elements; 0 = n_q*n_head*512                    */
  const int32_t* kv_len;    /* HOST, optional                                  */
  const int32_t* idx;       /* DEVICE, optional (sparse)                       */
  const int32_t* idx_count; /* DEVICE, required with idx                       */
  int64_t idx_seq_stride;   /* entries;  0 = n_kv                              */
  const void* wv;           /* DEVICE, optional: fused value up-projection     */
  int proj_dim;             /* MLA_PROJ_DIM when wv is set                     */
  float* out_proj;          /* DEVICE, required with wv                        */
  int64_t out_proj_seq_stride; /* elements; 0 = n_q*n_head*proj_dim            */
  const float* sinks;       /* DEVICE fp32 [n_head], optional                  */
  const float* alibi_slopes; /* DEVICE fp32 [n_head], optional                 */
  float softcap;            /* > 0 enables the logit softcap                   */
  int mask_gather;          /* 1: gather the mask's kept cells (no idx)        */
  float* out_lse;           /* DEVICE, optional: natural log-sum-exp per row   */
  int head_dim;             /* 0 / MLA_DK: 576-wide heads; MLA_DV: 512;
                               MLA_HEADS_DK: 192 (K and V per KV head)          */
  const void* v;            /* DEVICE f16, head_dim = MLA_HEADS_DK only        */
  int64_t v_seq_stride;     /* rows; 0 = n_kv                                  */
  int n_kv_head;            /* head_dim = MLA_HEADS_DK only: KV heads          */
} mla_fa_args;

/* Forward pass with the sizes of the single-sequence call:
 *   q [n_q][n_head][576] f16, kcache [n_kv] rows of kcache_type,
 *   mask [n_q][n_kv] f16 or NULL, out [n_q][n_head][512] fp32.
 * Uses the stream set by mla_set_stream (per host thread, default NULL) and a
 * workspace the library allocates on first use and keeps (grown as needed).
 * Constraints: 1 <= n_head <= 128, n_q >= 1, n_kv >= 1; q, kcache, out 16-byte aligned.
 * Returns MLA_OK or the first argument error. */
int mla_fa_forward(const void* q, const void* kcache, int kcache_type, const void* mask, int n_q,
                   int n_head, int n_kv, float scale, float* out);

/* Select the stream mla_fa_forward and mla_compact_mask launch on (this thread). */
int mla_set_stream(void* cuda_stream);

/* Bytes of workspace mla_fa_forward_ex needs for these arguments (0 when the
 * pass needs no split-KV partials). Returns 0 as well for invalid arguments.
 * A sparse pass (idx, or mask_gather) whose sequences have a single 128-row group
 * also keeps in the workspace the rows it attends, gathered into a dense f16 buffer
 * (head width x 2 bytes per row, for as many rows per sequence as its list can hold:
 * the smaller of idx_seq_stride and its length), and their mask values. */
size_t mla_fa_workspace_size(const mla_fa_args* a);

/* Batched / sparse forward pass into caller-owned workspace (device memory of
 * at least mla_fa_workspace_size(a) bytes, 256-byte aligned; may be NULL when
 * that size is 0). Split-KV partials go to the workspace and are merged by the
 * log-sum-exp combine before the call's last kernel ends. With wv set, every
 * sequence writes partials (so the workspace is never 0 bytes) and the combine
 * applies the projection. Errors: wv without out_proj MLA_ERR_NULL, proj_dim other
 * than MLA_PROJ_DIM MLA_ERR_UNSUPPORTED, misaligned wv / out_proj / stride
 * MLA_ERR_ALIGN. */
int mla_fa_forward_ex(const mla_fa_args* a, void* workspace, size_t ws_bytes, void* stream);

/* Forward pass for callers that cannot allocate device memory. The paper has no
 * counterpart to this entry point; it exists for users of this library.
 *
 * Some callers can't let a library call cudaMalloc: an inference engine that
 * reserves almost all of the GPU's memory for its KV cache at start-up (so a
 * later cudaMalloc fails or overcommits), a framework whose own allocator must
 * account for every byte, or a decode loop that cannot afford the device-wide
 * synchronisation cudaMalloc and cudaFree may cause. This call takes the same
 * arguments and gives the same results as mla_fa_forward_ex, but allocates
 * nothing: its split-KV partials go to a scratch array of
 * MLA_NOALLOC_SCRATCH_BYTES that the library declares in static device memory.
 * Every GPU that loads the library holds that array until the process exits.
 * The caller still passes q, kcache, mask and out.
 *
 * - A sparse pass whose gathered rows (see mla_fa_workspace_size) do not fit the
 *   scratch attends over its list with the gather inside the attention kernel,
 *   which keeps only the partials in the scratch.
 * - If the pass needs more scratch than MLA_NOALLOC_SCRATCH_BYTES even so, it
 *   returns MLA_ERR_WORKSPACE before launching anything.
 * - The first call on a device looks up the array's device address once
 *   (cudaGetSymbolAddress) with that device current; make that first call before
 *   any stream capture. The address is kept for the life of the process, so do
 *   not use this call after cudaDeviceReset or from another context on the same
 *   device (either one reloads the module and moves the array).
 * - All calls share the one array and it keeps the last call's contents. Nothing
 *   in it needs to start at zero: each call writes every partial it reads. Calls
 *   that overlap on the GPU (on different streams, or different host threads
 *   without ordering) race on it and give wrong results. */
#define MLA_NOALLOC_SCRATCH_BYTES (24u << 20)
int mla_fa_forward_noalloc(const mla_fa_args* a, void* stream);

/* Merge of partial results of the same query rows over disjoint key sets (the
 * log-sum-exp rule of the split-KV combine, applied across calls, e.g. a cache
 * split across devices whose per-device results were gathered):
 *   M = max_p lse_p[r],  w_p = exp(lse_p[r] - M),
 *   out[r] = sum_p w_p o_p[r] / sum_p w_p,   out_lse[r] = M + log(sum_p w_p).
 * A row whose parts are all -inf gets out = 0 and out_lse = -inf.
 * o_parts DEVICE fp32 [n_parts][rows][512], part p at o_parts + p*rows*512;
 * lse_parts DEVICE fp32 [n_parts][rows] (natural log, as out_lse of
 * mla_fa_forward_ex writes it); out DEVICE fp32 [rows][512]; out_lse DEVICE fp32
 * [rows] or NULL. 1 <= n_parts <= MLA_COMBINE_MAX_PARTS, rows >= 1; o_parts and
 * out 16-byte aligned, the lse arrays 4-byte aligned. out may not overlap the
 * inputs. Runs on `stream` (NULL: the legacy default stream); no host sync. */
#define MLA_COMBINE_MAX_PARTS 1024
int mla_fa_combine(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows,
                   float* out, float* out_lse, void* stream);

/* The same merge with the parts at any spacing: part p's O rows start at
 * o_parts + p*o_part_stride and its lse at lse_parts + p*lse_part_stride (floats), so the
 * parts can travel as one packed buffer each (rows x 512 values of O, then the rows'
 * lse), gathered across devices by a single all-gather. o_part_stride >= rows*512 and a
 * multiple of 4, lse_part_stride >= rows (else MLA_ERR_SHAPE / MLA_ERR_ALIGN); the rest as
 * mla_fa_combine, which is this call with o_part_stride = rows*512, lse_part_stride = rows. */
int mla_fa_combine_strided(const float* o_parts, int64_t o_part_stride, const float* lse_parts,
                           int64_t lse_part_stride, int n_parts, int64_t rows, float* out,
                           float* out_lse, void* stream);

/* The same plan for a GPU with sm_count SMs, computed on the host alone (no device is
 * queried, nothing is launched): units, max_splits as mla_fa_query_plan, and the
 * workspace bytes mla_fa_workspace_size would return on such a GPU. Any pointer may be
 * NULL. Errors: those of argument validation; sm_count < 1 MLA_ERR_SHAPE. */
int mla_fa_plan_for_sms(const mla_fa_args* a, int sm_count, int* units, int* max_splits,
                        size_t* workspace_bytes);

/* How the pass is divided: units = CTA pairs launched, max_splits = largest
 * number of KV splits of one (sequence, 128-row group). For tests and tools. */
int mla_fa_query_plan(const mla_fa_args* a, int* units, int* max_splits);

/* Single-scan mask compaction (llama.cpp b11413 release note, "single-scan
 * sparse FA index compaction"): writes, in ascending order, the index of every
 * cell of the f16 mask row whose value is not -inf (bits 0xFC00), and the number
 * of such cells to *count_out -- both on the device, with no host sync.
 * mask_row: DEVICE f16[n_kv]; idx_out: DEVICE int32[n_kv]; count_out: DEVICE int32.
 * Uses a small library-owned workspace (allocated once per device). */
int mla_compact_mask(const void* mask_row, int n_kv, int32_t* idx_out, int32_t* count_out,
                     void* stream);

/* Multi-row form with caller workspace: row r of `mask` starts at
 * mask + r*mask_row_stride (elements); its indices go to idx_out + r*idx_row_stride
 * and its count to count_out[r]. workspace: DEVICE, >= mla_compact_workspace_size
 * bytes, 256-byte aligned, zero-filled by the caller before its first use; each
 * call leaves it ready for the next (calls sharing one workspace must not overlap). */
size_t mla_compact_workspace_size(int n_rows, int n_kv);
int mla_compact_mask_ex(const void* mask, int n_rows, int64_t mask_row_stride, int n_kv,
                        int32_t* idx_out, int64_t idx_row_stride, int32_t* count_out,
                        void* workspace, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then return and clear this device's run-time status:
 * MLA_OK, MLA_ERR_TIMEOUT (a bounded wait in a kernel gave up; that kernel's
 * results are invalid) or MLA_ERR_INDEX; MLA_ERR_CUDA if the sync failed. */
int mla_get_device_status(void* stream);

/* Launch a one-CTA kernel that waits on a barrier nothing ever signals, with a
 * wait limit of timeout_ns; it records MLA_ERR_TIMEOUT and returns. Lets a test
 * exercise the bounded-wait error path without a fault. */
int mla_debug_wait_timeout(uint64_t timeout_ns, void* stream);

/* Per-kernel device timing. Between mla_profile_begin and mla_profile_end the
 * library records a pair of CUDA events around every kernel it launches (on
 * that launch's stream) and counts the launches. mla_profile_end synchronises
 * those events and fills up to max_entries records, one per kernel that ran;
 * *n_entries gets the number filled. Profiling state is per process. */
typedef struct mla_profile_entry {
  char name[48];     /* kernel name, e.g. "mla_fwd_f16" */
  int launches;      /* launches recorded                */
  double total_ms;   /* sum of event-timed durations     */
} mla_profile_entry;
int mla_profile_begin(void);
int mla_profile_end(mla_profile_entry* entries, int max_entries, int* n_entries);

/* Human-readable name of a status code (static string). */
const char* mla_status_string(int status);

/* Library version: major*10000 + minor*100 + patch. */
int mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_FA_H */
