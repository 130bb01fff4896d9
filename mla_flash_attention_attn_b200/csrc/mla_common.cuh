// Shared definitions of the MLA attention kernels: sizes, the launch plan and
// the per-device run-time status word.
#pragma once
#include <cstdint>

namespace mla {

constexpr int kDK = 576;             // cache row / query width (512 latent + 64 rope)
constexpr int kDV = 512;             // value width: first 512 columns of the row
constexpr int kRowsPerGroup = 128;   // M of the 2-SM MMA (64 rows in each CTA)
constexpr int kRowsPerCta = 64;
constexpr int kPlanMaxSeq = 128;     // sequences per launch (larger batches are chunked)
constexpr int kQ8RowBytes = 612;     // q8_0: 18 blocks of {f16 d; int8 q[32]}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Status codes written by kernels (same values as mla_status in mla_fa.h).
constexpr int kStatusLaunch = -6;   // launched with less dynamic shared memory than it needs
constexpr int kStatusTimeout = -7;
constexpr int kStatusIndex = -9;

// How one launch divides its sequences. A unit is one CTA pair: a 128-row
// group of one sequence over one contiguous range of key tiles (a KV split).
struct Plan {
  int n_seq;                         // sequences in this launch
  int seq_offset;                    // index of the launch's first sequence
  int groups;                        // 128-row groups per sequence
  int rows;                          // query rows per sequence (n_q * n_head)
  int n_head;
  int n_q;
  int n_kv;
  int total_units;
  int unit_base[kPlanMaxSeq + 1];    // first unit of each sequence
  int n_split[kPlanMaxSeq];          // KV splits of each sequence
  int kv_len[kPlanMaxSeq];           // dense: cells read for each sequence
  int ws_base[kPlanMaxSeq];          // first partial slot (-1: no split, direct output)
  int tile_keys;                     // keys of a plan tile: the attention kernel's step (128 or 256)
};

}  // namespace mla
