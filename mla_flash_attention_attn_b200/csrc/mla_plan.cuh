// Tile ranges from the mask, and the split plan built from them on the device.
//
// The mask drops every cell it sets to -inf, so a key tile whose cells are -inf for every
// query row of a 128-row group contributes nothing to that group (Vulkan FA for DeepSeek
// MLA article, section 2.2: work the mask removes is skipped; a causal chunk ends each
// token's keys at its own position, and padded cells past a sequence's length are -inf).
// Without host lengths, or with several query tokens per group, the host cannot know
// those ranges; two small kernels find them on the device before the attention kernel:
//  * mla_scan_kernel: one CTA per (sequence, 128-row group) finds the first and the last
//    kept cell of the group's token rows and records the group's 256-key tile range;
//  * mla_device_plan_kernel: one CTA turns the ranges into work units. With as many
//    groups as SM pairs or more, a unit is a group; with fewer, each group gets KV splits
//    in proportion to its tiles (never more units than SM pairs, the rounding taken back
//    from the group whose units grow least, as in the host plan), and its split partials
//    a run of slots that the combine reads through the per-group table.
// Both run as programmatic dependents of the kernel before them; nothing reads their
// output before griddepcontrol.wait.
#pragma once
#include <cstdint>

#include "mla_common.cuh"

namespace mla {

// One work unit of the device plan (8 ints): sequence in the launch (-1: the unit is idle
// and writes nothing), 128-row group, split, splits of the group, first tile, tiles, and
// the unit's partial slot (-1: the unit writes the output rows).
struct DevUnit {
  int b, g, s, n_split, tile_begin, n_tiles, slot, pad;
};
static_assert(sizeof(DevUnit) == 32, "device unit descriptor size");

constexpr int kDevPlanMaxGroups = 128;  // groups the split branch handles (fewer than SM pairs)

__global__ void __launch_bounds__(256)
    mla_scan_kernel(const __grid_constant__ Plan plan, const uint16_t* __restrict__ mask,
                    int64_t mask_seq_stride, int64_t mask_row_stride, int vec_ok,
                    int2* __restrict__ ranges) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int red[2][8];
  const int bg = blockIdx.x;
  const int b = bg / plan.groups, g = bg % plan.groups;
  const int len = plan.kv_len[b];
  const int row_lo = g * kRowsPerGroup;
  const int t_lo = row_lo / plan.n_head;
  const int t_hi = min(plan.rows - 1, row_lo + kRowsPerGroup - 1) / plan.n_head;
  int first = 0x7fffffff, last = -1;
  auto note = [&](int cell0, uint32_t keep) {
    if (keep) {
      first = min(first, cell0 + __ffs(keep) - 1);
      last = max(last, cell0 + 31 - __clz(keep));
    }
  };
  // chunks of 8 cells; with 16-byte rows a thread issues kBatch chunk loads at once (one
  // round trip to memory per kBatch x 256 chunks), the cells past the last whole chunk go
  // one by one
  constexpr int kBatch = 16;
  const int n_vec = vec_ok ? (len >> 3) : 0;
  for (int t = t_lo; t <= t_hi; ++t) {
    const uint16_t* mr = mask + (int64_t)(plan.seq_offset + b) * mask_seq_stride + (int64_t)t * mask_row_stride;
    const uint4* mv = reinterpret_cast<const uint4*>(mr);
    for (int c0 = 0; c0 < n_vec; c0 += kBatch * (int)blockDim.x) {
      uint4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int c = c0 + (int)threadIdx.x + u * (int)blockDim.x;
        v[u] = c < n_vec ? __ldg(mv + c) : make_uint4(0xFC00FC00u, 0xFC00FC00u, 0xFC00FC00u, 0xFC00FC00u);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t keep = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if ((w[k] & 0xFFFFu) != 0xFC00u) keep |= 1u << (2 * k);
          if ((w[k] >> 16) != 0xFC00u) keep |= 2u << (2 * k);
        }
        note(8 * (c0 + (int)threadIdx.x + u * (int)blockDim.x), keep);
      }
    }
    for (int cell = 8 * n_vec + (int)threadIdx.x; cell < len; cell += blockDim.x)
      if (__ldg(mr + cell) != 0xFC00u) note(cell, 1u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
  }
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][warp] = first;
    red[1][warp] = last;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < nw; ++w) {
      first = min(first, red[0][w]);
      last = max(last, red[1][w]);
    }
    ranges[bg] = last < 0 ? make_int2(0, 0) : make_int2(first / plan.tile_keys, last / plan.tile_keys + 1);
  }
}

// ranges [groups of the launch]: tile ranges from mla_scan_kernel; units [grid_units]:
// the descriptors the attention kernel reads (grid_units = the groups when there are at
// least `pairs` of them, else `pairs`); gsplit [groups]: {first partial slot or -1,
// splits} for the combine.
// max_split caps the splits of a group (the combine the host launches for them reads at
// most that many partials in one round trip).
__global__ void __launch_bounds__(256)
    mla_device_plan_kernel(const __grid_constant__ Plan plan, const int2* __restrict__ ranges, int pairs,
                           int max_split, int grid_units, DevUnit* __restrict__ units,
                           int2* __restrict__ gsplit) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int n_groups = plan.n_seq * plan.groups;
  if (n_groups >= pairs || n_groups > kDevPlanMaxGroups) {
    // a unit per group, no splits
    for (int u = threadIdx.x; u < grid_units; u += blockDim.x) {
      DevUnit d;
      if (u < n_groups) {
        const int2 r = ranges[u];
        d = {u / plan.groups, u % plan.groups, 0, 1, r.x, r.y - r.x, -1, 0};
        gsplit[u] = make_int2(-1, 1);
      } else {
        d = {-1, 0, 0, 1, 0, 0, -1, 0};
      }
      units[u] = d;
    }
    return;
  }
  __shared__ int tiles[kDevPlanMaxGroups];
  __shared__ int ns[kDevPlanMaxGroups];
  __shared__ int base[kDevPlanMaxGroups + 1];
  for (int i = threadIdx.x; i < n_groups; i += blockDim.x) {
    const int2 r = ranges[i];
    tiles[i] = r.y - r.x;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t sum = 0;
    for (int i = 0; i < n_groups; ++i) sum += tiles[i];
    int total = 0;
    for (int i = 0; i < n_groups; ++i) {
      int n = 1;
      if (sum > 0) {
        const float want = (float)pairs * (float)tiles[i] / (float)sum;
        n = max(1, min(min((int)floorf(want + 0.5f), max(1, tiles[i])), max_split));
      }
      ns[i] = n;
      total += n;
    }
    // rounding can ask for more units than SM pairs: take splits back one at a time from
    // the group whose units grow least (in tiles per unit) by losing one
    while (total > pairs) {
      int best = -1, best_load = 0;
      for (int i = 0; i < n_groups; ++i) {
        if (ns[i] <= 1) continue;
        const int load = (tiles[i] + ns[i] - 2) / (ns[i] - 1);
        if (best < 0 || load < best_load) {
          best = i;
          best_load = load;
        }
      }
      if (best < 0) break;
      --ns[best];
      --total;
    }
    int u = 0, slots = 0;
    for (int i = 0; i < n_groups; ++i) {
      base[i] = u;
      u += ns[i];
      gsplit[i] = make_int2(ns[i] > 1 ? slots : -1, ns[i]);
      if (ns[i] > 1) slots += ns[i];
    }
    base[n_groups] = u;
  }
  __syncthreads();
  for (int u = threadIdx.x; u < grid_units; u += blockDim.x) {
    DevUnit d = {-1, 0, 0, 1, 0, 0, -1, 0};
    if (u < base[n_groups]) {
      int i = 0;
      while (base[i + 1] <= u) ++i;
      const int s = u - base[i], n = ns[i];
      const int2 r = ranges[i];
      const int t0 = (int)((int64_t)s * tiles[i] / n), t1 = (int)((int64_t)(s + 1) * tiles[i] / n);
      const int2 gs = gsplit[i];
      d = {i / plan.groups, i % plan.groups, s, n, r.x + t0, t1 - t0, gs.x >= 0 ? gs.x + s : -1, 0};
    }
    units[u] = d;
  }
}

}  // namespace mla
