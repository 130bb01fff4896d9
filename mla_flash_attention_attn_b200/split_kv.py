"""Split-KV decode across ranks (one process per GPU, torch.distributed over NCCL).

Every rank holds a contiguous range of each sequence's cache cells. A step runs the
attention over the local range with each row's log-sum-exp (mla_fa_forward_ex with
out_lse), gathers the ranks' (O, lse) pairs with one all-gather, and merges them by
the log-sum-exp rule (mla_fa_combine): with M = max_r lse_r,
    out = sum_r e^{lse_r - M} O_r / sum_r e^{lse_r - M},
which equals attention over the whole cache because each O_r is the softmax-weighted
mean over the rank's cells. The split-KV combine within one call does the same across
the CTAs of a sequence; this module applies it across devices. torch.distributed is
the plumbing here: the attention and the merge run in this library's kernels.
"""
from . import binding

DV = binding.DV


def shard_bounds(n_kv, world):
    """Contiguous cache ranges [lo, hi) of the ranks, equal to within one cell."""
    if world < 1 or n_kv < world:
        raise ValueError("every rank needs at least one cache cell")
    return [(n_kv * r // world, n_kv * (r + 1) // world) for r in range(world)]


def shard_lengths(kv_len, lo, hi):
    """Valid cells of each sequence inside the range [lo, hi): the sequence's first
    kv_len cells are valid, so the range holds clamp(kv_len - lo, 0, hi - lo)."""
    return [max(0, min(int(n) - lo, hi - lo)) for n in kv_len]


def decode(q, kcache_shard, kv_type, mask_shard, scale, kv_len_shard=None, group=None,
           forward=None, combine=None):
    """One attention step over a cache split across the ranks of `group`.

    q: f16 [n_seq][n_q][n_head][576], the same on every rank; kcache_shard: this rank's
    cells of every sequence's cache, [n_seq][cells][576] f16 (or [..][612] q8_0);
    mask_shard: the mask's columns for those cells, f16 [n_seq][n_q][cells] or None;
    kv_len_shard: valid cells of each sequence in the shard (host ints), or None for all.
    Returns the merged out, fp32 [n_seq][n_q][n_head][512], on every rank.

    The rank writes its O rows and their lse straight into one packed buffer
    (binding.packed_width(rows) floats: O, then lse), and a single all-gather brings the
    ranks' buffers together in rank order: rows x (512 + 1) x 4 bytes sent per rank and
    step. `forward` and `combine` default to this library's calls (binding.forward,
    binding.combine_packed); tests of the orchestration on CPU pass stand-ins with the
    same signatures."""
    import torch
    import torch.distributed as dist

    forward = forward or binding.forward
    combine = combine or binding.combine_packed
    world = dist.get_world_size(group)
    n_seq, n_q, n_head = q.shape[:3]
    rows = n_seq * n_q * n_head
    width = binding.packed_width(rows)
    mine = torch.empty((width,), dtype=torch.float32, device=q.device)
    forward(q, kcache_shard, kv_type, mask_shard, scale,
            out=mine[: rows * DV].view(n_seq, n_q, n_head, DV), kv_len=kv_len_shard,
            out_lse=mine[rows * DV:].view(n_seq, n_q, n_head))
    parts = torch.empty((world * width,), dtype=torch.float32, device=q.device)
    dist.all_gather_into_tensor(parts, mine, group=group)
    out = combine(parts.view(world, width), rows)
    return out.view(n_seq, n_q, n_head, DV)
