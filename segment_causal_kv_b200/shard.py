"""Spreading one layer-step of segment attention over ranks (one process per GPU).

Heads share nothing on this path (Hy-Nomas model card, "Segment-Autoregressive
Diffusion Transformer": 16 heads of 128 dimensions, each with its own keys,
values and softmax; the per-(token, head) INT8 scales are per head too). So a
layer's cache and its attention split by head with no exchange at all when the
projections hand every rank the Q/K/V of its own heads: each rank owns a cache
of its heads and calls nomas_kv_commit / nomas_seg_attn on them.

When the inputs arrive split by sequence instead (the model card's "Standard
Inference" runs 8-way sequence parallelism), one all-to-all per tensor turns
token shards into head shards before the commit and the attention, and one
turns the head-sharded output back into token shards (the Ulysses scheme).
Those exchanges are the only collectives; they go through torch.distributed
(NCCL over NVLink on GPUs, gloo on the host). The exchange moves raw bytes, so
it is exact for every element type and backend.

Layouts: a token shard is [n_r][heads][128] (tokens of rank r, all heads); a
head shard is [N][nh_r][128] (all tokens, heads of rank r). Ranks own
contiguous ranges of tokens and of heads, the first (count mod world) ranks one
more than the rest.
"""

from __future__ import annotations

HEAD_DIM = 128


def split_counts(n: int, world: int) -> list[int]:
    """Sizes of `world` contiguous ranges covering [0, n); the first n % world ranges are one longer."""
    if world < 1 or n < 0:
        raise ValueError((n, world))
    base, extra = divmod(n, world)
    return [base + (1 if r < extra else 0) for r in range(world)]


def split_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """(first, count) of rank's contiguous range of [0, n)."""
    if not 0 <= rank < world:
        raise ValueError((rank, world))
    c = split_counts(n, world)
    return sum(c[:rank]), c[rank]


def head_range(heads: int, world: int, rank: int) -> tuple[int, int]:
    """(first head, heads) owned by rank; every rank must own at least one head."""
    if heads < world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks")
    return split_range(heads, world, rank)


def _dist():
    import torch.distributed as dist
    return dist


def _world_rank(group):
    dist = _dist()
    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def max_over_ranks(values, device=None, group=None) -> list[float]:
    """Element-wise maximum of a list of floats over the ranks (a no-op with one rank)."""
    import torch
    world, _ = _world_rank(group)
    vals = [float(x) for x in values]
    if world == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    _dist().all_reduce(t, op=_dist().ReduceOp.MAX, group=group)
    return [float(x) for x in t.tolist()]


def _bytes(x):
    """A [rows][heads][d] tensor as uint8 [rows][heads][d * element size] (a view when contiguous)."""
    import torch
    return x.contiguous().view(torch.uint8)


def seq_to_heads(x, heads: int, token_counts: list[int], group=None):
    """Token shard [n_r][heads][128] -> head shard [sum(token_counts)][nh_r][128].

    token_counts[j] is the number of tokens rank j holds, in token order.
    """
    import torch
    world, rank = _world_rank(group)
    if len(token_counts) != world or x.shape[0] != token_counts[rank] or x.shape[1] != heads:
        raise ValueError((tuple(x.shape), heads, token_counts, world, rank))
    if world == 1:
        return x
    xb = _bytes(x)
    row = xb.shape[2]  # bytes of one (token, head) vector
    hr = [head_range(heads, world, j) for j in range(world)]
    send = torch.cat([xb[:, h0:h0 + nh, :].reshape(-1) for h0, nh in hr])
    nh = hr[rank][1]
    recv = torch.empty(sum(token_counts) * nh * row, dtype=torch.uint8, device=x.device)
    _dist().all_to_all_single(recv, send,
                              output_split_sizes=[c * nh * row for c in token_counts],
                              input_split_sizes=[x.shape[0] * n * row for _, n in hr], group=group)
    return recv.view(sum(token_counts), nh, row).view(x.dtype)


def heads_to_seq(o, heads: int, token_counts: list[int], group=None):
    """Head shard [sum(token_counts)][nh_r][128] -> token shard [n_r][heads][128] (inverse of seq_to_heads)."""
    import torch
    world, rank = _world_rank(group)
    hr = [head_range(heads, world, j) for j in range(world)] if world > 1 else [(0, heads)]
    if len(token_counts) != world or o.shape[0] != sum(token_counts) or o.shape[1] != hr[rank][1]:
        raise ValueError((tuple(o.shape), heads, token_counts, world, rank))
    if world == 1:
        return o
    ob = _bytes(o)
    row = ob.shape[2]
    nh = hr[rank][1]
    n_r = token_counts[rank]
    recv = torch.empty(n_r * heads * row, dtype=torch.uint8, device=o.device)
    _dist().all_to_all_single(recv, ob.reshape(-1),
                              output_split_sizes=[n_r * n * row for _, n in hr],
                              input_split_sizes=[c * nh * row for c in token_counts], group=group)
    chunks, off = [], 0
    for _, n in hr:
        chunks.append(recv[off:off + n_r * n * row].view(n_r, n, row))
        off += n_r * n * row
    return torch.cat(chunks, dim=1).view(o.dtype)
