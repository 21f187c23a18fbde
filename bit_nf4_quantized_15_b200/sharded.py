"""NF4 double quantisation of one weight shared out over data-parallel ranks.

Quantisation is independent per group of 16384 weights: a group's 256
blocks of 64 share one second-level scale c1 and nothing crosses a group
boundary (nlp-lineage "QLoRA", section "The idea": blocks of 64, their
scales quantised again).  So each rank quantises a contiguous run of whole
groups of the flattened weight with the library's own kernel, and one
all-gather per buffer (codes, c2, c1) gives every rank the whole quantised
weight, byte for byte what a single-GPU quantisation produces.

The split and the gather are host logic; the quantisation of a rank's share
is a plain ``quantize`` call on a flat ``[1, len]`` view of its range.
"""

from __future__ import annotations

GROUP = 16384   # weights per second-level scale (256 blocks of 64)
BLOCK = 64


def shard_ranges(n_weights: int, world: int):
    """Flat weight range ``[w0, w1)`` of every rank: contiguous runs of whole
    groups, as equal in group count as possible, in rank order, covering
    ``[0, n_weights)`` once (only the last group may be partial; ranks beyond
    the group count get an empty range)."""
    if n_weights < 0 or n_weights % BLOCK or world < 1:
        raise ValueError("n_weights must be a non-negative multiple of 64 and world >= 1")
    groups = (n_weights + GROUP - 1) // GROUP
    out = []
    for r in range(world):
        g0, g1 = r * groups // world, (r + 1) * groups // world
        out.append((min(g0 * GROUP, n_weights), min(g1 * GROUP, n_weights)))
    return out


def part_sizes(w0: int, w1: int):
    """Elements of (codes uint8, c2 uint8, c1 fp32) for the flat range [w0, w1)."""
    n = w1 - w0
    return n // 2, n // BLOCK, (n + GROUP - 1) // GROUP


def gather_parts(local, ranges, rank, group=None):
    """All-gather every rank's (codes, c2, c1) part into the whole buffers.

    ``local``: this rank's three 1-D tensors (sizes from :func:`part_sizes`
    of its range).  Parts are padded to the largest rank's size for the
    collective and trimmed after it; the result is concatenated in rank
    order, i.e. in flat weight order."""
    import torch
    import torch.distributed as dist

    world = len(ranges)
    sizes = [part_sizes(*r) for r in ranges]
    out = []
    for k, t in enumerate(local):
        if t.numel() != sizes[rank][k]:
            raise ValueError("local part size does not match this rank's range")
        mx = max(s[k] for s in sizes)
        pad = torch.zeros(max(mx, 1), dtype=t.dtype, device=t.device)
        pad[: t.numel()] = t
        bufs = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(bufs, pad, group=group)
        out.append(torch.cat([bufs[r][: sizes[r][k]] for r in range(world)]))
    return tuple(out)


def quantize_sharded(W, group=None, fmt: str = "nf4", scale: str = "e4m3", quantize_fn=None):
    """Quantise the bf16 weight ``W [N, K]`` (identical on every rank) with
    each rank doing its share of the groups, then all-gather.  Returns an
    ``NF4Weight`` holding the whole quantised weight on every rank.

    ``quantize_fn(flat_slice) -> (codes, c2, c1)`` replaces the per-rank step
    (default: the library's quantiser on the GPU)."""
    import torch.distributed as dist

    from . import NF4Weight, quantize

    N, K = W.shape
    n = N * K
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    ranges = shard_ranges(n, world)
    w0, w1 = ranges[rank]
    flat = W.reshape(-1)[w0:w1]
    if quantize_fn is not None:
        local = quantize_fn(flat)
    elif w1 > w0:
        part = quantize(flat.view(1, -1), fmt=fmt, scale=scale)
        local = (part.codes, part.c2, part.c1)
    else:
        import torch
        local = (torch.empty(0, dtype=torch.uint8, device=W.device), torch.empty(0, dtype=torch.uint8, device=W.device),
                 torch.empty(0, dtype=torch.float32, device=W.device))
    if world == 1:
        codes, c2, c1 = local
    else:
        codes, c2, c1 = gather_parts(local, ranges, rank, group)
    return NF4Weight(codes, c2, c1, N, K, fmt, scale)
