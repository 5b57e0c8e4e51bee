"""Which independent units of a gated-retention prefill each rank takes.

Every (sequence, head) pair is its own recurrence chain (page "YOCO 完全拆解：Decoder-Decoder
架构如何让 KV Cache 只存一次", section "路线二：Multi-Head Gated Retention": one state per head,
no interaction between heads or sequences), so N ranks, one per GPU, split the chains with no
exchange on the data path: each rank prefills its own heads or its own sequences and no
collective is needed.  These helpers only decide the split; the prefill itself is the regular
call on the rank's slice.
"""
from typing import List, Sequence, Tuple


def head_range(H: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous heads [h0, h1) of rank `rank` among `world`: sizes differ by at most one."""
    if not (0 <= rank < world) or H < 0:
        raise ValueError("need 0 <= rank < world and H >= 0")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def sequence_assignment(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Packed sequences to ranks, balancing tokens: longest first, each to the rank with the
    fewest tokens so far (ties to the lower rank).  Returns, per rank, the indices of its
    sequences in their original order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if any(n < 0 for n in lengths):
        raise ValueError("sequence lengths must be >= 0")
    load = [0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(lengths)), key=lambda i: (-lengths[i], i)):
        r = min(range(world), key=lambda r: (load[r], r))
        out[r].append(i)
        load[r] += lengths[i]
    return [sorted(x) for x in out]


def packed_subset(cu_seqlens: Sequence[int], indices: Sequence[int]):
    """The token rows of sequences `indices` of a packed batch, and the cu_seqlens of the packed
    sub-batch they form.  Returns (rows, sub_cu): rows is a list of (start, end) token ranges in
    the original batch, in the order of `indices`."""
    rows, sub_cu = [], [0]
    for i in indices:
        a, b = int(cu_seqlens[i]), int(cu_seqlens[i + 1])
        rows.append((a, b))
        sub_cu.append(sub_cu[-1] + (b - a))
    return rows, sub_cu
