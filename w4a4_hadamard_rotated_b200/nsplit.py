"""The W4A4 layer split over GPUs along its output features (N-split).

Rows of the layer are independent, and so are its output columns: column n
needs only weight row n, its scale sw[n] and bias[n].  With P ranks, rank r
holds a contiguous block of weight rows [n0_r, n1_r) (packed codes, scales,
bias), computes the fused layer for every activation row into its own
[M, n1_r - n0_r] block of y with the library's kernels, and an all-gather
over the process group (NCCL over NVLink on GPUs) assembles the full
[M, N] output on every rank.  Every rank quantises the whole activation
itself (the activation pass is cheap next to the GEMM, and quantising
locally avoids a second collective).

The blocks are multiples of 8 columns (the library's N % 8 rule keeps every
block's first column 16-byte aligned in a row-major y); when N / P is not a
multiple of 8 the last blocks are narrower, and the all-gather moves blocks
padded to the widest one.

Only plumbing lives here -- partitioning, slicing and the collective; the
layer itself runs in the C-ABI library on each rank.
"""

import torch

ALIGN = 8


def column_blocks(N, world):
    """[(n0, n1)] for every rank: contiguous, disjoint blocks of output
    columns that cover [0, N), each a multiple of 8 wide (the last ones may
    be narrower, or empty when N is small)."""
    if N % ALIGN != 0:
        raise ValueError("N must be a multiple of 8")
    if world < 1:
        raise ValueError("world must be at least 1")
    units = N // ALIGN
    per = -(-units // world)
    out = []
    for r in range(world):
        a = min(units, r * per)
        b = min(units, (r + 1) * per)
        out.append((a * ALIGN, b * ALIGN))
    return out


def shard_weight(Wq, sw, bias, world, rank):
    """This rank's rows of the packed weight, its scales and its bias (views
    of contiguous row blocks, so they stay contiguous)."""
    n0, n1 = column_blocks(Wq.shape[0], world)[rank]
    return Wq[n0:n1], sw[n0:n1], (bias[n0:n1] if bias is not None else None)


def _place_blocks(recv, out, blocks, M, width):
    """Copy the gathered blocks (recv viewed as [world, M, width]) into their
    column slices of out [M, N]: one strided copy when every block is
    `width` wide and out is contiguous, else one copy per block."""
    world = len(blocks)
    N = blocks[-1][1]
    r3 = recv.view(world, M, width)
    if N == world * width and out.is_contiguous():
        out.view(M, world, width).copy_(r3.permute(1, 0, 2))
        return out
    for r, (a, b) in enumerate(blocks):
        if b > a:
            out[:, a:b].copy_(r3[r, :, : b - a])
    return out


def gather_columns(y_local, N, world, rank, group=None, out=None):
    """All-gather the ranks' column blocks into the full y [M, N].

    y_local is this rank's [M, n1 - n0] block.  The blocks travel padded to
    the widest block through one all_gather_into_tensor, then land in their
    column slices of `out` (allocated when not given)."""
    import torch.distributed as dist

    blocks = column_blocks(N, world)
    width = max(b - a for a, b in blocks)
    M = y_local.shape[0]
    n0, n1 = blocks[rank]
    if y_local.shape[1] != n1 - n0:
        raise ValueError(f"rank {rank} holds columns [{n0}, {n1}), got a block of {y_local.shape[1]}")
    send = torch.zeros(M, width, dtype=y_local.dtype, device=y_local.device)
    send[:, : n1 - n0] = y_local
    # the blocks concatenated along rows (the form every backend accepts)
    recv = torch.empty(world * M, width, dtype=y_local.dtype, device=y_local.device)
    if world > 1:
        dist.all_gather_into_tensor(recv, send, group=group)
    else:
        recv.copy_(send)
    if out is None:
        out = torch.empty(M, N, dtype=y_local.dtype, device=y_local.device)
    return _place_blocks(recv, out, blocks, M, width)


class NSplitLinear:
    """One W4A4 layer whose weight rows are split over the ranks of a process
    group.  Construct it on every rank with the full prepared weight (Wq
    [N, K/2], sw [N], bias [N] or None; each rank keeps only its block) or
    with `pre_sharded=True` and this rank's block.  Calling it with the
    activation x [M, K] (bf16, the same on every rank) returns the full
    y [M, N] on every rank.

    Each rank writes its block of y straight into its all-gather send buffer
    (a row stride of the widest block), and the send and receive buffers are
    kept per batch size and device, so a call allocates nothing after the
    first one of its shape (besides `out`, when not given).  With one rank
    the layer writes y directly."""

    def __init__(self, Wq, sw, bias=None, g=128, group=None, pre_sharded=False, N=None):
        import torch.distributed as dist

        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.g = g
        if pre_sharded:
            if N is None:
                raise ValueError("pre_sharded weights need the full N")
            self.N = int(N)
            n0, n1 = column_blocks(self.N, self.world)[self.rank]
            if Wq.shape[0] != n1 - n0:
                raise ValueError(f"rank {self.rank} expects {n1 - n0} weight rows, got {Wq.shape[0]}")
            self.Wq, self.sw, self.bias = Wq, sw, bias
        else:
            self.N = Wq.shape[0]
            self.Wq, self.sw, self.bias = shard_weight(Wq, sw, bias, self.world, self.rank)
        self.blocks = column_blocks(self.N, self.world)
        self.width = max(b - a for a, b in self.blocks)
        self._bufs = {}

    def _buffers(self, M, device):
        key = (M, device)
        if key not in self._bufs:
            # padding columns of send are never written: they stay zero
            send = torch.zeros(M, self.width, dtype=torch.bfloat16, device=device)
            recv = torch.empty(self.world * M, self.width, dtype=torch.bfloat16, device=device)
            self._bufs[key] = (send, recv)
        return self._bufs[key]

    def __call__(self, x, act=0, out=None):
        import torch.distributed as dist
        from . import linear_fused

        M = x.shape[0]
        if self.world == 1:
            return linear_fused(x, self.Wq, self.sw, self.bias, self.g, act, out=out)
        n0, n1 = self.blocks[self.rank]
        send, recv = self._buffers(M, x.device)
        if n1 > n0:
            linear_fused(x, self.Wq, self.sw, self.bias, self.g, act, out=send[:, : n1 - n0])
        dist.all_gather_into_tensor(recv, send, group=self.group)
        if out is None:
            out = torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
        return _place_blocks(recv, out, self.blocks, M, self.width)
