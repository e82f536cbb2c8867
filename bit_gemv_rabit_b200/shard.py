"""Row sharding of the residual-binary layer over ranks (one process per GPU).

Each rank owns one contiguous block of output rows.  In RABIT_LAYOUT_V2 a row's words are
contiguous and rows follow one another, so a rank's part of the packed signs is a single
contiguous range of the buffer (a view, no copy); it also owns the same columns of a and
needs all of b and x.  derive_pack and the GEMV run on the block with the library's kernels;
the per-rank outputs meet in one all-gather (torch.distributed: NCCL between GPUs), the only
exchange the layer has, and are laid out as [batch][N].

This module is plumbing around the C ABI: it slices, launches and gathers, and computes
nothing of the layer itself.
"""
from __future__ import annotations

import torch

from . import rabit


def row_block(N: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous rows [begin, end) of rank `rank`: sizes differ by at most one row."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    base, extra = divmod(N, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def words_per_row(K: int, P: int) -> int:
    """uint32 words of one row of the packed layout (G words per 32-column group)."""
    return rabit.rabit_packed_words(1, K, P)


class RowShard:
    """One rank's rows of an N x K layer with P paths."""

    def __init__(self, N: int, K: int, P: int, rank: int, world: int, device=None):
        self.N, self.K, self.P, self.rank, self.world = N, K, P, rank, world
        self.begin, self.end = row_block(N, world, rank)
        self.rows = self.end - self.begin
        self.max_rows = -(-N // world)
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.packed = None
        self.a = None
        self.b = None

    def attach(self, packed_full: torch.Tensor, a: torch.Tensor, b: torch.Tensor) -> "RowShard":
        """Use this rank's rows of an already packed layer (packed_full holds all N rows)."""
        w = words_per_row(self.K, self.P)
        self.packed = packed_full[self.begin * w:self.end * w]
        self.a = a[:, self.begin:self.end].contiguous()
        self.b = b
        return self

    def derive(self, W_rows: torch.Tensor, a: torch.Tensor, b: torch.Tensor) -> "RowShard":
        """Derive and pack this rank's rows: W_rows = W[begin:end] ([rows][K], pitch allowed),
        a the full [P][N] scales, b [P][K]."""
        if W_rows.shape[0] != self.rows:
            raise ValueError(f"W_rows has {W_rows.shape[0]} rows, this rank owns {self.rows}")
        self.a = a[:, self.begin:self.end].contiguous()
        self.b = b
        self.packed = rabit.alloc_packed(max(self.rows, 1), self.K, P=self.P, device=self.device)
        if self.rows:
            rabit.rabit_derive_pack(W_rows, self.a, b, self.packed, P=self.P)
        return self

    def local(self, x: torch.Tensor) -> torch.Tensor:
        """This rank's outputs, [batch][max_rows] fp32 (columns past its rows are zero)."""
        batch = x.shape[0]
        local = torch.zeros((batch, self.max_rows), dtype=torch.float32, device=x.device)
        if self.rows:
            rabit.rabit_gemv(self.packed, self.a, self.b, self.rows, self.K, x, local[:, :self.rows], P=self.P)
        return local

    def gemv(self, x: torch.Tensor, y: torch.Tensor, group=None, check_fault: bool = True) -> torch.Tensor:
        """y[:, n] for all n of the layer, from this rank's rows and one all-gather.
        Every rank of the group must call it (ranks without rows still join the gather).
        With check_fault, a rank whose kernel had a bounded wait expire raises RabitError
        after the gather (so every rank still takes the same collective steps); this
        synchronises the rank's stream once per call."""
        import torch.distributed as dist
        batch = x.shape[0]
        local = self.local(x)
        # ranks' blocks concatenated along dim 0, the form every backend accepts
        gathered = torch.empty((self.world * batch, self.max_rows), dtype=torch.float32, device=y.device)
        dist.all_gather_into_tensor(gathered, local, group=group)
        gathered = gathered.view(self.world, batch, self.max_rows)
        for r in range(self.world):
            b0, b1 = row_block(self.N, self.world, r)
            y[:, b0:b1] = gathered[r, :, :b1 - b0]
        if check_fault and self.rows:
            fault = rabit.rabit_read_fault(clear=True)
            if fault:
                raise rabit.RabitError(-8, f"RowShard.gemv (rank {self.rank}, fault word {fault:#x})")
        return y
