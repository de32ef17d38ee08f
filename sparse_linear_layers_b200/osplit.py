"""Output-row split of a Sparse-BitLinear layer across the GPUs of a process group.

Row o of y = dequant(x_q . W_t^T) depends on row o of the latent weights alone
(its N:M mask, its absmean scale and its codes are all per row: Sparse-BitNet
Guide, "Mathematical Formulation of Sparse-BitLinear", and the per-row scale
of the halo-sparse-bitnet-3:4-500m card's "Recipe"), so G GPUs can each own a
contiguous block of output rows.  Preparing a block of latent rows gives
exactly the codes and scales those rows get in the whole matrix; x is
replicated (each GPU quantises it itself, the same bits everywhere); every
GPU contracts its block with sbl_linear and one all-gather assembles y.  This
is the natural partition for decode, where a layer is a stream of weights and
splitting the rows splits the bytes each GPU reads.  (The pages' own
multi-GPU setup is data-parallel training: the Sparse-BitNet README,
"Features", distributed training with DDP.)

Only the global-scale convention (one scale for the whole matrix) does not
split this way; OSplitLinear does not offer it.  All arithmetic runs in the
library's kernels; this module slices, pads and gathers.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import api


def row_block(O: int, world: int, rank: int, align: int = 128):
    """[start, stop) of the output rows rank `rank` owns: blocks of
    ceil(O / world) rows rounded up to a multiple of `align` (the prefill
    kernels' output tile), the last ones shorter or empty."""
    if world < 1 or not 0 <= rank < world or O < 0:
        raise ValueError("bad world, rank or O")
    blk = block_rows(O, world, align)
    start = min(O, rank * blk)
    return start, min(O, start + blk)


def block_rows(O: int, world: int, align: int = 128) -> int:
    per = -(-O // world) if O else 0
    return -(-per // align) * align if per else 0


def gather_rows(y_block: torch.Tensor, O: int, world: int, rank: int, group=None, align: int = 128) -> torch.Tensor:
    """Assemble y [T, O] from every rank's y_block [T, rows of its block] with
    one all-gather (each rank's block padded to the common block width).  For
    T == 1 the result is a view of the gathered buffer; for T > 1 the blocks
    are interleaved into rows by one layout copy."""
    T = y_block.shape[0]
    blk = block_rows(O, world, align)
    start, stop = row_block(O, world, rank, align)
    if y_block.shape != (T, stop - start):
        raise ValueError(f"rank {rank} holds rows [{start}, {stop}) but y_block is {tuple(y_block.shape)}")
    if stop - start == blk:
        stage = y_block.contiguous()
    else:
        stage = torch.zeros((T, blk), dtype=y_block.dtype, device=y_block.device)
        stage[:, :stop - start] = y_block
    out = torch.empty((world * T * blk,), dtype=y_block.dtype, device=y_block.device)
    dist.all_gather_into_tensor(out, stage.reshape(-1), group=group)
    return out.view(world, T, blk).transpose(0, 1).reshape(T, world * blk)[:, :O]


class OSplitLinear:
    """One rank's share of an output-row-split layer: the latent rows of its
    block, prepared once (prepare() again after the latent weights change),
    and a forward that contracts them and all-gathers y.

    W is this rank's block of latent fp32 weights [rows, K] (or the whole
    matrix with `full=True`, from which the block is sliced), on this rank's
    GPU."""

    def __init__(self, W: torch.Tensor, O: int, n: int, m: int, group=None, full: bool = False,
                 align: int = 128):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.O, self.n, self.m, self.align = O, n, m, align
        self.start, self.stop = row_block(O, self.world, self.rank, align)
        if full:
            if W.shape[0] != O:
                raise ValueError("full=True needs the whole [O, K] matrix")
            W = W[self.start:self.stop]
        if W.shape[0] != self.stop - self.start:
            raise ValueError(f"rank {self.rank} owns rows [{self.start}, {self.stop}), got {W.shape[0]} rows")
        self.latent = W.contiguous()
        self.w: Optional[api.PreparedWeights] = None
        self.prepare()

    def prepare(self) -> None:
        self.w = api.sbl_prepare_weights(self.latent, self.n, self.m)

    def __call__(self, x: torch.Tensor, out_dtype: torch.dtype = torch.float32) -> torch.Tensor:
        """y [T, O] = dequant(int8(x) . W_t^T) over all ranks' rows; x bf16 [T, K]
        is the same on every rank."""
        y_block = api.sbl_linear(x, self.w, out_dtype=out_dtype)
        return gather_rows(y_block, self.O, self.world, self.rank, self.group, self.align)
