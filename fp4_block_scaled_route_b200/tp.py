"""Tensor parallelism over the expert intermediate size I, one process per GPU.

Rank r of G holds, for every expert (the shared expert included), the I/G
channels c in [r*I/G, (r+1)*I/G): the gate rows c and up rows I + c of w13,
the columns c of w2, and their scales.  I/G must be a multiple of 128, the
FP8 weight-block and activation-requant group, so no quantisation group
straddles two ranks and a rank's SwiGLU channels are exactly those of the
whole layer.  GEMM2 and the top-k combine are linear in the channels, so the
layer's fp32 result is the sum over ranks of the partial results that
``moe_forward_partial`` writes; one all-reduce (sum) over the ranks, then
``moe_finalize_bf16``, gives the layer output.

This module only slices tensors and calls torch.distributed for the sum;
every step of the layer runs in the library's kernels.
"""
from __future__ import annotations

from . import moe

WFMT_FP8 = 0
WFMT_MXFP4 = 1
WFMT_NVFP4 = 2
WFMT_MXFP4_A4 = 3
WFMT_MXFP8 = 4


def shard_weights(w13, s13, w2, s2, wfmt: int, I: int, rank: int, world: int, g13=None, g2=None) -> dict:
    """The slice of rank ``rank`` (of ``world``) of one layer's expert weights.

    Layouts as in include/moe.h, with the MXFP4 / NVFP4 / MXFP8 scales in
    their plain layouts (pack each rank's slice with pack_shard).  Returns a dict w13,
    s13, w2, s2 (contiguous) and, for NVFP4, g13, g2 (unchanged: the
    per-expert global scales apply to every slice)."""
    import torch
    if I % world or (I // world) % 128:
        raise ValueError(f"I/G = {I}/{world} must be a multiple of 128")
    Is = I // world
    c0, c1 = rank * Is, (rank + 1) * Is

    def gate_up(t, a, b, off):
        # rows a..b of the gate half and the same rows of the up half (dim 1)
        return torch.cat([t[:, a:b], t[:, off + a:off + b]], dim=1).contiguous()

    if wfmt == WFMT_FP8:
        b0, b1 = c0 // 128, c1 // 128                          # 128-row / 128-column scale blocks
        return dict(w13=gate_up(w13, c0, c1, I),                # [NE, 2I, H] -> [NE, 2Is, H]
                    s13=gate_up(s13, b0, b1, I // 128),         # [NE, 2I/128, H/128]
                    w2=w2[:, :, c0:c1].contiguous(),            # [NE, H, I] -> [NE, H, Is]
                    s2=s2[:, :, b0:b1].contiguous())            # [NE, H/128, I/128]
    if wfmt in (WFMT_MXFP4, WFMT_MXFP4_A4, WFMT_NVFP4):
        per = 16 if wfmt == WFMT_NVFP4 else 32                  # elements per scale code along K
        out = dict(w13=gate_up(w13, c0, c1, I),                 # [NE, 2I, H/2] packed nibbles
                   s13=gate_up(s13, c0, c1, I),                 # [NE, 2I, H/per]
                   w2=w2[:, :, c0 // 2:c1 // 2].contiguous(),   # [NE, H, I/2]
                   s2=s2[:, :, c0 // per:c1 // per].contiguous())  # [NE, H, I/per]
        if wfmt == WFMT_NVFP4:
            out.update(g13=g13, g2=g2)
        return out
    if wfmt == WFMT_MXFP8:
        return dict(w13=gate_up(w13, c0, c1, I),                # [NE, 2I, H] E4M3 bytes
                    s13=gate_up(s13, c0, c1, I),                # [NE, 2I, H/32]
                    w2=w2[:, :, c0:c1].contiguous(),            # [NE, H, I]
                    s2=s2[:, :, c0 // 32:c1 // 32].contiguous())  # [NE, H, I/32]
    raise ValueError(f"unknown weight format {wfmt}")


def allreduce_partial(partial, group=None):
    """Sum the ranks' fp32 partial results in place (torch.distributed, SUM);
    the identity without an initialised process group or with one rank."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


class TPMoeLayer:
    """One rank's share of a tensor-parallel MoE layer on its own GPU.

    ``forward`` runs the rank's I slice through the library
    (moe_forward_partial), all-reduces the fp32 partial over the process
    group, and rounds it to bf16 (moe_finalize_bf16).  Weights are given
    already sharded (shard_weights) and, for MXFP4 / NVFP4 / MXFP8, packed."""

    def __init__(self, H, I, E, k, wfmt, world: int, max_T=4096, n_shared=0, group=None):
        if I % world or (I // world) % 128:
            raise ValueError(f"I/G = {I}/{world} must be a multiple of 128")
        self.H, self.I, self.world, self.group = H, I, world, group
        self.layer = moe.MoeLayer(H, I // world, E, k, wfmt, max_T=max_T, n_shared=n_shared)

    def forward(self, x, topk_ids, topk_w, shard: dict, out=None, stream=None):
        acc = self.layer.forward_partial(x, topk_ids, topk_w, shard["w13"], shard["s13"], shard["w2"],
                                         shard["s2"], stream=stream, g13=shard.get("g13"), g2=shard.get("g2"))
        allreduce_partial(acc, self.group)
        return moe.finalize_bf16(acc, out=out, stream=stream)

    def close(self):
        self.layer.close()


def pack_shard(shard: dict, wfmt: int, stream=None) -> dict:
    """A rank's slice with its MXFP4 / NVFP4 / MXFP8 scales converted to the
    layout the library reads (FP8 scales are used as they are)."""
    out = dict(shard)
    if wfmt in (WFMT_MXFP4, WFMT_MXFP4_A4, WFMT_MXFP8):
        out["s13"], out["s2"] = moe.pack_mxfp4_scales(shard["s13"], stream), moe.pack_mxfp4_scales(shard["s2"], stream)
    elif wfmt == WFMT_NVFP4:
        out["s13"], out["s2"] = moe.pack_nvfp4_scales(shard["s13"], stream), moe.pack_nvfp4_scales(shard["s2"], stream)
    return out


__all__ = ["shard_weights", "allreduce_partial", "pack_shard", "TPMoeLayer"]
