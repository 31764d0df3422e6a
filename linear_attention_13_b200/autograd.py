"""torch.autograd entry for training: o = lightning_attention(q, k, v) with the
forward and backward passes in the library's kernels (la_prefill,
la_prefill_backward)."""
import torch

import linear_attention_13_b200 as la


class LightningAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, blk):
        o, _ = la.prefill(q, k, v, blk=blk, want_state=False)
        ctx.save_for_backward(q, k, v)
        ctx.blk = blk
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v = ctx.saved_tensors
        dq, dk, dv = la.prefill_backward(q, k, v, do.contiguous(), blk=ctx.blk)
        return dq, dk, dv, None


def lightning_attention(q, k, v, blk: int = 128):
    """Causal linear attention of contiguous [B,H,N,d] CUDA tensors, differentiable."""
    return LightningAttention.apply(q, k, v, blk)
