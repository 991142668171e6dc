"""The Transformer block under sequence parallelism: linear layers on the rank's rows around
Ring Self-Attention.

"Sequence Parallelism: Making 4D Parallelism Possible" (review page, Abstract) splits the
whole block by the sequence: every device holds a chunk of the rows, its linear layers (the
query/key/value projection, the output projection and the two layers of the MLP) work on those
rows alone with the weights every device holds, and only self-attention exchanges data, around
the ring. On rank r with rows X_r [c, hidden] (B = 1: the block's rows are one sequence's):

    [Q; K; V] = X_r Wqkv^T + bqkv               written as [3H, c, d] for attention
    O_r       = RingSelfAttention(Q, K, V)       the ring (sequence_ring_self_b200.ring)
    Y_r       = O_r Wo^T + bo + X_r              O read from [H, c, d] as [c, H d]
    Z_r       = GELU(Y_r W1^T + b1) W2^T + b2 + Y_r

The linear layers run in the library's tensor-core kernel (rsa_linear); the head split of the
projection and the head merge of the attention output are part of its tensor maps, so no copy
is made between the layers. Layer normalisation is not part of the linear layers and is left
out; dropout is absent, as in the attention.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import ring as ringmod
from . import rsa


@dataclass
class BlockWeights:
    """Weights of one block, replicated on every rank: wqkv [3 H d, hidden], wo [hidden, H d],
    w1 [ffn, hidden], w2 [hidden, ffn] (bf16, out x in); biases fp32."""
    wqkv: torch.Tensor
    bqkv: torch.Tensor
    wo: torch.Tensor
    bo: torch.Tensor
    w1: torch.Tensor
    b1: torch.Tensor
    w2: torch.Tensor
    b2: torch.Tensor
    heads: int
    head_dim: int


def gpu_linear(x, w, bias=None, residual=None, gelu=False, x_kin=None, y_kin=None):
    """The block's linear layer on the GPU (rsa_linear)."""
    return rsa.linear(x, w, bias, residual, gelu, x_kin=x_kin, y_kin=y_kin)


def block_forward(x, wts: BlockWeights, causal: bool = False, ring=None, comp=None,
                  lin=gpu_linear):
    """One rank's block forward on its rows x [c, hidden]. Returns (Z [c, hidden], parts) with
    parts the intermediate tensors (qkv [3H, c, d], the attention state, Y, the MLP hidden)."""
    H, d = wts.heads, wts.head_dim
    qkv = lin(x, wts.wqkv, wts.bqkv, y_kin=d)                  # [3H, c, d]
    q, k, v = (qkv[i * H:(i + 1) * H].unsqueeze(0) for i in range(3))  # [1, H, c, d] views
    st = ringmod.attention(q, k.contiguous(), v.contiguous(), causal, ring=ring, comp=comp)
    y = lin(st.o[0], wts.wo, wts.bo, x, x_kin=d)               # [c, hidden]
    h = lin(y, wts.w1, wts.b1, gelu=True)                       # [c, ffn]
    z = lin(h, wts.w2, wts.b2, y)                               # [c, hidden]
    return z, {"qkv": qkv, "attn": st, "y": y, "h": h}
