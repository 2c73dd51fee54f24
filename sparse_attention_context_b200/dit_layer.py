"""A DiT self-attention layer around the ISA forward, for end-to-end timing.

x [N, C] (the source-video tokens followed by the context tokens of one
sample, C = H * d channels) -> QKV projection -> per-head attention -> output
projection.  The projections are plain library GEMMs (torch.matmul, cuBLAS)
on random weights; the attention is the ISA forward of this library (its C
ABI) or, for comparison, the in-house dense kernel.  The layer has no
normalisation, bias or positional encoding: it is the attention module whose
latency ISA reduces, not a trained model.
"""
from __future__ import annotations

import torch

from . import api


def random_weights(C: int, device="cuda", seed: int = 0):
    """Random projection weights (std 1/sqrt(C)), bf16: w_qkv [3C, C], w_o [C, C]."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    w_qkv = (torch.randn(3 * C, C, generator=g) / C ** 0.5).to(device=device, dtype=torch.bfloat16)
    w_o = (torch.randn(C, C, generator=g) / C ** 0.5).to(device=device, dtype=torch.bfloat16)
    return w_qkv, w_o


def split_heads(qkv: torch.Tensor, H: int):
    """[N, 3C] -> three contiguous [1, H, N, d] tensors (q, k, v)."""
    N, C3 = qkv.shape
    d = C3 // (3 * H)
    t = qkv.view(N, 3, H, d).permute(1, 2, 0, 3)  # [3, H, N, d]
    return tuple(t[j].unsqueeze(0).contiguous() for j in range(3))


def merge_heads(o: torch.Tensor) -> torch.Tensor:
    """[1, H, N, d] -> [N, H*d]."""
    _, H, N, d = o.shape
    return o[0].permute(1, 0, 2).reshape(N, H * d)


def attention_layer(x: torch.Tensor, w_qkv: torch.Tensor, w_o: torch.Tensor, H: int, N_src: int, block: int,
                    keep: float, rho: float, attention: str = "isa", ws=None, dense_ws=None) -> torch.Tensor:
    """y = merge(attn(split(x w_qkv^T))) w_o^T with attn = the ISA forward
    (attention="isa") or the in-house dense kernel (attention="dense")."""
    q, k, v = split_heads(x @ w_qkv.t(), H)
    if attention == "isa":
        o = api.isa_forward(q, k, v, N_src, block, keep, rho, ws=ws)
    elif attention == "dense":
        o = api.isa_dense_attn_fwd(q, k, v, ws=dense_ws)
    else:
        raise ValueError(attention)
    return merge_heads(o) @ w_o.t()
