"""The DiT self-attention layer harness (QKV projection, ISA through the C
ABI, output projection) against a float64 composition of the same steps:
the projections recomputed in float64 from the same bf16 operands, the
attention by the oracle on the layer's own q, k, v."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_context_b200.dit_layer import attention_layer, merge_heads, random_weights, split_heads
from workloads import CONFIGS

from _parity import check_out

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("attention", ["isa", "dense"])
def test_dit_layer_matches_float64_composition(cuda_ok, attention):
    cfg = CONFIGS["tiny"]
    H, N, d = cfg.H, cfg.N, cfg.d
    C = H * d
    g = torch.Generator(device="cpu").manual_seed(3)
    x = torch.randn(N, C, generator=g).to(device="cuda", dtype=torch.bfloat16)
    w_qkv, w_o = random_weights(C, seed=5)
    y = attention_layer(x, w_qkv, w_o, H, cfg.N_src, cfg.block, cfg.keep, cfg.rho, attention=attention)
    torch.cuda.synchronize()
    # the attention input the layer used (bf16 projection, as the harness computes it)
    q, k, v = (t[0].double().cpu().numpy() for t in split_heads(x @ w_qkv.t(), H))
    o = np.empty((H, N, d))
    for h in range(H):
        if attention == "isa":
            o[h] = oracle.isa_head(q[h], k[h], v[h], cfg.N_src, cfg.block, cfg.keep, cfg.rho)["out"]
        else:
            o[h] = oracle.dense_head(q[h], k[h], v[h])
    o_flat = o.transpose(1, 0, 2).reshape(N, C)
    y_ref = o_flat @ w_o.double().cpu().numpy().T
    check_out(y.double().cpu().numpy(), y_ref, f"DiT layer ({attention})")
    # the head split and merge are inverse permutations
    qkv = x @ w_qkv.t()
    qq, kk, vv = split_heads(qkv, H)
    assert torch.equal(merge_heads(qq), qkv[:, :C]) and torch.equal(merge_heads(vv), qkv[:, 2 * C:])
