"""In-house dense flash attention (tcgen05) against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_context_b200 import api
from workloads import CONFIGS, bf16_bits_to_f64, from_torch_bf16

from _parity import check_out, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,N_src,N_ctx,H", [
    (64, 128, 0, 1), (64, 256, 256, 2), (128, 200, 133, 2), (128, 1, 0, 1), (64, 777, 300, 3), (128, 1024, 1024, 2)])
def test_dense_matches_oracle(cuda_ok, d, N_src, N_ctx, H):
    cfg = CONFIGS["tiny"].replace(H=H, d=d, N_src=N_src, N_ctx=N_ctx)
    bits, (q, k, v) = inputs(cfg)
    ws = api.dense_workspace(q.shape[-1])
    out = api.isa_dense_attn_fwd(q, k, v, ws=ws)
    assert api.isa_read_device_status(ws) == 0
    o = bf16_bits_to_f64(from_torch_bf16(out))
    for h in range(H):
        qh, kh, vh = (bf16_bits_to_f64(x[0, h]) for x in bits)
        check_out(o[0, h], oracle.dense_head(qh, kh, vh), f"dense h{h}")


def test_dense_480p_sampled_rows(cuda_ok):
    """Full-size 480p-latent dense attention (24 heads, 40560 tokens), checked
    on sampled rows of two heads, including the ragged last query tile."""
    cfg = CONFIGS["480p"]
    bits, (q, k, v) = inputs(cfg)
    out = api.isa_dense_attn_fwd(q, k, v)
    torch.cuda.synchronize()
    o = from_torch_bf16(out)
    rows = np.array([0, 1, 127, 128, 20279, 20280, 30000, 40447, 40448, 40559])
    rows = np.concatenate([rows, np.random.default_rng(1).choice(cfg.N, 118, replace=False)])
    for h in (0, cfg.H - 1):
        qh, kh, vh = (bf16_bits_to_f64(x[0, h]) for x in bits)
        check_out(bf16_bits_to_f64(o[0, h, rows]), oracle.dense_head(qh, kh, vh, rows=rows), f"dense480 h{h}")
