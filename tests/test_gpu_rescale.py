"""Running-max rescaling in the attention engine.  Some query rows are set to
4 in every channel and a few keys to 2 or 4 in every channel, so those rows'
largest score jumps by 90-260 (base-2 units) in a later key tile: in the
first or the second half of a tile, once or twice, in the ragged last tile,
for some rows of a warp and not the others.  Such rows move the engine's
running reference past its 2^32 threshold, so O and l are rescaled by
2^(m_old - m_new) mid-sequence (by some warps of a tile and not others);
their outputs must still match the float64 oracle, in the dense engine and
in the full attention of ISA (128- and 64-key tiles)."""
import numpy as np
import pytest

import oracle
from sparse_attention_context_b200 import api
from workloads import CONFIGS, bf16_bits_to_f64, f32_to_bf16_bits, from_torch_bf16, make_inputs, to_torch_bf16

from _parity import check_out, compare_head, run_fused

pytestmark = pytest.mark.gpu

# (head, query rows, key row, key amplitude); N = 1050 tokens (700 + 350)
PLANTS = [
    (0, [3, 17, 40, 100, 129, 200, 600, 1049], 138, 2.0),  # key tile 1 (of 128), first half
    (0, [3, 17, 40, 100, 129, 200, 600, 1049], 740, 4.0),  # key tile 5, second half: a second jump
    (1, [5, 6, 7, 300, 301], 300, 2.0),                    # key tile 2, second quarter
    (1, [5, 6, 7, 300, 301], 1040, 4.0),                   # the ragged last tile (26 keys)
]


def planted_inputs(cfg):
    q, k, v = (b.copy() for b in make_inputs(cfg, 0))
    for h, rows, key, amp in PLANTS:
        q[0, h, rows, :] = f32_to_bf16_bits(np.full(cfg.d, 4.0, np.float32))
        k[0, h, key, :] = f32_to_bf16_bits(np.full(cfg.d, amp, np.float32))
    return (q, k, v), [to_torch_bf16(b).cuda() for b in (q, k, v)]


def planted_score_log2(cfg, amp):
    """Score of a planted row against a planted key, in base-2 units
    (4 * amp * d / sqrt(d) * log2 e): far past the 2^32 rescale threshold
    above the ordinary scores of the first key tile."""
    return 4.0 * amp * cfg.d ** 0.5 * np.log2(np.e)


@pytest.mark.parametrize("d", [64, 128])
def test_dense_rescale_matches_oracle(cuda_ok, d):
    cfg = CONFIGS["tiny"].replace(H=2, d=d, N_src=700, N_ctx=350)
    assert planted_score_log2(cfg, 2.0) > 90
    bits, (q, k, v) = planted_inputs(cfg)
    ws = api.dense_workspace(d)
    out = api.isa_dense_attn_fwd(q, k, v, ws=ws)
    assert api.isa_read_device_status(ws) == 0
    o = bf16_bits_to_f64(from_torch_bf16(out))
    for h in range(cfg.H):
        qh, kh, vh = (bf16_bits_to_f64(x[0, h]) for x in bits)
        ref = oracle.dense_head(qh, kh, vh)
        check_out(o[0, h], ref, f"dense d{d} h{h}")
        # the planted rows end on the strongest planted key's value row
        rows = PLANTS[2 * h][1]
        key = PLANTS[2 * h + 1][2]
        assert np.allclose(o[0, h, rows], vh[key], atol=2e-2)


@pytest.mark.parametrize("d,block", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_full_attention_rescale_matches_oracle(cuda_ok, d, block):
    """Every row routed (rho = 1), so the planted rows take the full-attention
    kernel over their source blocks (always kept) and the kept context."""
    cfg = CONFIGS["tiny"].replace(H=2, d=d, N_src=700, N_ctx=350, block=block, keep=0.5, rho=1.0)
    bits, (q, k, v) = planted_inputs(cfg)
    g = run_fused(cfg, q, k, v)
    assert g["status"] == 0
    for h in range(cfg.H):
        compare_head(cfg, bits, g, 0, h, cfg.keep, cfg.rho)
