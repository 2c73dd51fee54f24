"""First-order Taylor variant of stage 4 on the GPU (through the C ABI)
against the float64 oracle: the correction matrices C_b of the kept blocks,
the index sets, and the output rows (first-order Taylor rows and full
attention rows)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_context_b200 import api
from workloads import CONFIGS, bf16_bits_to_f64, from_torch_bf16

from _parity import check_out, check_set, inputs

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": CONFIGS["tiny"],
    "small": CONFIGS["small"],
    "ragged128": CONFIGS["tiny"].replace(H=2, d=128, N_src=300, N_ctx=77, block=64, keep=0.6, rho=0.3),
    "ragged64": CONFIGS["tiny"].replace(H=3, d=64, N_src=1000, N_ctx=1500, block=128, keep=0.4, rho=0.1,
                                        frame_hw=250),
    "all_taylor": CONFIGS["tiny"].replace(rho=0.0),
    "all_full": CONFIGS["tiny"].replace(rho=1.0),
    "no_ctx_kept": CONFIGS["tiny"].replace(keep=0.0),
    "many_tiles": CONFIGS["tiny"].replace(H=1, d=128, N_src=3000, N_ctx=2900, block=128, keep=0.35, rho=0.25),
    "two_key_tiles": CONFIGS["tiny"].replace(H=1, d=64, N_src=9000, N_ctx=9000, block=64, keep=0.5, rho=0.2),
    "batch2": CONFIGS["tiny"].replace(B=2, H=3, d=128, N_src=700, N_ctx=450, block=128, keep=0.5, rho=0.2),
}


def run_t1(cfg, q, k, v, fused=True):
    """The isa_forward_taylor1 sequence stage by stage (fused: the sharpness
    pass of isa_route_taylor_fwd, as the one-call entry point runs it; else
    isa_route_queries)."""
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    cws = api.taylor1_workspace(shape)
    out = torch.empty_like(q)
    kept, _ = api.isa_preselect_ctx(q, k, v, shape, ws)
    if fused:
        routed, taylor, sharp = api.isa_route_taylor_fwd(q, kept, shape, ws, out)
    else:
        routed, taylor, sharp = api.isa_route_queries(q, kept, shape, ws)
    api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, out)
    api.isa_taylor1_attn_fwd(q, k, v, kept, taylor, shape, ws, cws, out)
    status = api.isa_read_device_status(ws)
    nK = -(-cfg.N_src // cfg.block) + api.isa_n_keep(shape)
    C = cws[:cfg.B * cfg.H * nK * cfg.d * cfg.d * 2].view(torch.bfloat16).double()
    return dict(kept=kept.cpu().numpy(), routed=routed.cpu().numpy(), sharp=sharp.cpu().numpy(),
                C=C.view(cfg.B * cfg.H, nK, cfg.d, cfg.d).cpu().numpy(), out_t=out,
                out=bf16_bits_to_f64(from_torch_bf16(out)), status=status)


def compare_head_t1(cfg, bits, g, b, h, rows=None):
    q, k, v = (bf16_bits_to_f64(x[b, h]) for x in bits)
    kw = dict(taylor_order=1, rows=rows)
    ref = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, **kw)
    nk, nr = ref["n_keep"], ref["n_route"]
    kept = g["kept"][b, h] if nk else np.zeros(0, np.int64)
    if not check_set(kept, ref["kept_ctx"], ref["sal_ctx"], nk):
        ref = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, kept_override=kept, **kw)
    routed = g["routed"][b, h] if nr else np.zeros(0, np.int64)
    if not check_set(routed, ref["routed"], ref["sharp"], nr):
        ref = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, kept_override=kept,
                              routed_override=routed, **kw)
    if "C" in ref:
        Cg, Cr = g["C"][b * cfg.H + h], ref["C"]
        # bf16 storage of each entry: relative 2^-9, plus fp32 accumulation
        assert np.allclose(Cg, Cr, rtol=5e-3, atol=1e-3 * np.abs(Cr).max()), \
            f"C max err {np.abs(Cg - Cr).max():.3e} of max {np.abs(Cr).max():.2f}"
    sel = slice(None) if rows is None else rows
    return check_out(g["out"][b, h][sel], ref["out"][sel], f"taylor1 out b{b} h{h}")


@pytest.mark.parametrize("name", list(CASES))
def test_taylor1_matches_oracle(cuda_ok, name):
    cfg = CASES[name]
    bits, (q, k, v) = inputs(cfg)
    g = run_t1(cfg, q, k, v)
    assert g["status"] == 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            compare_head_t1(cfg, bits, g, b, h)
    # the one-call entry point runs the same kernels: identical bits
    out = api.isa_forward_taylor1(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), g["out_t"].view(torch.int16))


@pytest.mark.parametrize("name", ["tiny", "ragged128", "many_tiles"])
def test_taylor1_after_stage_by_stage_routing(cuda_ok, name):
    """isa_taylor1_attn_fwd after isa_route_queries (the stage-by-stage
    sharpness kernel) against the oracle."""
    cfg = CASES[name]
    bits, (q, k, v) = inputs(cfg)
    g = run_t1(cfg, q, k, v, fused=False)
    assert g["status"] == 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            compare_head_t1(cfg, bits, g, b, h)


def test_taylor1_480p_sampled(cuda_ok):
    """All 24 heads of the 480p latent workload in one launch; C_b of every
    kept block and sampled output rows checked on two heads."""
    cfg = CONFIGS["480p"]
    bits, (q, k, v) = inputs(cfg)
    g = run_t1(cfg, q, k, v)
    assert g["status"] == 0
    rng = np.random.default_rng(13)
    for h in (0, cfg.H - 1):
        rows = np.unique(np.concatenate([rng.choice(cfg.N, 160, replace=False),
                                         [0, cfg.N_src - 1, cfg.N_src, cfg.N - 1]]))
        compare_head_t1(cfg, bits, g, 0, h, rows=rows)


def test_taylor1_injected_timeout_is_reported(cuda_ok):
    cfg = CONFIGS["tiny"]
    _, (q, k, v) = inputs(cfg)
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    good = api.isa_forward_taylor1(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws).clone()
    assert api.isa_read_device_status(ws) == 0
    ws[4:8].view(torch.int32).fill_(1)
    api.isa_forward_taylor1(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws)
    assert api.isa_read_device_status(ws) == 5
    ws[4:8].view(torch.int32).fill_(0)
    again = api.isa_forward_taylor1(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws)
    assert api.isa_read_device_status(ws) == 0
    assert torch.equal(again.view(torch.int16), good.view(torch.int16))


def test_taylor1_720p_two_heads(cuda_ok):
    """Two of the 40 heads of the 720p latent workload (710 kept blocks: six
    key tiles per item); C_b of every kept block and sampled output rows."""
    cfg = CONFIGS["720p"]
    bits, (q, k, v) = inputs(cfg, heads=[0, 39])
    sub = cfg.replace(H=2)
    g = run_t1(sub, q, k, v)
    assert g["status"] == 0
    rng = np.random.default_rng(17)
    for h in range(2):
        rows = np.unique(np.concatenate([rng.choice(cfg.N, 96, replace=False),
                                         [0, cfg.N_src - 1, cfg.N_src, cfg.N - 1]]))
        compare_head_t1(sub, bits, g, 0, h, rows=rows)
