"""ISA forward on the GPU (through the C ABI) against the float64 oracle,
stage by stage: saliency and kept context blocks, sharpness and routed /
Taylor query sets, and the output rows of both attention paths."""
import numpy as np
import pytest
import torch

from sparse_attention_context_b200 import api
from workloads import CONFIGS, from_torch_bf16

from _parity import check_out, check_set, compare_head, inputs, run_fused, run_stages

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": CONFIGS["tiny"],
    "small": CONFIGS["small"],
    # ragged segments, d=128 with 64-token blocks, every partial block in play
    "ragged128": CONFIGS["tiny"].replace(H=2, d=128, N_src=300, N_ctx=77, block=64, keep=0.6, rho=0.3),
    "ragged64": CONFIGS["tiny"].replace(H=3, d=64, N_src=1000, N_ctx=1500, block=128, keep=0.4, rho=0.1,
                                        frame_hw=250),
    "no_ctx_kept": CONFIGS["tiny"].replace(keep=0.0),
    "all_taylor": CONFIGS["tiny"].replace(rho=0.0),
    "all_full": CONFIGS["tiny"].replace(rho=1.0),
    "keep_all": CONFIGS["tiny"].replace(keep=1.0, rho=0.5),
    "no_context": CONFIGS["tiny"].replace(N_ctx=0, N_src=300),
    "ctx_lt_block": CONFIGS["tiny"].replace(N_src=200, N_ctx=50, keep=1.0),
    "src_lt_block": CONFIGS["tiny"].replace(N_src=30, N_ctx=400, block=128, keep=0.5),
    "many_tiles": CONFIGS["tiny"].replace(H=1, d=128, N_src=3000, N_ctx=2900, block=128, keep=0.35, rho=0.25),
    "batch2": CONFIGS["tiny"].replace(B=2, H=3, d=128, N_src=700, N_ctx=450, block=128, keep=0.5, rho=0.2),
    # block saliency over several 128-block tiles at d=64 (282 blocks: 3 row
    # and column tiles, pad columns in the last)
    "sal_tiles64": CONFIGS["tiny"].replace(H=2, d=64, N_src=9000, N_ctx=9000, block=64, keep=0.4, rho=0.1),
    # the source segment ends exactly on a 128-block tile (nSB = 128): the
    # context columns start a tile
    "sal_edge128": CONFIGS["tiny"].replace(H=1, d=128, N_src=16384, N_ctx=10000, block=128, keep=0.3, rho=0.05),
}


@pytest.mark.parametrize("name", list(CASES))
def test_isa_stages_match_oracle(cuda_ok, name):
    """Stage-by-stage ABI (isa_route_queries, isa_attn_fwd) and the fused
    path of isa_forward (isa_route_taylor_fwd + isa_full_attn_fwd), each
    against the oracle."""
    cfg = CASES[name]
    bits, (q, k, v) = inputs(cfg)
    g = run_stages(cfg, q, k, v)
    f = run_fused(cfg, q, k, v)
    assert g["status"] == 0 and f["status"] == 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            compare_head(cfg, bits, g, b, h, cfg.keep, cfg.rho)
            compare_head(cfg, bits, f, b, h, cfg.keep, cfg.rho)
    # the one-call entry point runs the fused path's kernels: identical bits
    out = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), f["out_t"].view(torch.int16))


def test_keep1_rho1_equals_dense_kernel_path(cuda_ok):
    """keep = rho = 1 reduces ISA to dense attention (up to rounding)."""
    cfg = CONFIGS["tiny"].replace(keep=1.0, rho=1.0, N_src=300, N_ctx=212)
    bits, (q, k, v) = inputs(cfg)
    out = api.isa_forward(q, k, v, cfg.N_src, cfg.block, 1.0, 1.0)
    dense = api.isa_dense_attn_fwd(q, k, v)
    torch.cuda.synchronize()
    check_out(out.double().cpu().numpy(), dense.double().cpu().numpy(), "isa vs dense")


@pytest.mark.parametrize("name,heads", [("480p", None), ("720p", [0, 5, 11, 16, 22, 27, 33, 39])])
def test_isa_full_size_sampled(cuda_ok, name, heads):
    """Full-size DiT latents through the fused path that isa_forward and the
    bench run.  480p runs all 24 heads in the launch configuration the bench
    times and checks every head; 720p runs 8 of its 40 heads (heads are
    independent units).  Per head the saliency, kept set, sharpness and
    routed / Taylor sets are checked whole against the oracle, the outputs
    on sampled rows of both paths plus the segment edges."""
    cfg = CONFIGS[name]
    bits, (q, k, v) = inputs(cfg, heads=heads)
    H = q.shape[1]
    g = run_fused(cfg.replace(H=H), q, k, v)
    assert g["status"] == 0
    rng = np.random.default_rng(7)
    per_head = 48 if H > 8 else 96
    for h in range(H):
        nr = g["routed"].shape[-1]
        routed = g["routed"][0, h]
        taylor = g["taylor"][0, h]
        rows = np.unique(np.concatenate([
            rng.choice(routed, min(per_head, nr), replace=False), rng.choice(taylor, per_head, replace=False),
            [0, cfg.N_src - 1, cfg.N_src, cfg.N - 1]]))
        compare_head(cfg.replace(H=H), bits, g, 0, h, cfg.keep, cfg.rho, rows=rows)


@pytest.mark.parametrize("groups", [1, 2, 5, None])
def test_host_buffer_path(cuda_ok, groups):
    """isa_forward_host (the end-to-end path: head slices pipelined over
    copy-in, compute and copy-out streams through a staging ring) gives the
    device path's output: index sets are per head, so only the key-split
    merge of the full-attention tail (which depends on how many heads share
    a launch) may round differently.  Two calls in a row reuse the staging
    buffer."""
    cfg = CONFIGS["small"]
    bits, (q, k, v) = inputs(cfg)
    ref = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    shape = api.make_shape(hq, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    staging = torch.zeros(api.host_staging_size(shape, groups), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        got = api.isa_forward(hq, hk, hv, cfg.N_src, cfg.block, cfg.keep, cfg.rho, groups=groups, staging=staging)
        assert not got.is_cuda and got.shape == q.shape
        assert api.isa_read_device_status(staging) == 0
        check_out(got.double().numpy(), ref.double().cpu().numpy(), f"host path, groups={groups}")
        if groups == 1:
            assert torch.equal(got.view(torch.int16), ref.cpu().view(torch.int16))  # same launches: same bits


def test_host_buffer_path_pageable_and_batch(cuda_ok):
    """Pageable host memory (synchronous copies) and B > 1 (slices cut
    across the batch dimension): each head's output as on the device path."""
    cfg = CONFIGS["tiny"].replace(B=2, H=5, d=128, N_src=700, N_ctx=450, block=128, keep=0.5, rho=0.2)
    bits, (q, k, v) = inputs(cfg)
    ref = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    got = api.isa_forward(q.cpu(), k.cpu(), v.cpu(), cfg.N_src, cfg.block, cfg.keep, cfg.rho, groups=3)
    check_out(got.double().numpy(), ref.double().cpu().numpy(), "pageable host path")
    for b in range(cfg.B):
        for h in range(cfg.H):
            compare_head(cfg, bits, dict(out=got.double().numpy(), **_sets(q, k, v, cfg)), b, h, cfg.keep, cfg.rho)


def _sets(q, k, v, cfg):
    """Index sets and statistics of the device path (per head they are what
    the host path computes too)."""
    g = run_fused(cfg, q, k, v)
    return {key: g[key] for key in ("kept", "sal", "sharp", "routed", "taylor")}


def test_other_kept_set_is_reported(cuda_ok):
    """The mean of v over a context block is pooled only when the
    pre-selection keeps that block: a later stage given another (valid)
    kept set reports ISA_ERR_INVALID_ARG in the device status word instead
    of computing on means that were never pooled."""
    cfg = CASES["many_tiles"]
    _, (q, k, v) = inputs(cfg)
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    kept, _ = api.isa_preselect_ctx(q, k, v, shape, ws)
    torch.cuda.synchronize()
    assert api.isa_read_device_status(ws) == 0
    api.isa_route_queries(q, kept, shape, ws)  # the same set: fine
    torch.cuda.synchronize()
    assert api.isa_read_device_status(ws) == 0
    nCB = -(-cfg.N_ctx // cfg.block)
    chosen = kept[0, 0].cpu().tolist()
    unused = next(c for c in range(nCB) if c not in chosen)
    other = kept.clone()
    other[0, 0] = torch.tensor(sorted(chosen[1:] + [unused]), dtype=kept.dtype, device=kept.device)
    api.isa_route_queries(q, other, shape, ws)
    torch.cuda.synchronize()
    assert api.isa_read_device_status(ws) == 1  # ISA_ERR_INVALID_ARG

