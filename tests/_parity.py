"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the float64 oracle on the same seeded bf16 inputs, compare.

Tolerances (stated for the ISA forward with bf16 inputs and fp32
accumulation): index sets bit-exact except members whose oracle score lies
within 1e-5 of the oracle's k-th score; outputs max |o - o_ref| <= 2e-2 and
sum|o - o_ref| / sum|o_ref| <= 5e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_attention_context_b200 import api
from workloads import Config, bf16_bits_to_f64, from_torch_bf16, make_inputs, to_torch_bf16

TIE_WINDOW = 1e-5
MAX_ABS = 2e-2
MEAN_REL = 5e-3


def inputs(cfg: Config, seed=0, heads=None):
    """(numpy bf16 bits, torch CUDA bf16 tensors) of q, k, v."""
    bits = make_inputs(cfg, seed, heads)
    dev = [to_torch_bf16(b).cuda() for b in bits]
    return bits, dev


def check_set(gpu_idx, ref_idx, scores, k, window=TIE_WINDOW):
    """Equal size; may differ only in members whose oracle score is within
    `window` of the oracle's k-th score.  Returns True if identical."""
    gpu_idx = np.sort(np.asarray(gpu_idx))
    ref_idx = np.sort(np.asarray(ref_idx))
    assert len(gpu_idx) == len(ref_idx) == k, (len(gpu_idx), len(ref_idx), k)
    assert len(np.unique(gpu_idx)) == k
    diff = np.setxor1d(gpu_idx, ref_idx)
    if len(diff):
        kth = oracle.kth_value(np.asarray(scores), k)
        dev = np.abs(np.asarray(scores)[diff] - kth)
        assert np.all(dev <= window), f"set mismatch outside the tie window: {diff[:8]} dev {dev.max()}"
    return len(diff) == 0


def check_out(o_gpu, o_ref, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    mx = float(err.max())
    rel = float(err.sum() / max(np.abs(o_ref).sum(), 1e-30))
    assert mx <= MAX_ABS and rel <= MEAN_REL, f"{what}: max abs {mx:.3e}, mean rel {rel:.3e}"
    return mx, rel


def run_stages(cfg: Config, q, k, v, keep=None, rho=None):
    """All stages through the C ABI, one call each; returns host copies."""
    keep = cfg.keep if keep is None else keep
    rho = cfg.rho if rho is None else rho
    shape = api.make_shape(q, cfg.N_src, cfg.block, keep, rho)
    ws = api.new_workspace(shape)
    kept, sal = api.isa_preselect_ctx(q, k, v, shape, ws)
    routed, taylor, sharp = api.isa_route_queries(q, kept, shape, ws)
    out = api.isa_attn_fwd(q, k, v, kept, routed, taylor, shape, ws)
    status = api.isa_read_device_status(ws)
    return dict(shape=shape, ws=ws, kept=kept.cpu().numpy(), sal=None if sal is None else sal.cpu().numpy(),
                routed=routed.cpu().numpy(), taylor=taylor.cpu().numpy(), sharp=sharp.cpu().numpy(),
                out=bf16_bits_to_f64(from_torch_bf16(out)), out_t=out, status=status)


def run_fused(cfg: Config, q, k, v, keep=None, rho=None):
    """The isa_forward path, one call per stage: pre-selection, the fused
    sharpness + Taylor pass with routing, then full attention."""
    keep = cfg.keep if keep is None else keep
    rho = cfg.rho if rho is None else rho
    shape = api.make_shape(q, cfg.N_src, cfg.block, keep, rho)
    ws = api.new_workspace(shape)
    out = torch.empty_like(q)
    kept, sal = api.isa_preselect_ctx(q, k, v, shape, ws)
    routed, taylor, sharp = api.isa_route_taylor_fwd(q, kept, shape, ws, out)
    api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, out)
    status = api.isa_read_device_status(ws)
    return dict(shape=shape, ws=ws, kept=kept.cpu().numpy(), sal=None if sal is None else sal.cpu().numpy(),
                routed=routed.cpu().numpy(), taylor=taylor.cpu().numpy(), sharp=sharp.cpu().numpy(),
                out=bf16_bits_to_f64(from_torch_bf16(out)), out_t=out, status=status)


def compare_head(cfg: Config, bits, g, b, h, keep, rho, rows=None):
    """Check one (b, h) of a GPU run `g` against the oracle, stage by stage.
    `rows` restricts the output comparison to a sample of rows."""
    q, k, v = (bf16_bits_to_f64(x[b, h]) for x in bits)
    H = bits[0].shape[1]
    bh = b * H + h
    # the sets are decided on all rows either way; `rows` only limits the outputs
    ref = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, keep, rho, rows=rows)
    # stage 1
    if g["sal"] is not None and ref["nCB"] > 0:
        s_gpu = g["sal"].reshape(-1, ref["nCB"])[bh]
        assert np.allclose(s_gpu, ref["sal_ctx"], rtol=1e-4, atol=1e-7), "saliency"
    kept_gpu = g["kept"].reshape(-1, ref["n_keep"])[bh] if ref["n_keep"] else np.zeros(0, np.int64)
    same_kept = check_set(kept_gpu, ref["kept_ctx"], ref["sal_ctx"], ref["n_keep"])
    assert np.all(np.diff(kept_gpu) > 0), "kept not ascending"
    if not same_kept:
        ref = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, keep, rho, kept_override=kept_gpu, rows=rows)
    # stage 2
    sh_gpu = g["sharp"].reshape(-1, cfg.N)[bh]
    assert np.allclose(sh_gpu, ref["sharp"], rtol=1e-4, atol=1e-7), \
        f"sharpness max rel {np.max(np.abs(sh_gpu - ref['sharp']) / ref['sharp']):.2e}"
    nr = ref["n_route"]
    routed_gpu = g["routed"].reshape(-1, nr)[bh] if nr else np.zeros(0, np.int64)
    taylor_gpu = g["taylor"].reshape(-1, cfg.N - nr)[bh] if cfg.N - nr else np.zeros(0, np.int64)
    same_routed = check_set(routed_gpu, ref["routed"], ref["sharp"], nr)
    assert np.all(np.diff(routed_gpu) > 0) and np.all(np.diff(taylor_gpu) > 0), "buckets not ascending"
    assert sorted(np.concatenate([routed_gpu, taylor_gpu]).tolist()) == list(range(cfg.N)), "not a partition"
    if not same_routed:
        ref = oracle.isa_head(q, k, v, cfg.N_src, cfg.block, keep, rho, kept_override=kept_gpu,
                              routed_override=routed_gpu, rows=rows)
    # stages 3 + 4
    o_gpu = g["out"][b, h]
    sel = slice(None) if rows is None else rows
    return check_out(o_gpu[sel], ref["out"][sel], f"out b{b} h{h}"), same_kept, same_routed
