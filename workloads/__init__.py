"""Seeded synthetic inputs for the ISA attention forward.

This module is shared by the oracle tests, the GPU parity tests and the bench.
It draws random numbers and casts them to bf16; it contains none of the
attention method's arithmetic (no pooling, no scores, no softmax).

Workload shapes follow the DiT-latent shapes of the ISA problem statement
(Lightning Unified Video Editing via In-Context Sparse Attention, abstract):
a sequence of source-video tokens followed by the same number of context
tokens, bidirectional attention per head.  No benchmark or dataset from the
pages is available here; these synthetic tensors stand in for the real
LIVEditor activations.

Draw recipe, per (b, h), from ``numpy.random.default_rng([seed, b, h])``
(one independent stream per head, so any subset of heads can be regenerated
on its own):

1. q, k, v ~ N(0, 1), float32, each [N, d], drawn in that order.
2. q row scale ~ lognormal(mean=0, sigma=0.5), one per row, multiplied in.
3. Planted sharp rows (if enabled): 10 % of the N rows, a uniform sample
   without replacement, multiplied by 4.
4. Per-frame key offset (if the config has frames): one N(0, 0.3^2)
   d-vector per latent frame of ``fh*fw`` tokens, added to every key row of
   that frame, separately in the source and in the context segment.
5. Context keys (rows N_src..N-1) multiplied by 0.5 (lower saliency).
6. Round to bf16 (round to nearest even).
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    d: int
    N_src: int
    N_ctx: int
    block: int
    keep: float
    rho: float
    planted: bool = True
    frame_hw: int | None = None  # tokens per latent frame (h*w); None = no offset

    @property
    def N(self) -> int:
        return self.N_src + self.N_ctx

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    # tiny: B=1, H=2, d=64, 256+256 tokens, block 64, keep .5, rho .25
    "tiny": Config("tiny", 1, 2, 64, 256, 256, 64, 0.5, 0.25, planted=True, frame_hw=None),
    # small: 4 latent frames of 32x32 per segment, block 128
    "small": Config("small", 1, 12, 64, 4096, 4096, 128, 0.3, 0.2, planted=False, frame_hw=32 * 32),
    # 480p latent: 13 frames of 30x52 per segment
    "480p": Config("480p", 1, 24, 128, 20280, 20280, 128, 0.25, 0.2, planted=True, frame_hw=30 * 52),
    # 720p latent: 21 frames of 45x80 per segment
    "720p": Config("720p", 1, 40, 128, 75600, 75600, 128, 0.2, 0.15, planted=True, frame_hw=45 * 80),
    # sweep shape (keep, rho varied by the caller)
    "sweep": Config("sweep", 1, 24, 128, 32768, 32768, 128, 0.25, 0.2, planted=True, frame_hw=None),
}

SWEEP_KEEP = (0.1, 0.25, 0.5, 1.0)
SWEEP_RHO = (0.0, 0.1, 0.2, 0.5, 1.0)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def head_inputs(cfg: Config, b: int, h: int, seed: int = 0):
    """bf16 bit patterns (uint16) of q, k, v for one (b, h); each [N, d]."""
    rng = np.random.default_rng([seed, b, h])
    N, d = cfg.N, cfg.d
    q = rng.standard_normal((N, d), dtype=np.float32)
    k = rng.standard_normal((N, d), dtype=np.float32)
    v = rng.standard_normal((N, d), dtype=np.float32)
    scale = rng.lognormal(mean=0.0, sigma=0.5, size=N).astype(np.float32)
    q *= scale[:, None]
    if cfg.planted:
        n_plant = int(round(0.1 * N))
        rows = rng.choice(N, size=n_plant, replace=False)
        q[rows] *= np.float32(4.0)
    if cfg.frame_hw:
        for seg_start, seg_len in ((0, cfg.N_src), (cfg.N_src, cfg.N_ctx)):
            n_frames = math.ceil(seg_len / cfg.frame_hw)
            offs = (0.3 * rng.standard_normal((n_frames, d))).astype(np.float32)
            for f in range(n_frames):
                a = seg_start + f * cfg.frame_hw
                e = min(seg_start + seg_len, a + cfg.frame_hw)
                k[a:e] += offs[f]
    k[cfg.N_src:] *= np.float32(0.5)
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def make_inputs(cfg: Config, seed: int = 0, heads=None, threads: int = 8):
    """All (b, h) of a config as uint16 bf16 bit arrays [B, H, N, d].

    ``heads`` optionally restricts to a list of head indices (every batch
    element); the result then has that many heads, in that order.
    """
    hs = list(range(cfg.H)) if heads is None else list(heads)
    B, N, d = cfg.B, cfg.N, cfg.d
    out = [np.empty((B, len(hs), N, d), dtype=np.uint16) for _ in range(3)]
    jobs = [(b, i, h) for b in range(B) for i, h in enumerate(hs)]

    def work(job):
        b, i, h = job
        for t, arr in zip(out, head_inputs(cfg, b, h, seed)):
            t[b, i] = arr

    if threads > 1 and len(jobs) > 1:
        with ThreadPoolExecutor(min(threads, len(jobs))) as ex:
            list(ex.map(work, jobs))
    else:
        for j in jobs:
            work(j)
    return tuple(out)


def to_torch_bf16(bits: np.ndarray):
    """View uint16 bf16 bit patterns as a torch.bfloat16 CPU tensor (no copy)."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def from_torch_bf16(t) -> np.ndarray:
    """torch.bfloat16 tensor (any device) -> uint16 bit patterns on the host."""
    import torch

    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
