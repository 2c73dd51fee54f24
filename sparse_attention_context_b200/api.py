"""Python binding of libisa.so: argument marshalling only.

Every function takes torch tensors for device memory and the current torch
CUDA stream, and calls the C entry point of the same name (include/isa.h);
no step of the ISA path runs in Python or torch.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import IsaShape, check, lib


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _check_qkv(*ts):
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
            raise ValueError("q, k, v, out must be contiguous CUDA bf16 tensors [B, H, N, d]")


def make_shape(q: torch.Tensor, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0) -> IsaShape:
    B, H, N, d = q.shape
    return IsaShape(B, H, int(N_src), int(N - N_src), d, int(block), float(keep), float(rho), float(scale))


def isa_n_keep(shape: IsaShape) -> int:
    return lib().isa_n_keep(ctypes.byref(shape))


def isa_n_route(shape: IsaShape) -> int:
    return lib().isa_n_route(ctypes.byref(shape))


def isa_n_route_blocks(shape: IsaShape) -> int:
    return lib().isa_n_route_blocks(ctypes.byref(shape))


def isa_workspace_size(shape: IsaShape) -> int:
    return lib().isa_workspace_size(ctypes.byref(shape))


def new_workspace(shape: IsaShape, device="cuda") -> torch.Tensor:
    """Zeroed workspace (control block included) for every call on `shape`."""
    n = isa_workspace_size(shape)
    if n == 0:
        raise ValueError("invalid or unsupported shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def isa_preselect_ctx(q, k, v, shape: IsaShape, ws, kept=None, saliency=None, want_saliency=True, stream=None):
    """Stage 1.  Returns (kept_ctx_idx [B,H,n_keep] int32, saliency [B,H,nCB] or None)."""
    _check_qkv(q, k, v)
    B, H = shape.B, shape.H
    nk = isa_n_keep(shape)
    nCB = -(-shape.N_ctx // shape.block)
    if kept is None:
        kept = torch.empty((B, H, nk), dtype=torch.int32, device=q.device)
    if saliency is None and want_saliency:
        saliency = torch.empty((B, H, nCB), dtype=torch.float32, device=q.device)
    rc = lib().isa_preselect_ctx(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 _ptr(kept) if nk > 0 else None, _ptr(saliency), ws.data_ptr(), ws.numel(),
                                 _stream(stream))
    check("isa_preselect_ctx", rc)
    return kept, saliency


def isa_route_queries(q, kept, shape: IsaShape, ws, routed=None, taylor=None, sharpness=None, want_sharpness=True,
                      stream=None):
    """Stage 2.  Returns (routed_idx [B,H,n_route], taylor_idx [B,H,N-n_route], sharpness [B,H,N] or None)."""
    _check_qkv(q)
    B, H, N = shape.B, shape.H, shape.N_src + shape.N_ctx
    nr = isa_n_route(shape)
    if routed is None:
        routed = torch.empty((B, H, nr), dtype=torch.int32, device=q.device)
    if taylor is None:
        taylor = torch.empty((B, H, N - nr), dtype=torch.int32, device=q.device)
    if sharpness is None and want_sharpness:
        sharpness = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = lib().isa_route_queries(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                 _ptr(routed) if nr > 0 else None, _ptr(taylor) if N - nr > 0 else None,
                                 _ptr(sharpness), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_route_queries", rc)
    return routed, taylor, sharpness


def isa_route_taylor_fwd(q, kept, shape: IsaShape, ws, out, routed=None, taylor=None, sharpness=None,
                         want_sharpness=True, stream=None):
    """Stages 2 + 4 fused: sharpness, routing, and the Taylor output of every
    row of `out`.  Returns (routed_idx, taylor_idx, sharpness or None)."""
    _check_qkv(q, out)
    B, H, N = shape.B, shape.H, shape.N_src + shape.N_ctx
    nr = isa_n_route(shape)
    if routed is None:
        routed = torch.empty((B, H, nr), dtype=torch.int32, device=q.device)
    if taylor is None:
        taylor = torch.empty((B, H, N - nr), dtype=torch.int32, device=q.device)
    if sharpness is None and want_sharpness:
        sharpness = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = lib().isa_route_taylor_fwd(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                    _ptr(routed) if nr > 0 else None, _ptr(taylor) if N - nr > 0 else None,
                                    _ptr(sharpness), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_route_taylor_fwd", rc)
    return routed, taylor, sharpness


def isa_attn_fwd(q, k, v, kept, routed, taylor, shape: IsaShape, ws, out=None, stream=None):
    """Stages 3 and 4.  Returns out [B,H,N,d] bf16."""
    if out is None:
        out = torch.empty_like(q)
    _check_qkv(q, k, v, out)
    rc = lib().isa_attn_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                            _ptr(kept) if kept.numel() else None, _ptr(routed) if routed.numel() else None,
                            _ptr(taylor) if taylor.numel() else None, out.data_ptr(), ws.data_ptr(), ws.numel(),
                            _stream(stream))
    check("isa_attn_fwd", rc)
    return out


def isa_full_attn_fwd(q, k, v, kept, routed, shape: IsaShape, ws, out, stream=None):
    """Stage 3 only: full attention for the routed rows of `out`."""
    _check_qkv(q, k, v, out)
    rc = lib().isa_full_attn_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 _ptr(kept) if kept.numel() else None, _ptr(routed) if routed.numel() else None,
                                 out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_full_attn_fwd", rc)
    return out


def isa_taylor_attn_fwd(q, kept, taylor, shape: IsaShape, ws, out, stream=None):
    """Stage 4 only: 0-th order Taylor attention for the taylor rows of `out`."""
    _check_qkv(q, out)
    rc = lib().isa_taylor_attn_fwd(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                   _ptr(taylor) if taylor.numel() else None, out.data_ptr(), ws.data_ptr(),
                                   ws.numel(), _stream(stream))
    check("isa_taylor_attn_fwd", rc)
    return out


def isa_full_attn_rows_fwd(q, k, v, kept, rows, shape: IsaShape, ws, out, stream=None):
    """Stage 3 for an explicit row list rows [B,H,n_rows] (-1 entries are padding)."""
    _check_qkv(q, k, v, out)
    n_rows = rows.shape[-1]
    rc = lib().isa_full_attn_rows_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      _ptr(kept) if kept.numel() else None, _ptr(rows) if rows.numel() else None,
                                      int(n_rows), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_full_attn_rows_fwd", rc)
    return out


def isa_route_blocks_taylor_fwd(q, kept, shape: IsaShape, ws, out, want_scores=True, want_sharpness=True,
                                stream=None):
    """Stages 2 + 4 with whole query blocks routed.  Returns (routed block
    indices [B,H,n_rb], routed rows [B,H,n_rb*block] with -1 pads, block
    scores [B,H,nB] or None, sharpness [B,H,N] or None)."""
    _check_qkv(q, out)
    B, H, N = shape.B, shape.H, shape.N_src + shape.N_ctx
    nB = -(-shape.N_src // shape.block) + -(-shape.N_ctx // shape.block)
    nrb = isa_n_route_blocks(shape)
    rblk = torch.empty((B, H, nrb), dtype=torch.int32, device=q.device)
    rows = torch.empty((B, H, nrb * shape.block), dtype=torch.int32, device=q.device)
    score = torch.empty((B, H, nB), dtype=torch.float32, device=q.device) if want_scores else None
    sharp = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if want_sharpness else None
    rc = lib().isa_route_blocks_taylor_fwd(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                           _ptr(rblk) if nrb else None, _ptr(rows) if nrb else None, _ptr(score),
                                           _ptr(sharp), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_route_blocks_taylor_fwd", rc)
    return rblk, rows, score, sharp


def isa_forward_blocks(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, ws=None,
                       out=None, stream=None):
    """The ISA forward with block-granular query grouping (CUDA tensors)."""
    shape = make_shape(q, N_src, block, keep, rho, scale)
    if ws is None:
        ws = new_workspace(shape, q.device)
    o = torch.empty_like(q) if out is None else out
    _check_qkv(q, k, v, o)
    rc = lib().isa_forward_blocks(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_forward_blocks", rc)
    return o


def taylor1_workspace(shape: IsaShape, device="cuda") -> torch.Tensor:
    """Buffer for the correction matrices of the first-order Taylor variant."""
    n = lib().isa_taylor1_workspace_size(ctypes.byref(shape))
    if n == 0:
        raise ValueError("invalid or unsupported shape")
    return torch.empty(n, dtype=torch.uint8, device=device)


def isa_taylor1_attn_fwd(q, k, v, kept, taylor, shape: IsaShape, ws, cws, out, stream=None):
    """First-order Taylor output for the taylor rows of `out` (C_b land in cws)."""
    _check_qkv(q, k, v, out)
    rc = lib().isa_taylor1_attn_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    _ptr(kept) if kept.numel() else None, _ptr(taylor) if taylor.numel() else None,
                                    out.data_ptr(), ws.data_ptr(), ws.numel(), cws.data_ptr(), cws.numel(),
                                    _stream(stream))
    check("isa_taylor1_attn_fwd", rc)
    return out


def isa_forward_taylor1(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, ws=None,
                        cws=None, out=None, stream=None):
    """The ISA forward with first-order Taylor attention for the rows that are not routed."""
    shape = make_shape(q, N_src, block, keep, rho, scale)
    if ws is None:
        ws = new_workspace(shape, q.device)
    if cws is None:
        cws = taylor1_workspace(shape, q.device)
    o = torch.empty_like(q) if out is None else out
    _check_qkv(q, k, v, o)
    rc = lib().isa_forward_taylor1(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   ws.data_ptr(), ws.numel(), cws.data_ptr(), cws.numel(), _stream(stream))
    check("isa_forward_taylor1", rc)
    return o


def isa_forward(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, ws=None, out=None,
                stream=None, groups=None, staging=None, sync=True):
    """All ISA stages in one call.

    CUDA inputs: isa_forward on the current stream; returns a CUDA tensor.
    CPU inputs (the host-buffer path): isa_forward_host, which copies q, k, v
    in, runs the forward and copies the output back into a (pinned) CPU
    tensor, head slices pipelined over a copy-in stream, the current stream
    and a copy-out stream (`groups` slices; None lets the library choose).
    `staging` is the device buffer the library works in (allocated here when
    None or too small).  With sync=True (default) the call returns once the
    output is in host memory; with sync=False it returns at once and the
    output is complete when the current stream is.  Pass pinned host tensors
    for the copies to be asynchronous.
    """
    if q.is_cuda:
        shape = make_shape(q, N_src, block, keep, rho, scale)
        if ws is None:
            ws = new_workspace(shape, q.device)
        o = torch.empty_like(q) if out is None else out
        _check_qkv(q, k, v, o)
        rc = lib().isa_forward(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               ws.data_ptr(), ws.numel(), _stream(stream))
        check("isa_forward", rc)
        return o
    return isa_forward_host(q, k, v, N_src, block, keep, rho, scale, out=out, groups=groups, staging=staging,
                            stream=stream, sync=sync)


_COPY_STREAMS = {}


def _copy_streams(device):
    """One copy-in and one copy-out stream per device, made once."""
    key = torch.device(device).index
    if key not in _COPY_STREAMS:
        with torch.cuda.device(key):
            _COPY_STREAMS[key] = (torch.cuda.Stream(), torch.cuda.Stream())
    return _COPY_STREAMS[key]


def host_staging_size(shape: IsaShape, groups=None) -> int:
    return lib().isa_host_staging_size(ctypes.byref(shape), 0 if groups is None else int(groups))


def isa_forward_host(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, out=None,
                     groups=None, staging=None, stream=None, sync=True):
    """The C entry point isa_forward_host on CPU bf16 tensors [B, H, N, d].
    Returns the output as a CPU tensor (pinned unless `out` is given)."""
    for t in (q, k, v) + ((out,) if out is not None else ()):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("host path: q, k, v, out must be contiguous CPU bf16 tensors [B, H, N, d]")
    shape = make_shape(q, N_src, block, keep, rho, scale)
    G = 0 if groups is None else int(groups)
    n = lib().isa_host_staging_size(ctypes.byref(shape), G)
    if n == 0:
        raise ValueError("invalid or unsupported shape")
    comp = torch.cuda.current_stream() if stream is None else stream
    dev = comp.device
    if staging is None or staging.numel() < n:
        staging = torch.empty(n, dtype=torch.uint8, device=dev)
    dst = out if out is not None else torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    s_in, s_out = _copy_streams(dev)
    rc = lib().isa_forward_host(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), dst.data_ptr(),
                                staging.data_ptr(), staging.numel(), G, comp.cuda_stream, s_in.cuda_stream,
                                s_out.cuda_stream)
    check("isa_forward_host", rc)
    staging.record_stream(comp)  # the caching allocator keeps it until the enqueued work is done
    if sync:
        comp.synchronize()
    return dst


def isa_forward_static(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, out=None,
                       stream=None):
    """All ISA stages with the library's fixed device scratch (no workspace,
    nothing allocated by the library).  CUDA tensors only; returns out."""
    if out is None:
        out = torch.empty_like(q)
    _check_qkv(q, k, v, out)
    shape = make_shape(q, N_src, block, keep, rho, scale)
    rc = lib().isa_forward_static(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  _stream(stream))
    check("isa_forward_static", rc)
    return out


def dense_workspace(d: int = 128, device="cuda") -> torch.Tensor:
    n = lib().isa_dense_workspace_size(int(d))
    if n == 0:
        raise ValueError("unsupported head dimension")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def isa_dense_attn_fwd(q, k, v, scale: float = 0.0, out=None, ws=None, stream=None):
    """In-house dense flash attention (the baseline).  Returns out [B,H,N,d] bf16."""
    if out is None:
        out = torch.empty_like(q)
    _check_qkv(q, k, v, out)
    B, H, N, d = q.shape
    if ws is None:
        ws = dense_workspace(d, q.device)
    rc = lib().isa_dense_attn_fwd(B, H, N, d, float(scale), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                  out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_dense_attn_fwd", rc)
    return out


def isa_read_device_status(ws, stream=None) -> int:
    """Synchronise, return the device status word of `ws` and reset it."""
    return lib().isa_read_device_status(ws.data_ptr(), _stream(stream))


def isa_selftest_umma(A, B, P, V, ws, stream=None):
    """Test-only: one-tile UMMA products S = A B^T, O = P V (P in shared
    memory) and O2 = P V (P in tensor memory), all fp32."""
    d, bn = A.shape[1], B.shape[0]
    S = torch.empty((128, bn), dtype=torch.float32, device=A.device)
    O = torch.empty((128, d), dtype=torch.float32, device=A.device)
    O2 = torch.empty((128, d), dtype=torch.float32, device=A.device)
    rc = lib().isa_selftest_umma(d, bn, A.data_ptr(), B.data_ptr(), P.data_ptr(), V.data_ptr(), S.data_ptr(),
                                 O.data_ptr(), O2.data_ptr(), ws.data_ptr(), _stream(stream))
    check("isa_selftest_umma", rc)
    return S, O, O2


def isa_selftest_ex2(x, stream=None):
    """Test-only: (FMA-pipe 2^x of the softmax, MUFU ex2, exp2f) of the fp32
    CUDA tensor x, each a tensor like x."""
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    yp, ym, yr = (torch.empty_like(x) for _ in range(3))
    rc = lib().isa_selftest_ex2(x.data_ptr(), yp.data_ptr(), ym.data_ptr(), yr.data_ptr(), x.numel(), _stream(stream))
    check("isa_selftest_ex2", rc)
    return yp, ym, yr


def isa_selftest_umma_pair(A, B, P, V, ws, stream=None):
    """Test-only: one M = 256 tile on a CTA pair: S = A B^T, O = P V (fp32)."""
    S = torch.empty((256, 128), dtype=torch.float32, device=A.device)
    O = torch.empty((256, 128), dtype=torch.float32, device=A.device)
    rc = lib().isa_selftest_umma_pair(A.data_ptr(), B.data_ptr(), P.data_ptr(), V.data_ptr(), S.data_ptr(),
                                      O.data_ptr(), ws.data_ptr(), _stream(stream))
    check("isa_selftest_umma_pair", rc)
    return S, O
