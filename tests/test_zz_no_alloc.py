"""isa_forward_static: the ISA forward for callers that cannot allocate
device memory (a framework allocator that owns the free memory, a serving
loop that must not allocate after start-up).  It runs on a fixed scratch
array inside the library instead of a caller workspace.

Checked through the C ABI against isa_forward with its own workspace, twice
in a row (the second call reuses a scratch that still holds the first
call's contents), and for the size limit.  Collected last on purpose."""
import ctypes

import pytest
import torch

from sparse_attention_context_b200 import api
from sparse_attention_context_b200._lib import lib
from workloads import CONFIGS

from _parity import check_out, inputs

pytestmark = pytest.mark.gpu


def call_static(q, k, v, out, cfg):
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    stream = torch.cuda.current_stream().cuda_stream
    return lib().isa_forward_static(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    stream)


@pytest.mark.parametrize("name", ["small", "480p"])
def test_static_scratch_matches_workspace_path(cuda_ok, name):
    cfg = CONFIGS[name]
    _, (q, k, v) = inputs(cfg)
    ref = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        assert call_static(q, k, v, out, cfg) == 0
        torch.cuda.synchronize()
        check_out(out.double().cpu().numpy(), ref.double().cpu().numpy(), f"static scratch {name}")


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_ok):
    cfg = CONFIGS["720p"]  # needs far more than the fixed scratch holds
    shape = api.make_shape(torch.empty((cfg.B, cfg.H, cfg.N, cfg.d), device="meta"), cfg.N_src, cfg.block,
                           cfg.keep, cfg.rho)
    assert lib().isa_workspace_size(ctypes.byref(shape)) > (64 << 20)
    buf = torch.zeros(16, dtype=torch.uint8, device="cuda")  # never read: rejected before any launch
    p = buf.data_ptr()
    assert lib().isa_forward_static(ctypes.byref(shape), p, p, p, p, None) == 3
