"""The ISA forward captured in a CUDA graph (torch.cuda.graph around the C
ABI calls on the capturing stream) replays to the same bits as the direct
calls, and keeps working when the inputs change in place between replays
(the graph holds pointers, not values)."""
import pytest
import torch

from sparse_attention_context_b200 import api
from workloads import CONFIGS

from _parity import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "many_tiles"])
def test_forward_replays_from_a_cuda_graph(cuda_ok, name):
    cfg = CONFIGS["tiny"] if name == "tiny" else CONFIGS["tiny"].replace(H=2, d=128, N_src=3000, N_ctx=2900,
                                                                         block=128, keep=0.35, rho=0.25)
    _, (q, k, v) = inputs(cfg)
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    out = torch.empty_like(q)
    ref = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws).clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream (sets kernel attributes before capture)
        api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert api.isa_read_device_status(ws) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # new inputs written in place: the replay computes on them
    q2 = torch.flip(q, dims=[2]).contiguous()
    ref2 = api.isa_forward(q2, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho).clone()
    q.copy_(q2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))
