"""The per-call hot path (quantize X, then the GEMM) captured into a CUDA
graph and replayed: the library's entry points enqueue only stream work
(memsets and kernels, with tensor maps passed by value), so a replay gives
the same bytes as the eager calls and picks up new X contents."""
import pytest
import torch

import workloads
import w4a4_gemm_nvfp4_b200 as nv

pytestmark = pytest.mark.gpu


def test_quantize_gemm_graph_replay():
    wl = workloads.WORKLOADS["pr1"]
    x = wl.x.make().cuda()
    w = wl.w.make().cuda()
    qw = nv.quantize(w, "six", "max", 448.0)
    qx = nv.quantize(x, "four_over_six", "mse", 256.0)          # eager: buffers, caches, attributes
    y = torch.empty(x.shape[0], w.shape[0], dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    nv.gemm(qx, qw, out=y, workspace=ws)
    torch.cuda.synchronize()
    y_eager = y.clone()

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            nv.quantize(x, "four_over_six", "mse", 256.0, out=qx)
            nv.gemm(qx, qw, out=y, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)

    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(ws) == nv.OK
    assert torch.equal(y, y_eager)

    # new activations through the same graph
    x2 = workloads.Operand(**{**wl.x.__dict__, "seed": 77}).make().cuda()
    x.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    y2 = nv.gemm(nv.quantize(x2, "four_over_six", "mse", 256.0), qw)
    assert torch.equal(y, y2)
