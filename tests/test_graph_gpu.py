"""mxq_linear captured in a CUDA graph replays to exactly the eager result, including after the
input buffer's contents change (the graph keeps pointers, not values)."""
import pytest
import torch

from nvfp4_block_scaled_mx_b200 import mxq, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,fmt", [(300, 512, 1024, "mxfp4"), (32, 1024, 2048, "mxfp4"), (256, 384, 512, "nvfp4"),
                                       (200, 256, 512, "mxfp8"), (200, 96, 1024, "mxfp8"), (300, 128, 512, "nvfp4"),
                                       (8, 2048, 1024, "nvfp4")])
def test_linear_graph_replay_matches_eager(M, N, K, fmt):
    A1 = synth.random_bf16((M, K), 7).cuda()
    A2 = synth.random_bf16((M, K), 8, std=3.0).cuda()
    W = synth.random_bf16((N, K), 9, std=0.02).cuda()
    g_w = g_a = None
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(W)
        g_a, _ = mxq.global_scale(torch.cat([A1, A2]))
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w)
    rule = "even" if fmt == "mxfp8" else "ceil"
    ref1 = mxq.linear(A1, Wq, Wsf, N, fmt, act_rule=rule, g_W=g_w, g_A=g_a)
    ref2 = mxq.linear(A2, Wq, Wsf, N, fmt, act_rule=rule, g_W=g_w, g_A=g_a)
    A = A1.clone()
    ws = torch.empty(mxq.mxq_linear_workspace_size(M, K, mxq.FMT[fmt]), dtype=torch.uint8, device="cuda")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        mxq.linear(A, Wq, Wsf, N, fmt, act_rule=rule, g_W=g_w, g_A=g_a, workspace=ws, out=out)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref1)
    A.copy_(A2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref2)
    assert mxq.mxq_device_status(reset=True) == 0
