"""The fused forward inside a CUDA graph: the library's calls only enqueue
work on the caller's stream (no synchronisation, no allocation), so one
forward can be captured once and replayed; the replay must give the eager
result bit for bit, on each expert-GEMM form."""
import pytest
import torch

import moe_inputs

pytestmark = pytest.mark.gpu


# (path, weights, E, T, bias); path 5 (split) on Zipf-skewed groups launches
# a CTA-pair and a weight-row GEMM per projection; path 6 the token-N CTA-pair
# GEMMs; T = 2048 with E = 24 takes the router that selects in its epilogue
# (4-CTA clusters exchanging partials by bulk copies)
@pytest.mark.parametrize("path,w,E,T,bias", [(2, "bf16", 20, 300, None), (3, "bf16", 64, 300, None),
                                             (4, "bf16", 2, 2048, None), (0, "fp8", 12, 300, None),
                                             (5, "bf16", 24, 1536, "zipf"), (6, "bf16", 24, 1536, "zipf"),
                                             (0, "bf16", 24, 2048, "zipf")])
def test_forward_replays_from_a_cuda_graph(path, w, E, T, bias):
    import sparse_moe_layer_top_b200 as moe
    d, k, I, I_s = (256, 2, 256, 128) if E == 2 else (384, 3, 256, 128)
    inp = moe_inputs.make_inputs(T, d, E, k, I, I_s, act="bf16", w=w, bias=bias, seed=8, device="cuda")
    moe.set_path(path)
    try:
        layer = moe.MoELayer.from_inputs(inp, max_tokens=T)
        y_eager = layer(inp.x)
        torch.cuda.synchronize()
        x = inp.x.clone()
        y = torch.empty_like(y_eager)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            layer(x, y, stream=s)  # warm-up on the capture stream (device set-up, tensor maps)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            layer(x, y, stream=s)
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_eager)
        # a new input in the same buffer flows through the replay
        x.copy_(inp.x.flip(0))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, layer(inp.x.flip(0).contiguous()))
        status, detail = moe.device_status()
        assert status == 0, hex(detail)
    finally:
        moe.set_path(0)
