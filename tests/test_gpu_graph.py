"""The launch calls allocate nothing and never wait on the host, so a
quantize + forward pair can be captured into a CUDA graph and replayed: the
replays on new input data must equal eager runs bit for bit."""
import pytest

from qlutil import to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,epi", [("fp8", "bias_gelu"), ("nvfp4", "swiglu"),
                                     ("nvfp4", "split_bias_gelu"), ("w8a16", "bias")])
def test_quantize_and_forward_replay_from_a_cuda_graph(fmt, epi):
    import torch
    import precision_gemm_qlinear_b200 as ql
    M, N, K = 520, 1024, 512
    w = to_dev_bf16(draw("normal", (N, K), 31, "w", std=0.02))
    b = to_dev_bf16(draw("normal", (N,), 31, "bias", std=0.01))
    lay = ql.QLinear(fmt, epi, w, b, split_col=512 if epi == "split_bias_gelu" else 0)
    x = to_dev_bf16(draw("normal", (M, K), 31, "x"))
    codes, scales = lay.act_buffers(M)
    out = torch.empty((M, lay.Nout), dtype=torch.bfloat16, device="cuda")

    def run():
        lay.quantize(x, codes, scales)
        lay.forward_codes(codes, scales, M, out)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()  # eager warm-up on the side stream (kernel attributes set once)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for seed in (32, 33, 34):
        x.copy_(to_dev_bf16(draw("normal", (M, K), seed, "x")))
        g.replay()
        torch.cuda.synchronize()
        got = out.clone()
        run()  # eager, same inputs
        torch.cuda.synchronize()
        assert torch.equal(got, out)
    assert lay.check() == 0
