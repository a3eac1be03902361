"""The library allocates nothing and never synchronises the host, so a whole
relu^2 MLP step (forward + backward, eleven kernels) can be captured once into a
CUDA graph and replayed; replays must reproduce eager results bit for bit."""
import pytest
import torch

from fp8_gemms_b200 import synthetic

pytestmark = pytest.mark.gpu


def test_mlp_step_in_a_cuda_graph():
    from fp8_gemms_b200 import _lib, api
    w = synthetic.MlpWorkload("graph", 512, 256, 1024, True)
    t = {k: v.cuda() for k, v in w.tensors().items()}
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    Y = torch.empty(w.M, w.d, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty_like(Y)
    dWu = torch.empty(w.f, w.d, dtype=torch.bfloat16, device="cuda")
    dWd = torch.empty(w.d, w.f, dtype=torch.bfloat16, device="cuda")

    def step():
        mlp.forward(t["X"], t["W_up"], t["W_down"], Y=Y)
        mlp.backward(t["dY"], dX=dX, dW_up=dWu, dW_down=dWd)

    step()                      # eager (also completes one-time set-up before capture)
    torch.cuda.synchronize()
    eager = [x.clone() for x in (Y, dX, dWu, dWd)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    for x in (Y, dX, dWu, dWd):
        x.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    for a, b in zip(eager, (Y, dX, dWu, dWd)):
        assert torch.equal(a, b)
    # a new input is picked up by a replay (the graph reads the same buffers)
    t["X"].mul_(2.0)
    g.replay()
    mlp2 = api.Relu2Mlp(w.M, w.d, w.f)
    Y2 = mlp2.forward(t["X"], t["W_up"], t["W_down"])
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
