"""The host pipeline (copies of step i+1 and i-1 overlapped with step i) gives exactly
the results of plain in-line steps on the same host inputs."""
import numpy as np
import pytest

from poetx_inputs import LayerShape, layer_inputs

pytestmark = pytest.mark.gpu


def test_host_pipeline_matches_inline_steps():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    from orthogonal_reparameterized_cnp_b200.host_pipeline import HostPipeline

    s = LayerShape("pipe-512x384-b128", T=256, n=512, m=384, b=128, k=4, dtype="bf16",
                   config_id=9, std_theta=0.01)
    inp = layer_inputs(s)
    dev = torch.device("cuda")
    to = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)  # noqa: E731
    pP, _ = P.make_perm(inp.seed_P, s.n)
    pR, _ = P.make_perm(inp.seed_R, s.m)
    layer = P.PoetxLinear(to(inp.W0, torch.bfloat16), to(inp.theta_P, torch.float32),
                          to(inp.theta_R, torch.float32), pP, pR, s.b, s.k, s.T)
    steps = 5
    rng = np.random.default_rng(3)
    hx = [torch.from_numpy(rng.standard_normal((s.T, s.n)).astype(np.float32)).to(torch.bfloat16)
          .pin_memory() for _ in range(steps)]
    hdy = [torch.from_numpy(rng.standard_normal((s.T, s.m)).astype(np.float32))
           .to(torch.bfloat16).pin_memory() for _ in range(steps)]
    hth = [(layer.theta.cpu() * (1.0 + 0.1 * i)).pin_memory() for i in range(steps)]
    # in-line reference steps
    want = []
    y = torch.empty((s.T, s.m), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((s.T, s.n), dtype=torch.bfloat16, device=dev)
    for i in range(steps):
        layer.theta.copy_(hth[i].to(dev))
        layer.step(hx[i].to(dev), hdy[i].to(dev), y, dx)
        torch.cuda.synchronize()
        want.append((y.cpu().clone(), dx.cpu().clone(), layer.dtheta.cpu().clone()))
    # pipelined: every step to its own host outputs
    outs = [(torch.empty((s.T, s.m), dtype=torch.bfloat16).pin_memory(),
             torch.empty((s.T, s.n), dtype=torch.bfloat16).pin_memory(),
             torch.empty(tuple(layer.dtheta.shape), dtype=torch.float32).pin_memory())
            for _ in range(steps)]
    pipe = HostPipeline(layer, nbuf=2)
    for i in range(steps):
        pipe.submit(i, hx[i], hdy[i], hth[i], *outs[i])
    pipe.synchronize()
    assert P.device_status() == P.POETX_OK
    for i in range(steps):
        for got, ref in zip(outs[i], want[i]):
            assert torch.equal(got, ref), f"step {i}"
    # only the step's result (dtheta) to the host: y and dx stay on the device
    hdth = [torch.empty(tuple(layer.dtheta.shape), dtype=torch.float32).pin_memory()
            for _ in range(steps)]
    pipe = HostPipeline(layer, nbuf=2)
    for i in range(steps):
        pipe.submit(i, hx[i], hdy[i], hth[i], None, None, hdth[i])
    pipe.synchronize()
    assert P.device_status() == P.POETX_OK
    for i in range(steps):
        assert torch.equal(hdth[i], want[i][2]), f"step {i}"
