"""Shared helpers of the GPU parity tests: run the library on seeded inputs and return
float64 numpy results next to the oracle's."""
from __future__ import annotations

import numpy as np

from poetx_inputs import LayerInputs, LayerShape, layer_inputs


def norm_max_err(gpu, ref) -> float:
    """max|gpu - ref| / max|ref| (per output tensor)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max() if ref.size else 1.0
    return float(np.abs(gpu - ref).max() / (den if den > 0 else 1.0)) if ref.size else 0.0


def tensor(a, dtype):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def run_layer(inp: LayerInputs, save: bool = True, cnp_only_forward: bool = False):
    """Runs merge, CNP forward, layer forward + backward and CNP backward on the GPU."""
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P

    s = inp.shape
    act = torch.float32 if s.dtype == "f32" else torch.bfloat16
    perm_P, inv_P = P.make_perm(inp.seed_P, s.n)
    perm_R, inv_R = P.make_perm(inp.seed_R, s.m)
    W0 = tensor(inp.W0, act)
    layer = P.PoetxLinear(W0, tensor(inp.theta_P, torch.float32),
                          tensor(inp.theta_R, torch.float32), perm_P, perm_R, s.b, s.k, s.T,
                          save_activations=save)
    x = tensor(inp.x, act)
    dy = tensor(inp.dy, act)
    y = torch.empty((s.T, s.m), dtype=act, device="cuda")
    dx = torch.empty((s.T, s.n), dtype=act, device="cuda")
    layer.step(x, dy, y, dx)
    torch.cuda.synchronize()
    assert P.device_status() == P.POETX_OK
    out = dict(perm_P=perm_P, perm_R=perm_R, inv_P=inv_P, inv_R=inv_R,
               W0p=host(layer.W0p), G=host(layer.G), y=host(y), dx=host(dx),
               dG_P=host(layer.dG[: layer.nP]), dG_R=host(layer.dG[layer.nP:]),
               dtheta_P=host(layer.dtheta[: layer.nP]), dtheta_R=host(layer.dtheta[layer.nP:]))
    if layer.G_lp is not None:
        out["G_lp"] = host(layer.G_lp)
    out["layer"] = layer
    return out


def run_group(inps, save: bool = True):
    """Runs one step of a PoetxLinearGroup (one CNP forward over every block, every
    linear's forward and backward, one CNP backward) on the GPU; returns per-linear outputs
    like run_layer's, plus "group"."""
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P

    s0 = inps[0].shape
    act = torch.float32 if s0.dtype == "f32" else torch.bfloat16
    specs, xs, dys, ys, dxs, perms = [], [], [], [], [], []
    for inp in inps:
        s = inp.shape
        perm_P, inv_P = P.make_perm(inp.seed_P, s.n)
        perm_R, inv_R = P.make_perm(inp.seed_R, s.m)
        perms.append((perm_P, perm_R, inv_P, inv_R))
        specs.append((tensor(inp.W0, act), tensor(inp.theta_P, torch.float32),
                      tensor(inp.theta_R, torch.float32), perm_P, perm_R))
        xs.append(tensor(inp.x, act))
        dys.append(tensor(inp.dy, act))
        ys.append(torch.empty((s.T, s.m), dtype=act, device="cuda"))
        dxs.append(torch.empty((s.T, s.n), dtype=act, device="cuda"))
    g = P.PoetxLinearGroup(specs, s0.b, s0.k, s0.T, save_activations=save)
    g.step(xs, dys, ys, dxs)
    torch.cuda.synchronize()
    assert P.device_status() == P.POETX_OK
    outs = []
    for L, y, dx, (perm_P, perm_R, inv_P, inv_R) in zip(g.layers, ys, dxs, perms):
        o = dict(perm_P=perm_P, perm_R=perm_R, inv_P=inv_P, inv_R=inv_R, W0p=host(L.W0p),
                 G=host(L.G), y=host(y), dx=host(dx), dG_P=host(L.dG[: L.nP]),
                 dG_R=host(L.dG[L.nP:]), dtheta_P=host(L.dtheta[: L.nP]),
                 dtheta_R=host(L.dtheta[L.nP:]))
        if L.G_lp is not None:
            o["G_lp"] = host(L.G_lp)
        outs.append(o)
    del xs, dys, ys, dxs
    return outs, g


__all__ = ["LayerShape", "layer_inputs", "norm_max_err", "tensor", "host", "run_layer",
           "run_group"]
