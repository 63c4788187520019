"""Seeded synthetic inputs shared by the oracle-side tests and the CUDA-side harness.

This module holds no arithmetic of the layer itself: it only draws numbers and rounds
them to the storage precision the GPU path receives.  Both sides (the float64 oracle
and the CUDA library) consume exactly the same host arrays.

Recipe
------
* Values: ``numpy.random.Generator(PCG64(SeedSequence([config_id, linear_id, tensor_id])))``,
  ``standard_normal`` in float64, multiplied by the stated standard deviation, then
  rounded to the storage dtype.  ``tensor_id``: x=0, W0=1, theta_P=2, theta_R=3, dy=4, dG=5.
* Rounding: fp32 storage is float64 -> float32 (round to nearest even).  bf16 storage is
  float64 -> float32 -> bf16 (both steps round to nearest even).  The oracle receives the
  rounded values widened back to float64, so it never sees a value the GPU did not get.
* theta is drawn directly in its packed form (strict upper triangle per block).
* Permutations are NOT drawn here: the permutation generator is part of the method and
  each side implements it separately (see ``oracle.poetx_ref.make_perm`` and
  ``poetx_make_perm`` in the C library).  This module only provides the seed convention
  ``(config_id << 32) | (linear_id << 8) | side`` with side 0 = P (input), 1 = R (output).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

TENSOR_IDS = {"x": 0, "W0": 1, "theta_P": 2, "theta_R": 3, "dy": 4, "dG": 5}


def _rng(config_id: int, linear_id: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([config_id, linear_id, tensor_id])))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """float -> float32 (RNE) -> bf16 (RNE); returned as float32 holding bf16-exact values."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(a_bf16_exact_f32: np.ndarray) -> np.ndarray:
    """The uint16 bit pattern of float32 values that are already bf16-exact."""
    u = np.ascontiguousarray(a_bf16_exact_f32, dtype=np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)


def draw(config_id: int, linear_id: int, tensor: str, shape, std: float, storage: str) -> np.ndarray:
    """One seeded N(0, std^2) tensor rounded to ``storage`` ('f32' or 'bf16').

    Returns float32 holding exactly the stored values.
    """
    g = _rng(config_id, linear_id, TENSOR_IDS[tensor])
    a = g.standard_normal(size=shape) * std
    if storage == "f32":
        return a.astype(np.float32)
    if storage == "bf16":
        return round_to_bf16(a)
    raise ValueError(storage)


def perm_seed(config_id: int, linear_id: int, side: int) -> int:
    return (config_id << 32) | (linear_id << 8) | side


@dataclass
class LayerShape:
    """One POET-X linear: T tokens, n inputs, m outputs, block size b, Neumann order k."""
    name: str
    T: int
    n: int
    m: int
    b: int
    k: int
    dtype: str  # 'f32' (everything fp32) or 'bf16' (bf16 activations/W0, fp32 theta/CNP)
    config_id: int
    linear_id: int = 0
    std_x: float = 1.0
    std_theta: float = 0.01
    std_w0: float | None = None  # default 1/sqrt(n)
    std_dy: float = 1.0

    @property
    def nblk_P(self) -> int:
        return self.n // self.b

    @property
    def nblk_R(self) -> int:
        return self.m // self.b

    @property
    def ntri(self) -> int:
        return self.b * (self.b - 1) // 2


@dataclass
class LayerInputs:
    shape: LayerShape
    x: np.ndarray        # [T, n]  (float32 holding storage-exact values)
    W0: np.ndarray       # [m, n]
    theta_P: np.ndarray  # [n/b, b(b-1)/2] float32
    theta_R: np.ndarray  # [m/b, b(b-1)/2] float32
    dy: np.ndarray       # [T, m]
    seed_P: int = 0
    seed_R: int = 0
    extra: dict = field(default_factory=dict)


def layer_inputs(s: LayerShape) -> LayerInputs:
    act = "f32" if s.dtype == "f32" else "bf16"
    std_w0 = s.std_w0 if s.std_w0 is not None else 1.0 / np.sqrt(s.n)
    x = draw(s.config_id, s.linear_id, "x", (s.T, s.n), s.std_x, act)
    W0 = draw(s.config_id, s.linear_id, "W0", (s.m, s.n), std_w0, act)
    tP = draw(s.config_id, s.linear_id, "theta_P", (s.nblk_P, s.ntri), s.std_theta, "f32")
    tR = draw(s.config_id, s.linear_id, "theta_R", (s.nblk_R, s.ntri), s.std_theta, "f32")
    dy = draw(s.config_id, s.linear_id, "dy", (s.T, s.m), s.std_dy, act)
    return LayerInputs(s, x, W0, tP, tR, dy,
                       perm_seed(s.config_id, s.linear_id, 0), perm_seed(s.config_id, s.linear_id, 1))


def cnp_inputs(config_id: int, linear_id: int, nblk: int, b: int, std_theta: float = 0.01,
               std_dG: float = 1.0, chunk_blocks: int = 256):
    """theta [nblk, b(b-1)/2] and an upstream gradient dG [nblk, b, b], both fp32.

    Drawn in chunks of blocks from one stream per tensor (the same values as a single
    draw), so large block counts never hold a float64 copy of the whole tensor.
    """
    ntri = b * (b - 1) // 2
    out = []
    for name, shape, std in [("theta_P", (ntri,), std_theta), ("dG", (b, b), std_dG)]:
        g = _rng(config_id, linear_id, TENSOR_IDS[name])
        a = np.empty((nblk,) + shape, dtype=np.float32)
        for c0 in range(0, nblk, chunk_blocks):
            c1 = min(nblk, c0 + chunk_blocks)
            a[c0:c1] = (g.standard_normal(size=(c1 - c0,) + shape) * std).astype(np.float32)
        out.append(a)
    return out[0], out[1]


# ---------------------------------------------------------------- named workloads
# The five workloads the layer is measured and checked on (shapes only).

def workload_small_fp32() -> LayerShape:
    """Single POET-X linear, all fp32: n=m=256, b=32, k=4, T=512, theta~N(0, 0.02^2)."""
    return LayerShape("fp32-256x256-b32-T512", T=512, n=256, m=256, b=32, k=4, dtype="f32",
                      config_id=1, std_theta=0.02)


def workload_llama1b_attn() -> LayerShape:
    """Llama-1B-shaped attention projection: n=m=2048, b=256, k=4, T=8192, bf16 activations."""
    return LayerShape("llama1b-attn-2048x2048-b256-T8192", T=8192, n=2048, m=2048, b=256, k=4,
                      dtype="bf16", config_id=2, std_theta=0.01)


def workload_llama8b_up() -> LayerShape:
    """Llama-8B-shaped MLP up-projection: n=4096 -> m=14336, b=256, k=4, T=16384, bf16."""
    return LayerShape("llama8b-up-4096x14336-b256-T16384", T=16384, n=4096, m=14336, b=256, k=4,
                      dtype="bf16", config_id=3, std_theta=0.01)


LLAMA13B_LINEARS = [  # (name, n_in, n_out) for d=5120, ffn=13824
    ("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120), ("o", 5120, 5120),
    ("gate", 5120, 13824), ("up", 5120, 13824), ("down", 13824, 5120),
]


def workload_llama13b_block(T: int = 8192):
    """All 7 linears of a Llama-13B-shaped decoder block as POET-X layers, b=256, k=4."""
    return [LayerShape(f"llama13b-{nm}-{n}x{m}-b256-T{T}", T=T, n=n, m=m, b=256, k=4, dtype="bf16",
                       config_id=5, linear_id=i, std_theta=0.01)
            for i, (nm, n, m) in enumerate(LLAMA13B_LINEARS)]


LLAMA8B_LINEAR_DIMS = [(4096, 4096)] * 4 + [(4096, 14336)] * 2 + [(14336, 4096)]


def cnp_sweep_blocks(b: int, layers: int = 32) -> int:
    """Block count of the CNP sweep: both sides of all 7 linears x 32 layers of Llama-8B shapes."""
    dims = sum(n + m for n, m in LLAMA8B_LINEAR_DIMS) * layers
    assert dims % b == 0
    return dims // b
