"""Thin ctypes binding of libpoetx (the C ABI declared in include/poetx.h).

Argument marshalling only: tensors are passed as raw device pointers, the stream as the
torch stream handle.  Every step of the layer runs in the library's CUDA kernels; there is
no fallback.  A missing library or a call without a CUDA device raises immediately.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpoetx.so")

POETX_OK = 0
POETX_ERR_INVALID_ARG = 1
POETX_ERR_SHAPE = 2
POETX_ERR_DTYPE = 3
POETX_ERR_ALIGN = 4
POETX_ERR_WORKSPACE = 5
POETX_ERR_CUDA = 6
POETX_ERR_TIMEOUT = 7

POETX_F32 = 0
POETX_BF16 = 1

_c_int = ctypes.c_int
_c_i32 = ctypes.c_int32
_c_u64 = ctypes.c_uint64
_c_size = ctypes.c_size_t
_vp = ctypes.c_void_p
_i32p = ctypes.POINTER(ctypes.c_int32)


class LinearDesc(ctypes.Structure):
    _fields_ = [("T", _c_i32), ("n", _c_i32), ("m", _c_i32), ("b", _c_i32), ("dtype", _c_i32),
                ("perm_P", _vp), ("inv_P", _vp), ("perm_R", _vp), ("inv_R", _vp)]


# name -> (restype, argtypes); the same list is checked against include/poetx.h by the tests
SIGNATURES = {
    "poetx_status_string": (ctypes.c_char_p, [_c_int]),
    "poetx_last_error": (ctypes.c_char_p, []),
    "poetx_version": (ctypes.c_char_p, []),
    "poetx_make_perm": (_c_int, [_c_u64, _c_i32, _i32p, _i32p]),
    "poetx_invert_perm": (_c_int, [_i32p, _c_i32, _i32p]),
    "poetx_merge_perm": (_c_int, [_vp, _vp, _c_i32, _c_i32, _vp, _vp, _c_int, _vp]),
    "poetx_permute_cols": (_c_int, [_vp, _vp, _vp, _c_i32, _c_i32, _c_int, _vp]),
    "poetx_outer_merge_workspace": (_c_size, [_c_i32, _c_i32, _c_int]),
    "poetx_outer_merge": (_c_int, [_vp, _vp, _vp, _c_i32, _c_i32, _c_i32, _vp, _vp, _vp, _vp,
                                   _vp, _c_int, _vp, _c_size, _vp]),
    "poetx_cnp_workspace": (_c_size, [_c_i32, _c_i32, _c_i32]),
    "poetx_cnp_fwd": (_c_int, [_vp, _vp, _vp, _c_i32, _c_i32, _c_i32, _vp, _c_size, _vp]),
    "poetx_cnp_bwd": (_c_int, [_vp, _vp, _vp, _c_i32, _c_i32, _c_i32, _vp, _c_size, _vp]),
    "poetx_cnp_fwd_static": (_c_int, [_vp, _vp, _vp, _c_i32, _c_i32, _c_i32, _vp]),
    "poetx_cnp_fwd_save": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_i32, _c_i32, _c_i32, _vp,
                                    _c_size, _vp]),
    "poetx_cnp_bwd_saved": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_i32, _c_i32, _c_i32, _vp,
                                     _c_size, _vp]),
    "poetx_linear_fwd_workspace": (_c_size, [ctypes.POINTER(LinearDesc), _c_int, _c_int]),
    "poetx_linear_bwd_workspace": (_c_size, [ctypes.POINTER(LinearDesc), _c_int, _c_int]),
    "poetx_linear_fwd": (_c_int, [ctypes.POINTER(LinearDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _c_size, _vp]),
    "poetx_linear_bwd": (_c_int, [ctypes.POINTER(LinearDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _vp, _vp, _c_int, _vp, _c_size, _vp]),
    "poetx_device_status": (_c_int, [_vp]),
    "poetx_set_wait_limit": (_c_int, [_c_u64, ctypes.POINTER(_c_u64)]),
    "poetx_set_gemm_pairs": (_c_int, [_c_int, ctypes.POINTER(_c_int)]),
    "poetx_selftest_wait_timeout": (_c_int, [_vp, _vp, _c_i32, _c_i32, _c_i32, _vp, _c_size,
                                             _vp]),
    "poetx_fma_probe": (_c_int, [_vp, _c_i32, _c_i32, _vp]),
    "poetx_quantize_rows": (_c_int, [_vp, _vp, _vp, _c_i32, _c_i32, _c_int, _vp]),
    "poetx_merge_perm_q8": (_c_int, [_vp, _vp, _vp, _c_i32, _c_i32, _vp, _vp, _c_int, _vp]),
    "poetx_linear_q8_scratch": (_c_size, [ctypes.POINTER(LinearDesc)]),
    "poetx_linear_fwd_q8": (_c_int, [ctypes.POINTER(LinearDesc), _vp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _vp, _c_size, _vp]),
    "poetx_linear_bwd_q8": (_c_int, [ctypes.POINTER(LinearDesc), _vp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_size, _vp]),
    "poetx_launch_count": (_c_u64, []),
    "poetx_profile_begin": (_c_int, [ctypes.c_char_p]),
    "poetx_profile_end": (_c_int, [_i32p, ctypes.POINTER(ctypes.c_double)]),
}

_lib = None


class PoetxError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        lib = _load()
        super().__init__(f"{where}: {lib.poetx_status_string(status).decode()} "
                         f"({status}): {lib.poetx_last_error().decode()}")


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libpoetx.so not built ({LIB_PATH}); run "
                               "`python -m orthogonal_reparameterized_cnp_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def lib():
    return _load()


def _check(status: int, where: str):
    if status != POETX_OK:
        raise PoetxError(status, where)


# ------------------------------------------------------------------------ helpers
def _ptr(t) -> int | None:
    """Device pointer of a torch tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return POETX_F32
    if t.dtype == torch.bfloat16:
        return POETX_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------------ host calls
def make_perm(seed: int, n: int):
    """Seeded permutation and its inverse (numpy int32), computed by the library."""
    L = _load()
    perm = np.empty(n, dtype=np.int32)
    inv = np.empty(n, dtype=np.int32)
    _check(L.poetx_make_perm(seed & ((1 << 64) - 1), n,
                             perm.ctypes.data_as(_i32p), inv.ctypes.data_as(_i32p)),
           "poetx_make_perm")
    return perm, inv


def invert_perm(perm) -> np.ndarray:
    """Inverse of an index map (numpy int32), computed and validated by the library: a map
    that is not a bijection of range(n) raises PoetxError (POETX_ERR_INVALID_ARG)."""
    L = _load()
    p = np.ascontiguousarray(np.asarray(perm), dtype=np.int32)
    if p.ndim != 1:
        raise ValueError("an index map is a 1-D array")
    inv = np.empty_like(p)
    _check(L.poetx_invert_perm(p.ctypes.data_as(_i32p), len(p), inv.ctypes.data_as(_i32p)),
           "poetx_invert_perm")
    return inv


def set_wait_limit(ns: int) -> int:
    """Sets the kernels' bounded-wait limit (0: the 2 s default); returns the previous one."""
    prev = _c_u64(0)
    _check(_load().poetx_set_wait_limit(int(ns), ctypes.byref(prev)), "poetx_set_wait_limit")
    return int(prev.value)


def set_gemm_pairs(enable: bool) -> bool:
    """Merged-weight GEMMs on CTA pairs (True, the default) or single CTAs; returns the
    previous setting."""
    prev = ctypes.c_int(0)
    _check(_load().poetx_set_gemm_pairs(int(bool(enable)), ctypes.byref(prev)),
           "poetx_set_gemm_pairs")
    return bool(prev.value)


def cnp_workspace(nblk: int, b: int, k: int) -> int:
    return int(_load().poetx_cnp_workspace(nblk, b, k))


def linear_desc(T, n, m, b, dtype_code, perm_P, inv_P, perm_R, inv_R) -> LinearDesc:
    return LinearDesc(T, n, m, b, dtype_code, _ptr(perm_P), _ptr(inv_P), _ptr(perm_R),
                      _ptr(inv_R))


def linear_fwd_workspace(desc: LinearDesc, has_save_u=True, has_save_w=True) -> int:
    return int(_load().poetx_linear_fwd_workspace(ctypes.byref(desc), int(has_save_u),
                                                  int(has_save_w)))


def linear_bwd_workspace(desc: LinearDesc, has_save_u=True, has_save_w=True) -> int:
    return int(_load().poetx_linear_bwd_workspace(ctypes.byref(desc), int(has_save_u),
                                                  int(has_save_w)))


def launch_count() -> int:
    return int(_load().poetx_launch_count())


def profile_begin(name: str | None):
    _check(_load().poetx_profile_begin(name.encode() if name else None), "poetx_profile_begin")


def profile_end():
    n = ctypes.c_int32(0)
    ms = ctypes.c_double(0.0)
    _check(_load().poetx_profile_end(ctypes.byref(n), ctypes.byref(ms)), "poetx_profile_end")
    return int(n.value), float(ms.value)


# ------------------------------------------------------------------------ device calls
def _require_cuda():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("libpoetx needs a CUDA device (sm_100a); none is available")


def merge_perm(W0, W0p, perm_R, perm_P, stream=None):
    _require_cuda()
    m, n = W0.shape
    _check(_load().poetx_merge_perm(_ptr(W0), _ptr(W0p), m, n, _ptr(perm_R), _ptr(perm_P),
                                    _dtype_code(W0), _stream(stream)), "poetx_merge_perm")


def outer_merge_workspace(m: int, n: int, dtype_code: int) -> int:
    return int(_load().poetx_outer_merge_workspace(m, n, dtype_code))


def outer_merge(W0p, G_P, G_R, b: int, inv_P, inv_R, perm_P_new, perm_R_new, W0p_new, ws,
                stream=None):
    """W0p_new = merged weight, under the new permutations, of R W0 P (see the header)."""
    _require_cuda()
    m, n = W0p.shape
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_outer_merge(_ptr(W0p), _ptr(G_P), _ptr(G_R), m, n, b, _ptr(inv_P),
                                     _ptr(inv_R), _ptr(perm_P_new), _ptr(perm_R_new),
                                     _ptr(W0p_new), _dtype_code(W0p), _ptr(ws), ws_bytes,
                                     _stream(stream)), "poetx_outer_merge")


def permute_cols(x, out, idx, stream=None):
    _require_cuda()
    rows, cols = x.shape
    _check(_load().poetx_permute_cols(_ptr(x), _ptr(out), _ptr(idx), rows, cols, _dtype_code(x),
                                      _stream(stream)), "poetx_permute_cols")


def cnp_fwd(theta, G, G_bf16, b: int, k: int, ws, stream=None):
    _require_cuda()
    nblk = theta.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_cnp_fwd(_ptr(theta), _ptr(G), _ptr(G_bf16), nblk, b, k, _ptr(ws),
                                 ws_bytes, _stream(stream)), "poetx_cnp_fwd")


def cnp_fwd_static(theta, G, G_bf16, b: int, k: int, stream=None):
    """CNP forward with the library's fixed device scratch (no caller buffer; see the
    header for the size limit and the sharing rules)."""
    _require_cuda()
    nblk = theta.shape[0]
    _check(_load().poetx_cnp_fwd_static(_ptr(theta), _ptr(G), _ptr(G_bf16), nblk, b, k,
                                        _stream(stream)), "poetx_cnp_fwd_static")


def cnp_bwd(theta, dG, dtheta, b: int, k: int, ws, stream=None):
    _require_cuda()
    nblk = theta.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_cnp_bwd(_ptr(theta), _ptr(dG), _ptr(dtheta), nblk, b, k, _ptr(ws),
                                 ws_bytes, _stream(stream)), "poetx_cnp_bwd")


def cnp_fwd_save(theta, G, G_bf16, Q_save, S_save, F_save, b: int, k: int, ws, stream=None):
    """CNP forward that also keeps Q, S = Q^2 and F' for poetx_cnp_bwd_saved."""
    _require_cuda()
    nblk = theta.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_cnp_fwd_save(_ptr(theta), _ptr(G), _ptr(G_bf16), _ptr(Q_save),
                                      _ptr(S_save), _ptr(F_save), nblk, b, k, _ptr(ws), ws_bytes,
                                      _stream(stream)), "poetx_cnp_fwd_save")


def cnp_bwd_saved(theta, dG, Q_saved, S_saved, F_saved, dtheta, b: int, k: int, ws,
                  stream=None):
    """CNP backward reading the forward's Q, S and F' (theta unchanged since)."""
    _require_cuda()
    nblk = theta.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_cnp_bwd_saved(_ptr(theta), _ptr(dG), _ptr(Q_saved), _ptr(S_saved),
                                       _ptr(F_saved), _ptr(dtheta), nblk, b, k, _ptr(ws),
                                       ws_bytes, _stream(stream)), "poetx_cnp_bwd_saved")


def linear_fwd(desc: LinearDesc, x, G_P, G_R, W0p, y, save_u, save_w, ws, stream=None):
    _require_cuda()
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_linear_fwd(ctypes.byref(desc), _ptr(x), _ptr(G_P), _ptr(G_R),
                                    _ptr(W0p), _ptr(y), _ptr(save_u), _ptr(save_w), _ptr(ws),
                                    ws_bytes, _stream(stream)), "poetx_linear_fwd")


def linear_bwd(desc: LinearDesc, x, dy, G_P, G_R, W0p, save_u, save_w, dx, dG_P, dG_R,
               accumulate: int, ws, stream=None):
    _require_cuda()
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_linear_bwd(ctypes.byref(desc), _ptr(x), _ptr(dy), _ptr(G_P), _ptr(G_R),
                                    _ptr(W0p), _ptr(save_u), _ptr(save_w), _ptr(dx), _ptr(dG_P),
                                    _ptr(dG_R), int(accumulate), _ptr(ws), ws_bytes,
                                    _stream(stream)), "poetx_linear_bwd")


def quantize_rows(W, q, scales, stream=None):
    """Per-row symmetric int8 codes and fp32 scales of W (see the header)."""
    _require_cuda()
    m, n = W.shape
    _check(_load().poetx_quantize_rows(_ptr(W), _ptr(q), _ptr(scales), m, n, _dtype_code(W),
                                       _stream(stream)), "poetx_quantize_rows")


def merge_perm_q8(W0, q, scales, perm_R, perm_P, stream=None):
    """Int8 codes and per-row scales of W0' = W0[perm_R][:, perm_P], without forming W0'."""
    _require_cuda()
    m, n = W0.shape
    _check(_load().poetx_merge_perm_q8(_ptr(W0), _ptr(q), _ptr(scales), m, n, _ptr(perm_R),
                                       _ptr(perm_P), _dtype_code(W0), _stream(stream)),
           "poetx_merge_perm_q8")


def linear_q8_scratch(desc: LinearDesc) -> int:
    return int(_load().poetx_linear_q8_scratch(ctypes.byref(desc)))


def linear_fwd_q8(desc: LinearDesc, x, G_P, G_R, W0q, scales, y, save_u, save_w, ws,
                  stream=None):
    _require_cuda()
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_linear_fwd_q8(ctypes.byref(desc), _ptr(x), _ptr(G_P), _ptr(G_R),
                                       _ptr(W0q), _ptr(scales), _ptr(y), _ptr(save_u),
                                       _ptr(save_w), _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_linear_fwd_q8")


def linear_bwd_q8(desc: LinearDesc, x, dy, G_P, G_R, W0q, scales, save_u, save_w, dx, dG_P,
                  dG_R, accumulate: int, ws, stream=None):
    _require_cuda()
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_linear_bwd_q8(ctypes.byref(desc), _ptr(x), _ptr(dy), _ptr(G_P),
                                       _ptr(G_R), _ptr(W0q), _ptr(scales), _ptr(save_u),
                                       _ptr(save_w), _ptr(dx), _ptr(dG_P), _ptr(dG_R),
                                       accumulate, _ptr(ws), ws_bytes, _stream(stream)),
           "poetx_linear_bwd_q8")


def selftest_wait_timeout(theta, G, b: int, k: int, ws, stream=None):
    """Runs the CNP forward with a dependency that is never met (see the header)."""
    _require_cuda()
    nblk = theta.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().poetx_selftest_wait_timeout(_ptr(theta), _ptr(G), nblk, b, k, _ptr(ws),
                                               ws_bytes, _stream(stream)),
           "poetx_selftest_wait_timeout")


def fma_probe(out, ctas: int, iters: int, stream=None):
    """FP32 FMA throughput probe: ctas * 512 * 16 * iters * 2 FLOPs into out[ctas * 512]."""
    _require_cuda()
    _check(_load().poetx_fma_probe(_ptr(out), ctas, iters, _stream(stream)), "poetx_fma_probe")


def device_status(stream=None) -> int:
    _require_cuda()
    return int(_load().poetx_device_status(_stream(stream)))


# ------------------------------------------------------------------------ layer objects
class CnpBuffers:
    """Device buffers of the Cayley-Neumann parameterisation of nblk b x b blocks: theta,
    G (fp32 and, for the bf16 layer, its bf16 copy), the upstream dG, dtheta, and the Q,
    S = Q^2 and F' that the forward keeps for the backward.  One forward call and one
    backward call cover every block, whichever layers the blocks belong to."""

    def __init__(self, nblk: int, b: int, k: int, device, lowp_dtype=None):
        import torch
        self.nblk, self.b, self.k = nblk, b, k
        f32 = dict(dtype=torch.float32, device=device)
        ntri = b * (b - 1) // 2
        self.theta = torch.zeros((nblk, ntri), **f32)
        self.G = torch.empty((nblk, b, b), **f32)
        self.G_lp = torch.empty((nblk, b, b), dtype=lowp_dtype, device=device) \
            if lowp_dtype is not None else None
        self.dG = torch.zeros((nblk, b, b), **f32)
        self.dtheta = torch.empty((nblk, ntri), **f32)
        self.Q_save = torch.empty((nblk, b, b), **f32)
        self.S_save = torch.empty((nblk, b, b), **f32)
        self.F_save = torch.empty((nblk, b, b), **f32)
        self.ws = None
        self.set_order(k)

    def set_order(self, k: int):
        """Neumann order of the following calls (the scratch is resized to it)."""
        import torch
        self.k = k
        self.ws = None
        self.ws = torch.empty(max(cnp_workspace(self.nblk, self.b, k), 16), dtype=torch.uint8,
                              device=self.G.device)

    def forward(self, stream=None):
        cnp_fwd_save(self.theta, self.G, self.G_lp, self.Q_save, self.S_save, self.F_save,
                     self.b, self.k, self.ws, stream)

    def backward(self, stream=None):
        """dtheta from dG; reads the Q, S and F' of the last forward (theta unchanged)."""
        cnp_bwd_saved(self.theta, self.dG, self.Q_save, self.S_save, self.F_save, self.dtheta,
                      self.b, self.k, self.ws, stream)


def _layer_scratch_bytes(desc, save: bool, int8: bool) -> int:
    q8 = linear_q8_scratch(desc) if int8 else 0
    return max(linear_fwd_workspace(desc, save, save), linear_bwd_workspace(desc, save, save),
               16) + q8


class PoetxLinear:
    """One POET-X linear on the GPU: merged weight, CNP blocks, forward and backward.

    All buffers are torch tensors on the current device; every computation is a libpoetx
    call.  The CNP blocks are the input-side blocks first, then the output-side blocks, in
    ``cnp`` (a CnpBuffers of this layer alone unless one is shared, see PoetxLinearGroup);
    ``theta``, ``G``, ``dG``, ``dtheta`` are this layer's rows of it.  The inverse index
    maps come from the library, which rejects a perm_P or perm_R that is not a bijection.
    The permutations are merged into W0' once, at construction (and again by merge()).
    """

    def __init__(self, W0, theta_P, theta_R, perm_P, perm_R, b: int, k: int, T: int,
                 save_activations: bool = True, int8_weight: bool = False, cnp=None,
                 first_block: int = 0, ws=None):
        import torch
        self.m, self.n = W0.shape
        # the index maps are checked (bijections) and inverted by the library, on the host,
        # before any device work
        pP = np.ascontiguousarray(np.asarray(perm_P), dtype=np.int32)
        pR = np.ascontiguousarray(np.asarray(perm_R), dtype=np.int32)
        if pP.shape != (self.n,) or pR.shape != (self.m,):
            raise ValueError("perm_P must have n entries and perm_R m entries")
        iP, iR = invert_perm(pP), invert_perm(pR)
        _require_cuda()
        dev = W0.device
        self.b, self.k, self.T = b, k, T
        self.bf16 = W0.dtype == torch.bfloat16
        self.nP, self.nR = self.n // b, self.m // b
        nblk = self.nP + self.nR
        i32 = dict(dtype=torch.int32, device=dev)
        self.perm_P, self.inv_P = torch.as_tensor(pP, **i32), torch.as_tensor(iP, **i32)
        self.perm_R, self.inv_R = torch.as_tensor(pR, **i32), torch.as_tensor(iR, **i32)
        self.W0 = W0
        self.W0p = None if int8_weight else torch.empty_like(W0)
        if cnp is None:
            cnp = CnpBuffers(nblk, b, k, dev, W0.dtype if self.bf16 else None)
            first_block = 0
        if cnp.b != b or cnp.k != k or first_block + nblk > cnp.nblk:
            raise ValueError("the CNP buffers do not hold this layer's blocks")
        self.cnp = cnp
        rows = slice(first_block, first_block + nblk)
        self.theta, self.G, self.dG, self.dtheta = (cnp.theta[rows], cnp.G[rows], cnp.dG[rows],
                                                    cnp.dtheta[rows])
        self.G_lp = cnp.G_lp[rows] if cnp.G_lp is not None else None
        self.theta[: self.nP] = theta_P
        self.theta[self.nP:] = theta_R
        self.desc = linear_desc(T, self.n, self.m, b, POETX_BF16 if self.bf16 else POETX_F32,
                                self.perm_P, self.inv_P, self.perm_R, self.inv_R)
        act = W0.dtype
        self.save = save_activations
        if save_activations:
            self.U = torch.empty((T, self.n), dtype=act, device=dev)
            self.Wsave = torch.empty((T, self.m), dtype=act, device=dev)
        else:
            self.U = self.Wsave = None
        # int8 merged weight (POET-XQ): codes + per-row scales; the bf16 weight exists only
        # inside each layer call's scratch
        self.int8 = int8_weight
        if int8_weight:
            if not self.bf16:
                raise ValueError("the int8 base weight needs the bf16 layer")
            self.W0q = torch.empty((self.m, self.n), dtype=torch.int8, device=dev)
            self.scales = torch.empty((self.m,), dtype=torch.float32, device=dev)
        need = _layer_scratch_bytes(self.desc, self.save, int8_weight)
        if ws is None:
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
        elif ws.numel() * ws.element_size() < need:
            raise ValueError("shared layer scratch too small")
        self.ws = ws
        if int8_weight:  # the merged weight exists only as int8 codes (merge_perm_q8)
            self.W0p = None
        self.merge()

    def G_ops(self):
        G = self.G_lp if self.bf16 else self.G
        return G[: self.nP], G[self.nP:]

    def merge(self, stream=None):
        """W0' = Pi_R W0 Pi_P^T (and its int8 codes): once per set of permutations."""
        if self.int8:
            merge_perm_q8(self.W0, self.W0q, self.scales, self.perm_R, self.perm_P, stream)
        else:
            merge_perm(self.W0, self.W0p, self.perm_R, self.perm_P, stream)

    def cnp_forward(self, stream=None):
        self.cnp.forward(stream)

    def forward(self, x, y, stream=None):
        GP, GR = self.G_ops()
        if self.int8:
            linear_fwd_q8(self.desc, x, GP, GR, self.W0q, self.scales, y, self.U, self.Wsave,
                          self.ws, stream)
        else:
            linear_fwd(self.desc, x, GP, GR, self.W0p, y, self.U, self.Wsave, self.ws, stream)

    def backward(self, x, dy, dx, accumulate=0, stream=None):
        GP, GR = self.G_ops()
        if self.int8:
            linear_bwd_q8(self.desc, x, dy, GP, GR, self.W0q, self.scales, self.U, self.Wsave,
                          dx, self.dG[: self.nP], self.dG[self.nP:], accumulate, self.ws,
                          stream)
        else:
            linear_bwd(self.desc, x, dy, GP, GR, self.W0p, self.U, self.Wsave, dx,
                       self.dG[: self.nP], self.dG[self.nP:], accumulate, self.ws, stream)

    def cnp_backward(self, stream=None):
        """dtheta from dG; reads Q, S and F' of the last cnp_forward (theta unchanged)."""
        self.cnp.backward(stream)

    def step(self, x, dy, y, dx, stream=None):
        """One pass of the per-step path: CNP forward, layer forward and backward, CNP
        backward (the merge of the permutations is per set of permutations, not per step)."""
        self.cnp_forward(stream)
        self.forward(x, y, stream)
        self.backward(x, dy, dx, 0, stream)
        self.cnp_backward(stream)


class PoetxLinearGroup:
    """Several POET-X linears (e.g. the seven of a decoder block) whose CNP forward and
    backward each run as one call over all of their blocks, and whose layer calls share one
    scratch buffer (they run one after another on one stream).

    specs: list of (W0, theta_P, theta_R, perm_P, perm_R) per linear.
    """

    def __init__(self, specs, b: int, k: int, T: int, save_activations: bool = True,
                 int8_weight: bool = False):
        import torch
        _require_cuda()
        W0s = [sp[0] for sp in specs]
        dev = W0s[0].device
        bf16 = W0s[0].dtype == torch.bfloat16
        nblks = [(W.shape[1] + W.shape[0]) // b for W in W0s]
        self.cnp = CnpBuffers(sum(nblks), b, k, dev, W0s[0].dtype if bf16 else None)
        need = 16
        for W in W0s:
            m, n = W.shape
            d = LinearDesc(T, n, m, b, POETX_BF16 if bf16 else POETX_F32, None, None, None, None)
            need = max(need, _layer_scratch_bytes(d, save_activations, int8_weight))
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        self.layers = []
        off = 0
        for sp, nb in zip(specs, nblks):
            W0, tP, tR, pP, pR = sp
            self.layers.append(PoetxLinear(W0, tP, tR, pP, pR, b, k, T, save_activations,
                                           int8_weight, cnp=self.cnp, first_block=off,
                                           ws=self.ws))
            off += nb
        self.b, self.k, self.T = b, k, T

    def merge(self, stream=None):
        for L in self.layers:
            L.merge(stream)

    def cnp_forward(self, stream=None):
        self.cnp.forward(stream)

    def forward(self, xs, ys, stream=None):
        for L, x, y in zip(self.layers, xs, ys):
            L.forward(x, y, stream)

    def backward(self, xs, dys, dxs, accumulate=0, stream=None):
        for L, x, dy, dx in reversed(list(zip(self.layers, xs, dys, dxs))):
            L.backward(x, dy, dx, accumulate, stream)

    def cnp_backward(self, stream=None):
        self.cnp.backward(stream)

    def step(self, xs, dys, ys, dxs, stream=None):
        """CNP forward (every block, one call), every layer's forward, every layer's
        backward (last layer first), CNP backward (one call)."""
        self.cnp_forward(stream)
        self.forward(xs, ys, stream)
        self.backward(xs, dys, dxs, 0, stream)
        self.cnp_backward(stream)
