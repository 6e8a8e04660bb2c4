"""Python binding of the Fourier-approximated KV cache library (sm_100a).

Argument marshalling only: every step of the hot path runs in the CUDA kernels of
``libfourier_attention.so`` behind the C ABI declared in ``include/fourier_attention.h``.
PyTorch is used for device memory and streams. The functions keep the C names:

    fa_plan_init, fa_plan_reserve, fa_build_basis, fa_compress, fa_decode_workspace_size,
    fa_decode_describe, fa_decode, fa_decode_noalloc, fa_append, fa_dim_sensitivity_workspace_size,
    fa_dim_sensitivity, fa_select_dims, fa_device_status, fa_last_error

There is no CPU fallback: if the shared library is missing or fails to load, importing
this package raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import _build

HEAD_DIM = 128
MAX_KV_HEADS = 64
MAX_K_DECODE = 2047
FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_DEVICE = range(5)
FA_BF16, FA_F32 = 0, 1
(FA_SPLIT_NONE, FA_SPLIT_CUDA_CORES, FA_SPLIT_TC_TOKEN_MAJOR, FA_SPLIT_WARP_MMA,
 FA_SPLIT_TC_CLUSTER) = range(5)

EXPORTED = ("fa_plan_init", "fa_plan_reserve", "fa_build_basis", "fa_compress",
            "fa_decode_workspace_size", "fa_decode", "fa_decode_noalloc", "fa_append",
            "fa_dim_sensitivity_workspace_size", "fa_dim_sensitivity", "fa_select_dims",
            "fa_device_status", "fa_watchdog_selftest", "fa_last_error", "fa_decode_describe")
NOISE_SCALE = 0.1
NOALLOC_SCRATCH_BYTES = 16 << 20


class FaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class fa_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "D", "L", "S", "R", "k")]


_H = MAX_KV_HEADS


class fa_plan(ctypes.Structure):
    _fields_ = [
        ("shape", fa_shape),
        ("S", ctypes.c_int32), ("R", ctypes.c_int32), ("M", ctypes.c_int32),
        ("kk", ctypes.c_int32), ("G", ctypes.c_int32), ("phi_ld", ctypes.c_int32),
        ("e_token_major", ctypes.c_int32), ("P", ctypes.c_int32), ("recent_head", ctypes.c_int32),
        ("dc", ctypes.c_int32 * _H), ("de", ctypes.c_int32 * _H),
        ("dc_ld", ctypes.c_int32 * _H), ("de_ld", ctypes.c_int32 * _H),
        ("e_pitch", ctypes.c_int32 * _H),
        ("c_off", ctypes.c_int64 * _H), ("e_off", ctypes.c_int64 * _H),
        ("c_batch", ctypes.c_int64), ("e_batch", ctypes.c_int64),
        ("f_elems", ctypes.c_int64), ("e_elems", ctypes.c_int64), ("c_elems", ctypes.c_int64),
        ("perm", (ctypes.c_uint8 * HEAD_DIM) * _H),
    ]


class fa_decode_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("split_kernel", "num_splits", "cluster", "launches")]


SPLIT_KERNELS = {0: "none (no middle span)", 1: "CUDA cores (decode_main_kernel)",
                 2: "tcgen05, token-major E (decode_tc_kernel)",
                 3: "warp MMA (decode_hmma_kernel)",
                 4: "tcgen05, slot-split cluster (decode_cl_kernel)"}


class fa_cache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("F_K", "F_V", "E_K", "E_V", "C_K", "C_V")]


def _load() -> ctypes.CDLL:
    path = _build.LIB
    if os.environ.get("FA_SKIP_BUILD") != "1":
        path = _build.build()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing; run fourier_basis_attention_b200._build.build()")
    return configure(ctypes.CDLL(path))


def configure(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the C signatures on a loaded copy of the library."""
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.fa_plan_init.argtypes = [ctypes.POINTER(fa_shape), P, ctypes.POINTER(fa_plan)]
    lib.fa_plan_reserve.argtypes = [ctypes.POINTER(fa_plan), I32]
    lib.fa_build_basis.argtypes = [I32, I32, I32, I32, P, I64, P]
    lib.fa_append.argtypes = [ctypes.POINTER(fa_plan), P, P, ctypes.POINTER(fa_cache), P]
    lib.fa_dim_sensitivity_workspace_size.argtypes = [ctypes.POINTER(fa_shape)]
    lib.fa_dim_sensitivity_workspace_size.restype = SZ
    lib.fa_dim_sensitivity.argtypes = [ctypes.POINTER(fa_shape), P, P, P, P, P, SZ, P]
    lib.fa_select_dims.argtypes = [P, I32, I32, P]
    lib.fa_compress.argtypes = [ctypes.POINTER(fa_plan), P, P, P, ctypes.POINTER(fa_cache), P]
    lib.fa_decode_workspace_size.argtypes = [ctypes.POINTER(fa_plan), I32]
    lib.fa_decode_workspace_size.restype = SZ
    lib.fa_decode_describe.argtypes = [ctypes.POINTER(fa_plan), I32, ctypes.POINTER(fa_decode_info)]
    lib.fa_decode.argtypes = [ctypes.POINTER(fa_plan), P, ctypes.POINTER(fa_cache), P, I32, P, SZ,
                              I32, P]
    lib.fa_decode_noalloc.argtypes = [ctypes.POINTER(fa_plan), P, ctypes.POINTER(fa_cache), P, I32,
                                      I32, P]
    lib.fa_device_status.argtypes = [P]
    lib.fa_watchdog_selftest.argtypes = [ctypes.c_uint32, P]
    lib.fa_last_error.argtypes = []
    lib.fa_last_error.restype = ctypes.c_char_p
    for name in ("fa_plan_init", "fa_plan_reserve", "fa_build_basis", "fa_compress", "fa_decode",
                 "fa_decode_noalloc", "fa_append", "fa_dim_sensitivity", "fa_select_dims",
                 "fa_device_status", "fa_watchdog_selftest", "fa_decode_describe"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


LIB = _load()
LIB_PATH = _build.LIB


def fa_last_error() -> str:
    return LIB.fa_last_error().decode()


def _check(code: int) -> None:
    if code != FA_OK:
        raise FaError(code, fa_last_error())


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


# ----------------------------------------------------------------------------- C entry points

def fa_plan_init(B, Hq, Hkv, L, S, R, k, mask, D=HEAD_DIM) -> fa_plan:
    """Host-side plan of one layer. ``mask``: uint8-like [Hkv, 128], nonzero = compressed."""
    m = np.ascontiguousarray(np.asarray(mask) != 0, dtype=np.uint8)
    if m.shape != (Hkv, D):
        raise FaError(FA_ERR_INVALID, f"mask shape {m.shape} != ({Hkv}, {D})")
    shape = fa_shape(B, Hq, Hkv, D, L, S, R, k)
    plan = fa_plan()
    _check(LIB.fa_plan_init(ctypes.byref(shape), m.ctypes.data, ctypes.byref(plan)))
    return plan


def fa_plan_reserve(plan: fa_plan, L_max: int) -> fa_plan:
    """Room for tokens appended while decoding: basis period P = L_max - S - R (in place)."""
    _check(LIB.fa_plan_reserve(ctypes.byref(plan), int(L_max)))
    return plan


def fa_build_basis(M: int, k: int, phiT, ld: int | None = None, normalized: bool = False,
                   stream=None) -> None:
    """Fill device tensor ``phiT`` ([k, ld], bf16 or fp32) with the transposed basis
    (``normalized=False``: the unit-amplitude table fa_compress reads)."""
    import torch
    dtype = FA_BF16 if phiT.dtype == torch.bfloat16 else FA_F32
    if ld is None:
        ld = phiT.shape[-1]
    _check(LIB.fa_build_basis(M, k, dtype, int(bool(normalized)), _ptr(phiT), ld,
                              _stream(stream)))


def fa_compress(plan: fa_plan, K, V, phiT, cache: "Cache", stream=None) -> None:
    _check(LIB.fa_compress(ctypes.byref(plan), _ptr(K), _ptr(V), _ptr(phiT),
                           ctypes.byref(cache.c), _stream(stream)))


def fa_decode_workspace_size(plan: fa_plan, num_splits: int = 0) -> int:
    return int(LIB.fa_decode_workspace_size(ctypes.byref(plan), num_splits))


def fa_decode_describe(plan: fa_plan, num_splits: int = 0) -> fa_decode_info:
    """How fa_decode runs this plan: split kernel, split count, cluster size, launches."""
    info = fa_decode_info()
    _check(LIB.fa_decode_describe(ctypes.byref(plan), num_splits, ctypes.byref(info)))
    return info


def fa_decode(plan: fa_plan, q, cache: "Cache", out, workspace, num_splits: int = 0,
              stream=None) -> None:
    """One decode step; ``out`` is a [B, Hq, 128] fp32 or bf16 device tensor."""
    import torch
    out_dtype = FA_F32 if out.dtype == torch.float32 else FA_BF16
    nbytes = workspace.numel() * workspace.element_size()
    _check(LIB.fa_decode(ctypes.byref(plan), _ptr(q), ctypes.byref(cache.c), _ptr(out),
                         out_dtype, _ptr(workspace), nbytes, num_splits, _stream(stream)))


def fa_decode_noalloc(plan: fa_plan, q, cache: "Cache", out, num_splits: int = 0,
                      stream=None) -> None:
    """fa_decode without a workspace argument, for callers that cannot allocate device
    memory: the library's own fixed scratch array is used (see the C header)."""
    import torch
    out_dtype = FA_F32 if out.dtype == torch.float32 else FA_BF16
    _check(LIB.fa_decode_noalloc(ctypes.byref(plan), _ptr(q), ctypes.byref(cache.c), _ptr(out),
                                 out_dtype, num_splits, _stream(stream)))


def fa_append(plan: fa_plan, k_new, v_new, cache: "Cache", stream=None) -> None:
    """Append one token per sequence (k_new, v_new: bf16 [B, Hkv, 128]); advances ``plan``."""
    _check(LIB.fa_append(ctypes.byref(plan), _ptr(k_new), _ptr(v_new), ctypes.byref(cache.c),
                         _stream(stream)))


def fa_dim_sensitivity_workspace_size(B, Hq, Hkv, L) -> int:
    return LIB.fa_dim_sensitivity_workspace_size(ctypes.byref(fa_shape(B, Hq, Hkv, HEAD_DIM, L, 0, 0, 1)))


def fa_dim_sensitivity(q, K, noise, scores, workspace, stream=None) -> None:
    """Sensitivity scores [Hkv, 128] (fp32, device) of every head dim under value noise.
    q: bf16 [B, Hq, 128]; K, noise: bf16 [B, Hkv, L, 128]."""
    B, Hkv, L, D = K.shape
    shape = fa_shape(B, q.shape[1], Hkv, D, L, 0, 0, 1)
    _check(LIB.fa_dim_sensitivity(ctypes.byref(shape), _ptr(q), _ptr(K), _ptr(noise), _ptr(scores),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream)))


def fa_select_dims(scores, n_compressed: int) -> np.ndarray:
    """Host: uint8 mask [Hkv, 128] compressing the n_compressed lowest-score dims per KV head."""
    sc = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    Hkv = sc.shape[0]
    mask = np.zeros((Hkv, HEAD_DIM), dtype=np.uint8)
    _check(LIB.fa_select_dims(sc.ctypes.data, Hkv, int(n_compressed), mask.ctypes.data))
    return mask


def fa_device_status(stream=None) -> None:
    _check(LIB.fa_device_status(_stream(stream)))


def fa_watchdog_selftest(wait_ns: int = 20_000_000, stream=None) -> None:
    """Launch a kernel whose bounded wait must expire (see the C header)."""
    _check(LIB.fa_watchdog_selftest(wait_ns, _stream(stream)))


# ----------------------------------------------------------------------------- marshalling helpers

class Cache:
    """Device buffers of one layer's hybrid cache (allocated by torch) + the C struct.
    F and E are bf16, C is fp32 (see fa_plan in the header)."""

    def __init__(self, plan: fa_plan, device="cuda"):
        import torch
        bf = torch.bfloat16
        self.plan = plan
        self.F_K = torch.empty(max(plan.f_elems, 8), dtype=bf, device=device)
        self.F_V = torch.empty_like(self.F_K)
        self.E_K = torch.empty(max(plan.e_elems, 8), dtype=bf, device=device)
        self.E_V = torch.empty_like(self.E_K)
        self.C_K = torch.empty(max(plan.c_elems, 8), dtype=torch.float32, device=device)
        self.C_V = torch.empty_like(self.C_K)
        self.c = fa_cache(*(t.data_ptr() for t in (self.F_K, self.F_V, self.E_K, self.E_V,
                                                  self.C_K, self.C_V)))

    # views in the documented layouts (for tests and callers that inspect the cache)
    def F(self, which: str):
        """[B, Hkv, S + R, 128]: sink rows, then the recent ring (oldest at S + recent_head)."""
        p = self.plan
        t = self.F_K if which == "K" else self.F_V
        return t[:p.f_elems].view(p.shape.B, p.shape.Hkv, p.S + p.R, HEAD_DIM)

    def F_tokens(self, which: str):
        """[B, Hkv, S + R, 128]: the sink rows, then the recent rows in token order (the ring
        rotated so that its oldest row comes first). A copy, not a view."""
        import torch
        p = self.plan
        F = self.F(which)
        if p.R == 0 or p.recent_head == 0:
            return F.clone()
        idx = list(range(p.S)) + [p.S + (p.recent_head + a) % p.R for a in range(p.R)]
        return F[:, :, torch.tensor(idx, device=F.device)]

    def E(self, which: str, b: int, g: int):
        return self.E_raw(which, b, g)[:, :self.plan.de[g]]

    def C(self, which: str, b: int, g: int):
        p = self.plan
        t = self.C_K if which == "K" else self.C_V
        off = b * p.c_batch + p.c_off[g]
        return t[off:off + p.kk * p.dc_ld[g]].view(p.kk, p.dc_ld[g])[:, :p.dc[g]]

    def E_raw(self, which: str, b: int, g: int):
        """[M, de_ld] view of KV head (b, g)'s middle rows (strided when E is token-major)."""
        p = self.plan
        t = self.E_K if which == "K" else self.E_V
        off = b * p.e_batch + p.e_off[g]
        return t.as_strided((p.M, p.de_ld[g]), (p.e_pitch[g], 1), t.storage_offset() + off)

    def C_raw(self, which: str, b: int, g: int):
        p = self.plan
        t = self.C_K if which == "K" else self.C_V
        off = b * p.c_batch + p.c_off[g]
        return t[off:off + p.kk * p.dc_ld[g]].view(p.kk, p.dc_ld[g])


def basis_table(plan: fa_plan, device="cuda", stream=None):
    """Allocate and fill the bf16 basis table (period P) fa_compress reads (None if M == 0)."""
    import torch
    if plan.M == 0:
        return None
    phiT = torch.empty(plan.shape.k, plan.phi_ld, dtype=torch.bfloat16, device=device)
    fa_build_basis(plan.P, plan.shape.k, phiT, plan.phi_ld, normalized=False, stream=stream)
    return phiT


def perm_lists(plan: fa_plan, g: int):
    """(compressed dims, retained dims) of KV head g, as the plan derived them."""
    perm = np.frombuffer(bytes(plan.perm[g]), dtype=np.uint8).astype(np.int64)
    return perm[:plan.dc[g]], perm[plan.dc[g]:]
