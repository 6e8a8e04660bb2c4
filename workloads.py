"""Seeded synthetic workloads: the five cache shapes and their input generators.

Shared by the tests, ``bench.py`` and ``__graft_entry__.smoke()``. This module holds
no Fourier-attention arithmetic: it only draws caches, queries and dim masks. The
caches stand in for LLaMA KV caches on long-context tasks (LongBench, NIAH), which
are not available here; the shapes follow the LLaMA attention layouts named below.

Generators (per batch b, KV head g, head dim d, and K / V separately):

* ``sinusoid``: sum of 4 sinusoids over the token index t, period ~ U[64, 2048]
  tokens, amplitude ~ N(0, 1), phase ~ U[0, 2 pi); plus ``noise`` * N(0, 1).
* ``trend``: the sinusoid mix, plus a rank-4 smooth trend (4 stationary AR(1) series
  with rho = 0.999 and unit variance, mixed into the D dims by a N(0, 1/4) D x 4
  matrix), plus 0.05 * N(0, 1).

Queries are N(0, 1). Everything is drawn in fp32 with torch generators seeded from
the workload seed and rounded to bf16 once. Tensors can be drawn directly on a CUDA
device (large shapes) or on the CPU (oracle-sized shapes); the two devices give
different streams, so parity tests copy device inputs back to the host.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch

D = 128


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    S: int
    R: int
    k: int
    mask: str          # "low96" | "rand96" | "rand64or96" | "none" | "all"
    gen: str           # "sinusoid" | "trend"
    noise: float = 0.1
    seed: int = 0
    layers: int = 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


# The five cache shapes of the hot path.
SINGLE_HEAD_2K = Workload("single_head_L2048_k63", B=1, Hq=4, Hkv=1, L=2048, S=32, R=64,
                          k=63, mask="low96", gen="sinusoid", noise=0.1, seed=0)
LLAMA2_7B_MHA_32K = Workload("llama2_7b_mha_b8_L32768_k255", B=8, Hq=32, Hkv=32, L=32768,
                             S=32, R=64, k=255, mask="rand96", gen="sinusoid", seed=1)
LLAMA3_8B_GQA_32K = Workload("llama3_8b_gqa_b16_L32768_k511", B=16, Hq=32, Hkv=8, L=32768,
                             S=32, R=1024, k=511, mask="rand64or96", gen="trend",
                             noise=0.05, seed=2)
LLAMA3_8B_GQA_128K = Workload("llama3_8b_gqa_b4_L131072_k1023", B=4, Hq=32, Hkv=8,
                              L=131072, S=32, R=2048, k=1023, mask="rand96",
                              gen="sinusoid", seed=3)
CONFIGS = [SINGLE_HEAD_2K, LLAMA2_7B_MHA_32K, LLAMA3_8B_GQA_32K, LLAMA3_8B_GQA_128K]

# Full 32-layer LLaMA-3-8B-shaped cache: decode sweep over batch x context length.
SWEEP_BATCH = (1, 8, 32, 64)
SWEEP_L = (8192, 32768, 131072)


def llama3_8b_layer(B: int, L: int, layer: int) -> Workload:
    """One layer of the 32-layer sweep: k = L/128 - 1 (odd), 75% of dims compressed."""
    return Workload(f"llama3_8b_layer{layer}_b{B}_L{L}_k{L // 128 - 1}", B=B, Hq=32, Hkv=8,
                    L=L, S=32, R=1024, k=L // 128 - 1, mask="rand96", gen="sinusoid",
                    seed=layer, layers=32)


def shrink(w: Workload, **kw) -> Workload:
    """Same generator and mask recipe at other sizes (for oracle-sized parity cases)."""
    return replace(w, **kw)


def dim_mask(w: Workload) -> np.ndarray:
    """uint8 [Hkv, D] mask, 1 = compressed dim, from numpy PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(1_000_003 + w.seed))
    m = np.zeros((w.Hkv, D), dtype=np.uint8)
    for g in range(w.Hkv):
        if w.mask == "low96":
            m[g, :96] = 1
        elif w.mask == "rand96":
            m[g, np.sort(rng.permutation(D)[:96])] = 1
        elif w.mask == "rand64or96":
            dc = 64 if rng.random() < 0.5 else 96
            m[g, np.sort(rng.permutation(D)[:dc])] = 1
        elif w.mask == "none":
            pass
        elif w.mask == "all":
            m[g, :] = 1
        else:
            raise ValueError(w.mask)
    return m


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _sinusoids(shape_bg, L, gen, device, chunk_t=8192):
    """[BH, L, D] fp32: per (head, dim) a sum of 4 sinusoids of the token index."""
    BH = shape_bg
    period = 64.0 + (2048.0 - 64.0) * torch.rand(BH, 1, D, 4, generator=gen, device=device)
    amp = torch.randn(BH, 1, D, 4, generator=gen, device=device)
    phase = 2.0 * np.pi * torch.rand(BH, 1, D, 4, generator=gen, device=device)
    out = torch.empty(BH, L, D, dtype=torch.float32, device=device)
    omega = (2.0 * np.pi) / period
    for t0 in range(0, L, chunk_t):
        t1 = min(L, t0 + chunk_t)
        t = torch.arange(t0, t1, device=device, dtype=torch.float32).view(1, -1, 1, 1)
        out[:, t0:t1] = (amp * torch.sin(omega * t + phase)).sum(-1)
    return out


def _ar1_trend(BH, L, gen, device, rho=0.999, rank=4, block=256):
    """[BH, L, rank] stationary AR(1) series (unit variance), via a blocked scan."""
    c = float(np.sqrt(1.0 - rho * rho))
    nb = (L + block - 1) // block
    eps = c * torch.randn(BH, rank, nb * block, generator=gen, device=device)
    z_prev = torch.randn(BH, rank, generator=gen, device=device)
    i = torch.arange(block, device=device, dtype=torch.float64)
    lag = (i[:, None] - i[None, :])
    T = torch.where(lag >= 0, torch.tensor(rho, dtype=torch.float64, device=device) ** lag.clamp(min=0),
                    torch.zeros((), dtype=torch.float64, device=device)).float()
    local = eps.view(BH, rank, nb, block) @ T.t()             # within-block partial sums
    decay = (rho ** (i + 1)).float()                             # rho^(i+1)
    z = torch.empty_like(local)
    for b in range(nb):
        z[:, :, b] = local[:, :, b] + decay * z_prev[..., None]
        z_prev = z[:, :, b, -1]
    return z.view(BH, rank, nb * block)[:, :, :L].transpose(1, 2)


def kv_cache(w: Workload, which: str, device="cpu", b_range=None) -> torch.Tensor:
    """bf16 [B, Hkv, L, D] K or V cache of workload ``w``, drawn on ``device``.

    ``b_range`` = (b0, b1) draws only those batch rows (same values as the full draw
    is NOT guaranteed; use it for memory-bounded generation of big caches).
    """
    assert which in ("K", "V")
    b0, b1 = b_range if b_range is not None else (0, w.B)
    out = torch.empty(b1 - b0, w.Hkv, w.L, D, dtype=torch.bfloat16, device=device)
    for b in range(b0, b1):
        seed = (w.seed * 1_000_003 + (0 if which == "K" else 500_009) + 7919 * b) & 0x7FFFFFFF
        gen = _gen(device, seed)
        x = _sinusoids(w.Hkv, w.L, gen, device)
        if w.gen == "trend":
            z = _ar1_trend(w.Hkv, w.L, gen, device)                    # [Hkv, L, 4]
            mix = 0.5 * torch.randn(w.Hkv, 4, D, generator=gen, device=device)
            x += z @ mix
            x += 0.05 * torch.randn(x.shape, generator=gen, device=device)
        else:
            x += w.noise * torch.randn(x.shape, generator=gen, device=device)
        out[b - b0] = x.to(torch.bfloat16)
        del x
    return out


def queries(w: Workload, device="cpu") -> torch.Tensor:
    """bf16 [B, Hq, D] decode queries, N(0, 1)."""
    gen = _gen(device, (w.seed * 1_000_003 + 424_242) & 0x7FFFFFFF)
    return torch.randn(w.B, w.Hq, D, generator=gen, device=device).to(torch.bfloat16)


def value_noise(w: Workload, device="cpu") -> torch.Tensor:
    """bf16 [B, Hkv, L, D] N(0, 1) draws: the noise of the head-dimension analysis."""
    gen = _gen(device, (w.seed * 1_000_003 + 777_767) & 0x7FFFFFFF)
    return torch.randn(w.B, w.Hkv, w.L, D, generator=gen, device=device).to(torch.bfloat16)


# ----------------------------------------------------------------------------- counter-based draws

_SM64_GAMMA = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1


def splitmix64(seed: int, n: int) -> np.ndarray:
    """The first n outputs (uint64) of SplitMix64 started at state ``seed`` (Steele, Lea
    and Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014, in the
    64-bit finaliser form Vigna distributes as splitmix64.c): output i mixes the state
    seed + (i + 1) * gamma. Counter-based, so a C program reproduces the same stream
    from the same published definition without sharing code with this module."""
    i = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & _M64) + i * np.uint64(_SM64_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def grid_values(seed: int, n: int) -> np.ndarray:
    """n values on the grid {-128, ..., 127} / 64 (exact in bf16), from the top byte of
    each SplitMix64 output read as a signed 8-bit integer."""
    top = (splitmix64(seed, n) >> np.uint64(56)).astype(np.int64)
    return np.where(top >= 128, top - 256, top).astype(np.float64) / 64.0
