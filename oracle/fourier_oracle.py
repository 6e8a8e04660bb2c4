"""fp64 CPU oracle for the Fourier-approximated KV cache (FourierAttention).

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously-correct statement of
what the hot path computes. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import it. The CUDA library never
calls it and shares no code, tables or helpers with it.

Sources (web pages, cited by title and section):

* [skill] agent-skills.jp, "Beyond homogeneous attention: memory-efficient LLMs via a
  Fourier-approximated KV cache" skill page -- "Core concept", "Architecture overview",
  Step 2 (``fourier_compress_kv_cache``), Step 3 (``selective_preserve_tokens``),
  Step 4 (``reconstruct_from_fourier``).
* [abstract] shd-paper.top summary of arXiv 2506.11886, "Beyond Homogeneous Attention:
  Memory-Efficient LLMs via Fourier-Approximated KV Cache" -- English abstract and
  "method details" ("projecting the long-context-insensitive dimensions onto orthogonal
  Fourier bases ... fixed-length spectral coefficients").

Readings of points the pages leave open (each is listed in the design notes):

* The basis is the real orthonormal Fourier basis over the middle span of M tokens,
  ordered [DC, cos_1, sin_1, cos_2, sin_2, ...]; ``k`` counts real basis functions.
  The skill page's Step 2 keeps the first k_b complex ``rfft`` bins, which spans the
  same space as the first 2*k_b - 1 real functions (tests pin this equality).
* For M even, frequency f = M/2 (Nyquist) has only a cosine, normalised by 1/sqrt(M).
  Every other cosine/sine has sqrt(2/M); DC has 1/sqrt(M). k must satisfy 1 <= k <= M.
* Only the masked (compressed) head dims of the middle span are projected; sink
  tokens [0, S), recent tokens [L-R, L) and the retained dims stay exact.
* When L <= S + R the middle is empty: the sink keeps min(S, L) tokens, the recent
  window keeps the remaining min(R, L - S) tokens, and every token is stored once.
* Decode: one query per sequence attends to all L cached tokens with softmax scale
  1/sqrt(D); query head h reads KV head h // (Hq / Hkv).
* Basis period. By default the basis period P equals the middle length M. A cache that
  takes appended tokens during decoding keeps a fixed period P >= M (its capacity):
  the middle tokens t < M are projected onto the period-P functions, which is the same
  as projecting the middle zero-padded to P tokens (pinned against a library FFT), and
  a token that leaves the recent window joins the middle at t = M. The pages say only
  that the spectral coefficients have a fixed length; they do not say how the cache is
  maintained while decoding.

* Dimension analysis ([skill] Step 1, ``analyze_head_dimensions``): each head dim d in
  turn gets 0.1 * N(0, 1) noise added to the VALUES of every token, and its sensitivity
  is the Frobenius norm of the change of the attention output. Scores are kept per KV
  head (the masks are per KV head), over all batch rows and the query heads of the group.
  The noise draws are an input. The dims with the lowest scores are the ones compressed.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
(closed forms, library FFT equality, orthonormality, Parseval, brute force).
"""
from __future__ import annotations

from dataclasses import dataclass
from functools import lru_cache

import numpy as np

__all__ = [
    "partition",
    "split_dims",
    "basis",
    "Hybrid",
    "compress",
    "reconstruct",
    "attention",
    "decode",
    "NOISE_SCALE",
    "dim_sensitivity",
    "select_dims",
]


def partition(L: int, S: int, R: int) -> tuple[int, int, int]:
    """Token partition of one sequence into sink / middle / recent.

    [skill] Step 3 (``selective_preserve_tokens``): the first ``preserve_initial`` and
    the last ``preserve_recent`` tokens stay uncompressed, the span between them is
    compressed, and nothing is compressed when the sequence is not longer than
    S + R. Returns (S_eff, R_eff, M) with S_eff + M + R_eff == L and each token in
    exactly one part.
    """
    if L < 0 or S < 0 or R < 0:
        raise ValueError("negative length")
    s_eff = min(S, L)
    r_eff = min(R, L - s_eff)
    m = L - s_eff - r_eff
    return s_eff, r_eff, m


def split_dims(mask_row) -> tuple[np.ndarray, np.ndarray]:
    """Compressed and retained head-dim index lists (both ascending) of one KV head.

    [abstract] and [skill] "Architecture overview": only the long-context-insensitive
    dims are Fourier-compressed; the others are kept in full. ``mask_row`` is a
    length-D array, nonzero = compressed.
    """
    m = np.asarray(mask_row).astype(bool)
    idx = np.arange(m.shape[0])
    return idx[m], idx[~m]


def _norm(f: np.ndarray, M: int) -> np.ndarray:
    """Orthonormal scale of frequency f over period M: 1/sqrt(M) for DC and Nyquist,
    else sqrt(2/M)."""
    single = (f == 0) | (2 * f == M)
    return np.where(single, 1.0 / np.sqrt(M), np.sqrt(2.0 / M))


@lru_cache(maxsize=2)
def _basis_full(P: int, k: int, M: int) -> np.ndarray:
    """Rows 0..M-1 of the period-P table, cached (read-only) so that one head's K, V and
    reconstruction share it; the values are those of ``basis``."""
    phi = basis(P, k, 0, M)
    phi.setflags(write=False)
    return phi


def basis(M: int, k: int, t0: int = 0, t1: int | None = None) -> np.ndarray:
    """Rows t0..t1-1 of Phi (M x k), Phi[t, j] = phi_j(t), in fp64; M is the period.

    [abstract]: "orthogonal Fourier bases"; [skill] "Architecture overview": a
    translation (shift) Fourier transform turns the span into k << L fixed-length
    spectral coefficients. Function j: j = 0 is the constant; for j >= 1 the frequency
    is f = (j + 1) // 2, odd j is the cosine and even j the sine of 2*pi*f*t/M.
    The phase f*t is reduced modulo M in exact integer arithmetic before the fp64
    cos/sin, so large M loses no accuracy. Rows past the period (t1 > M) are allowed;
    a cache with reserved room evaluates rows t < (its middle length) <= M.
    """
    if not (1 <= k <= M):
        raise ValueError(f"need 1 <= k <= M, got k={k}, M={M}")
    if t1 is None:
        t1 = M
    t = np.arange(t0, t1, dtype=np.int64)[:, None]
    j = np.arange(k, dtype=np.int64)[None, :]
    f = (j + 1) // 2
    r = (f * t) % M  # exact integer phase
    ang = (2.0 * np.pi / M) * r.astype(np.float64)
    is_sin = (j % 2 == 0) & (j > 0)
    vals = np.where(is_sin, np.sin(ang), np.cos(ang))
    return vals * _norm(f, M)


@dataclass
class Hybrid:
    """One KV head's hybrid cache (the dict of [skill] Step 3, made explicit).

    sink:   [S_eff, D]  tokens [0, S_eff), all dims, exact
    recent: [R_eff, D]  tokens [L - R_eff, L), all dims, exact
    E:      [M, De]     middle tokens, retained dims ``ed`` (ascending), exact
    C:      [k, Dc]     Fourier coefficients of the middle tokens' compressed dims ``cd``
    P:      basis period (P >= M; P == M unless room for appended tokens was reserved)
    """

    L: int
    D: int
    S: int
    R: int
    M: int
    k: int
    cd: np.ndarray
    ed: np.ndarray
    sink: np.ndarray
    recent: np.ndarray
    E: np.ndarray
    C: np.ndarray
    P: int = 0


def compress(X, mask_row, S: int, R: int, k: int, period: int | None = None) -> Hybrid:
    """Compress one KV head's cache X [L, D] into its hybrid form.

    [skill] Step 3 splits the tokens, Step 2 projects the middle span onto the basis
    (``fourier_compress_kv_cache``); [abstract] restricts the projection to the
    long-context-insensitive dims. C = Phi^T X[S:L-R, cd] (fp64 BLAS), with Phi the
    first M rows of the period-P basis (``period``; default P = M, and P >= M).
    A cache that had tokens appended while decoding is, by this reading, the cache of
    the longer sequence with the period it was created with.
    """
    X = np.asarray(X, dtype=np.float64)
    L, D = X.shape
    s_eff, r_eff, M = partition(L, S, R)
    P = M if period is None else int(period)
    if M > 0 and P < M:
        raise ValueError(f"period P={P} is shorter than the middle span M={M}")
    cd, ed = split_dims(mask_row)
    mid = X[s_eff:L - r_eff]
    if M > 0 and cd.size > 0:
        phi = _basis_full(P, k, M)
        C = phi.T @ mid[:, cd]
    else:
        C = np.zeros((k if M > 0 else 0, cd.size))
    return Hybrid(L=L, D=D, S=s_eff, R=r_eff, M=M, k=k, cd=cd, ed=ed,
                  sink=X[:s_eff].copy(), recent=X[L - r_eff:].copy(),
                  E=mid[:, ed].copy(), C=C, P=P)


def reconstruct(h: Hybrid) -> np.ndarray:
    """Approximate cache X~ [L, D]: X^ = Phi C on the compressed dims of the middle.

    [skill] Step 4 (``reconstruct_from_fourier``): zero-filled spectrum, inverse
    transform to the original length. Here written as the basis expansion Phi @ C,
    which equals that truncated inverse real FFT (pinned in the tests). With a period
    P > M the expansion is evaluated on the first M rows of the period-P basis.
    """
    Xt = np.zeros((h.L, h.D))
    Xt[:h.S] = h.sink
    Xt[h.L - h.R:] = h.recent
    if h.M > 0:
        mid = np.zeros((h.M, h.D))
        mid[:, h.ed] = h.E
        if h.cd.size > 0:
            mid[:, h.cd] = _basis_full(h.P or h.M, h.k, h.M) @ h.C
        Xt[h.S:h.S + h.M] = mid
    return Xt


def attention(q, K, V, scale: float) -> np.ndarray:
    """Naive softmax attention of query rows q [G, D] over K, V [L, D] (fp64)."""
    q = np.asarray(q, dtype=np.float64)
    s = scale * (q @ np.asarray(K, dtype=np.float64).T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.asarray(V, dtype=np.float64)


def decode(q, hk: Hybrid, hv: Hybrid, scale: float | None = None) -> np.ndarray:
    """One decode step of the G query heads that share one KV head.

    Reconstructs K~ and V~ explicitly ([skill] Step 4, "restore during decoding") and
    runs plain softmax attention over all L tokens. q is [G, D]; returns [G, D].
    """
    D = hk.D
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    return attention(q, reconstruct(hk), reconstruct(hv), scale)


NOISE_SCALE = 0.1


def dim_sensitivity(q, K, V, noise, scale: float | None = None) -> np.ndarray:
    """Sensitivity score of every head dim of one KV head ([skill] Step 1).

    q [B, G, D] (the query heads of the group in every batch row), K, V, noise [B, L, D].
    For each dim d, as the page's loop does: the unperturbed output, the output with
    V[:, :, d] += NOISE_SCALE * noise[:, :, d], and the norm of their difference over
    every batch row, query head and dim. Returns [D] (fp64).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    noise = np.asarray(noise, dtype=np.float64)
    B, _, D = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    base = np.stack([attention(q[b], K[b], V[b], scale) for b in range(B)])
    out = np.empty(D)
    for d in range(D):
        Vn = V.copy()
        Vn[:, :, d] += NOISE_SCALE * noise[:, :, d]
        noisy = np.stack([attention(q[b], K[b], Vn[b], scale) for b in range(B)])
        out[d] = np.linalg.norm(base - noisy)
    return out


def select_dims(scores, n_compressed: int) -> np.ndarray:
    """Mask row of one KV head: the n_compressed dims with the lowest sensitivity are
    compressed (1), the rest retained (0) ([skill] Step 1: low-sensitivity dims are the
    compression candidates). Equal scores are ranked by dim index (stable order)."""
    scores = np.asarray(scores, dtype=np.float64)
    if not 0 <= n_compressed <= scores.size:
        raise ValueError("n_compressed out of range")
    order = np.argsort(scores, kind="stable")
    mask = np.zeros(scores.size, dtype=np.uint8)
    mask[order[:n_compressed]] = 1
    return mask
