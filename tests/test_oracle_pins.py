"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each check compares the oracle with something it does not compute: hand-derived
values (tests/golden/hand_cases.txt), a library FFT (numpy.fft.rfft / irfft), closed
forms (orthonormality, Parseval, exact reconstruction at k = M, lossless integer
frequencies) and brute force on tiny inputs. The mutation tests at the end plant
plausible mistakes in copies of the oracle's basis and check that a pin catches each.
"""
import itertools

import numpy as np
import pytest
import torch

from oracle import fourier_oracle as fo

TOL = 1e-12


# ----------------------------------------------------------------------------- checks
# Written as functions of a basis generator so the mutation tests can reuse them.

def check_orthonormal(basis_fn, M, k):
    phi = basis_fn(M, k)
    return np.abs(phi.T @ phi - np.eye(k)).max()


def check_rfft_bins(basis_fn, M, k, rng):
    """C = Phi^T x against numpy's rfft R: C0 = R0/sqrt(M), C_{2f-1} = sqrt(2/M) Re R_f,
    C_{2f} = -sqrt(2/M) Im R_f (Nyquist: C = R_{M/2}/sqrt(M))."""
    x = rng.standard_normal(M)
    C = basis_fn(M, k).T @ x
    R = np.fft.rfft(x)
    ref = np.empty(k)
    for j in range(k):
        f = (j + 1) // 2
        if j == 0:
            ref[j] = R[0].real / np.sqrt(M)
        elif 2 * f == M:
            ref[j] = R[f].real / np.sqrt(M)
        elif j % 2 == 1:
            ref[j] = np.sqrt(2.0 / M) * R[f].real
        else:
            ref[j] = -np.sqrt(2.0 / M) * R[f].imag
    return np.abs(C - ref).max() / max(1.0, np.abs(ref).max())


def check_truncated_irfft(basis_fn, M, kb, rng):
    """Skill page Step 4: keep the first kb rfft bins, zero the rest, irfft(n=M).
    Must equal Phi Phi^T x with k = 2 kb - 1 real functions (kb < M/2)."""
    x = rng.standard_normal(M)
    R = np.fft.rfft(x)
    R[kb:] = 0
    ref = np.fft.irfft(R, n=M)
    phi = basis_fn(M, 2 * kb - 1)
    return np.abs(phi @ (phi.T @ x) - ref).max()


def check_period_rfft(basis_fn, P, M, k, rng):
    """Rows t < M of the period-P basis against numpy's rfft of the M samples zero-padded
    to P (n=P): the same bin relations as check_rfft_bins, with P in place of M."""
    x = rng.standard_normal(M)
    C = basis_fn(P, k, 0, M).T @ x
    R = np.fft.rfft(np.concatenate([x, np.zeros(P - M)]), n=P)
    ref = np.empty(k)
    for j in range(k):
        f = (j + 1) // 2
        if j == 0:
            ref[j] = R[0].real / np.sqrt(P)
        elif 2 * f == P:
            ref[j] = R[f].real / np.sqrt(P)
        elif j % 2 == 1:
            ref[j] = np.sqrt(2.0 / P) * R[f].real
        else:
            ref[j] = -np.sqrt(2.0 / P) * R[f].imag
    return np.abs(C - ref).max() / max(1.0, np.abs(ref).max())


# ----------------------------------------------------------------------------- partition

def test_partition_brute_force():
    for L, S, R in itertools.product(range(0, 12), range(0, 6), range(0, 6)):
        s, r, m = fo.partition(L, S, R)
        assert s + m + r == L and min(s, r, m) >= 0
        # brute force: label every token, each exactly once
        labels = ["sink" if t < s else ("recent" if t >= L - r else "mid") for t in range(L)]
        if L > S + R:  # the skill page compresses only when the sequence is longer than S+R
            assert (s, r, m) == (S, R, L - S - R)
            assert labels.count("mid") == L - S - R
        else:
            assert m == 0 and s == min(S, L)


def test_split_dims_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(50):
        mask = (rng.random(128) < rng.random()).astype(np.uint8)
        cd, ed = fo.split_dims(mask)
        assert list(cd) == [d for d in range(128) if mask[d]]
        assert list(ed) == [d for d in range(128) if not mask[d]]


# ----------------------------------------------------------------------------- basis

def test_basis_hand_values(hand_cases):
    for M in (4, 3):
        phi = fo.basis(M, M)
        for j in range(M):
            ref = np.array(hand_cases[f"basis_M{M}_j{j}"])
            assert np.abs(phi[:, j] - ref).max() < 1e-15


@pytest.mark.parametrize("M,k", [(1, 1), (2, 2), (3, 3), (4, 4), (7, 5), (8, 8), (8, 7),
                                 (64, 63), (127, 127), (128, 128), (1952, 63), (4099, 1023),
                                 (32672, 255)])
def test_basis_orthonormal(M, k):
    assert check_orthonormal(fo.basis, M, k) < TOL


def test_basis_orthonormal_large_M_compensated():
    """M = 128992 (the 128K-context middle span): Gram entries by exact fsum."""
    import math
    M, k = 128992, 1023
    rows = fo.basis(M, 8, 0, M)        # first 8 functions, all tokens
    last = fo.basis(M, k, 0, M)[:, -4:]  # and the last 4 (highest frequency)
    cols = np.concatenate([rows, last], axis=1)
    for a in range(cols.shape[1]):
        for b in range(a, cols.shape[1]):
            g = math.fsum(cols[:, a] * cols[:, b])
            assert abs(g - (1.0 if a == b else 0.0)) < TOL


def test_basis_chunk_rows_match():
    M, k = 1000, 31
    full = fo.basis(M, k)
    part = fo.basis(M, k, 300, 700)
    assert np.array_equal(full[300:700], part)


def test_basis_rejects_bad_k():
    with pytest.raises(ValueError):
        fo.basis(4, 5)
    with pytest.raises(ValueError):
        fo.basis(4, 0)


@pytest.mark.parametrize("M,k", [(16, 16), (17, 17), (16, 9), (1952, 63), (2047, 255),
                                 (4096, 4096)])
def test_rfft_bins(M, k):
    assert check_rfft_bins(fo.basis, M, k, np.random.default_rng(M + k)) < TOL


@pytest.mark.parametrize("M,kb", [(16, 3), (17, 8), (1952, 32), (2048, 128)])
def test_truncated_irfft_equals_projection(M, kb):
    assert check_truncated_irfft(fo.basis, M, kb, np.random.default_rng(M)) < TOL


# ----------------------------------------------------------------------------- compress

def test_compress_hand_example(hand_cases):
    x = np.array(hand_cases["compress_x"])[:, None]
    mask = np.ones(1)
    h4 = fo.compress(x, mask, 0, 0, 4)
    assert np.abs(h4.C[:, 0] - hand_cases["compress_C_k4"]).max() < 1e-15
    assert np.abs(fo.reconstruct(h4)[:, 0] - hand_cases["recon_k4"]).max() < 1e-14
    h3 = fo.compress(x, mask, 0, 0, 3)
    assert np.abs(fo.reconstruct(h3)[:, 0] - hand_cases["recon_k3"]).max() < 1e-14


@pytest.mark.parametrize("M", [1, 2, 5, 64, 127, 128, 255])
def test_k_equals_M_reconstructs_exactly(M):
    rng = np.random.default_rng(M)
    S, R, D = 3, 2, 128
    X = rng.standard_normal((S + M + R, D))
    mask = (rng.random(D) < 0.75).astype(np.uint8)
    h = fo.compress(X, mask, S, R, M)
    assert np.abs(fo.reconstruct(h) - X).max() < TOL * max(1.0, np.abs(X).max()) * 10


@pytest.mark.parametrize("M,k", [(500, 63), (1952, 63), (1000, 1000), (999, 2)])
def test_parseval(M, k):
    rng = np.random.default_rng(k)
    X = rng.standard_normal((M, 128))
    h = fo.compress(X, np.ones(128), 0, 0, k)
    resid = X - fo.reconstruct(h)
    lhs = (X ** 2).sum(0)
    rhs = (h.C ** 2).sum(0) + (resid ** 2).sum(0)
    assert np.abs(lhs - rhs).max() / lhs.max() < TOL


def test_lossless_integer_frequencies():
    """A sum of cosines with integer frequency f <= floor(k/2) lies in the span."""
    M, k = 1952, 63
    rng = np.random.default_rng(1)
    t = np.arange(M)
    X = np.zeros((M, 4))
    for col in range(4):
        for f in rng.integers(0, k // 2 + 1, size=3):
            X[:, col] += rng.standard_normal() * np.cos(2 * np.pi * f * t / M + rng.uniform(0, 2 * np.pi))
    h = fo.compress(X, np.ones(4), 0, 0, k)
    assert np.abs(fo.reconstruct(h) - X).max() < 1e-11


def test_sink_recent_retained_are_exact_copies():
    rng = np.random.default_rng(2)
    L, S, R, D = 300, 32, 64, 128
    X = rng.standard_normal((L, D))
    mask = (rng.random(D) < 0.75).astype(np.uint8)
    h = fo.compress(X, mask, S, R, 31)
    Xt = fo.reconstruct(h)
    cd, ed = fo.split_dims(mask)
    assert np.array_equal(Xt[:S], X[:S]) and np.array_equal(Xt[L - R:], X[L - R:])
    assert np.array_equal(Xt[S:L - R][:, ed], X[S:L - R][:, ed])
    assert np.array_equal(h.E, X[S:L - R][:, ed])
    # compressed dims changed (k < M), so the projection really ran on them
    assert np.abs(Xt[S:L - R][:, cd] - X[S:L - R][:, cd]).max() > 1e-3


@pytest.mark.parametrize("P,M,k", [(700, 500, 63), (701, 300, 255), (1024, 1023, 1024),
                                   (64, 1, 64), (4099, 4000, 255)])
def test_period_rows_equal_zero_padded_rfft(P, M, k):
    """A cache with reserved room projects its M middle tokens onto the period-P basis:
    that is the rfft of the middle zero-padded to P samples."""
    assert check_period_rfft(fo.basis, P, M, k, np.random.default_rng(P + M)) < TOL


@pytest.mark.parametrize("P,M", [(40, 31), (64, 63), (129, 100)])
def test_period_full_basis_reconstructs_exactly(P, M):
    """k = P functions of period P are a complete orthonormal basis of P samples, so the
    zero-padded middle, and with it every middle token, is reconstructed exactly."""
    rng = np.random.default_rng(P)
    S, R, D = 4, 3, 128
    X = rng.standard_normal((S + M + R, D))
    mask = (rng.random(D) < 0.75).astype(np.uint8)
    h = fo.compress(X, mask, S, R, P, period=P)
    assert h.P == P and h.M == M
    assert np.abs(fo.reconstruct(h) - X).max() < 1e-12
    q = rng.standard_normal((2, D))
    hv = fo.compress(X[::-1].copy(), mask, S, R, P, period=P)
    ref = fo.attention(q, X, X[::-1], 1 / np.sqrt(D))
    assert np.abs(fo.decode(q, h, hv) - ref).max() < 1e-12


def test_period_default_is_the_middle_length():
    rng = np.random.default_rng(9)
    X = rng.standard_normal((300, 128))
    mask = (rng.random(128) < 0.75).astype(np.uint8)
    a = fo.compress(X, mask, 16, 32, 31)
    b = fo.compress(X, mask, 16, 32, 31, period=a.M)
    assert a.P == a.M == 252 and np.array_equal(a.C, b.C)
    with pytest.raises(ValueError):
        fo.compress(X, mask, 16, 32, 31, period=a.M - 1)


# ----------------------------------------------------------------------------- attention

def test_attention_hand_case(hand_cases):
    q = np.array([hand_cases["attn_q"]])
    K = np.array([hand_cases["attn_K0"], hand_cases["attn_K1"]])
    V = np.array([hand_cases["attn_V0"], hand_cases["attn_V1"]])
    out = fo.attention(q, K, V, 1.0)
    assert np.abs(out[0] - hand_cases["attn_out"]).max() < 1e-14


def test_attention_matches_torch_softmax():
    rng = np.random.default_rng(3)
    q, K, V = rng.standard_normal((4, 128)), rng.standard_normal((200, 128)), rng.standard_normal((200, 128))
    sc = 1 / np.sqrt(128)
    p = torch.softmax(torch.from_numpy(q) @ torch.from_numpy(K).T * sc, dim=-1)
    ref = (p @ torch.from_numpy(V)).numpy()
    assert np.abs(fo.attention(q, K, V, sc) - ref).max() < 1e-13


@pytest.mark.parametrize("case", ["no_dims", "no_middle"])
def test_nothing_compressed_is_plain_attention(case):
    rng = np.random.default_rng(4)
    L, D = 400, 128
    K, V, q = rng.standard_normal((L, D)), rng.standard_normal((L, D)), rng.standard_normal((4, D))
    if case == "no_dims":
        mask, S, R = np.zeros(D), 32, 64
    else:
        mask, S, R = np.ones(D), 300, 200
    hk, hv = fo.compress(K, mask, S, R, 15), fo.compress(V, mask, S, R, 15)
    ref = fo.attention(q, K, V, 1 / np.sqrt(D))
    assert np.abs(fo.decode(q, hk, hv) - ref).max() < 1e-13


def test_coefficient_domain_identity():
    """Scores and values in the coefficient domain equal those on the reconstruction:
    q . X^_t = q_e . E_t + (Phi (C_K q_c))_t and p^T X^ = (Phi^T p)^T C_V."""
    rng = np.random.default_rng(6)
    L, S, R, D, k = 700, 32, 64, 128, 63
    mask = (rng.random(D) < 0.75).astype(np.uint8)
    K, V, q = rng.standard_normal((L, D)), rng.standard_normal((L, D)), rng.standard_normal(D)
    hk, hv = fo.compress(K, mask, S, R, k), fo.compress(V, mask, S, R, k)
    Kt, Vt = fo.reconstruct(hk), fo.reconstruct(hv)
    phi = fo.basis(hk.M, k)
    cd, ed = hk.cd, hk.ed
    s_ref = Kt[S:L - R] @ q
    s_coef = hk.E @ q[ed] + phi @ (hk.C @ q[cd])
    assert np.abs(s_ref - s_coef).max() < 1e-11
    p = rng.random(hk.M)
    v_ref = p @ Vt[S:L - R]
    assert np.abs(v_ref[cd] - (phi.T @ p) @ hv.C).max() < 1e-11
    assert np.abs(v_ref[ed] - p @ hv.E).max() < 1e-11


def test_gqa_head_grouping_matches_per_head_loop():
    rng = np.random.default_rng(7)
    L, D, G = 300, 128, 4
    K, V = rng.standard_normal((L, D)), rng.standard_normal((L, D))
    q = rng.standard_normal((G, D))
    mask = (rng.random(D) < 0.5).astype(np.uint8)
    hk, hv = fo.compress(K, mask, 8, 16, 41), fo.compress(V, mask, 8, 16, 41)
    joint = fo.decode(q, hk, hv)
    for h in range(G):
        assert np.abs(joint[h] - fo.decode(q[h:h + 1], hk, hv)[0]).max() < 1e-14


# ----------------------------------------------------------------------------- mutations
# Each mutant is a plausible slip in writing the basis; some pin above must reject it.

def _mutant(kind):
    def fn(M, k, t0=0, t1=None):
        phi = fo.basis(M, k, t0, t1).copy()
        t = np.arange(t0, M if t1 is None else t1)
        if kind == "sin_sign" and k > 2:
            phi[:, 2] *= -1
        elif kind == "swap_cos_sin" and k > 2:
            phi[:, [1, 2]] = phi[:, [2, 1]]
        elif kind == "norm_dc_like" and k > 1:
            phi[:, 1] *= np.sqrt(0.5)
        elif kind == "freq_off_by_one" and k > 1:
            phi[:, 1] = np.sqrt(2.0 / M) * np.cos(2 * np.pi * 2 * t / M)
        elif kind == "angle_no_reduce":      # phase computed in fp32 without reduction
            f = (np.arange(k) + 1) // 2
            ang = (np.float32(2 * np.pi / M) * (f[None, :] * t[:, None]).astype(np.float32)).astype(np.float64)
            base = np.where((np.arange(k) % 2 == 0) & (np.arange(k) > 0), np.sin(ang), np.cos(ang))
            phi = base * np.where((f == 0) | (2 * f == M), 1 / np.sqrt(M), np.sqrt(2.0 / M))
        return phi
    return fn


def _period_mutant(kind):
    """Slips in handling a period P longer than the M rows evaluated."""
    def fn(P, k, t0=0, t1=None):
        M = P if t1 is None else t1
        if kind == "period_is_rows":        # the row count used as the period
            return fo.basis(M, k, t0, t1)
        if kind == "norm_over_rows":        # right functions, scale of the M-row span
            return fo.basis(P, k, t0, t1) * np.sqrt(P / M)
        raise ValueError(kind)
    return fn


@pytest.mark.parametrize("kind", ["period_is_rows", "norm_over_rows"])
def test_period_pins_reject_planted_mistakes(kind):
    assert check_period_rfft(_period_mutant(kind), 700, 500, 63, np.random.default_rng(1)) > TOL


@pytest.mark.parametrize("kind", ["sin_sign", "swap_cos_sin", "norm_dc_like", "freq_off_by_one",
                                  "angle_no_reduce"])
def test_pins_reject_planted_mistakes(kind):
    fn = _mutant(kind)
    rng = np.random.default_rng(0)
    caught = (check_orthonormal(fn, 4099, 255) > TOL
              or check_rfft_bins(fn, 4099, 255, rng) > TOL
              or check_truncated_irfft(fn, 4099, 100, rng) > TOL)
    assert caught, kind


# ----------------------------------------------------------------------------- dim analysis

def _sens_case(seed, B=2, G=3, L=50, D=128):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, G, D)), rng.standard_normal((B, L, D)),
            rng.standard_normal((B, L, D)), rng.standard_normal((B, L, D)))


def test_sensitivity_equals_weighted_noise_closed_form():
    """Only V changes, so by linearity the output change of dim d is 0.1 * P n_d with P the
    (unchanged) softmax weights: written here with torch's softmax, not the oracle's."""
    q, K, V, n = _sens_case(1)
    s = fo.dim_sensitivity(q, K, V, n)
    qt, Kt, nt = (torch.from_numpy(x) for x in (q, K, n))
    P = torch.softmax(qt @ Kt.transpose(1, 2) / np.sqrt(128), dim=-1)     # [B, G, L]
    ref = 0.1 * torch.linalg.vector_norm(P @ nt, dim=(0, 1)).numpy()      # [D]
    assert np.abs(s - ref).max() < 1e-12 * ref.max()


def test_sensitivity_hand_case():
    """One token: softmax weight 1, so the change is exactly 0.1 * noise of that token."""
    q, K, V, n = _sens_case(2, B=1, G=2, L=1)
    s = fo.dim_sensitivity(q, K, V, n)
    assert np.abs(s - 0.1 * np.sqrt(2) * np.abs(n[0, 0])).max() < 1e-15


def test_sensitivity_ignores_values_and_zero_noise():
    q, K, V, n = _sens_case(3)
    a = fo.dim_sensitivity(q, K, V, n)
    assert np.abs(a - fo.dim_sensitivity(q, K, 5 * V + 3, n)).max() < 1e-12 * a.max()
    n[:, :, 7] = 0
    assert fo.dim_sensitivity(q, K, V, n)[7] < 1e-15


def test_select_dims_brute_force():
    rng = np.random.default_rng(4)
    for _ in range(50):
        sc = rng.integers(0, 6, size=12).astype(float)       # many ties
        nc = int(rng.integers(0, 13))
        m = fo.select_dims(sc, nc)
        assert m.sum() == nc
        # every compressed dim ranks below every retained one in (score, index) order
        key = [(sc[i], i) for i in range(12)]
        if 0 < nc < 12:
            assert max(key[i] for i in range(12) if m[i]) < min(key[i] for i in range(12) if not m[i])


def test_sensitivity_pin_rejects_planted_mistakes():
    q, K, V, n = _sens_case(5)
    qt, Kt, nt = (torch.from_numpy(x) for x in (q, K, n))
    P = torch.softmax(qt @ Kt.transpose(1, 2) / np.sqrt(128), dim=-1)
    ref = 0.1 * torch.linalg.vector_norm(P @ nt, dim=(0, 1)).numpy()
    good = fo.dim_sensitivity(q, K, V, n)
    # perturbing the keys instead, or dropping the 0.1 scale, is caught by the closed form
    keys = np.empty(128)
    base = np.stack([fo.attention(q[b], K[b], V[b], 1 / np.sqrt(128)) for b in range(2)])
    for d in range(128):
        Kn = K.copy()
        Kn[:, :, d] += 0.1 * n[:, :, d]
        keys[d] = np.linalg.norm(base - np.stack([fo.attention(q[b], Kn[b], V[b], 1 / np.sqrt(128))
                                                  for b in range(2)]))
    for wrong in (keys, good / 0.1):
        assert np.abs(wrong - ref).max() > 1e-6 * ref.max()


# ----------------------------------------------------------------------------- properties

from hypothesis import given, settings, strategies as st


@settings(max_examples=40, deadline=None)
@given(M=st.integers(1, 300), extra=st.integers(0, 200), kfrac=st.floats(0.0, 1.0),
       seed=st.integers(0, 2 ** 31 - 1))
def test_period_projection_bessel_and_linearity(M, extra, kfrac, seed):
    """For any period P >= M and k <= P the coefficients are an orthogonal projection of the
    middle zero-padded to P samples: Bessel's inequality holds (equality at k = P), and the
    map is linear."""
    P = M + extra
    k = max(1, min(P, int(round(kfrac * P))))
    rng = np.random.default_rng(seed)
    x, y = rng.standard_normal((M, 3)), rng.standard_normal((M, 3))
    mask = np.ones(3)
    cx = fo.compress(x, mask, 0, 0, k, period=P).C
    cy = fo.compress(y, mask, 0, 0, k, period=P).C
    energy = (x ** 2).sum(0)
    assert np.all((cx ** 2).sum(0) <= energy * (1 + 1e-12))
    if k == P:
        assert np.allclose((cx ** 2).sum(0), energy, rtol=1e-10)
    a, b = rng.standard_normal(2)
    cxy = fo.compress(a * x + b * y, mask, 0, 0, k, period=P).C
    assert np.abs(cxy - (a * cx + b * cy)).max() <= 1e-10 * max(1.0, np.abs(cxy).max())


def test_period_hand_example(hand_cases):
    """A middle of 2 tokens under period 4, then one appended token (hand-derived values)."""
    x = np.array(hand_cases["period4_x"])[:, None]
    h = fo.compress(x, np.ones(1), 0, 0, 4, period=4)
    assert h.P == 4 and h.M == 2
    assert np.abs(h.C[:, 0] - hand_cases["period4_C"]).max() < 1e-15
    x3 = np.array(hand_cases["period4_x_appended"])[:, None]
    h3 = fo.compress(x3, np.ones(1), 0, 0, 4, period=4)
    assert np.abs(h3.C[:, 0] - hand_cases["period4_C_appended"]).max() < 1e-15


def test_mask_agreement_check_rejects_a_swap_across_a_wide_cut():
    """The GPU mask check (tests/test_gpu_sensitivity.py) must reject a selection that swaps
    two dims whose oracle scores differ by more than the tolerance, and accept one that
    swaps only dims tied within it. The mistake is planted in the scores on the CPU."""
    from test_gpu_sensitivity import TOL, check_masks_agree
    so = np.linspace(1.0, 2.0, 128)            # cut gaps 1/127 > TOL * max
    check_masks_agree(so.copy(), so, 96)
    swapped = so.copy()
    swapped[[95, 96]] = swapped[[96, 95]]       # dim 96 compressed, dim 95 retained
    with pytest.raises(AssertionError):
        check_masks_agree(swapped, so, 96)
    tied = so.copy()
    tied[96] = tied[95] + 0.5 * TOL * tied.max()
    near = tied.copy()
    near[[95, 96]] = near[[96, 95]]
    check_masks_agree(near, tied, 96)
