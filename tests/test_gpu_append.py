"""GPU parity of decode-time cache maintenance (fa_plan_reserve + fa_append).

Definition checked (the oracle's reading): after n appends, the hybrid cache equals the
cache that the oracle compresses from the whole longer sequence with the period P fixed
by the reservation. Sink rows, recent rows (in ring order) and retained dims are
bit-exact; coefficients and decode output meet the 3e-3 bound of the other parity tests.
"""
import dataclasses

import numpy as np
import pytest
import torch

import fourier_basis_attention_b200 as fa
import workloads as wl
from oracle import fourier_oracle as fo

pytestmark = pytest.mark.gpu
TOL = 3e-3
D = 128


def close(gpu, ref, tol=TOL):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    err = np.abs(gpu - ref).max()
    scale = np.abs(ref).max()
    assert err <= tol * scale, f"max err {err:.3e} > {tol} * {scale:.3e}"


def ring_in_token_order(F, p):
    """F rows [S + R, D] with the recent rows rotated back to token order."""
    idx = list(range(p.S)) + [p.S + (p.recent_head + a) % p.R for a in range(p.R)]
    return F[idx]


def decode(p, cache, q, num_splits=0):
    ws = torch.empty(max(fa.fa_decode_workspace_size(p, num_splits), 16), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(p.shape.B, p.shape.Hq, D, dtype=torch.float32, device="cuda")
    fa.fa_decode(p, q, cache, out, ws, num_splits)
    fa.fa_device_status()
    return out


def run_append(w, n_app, extra, mask=None, heads=None, num_splits=0, gen_device="cpu"):
    """Compress the first w.L tokens into a cache with room for n_app + extra more, append
    n_app tokens one by one, then check every part of the cache (of the sampled heads) and
    a decode step."""
    mask = wl.dim_mask(w) if mask is None else mask
    L1 = w.L + n_app
    wf = dataclasses.replace(w, L=L1)
    K, V = wl.kv_cache(wf, "K", device=gen_device), wl.kv_cache(wf, "V", device=gen_device)
    q = wl.queries(w)
    Kd, Vd = K.cuda(), V.cuda()
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    M0 = p.M
    fa.fa_plan_reserve(p, L1 + extra)
    P = p.P
    assert P == M0 + n_app + extra
    cache = fa.Cache(p)
    fa.fa_compress(p, Kd[:, :, :w.L].contiguous(), Vd[:, :, :w.L].contiguous(), fa.basis_table(p),
                   cache)
    for i in range(n_app):
        fa.fa_append(p, Kd[:, :, w.L + i].contiguous(), Vd[:, :, w.L + i].contiguous(), cache)
    fa.fa_device_status()
    assert (p.shape.L, p.M, p.P) == (L1, M0 + n_app, P)
    assert p.recent_head == (n_app % p.R if p.R > 0 else 0)
    out = decode(p, cache, q.cuda(), num_splits).cpu().numpy()
    torch.cuda.synchronize()
    pairs = heads or [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    for b, g in pairs:
        cd, ed = fa.perm_lists(p, g)
        hyb = {}
        for which, X in (("K", K[b, g].cpu()), ("V", V[b, g].cpu())):
            ref = fo.compress(X.double().numpy(), mask[g], w.S, w.R, w.k, period=P)
            hyb[which] = ref
            F = ring_in_token_order(cache.F(which)[b, g].cpu(), p)
            assert torch.equal(F[:p.S], X[:p.S]) and torch.equal(F[p.S:], X[L1 - p.R:])
            assert torch.equal(cache.E(which, b, g).cpu(), X[p.S:p.S + p.M][:, torch.from_numpy(ed)])
            assert not cache.E_raw(which, b, g)[:, p.de[g]:].any().item()
            assert not cache.C_raw(which, b, g)[:, p.dc[g]:].any().item()
            if p.dc[g] > 0:
                close(cache.C(which, b, g).cpu().numpy(), ref.C)
        o = out[b, g * w.G:(g + 1) * w.G]
        q64 = q[b, g * w.G:(g + 1) * w.G].double().numpy()
        close(o, fo.decode(q64, hyb["K"], hyb["V"]))
    return p, cache, K, V


SMALL = wl.shrink(wl.llama3_8b_layer(1, 8192, 0), B=2, Hq=8, Hkv=2, L=700, S=32, R=64, k=63)


@pytest.mark.parametrize("n_app,extra", [(0, 0), (0, 300), (1, 0), (70, 30), (131, 5)],
                         ids=["none_P_eq_M", "none_P_gt_M", "one", "wraps_ring", "two_wraps"])
def test_append_cuda_core_decode(n_app, extra):
    """Blocked E, CUDA-core decode; n_app > R folds tokens that were themselves appended.
    n_app = 0 checks the period plumbing of fa_compress / fa_decode alone (P = M, P > M)."""
    p, _, _, _ = run_append(SMALL, n_app, extra)
    assert p.e_token_major == 0 and p.P == p.M + extra


def test_append_tensor_core_decode_token_major():
    w = wl.shrink(wl.llama3_8b_layer(1, 8192, 0), B=16, Hq=8, Hkv=2, L=1400, S=32, R=64, k=127)
    p, _, _, _ = run_append(w, 80, 20, heads=[(0, 0), (0, 1), (9, 1), (15, 0)])
    assert p.e_token_major == 1


def test_append_warp_mma_decode():
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=2, Hq=16, Hkv=4, L=2000, k=300)
    mask = np.ones((4, D), dtype=np.uint8)
    rng = np.random.default_rng(3)
    for g, r in enumerate([32, 0, 128, 5]):     # retained dims per KV head (none / all)
        mask[g, rng.permutation(D)[:r]] = 0
    p, _, _, _ = run_append(w, 67, 10, mask=mask)
    assert p.e_token_major == 0


def test_append_without_recent_window():
    """R = 0: each new token joins the middle directly."""
    w = wl.shrink(SMALL, B=1, Hq=4, Hkv=1, L=300, S=8, R=0, k=31)
    p, cache, K, V = run_append(w, 9, 3)
    assert p.R == 0 and p.recent_head == 0


def test_append_matches_gpu_compress_of_longer_sequence():
    """fa_compress of the longer sequence (same period) writes the same cache up to fp32
    rounding of the coefficients; E and the sink / recent rows are identical."""
    w = SMALL
    n_app, extra = 40, 24
    p, cache, K, V = run_append(w, n_app, extra, heads=[(0, 0)])
    mask = wl.dim_mask(w)
    p2 = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L + n_app, w.S, w.R, w.k, mask)
    fa.fa_plan_reserve(p2, w.L + n_app + extra)
    assert p2.P == p.P and p2.M == p.M
    c2 = fa.Cache(p2)
    fa.fa_compress(p2, K.cuda(), V.cuda(), fa.basis_table(p2), c2)
    fa.fa_device_status()
    for b in range(w.B):
        for g in range(w.Hkv):
            for which in ("K", "V"):
                assert torch.equal(cache.E(which, b, g), c2.E(which, b, g))
                assert torch.equal(ring_in_token_order(cache.F(which)[b, g], p), c2.F(which)[b, g])
                close(cache.C(which, b, g).cpu().numpy(), c2.C(which, b, g).cpu().numpy())


def test_append_until_full_then_refused():
    w = wl.shrink(SMALL, B=1, Hq=4, Hkv=1, L=400, k=31)
    mask = wl.dim_mask(w)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    fa.fa_plan_reserve(p, w.L + 3)
    cache = fa.Cache(p)
    K = wl.kv_cache(w, "K").cuda()
    fa.fa_compress(p, K, K, fa.basis_table(p), cache)
    x = torch.zeros(1, 1, D, dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        fa.fa_append(p, x, x, cache)
    assert p.M == p.P
    with pytest.raises(fa.FaError) as e:
        fa.fa_append(p, x, x, cache)
    assert e.value.code == fa.FA_ERR_UNSUPPORTED
    fa.fa_device_status()


@pytest.mark.parametrize("w,n_app", [(wl.LLAMA2_7B_MHA_32K, 16), (wl.LLAMA3_8B_GQA_128K, 16),
                                       (wl.llama3_8b_layer(64, 131072, 30), 1)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_append_full_size_sampled_heads(w, n_app):
    """The bench-sized caches and the largest point of the 32-layer cache (B = 64,
    L = 128K): appends, then the first and last (batch, KV head) against the oracle of the
    longer sequence."""
    p, cache, K, V = run_append(w, n_app, 8, heads=[(0, 0), (w.B - 1, w.Hkv - 1)],
                                gen_device="cuda")
    assert p.M == w.L - w.S - w.R + n_app
    idx = [p.S + (p.recent_head + a) % p.R for a in range(p.R)]
    assert torch.equal(cache.F("K")[:, :, idx], K[:, :, p.shape.L - p.R:])
