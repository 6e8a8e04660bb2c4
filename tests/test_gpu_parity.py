"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bars (from the method's tolerances):
* token / dim partition, sink/recent rows (F) and retained dims (E): bit-exact;
* floating point (basis table, coefficients C, decode output): max |err| <= 3e-3 * max |ref|
  over the compared tensor, for bf16 I/O with fp32 accumulation.

Three decode checks: "isolated" (oracle attention over the GPU-written hybrid cache),
"end-to-end" (oracle compress + attention from the original cache vs GPU compress +
decode), and the basis / coefficient checks of fa_compress itself. Oracle-sized cases
compare every element; the full-size workloads compare sampled (batch, KV head) pairs.
"""
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
    if ref.size == 0:
        return 0.0
    err = np.abs(gpu - ref).max()
    scale = np.abs(ref).max()
    assert err <= tol * scale, f"max err {err:.3e} > {tol} * {scale:.3e}"
    return err / scale


def run_path(w, K, V, q, mask, num_splits=0):
    """GPU compress + decode through the binding (inputs already on the device).

    Returns the fp32 decode output. The 3e-3 bound is tighter than bf16's unit roundoff
    (2^-8), so parity is judged on fp32; the bf16 output is checked here to be exactly
    that fp32 result rounded to nearest even."""
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    phiT = fa.basis_table(p)
    cache = fa.Cache(p)
    fa.fa_compress(p, K, V, phiT, cache)
    fa.fa_device_status()
    ws = torch.empty(max(fa.fa_decode_workspace_size(p, num_splits), 16), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(w.B, w.Hq, D, dtype=torch.float32, device="cuda")
    fa.fa_decode(p, q, cache, out, ws, num_splits)
    out_bf = torch.empty(w.B, w.Hq, D, dtype=torch.bfloat16, device="cuda")
    fa.fa_decode(p, q, cache, out_bf, ws, num_splits)
    fa.fa_device_status()
    torch.cuda.synchronize()
    assert torch.equal(out_bf, out.to(torch.bfloat16))
    return p, cache, out


def gpu_hybrid(p, cache, which, b, g, L):
    """The GPU-written hybrid cache of one head, as an oracle Hybrid (fp64)."""
    cd, ed = fa.perm_lists(p, g)
    F = cache.F(which)[b, g].float().cpu().numpy().astype(np.float64)
    C = cache.C(which, b, g).cpu().numpy().astype(np.float64) if p.M > 0 else np.zeros((0, len(cd)))
    E = cache.E(which, b, g).float().cpu().numpy().astype(np.float64) if p.M > 0 else np.zeros((0, len(ed)))
    return fo.Hybrid(L=L, D=D, S=p.S, R=p.R, M=p.M, k=p.shape.k, cd=cd, ed=ed,
                     sink=F[:p.S], recent=F[p.S:], E=E, C=C)


def check_head(w, p, cache, out, Kh, Vh, qh, mask_row, b, g):
    """All parity checks of one (b, g). Kh, Vh: bf16 [L, D] host tensors; qh: [G, D]."""
    Kd, Vd = Kh.double().numpy(), Vh.double().numpy()
    hk, hv = fo.compress(Kd, mask_row, w.S, w.R, w.k), fo.compress(Vd, mask_row, w.S, w.R, w.k)
    # bit-exact parts: sink/recent rows and retained dims
    for which, X in (("K", Kh), ("V", Vh)):
        F = cache.F(which)[b, g].cpu()
        assert torch.equal(F[:p.S], X[:p.S]) and torch.equal(F[p.S:], X[w.L - p.R:])
        if p.M > 0:
            ed = torch.from_numpy(fa.perm_lists(p, g)[1])
            assert torch.equal(cache.E(which, b, g).cpu(), X[p.S:p.S + p.M][:, ed])
            assert not cache.E_raw(which, b, g)[:, p.de[g]:].any().item()
            assert not cache.C_raw(which, b, g)[:, p.dc[g]:].any().item()
    # coefficients
    if p.M > 0 and p.dc[g] > 0:
        close(cache.C("K", b, g).cpu().numpy(), hk.C)
        close(cache.C("V", b, g).cpu().numpy(), hv.C)
    o = out[b, g * w.G:(g + 1) * w.G].float().cpu().numpy()
    q64 = qh.double().numpy()
    # isolated decode: oracle attention over the GPU-written hybrid cache
    ref_iso = fo.decode(q64, gpu_hybrid(p, cache, "K", b, g, w.L), gpu_hybrid(p, cache, "V", b, g, w.L))
    close(o, ref_iso)
    # end to end: oracle compress + attention from the original cache
    close(o, fo.decode(q64, hk, hv))


def run_small(w, mask=None, num_splits=0, heads=None):
    mask = wl.dim_mask(w) if mask is None else mask
    K, V, q = wl.kv_cache(w, "K"), wl.kv_cache(w, "V"), wl.queries(w)
    p, cache, out = run_path(w, K.cuda(), V.cuda(), q.cuda(), mask, num_splits)
    pairs = heads or [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    for b, g in pairs:
        check_head(w, p, cache, out, K[b, g], V[b, g], q[b, g * w.G:(g + 1) * w.G], mask[g], b, g)
    return p


# ----------------------------------------------------------------------------- basis table

@pytest.mark.parametrize("M,k", [(1, 1), (2, 2), (4, 4), (7, 7), (64, 63), (1952, 63),
                                 (4096, 4096), (32672, 255), (128992, 1023)])
def test_basis_table(M, k):
    ld = (M + 7) // 8 * 8
    rows = np.unique(np.linspace(0, k - 1, min(k, 64)).astype(int))
    cols = np.unique(np.concatenate([np.arange(min(M, 512)), np.linspace(0, M - 1, 2048).astype(int)]))
    ref = fo.basis(M, k)[np.ix_(cols, rows)].T                  # orthonormal phi_j(t)
    f = (rows + 1) // 2
    scale_j = np.where((f == 0) | (2 * f == M), 1 / np.sqrt(M), np.sqrt(2.0 / M))[:, None]
    for normalized in (True, False):
        t32 = torch.full((k, ld), 7.0, dtype=torch.float32, device="cuda")
        t16 = torch.full((k, ld), 7.0, dtype=torch.bfloat16, device="cuda")
        fa.fa_build_basis(M, k, t32, ld, normalized=normalized)
        fa.fa_build_basis(M, k, t16, ld, normalized=normalized)
        torch.cuda.synchronize()
        r = ref if normalized else ref / scale_j                  # unit amplitude when unscaled
        amp = np.abs(r).max()
        g32 = t32[rows][:, cols].double().cpu().numpy()
        g16 = t16[rows][:, cols].double().cpu().numpy()
        assert np.abs(g32 - r).max() <= 4e-6 * amp
        # bf16: round to nearest even, relative error at most 2^-8
        assert np.all(np.abs(g16 - r) <= 2.0 ** -8 * np.abs(r) + 1e-7 * amp)
        assert not t32[:, M:].any().item() and not t16[:, M:].any().item()
    # the unscaled DC row and the Nyquist row are exact in bf16
    assert (t16[0, :M] == 1).all().item()
    if M % 2 == 0 and k == M:
        alt = torch.tensor([1.0, -1.0], device="cuda").repeat(M // 2).to(torch.bfloat16)
        assert torch.equal(t16[M - 1, :M], alt)


# ----------------------------------------------------------------------------- oracle-sized cases

SMALL = [
    wl.SINGLE_HEAD_2K,
    wl.shrink(wl.LLAMA2_7B_MHA_32K, B=2, Hq=4, Hkv=4, L=1000),
    wl.shrink(wl.LLAMA3_8B_GQA_32K, B=2, Hq=8, Hkv=2, L=1800),
    wl.shrink(wl.LLAMA3_8B_GQA_128K, B=1, Hq=8, Hkv=2, L=4200),
    wl.shrink(wl.llama3_8b_layer(1, 8192, 7), B=2, Hq=8, Hkv=2, L=3000),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: f"{w.name}_B{w.B}_L{w.L}")
def test_small_workloads_all_heads(w):
    run_small(w)


@pytest.mark.parametrize("ns", [1, 3, 7, 1000])
def test_forced_split_counts(ns):
    run_small(wl.shrink(wl.LLAMA3_8B_GQA_32K, B=1, Hq=8, Hkv=2, L=2000), num_splits=ns)


@pytest.mark.parametrize("name,kw,mask", [
    ("no_middle", dict(L=90), "rand96"),                     # L <= S + R
    ("middle_of_one", dict(L=97, k=1), "rand96"),
    ("nothing_compressed", dict(L=700), "none"),
    ("everything_compressed", dict(L=700), "all"),
    ("k_equals_M", dict(L=96 + 127, k=127), "rand96"),
    ("k_even", dict(L=700, k=64), "rand96"),
    ("k_one_dc_only", dict(L=700, k=1), "rand96"),
    ("k_two", dict(L=700, k=2), "rand96"),
    ("single_ragged_tile", dict(L=96 + 40, k=17), "rand96"),
    ("group_2", dict(L=900, Hq=4, Hkv=2, k=31), "rand64or96"),
    ("group_8", dict(L=900, Hq=16, Hkv=2, k=31), "rand64or96"),
    ("mha_partial_head_set", dict(L=900, Hq=3, Hkv=3, k=31), "rand96"),
    ("no_sink", dict(L=800, S=0, k=63), "rand96"),
    ("no_recent", dict(L=800, R=0, k=63), "rand96"),
])
def test_edge_cases(name, kw, mask):
    base = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=1, Hq=2, Hkv=2, L=700, S=32, R=64, k=31)
    w = wl.shrink(base, mask=mask, **kw)
    run_small(w)


def test_ragged_mask_padding():
    """Popcounts that are not multiples of 8 exercise the padded C / E row strides."""
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=2, Hq=4, Hkv=4, L=600, k=47)
    rng = np.random.default_rng(11)
    mask = np.zeros((4, D), dtype=np.uint8)
    for g, dc in enumerate([37, 1, 127, 90]):
        mask[g, rng.permutation(D)[:dc]] = 1
    run_small(w, mask=mask)


# The plan puts E token-major and fa_decode runs the middle span on the tensor-core split
# kernel when k <= 255, G in {1, 2, 4}, k G >= 255, at least 128 query heads and at most 32
# exact dims per KV head; these cases cover its split counts, chunk layouts and head sets.
TC_BASE = wl.shrink(wl.llama3_8b_layer(1, 8192, 0), B=16, Hq=8, Hkv=2, L=1400, k=127)
TC_HEADS = [(0, 0), (0, 1), (7, 1), (15, 0), (15, 1)]


def test_tensor_core_shapes_are_token_major():
    masks = [wl.dim_mask(TC_BASE)] + [_ragged(dcs) for dcs, _ in TC_RAGGED]
    shapes = [TC_BASE] + [_ragged_shape(k) for _, k in TC_RAGGED] + [TC_WIDE]
    for w, m in zip(shapes, masks + [wl.dim_mask(TC_WIDE)]):
        assert fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, m).e_token_major == 1


@pytest.mark.parametrize("ns", [0, 1, 3, 7, 1000])
def test_split_counts_tensor_core(ns):
    run_small(TC_BASE, num_splits=ns, heads=TC_HEADS)


TC_RAGGED = [([97, 100, 123, 127], 255),   # 31, 28, 5, 1 exact dims: 32-element rows
             ([114, 120, 126, 124], 255),  # 14, 8, 2, 4: 16-element rows
             ([120, 124, 128, 127], 255),  # 8, 4, 0, 1: 8-element rows
             ([128, 96, 120, 112], 255)]   # 0, 32, 8, 16


def _ragged_shape(k):
    return wl.shrink(wl.LLAMA2_7B_MHA_32K, B=16, Hq=8, Hkv=4, L=1400, k=k)


def _ragged(dcs):
    rng = np.random.default_rng(5)
    mask = np.zeros((4, D), dtype=np.uint8)
    for g, dc in enumerate(dcs):
        mask[g, rng.permutation(D)[:dc]] = 1
    return mask


@pytest.mark.parametrize("dcs,k", TC_RAGGED, ids=lambda x: str(x))
def test_ragged_mask_tensor_core(dcs, k):
    """Exact-dim rows of 1, 2 or 4 sixteen-byte chunks, KV heads with 0 to 32 exact dims."""
    run_small(_ragged_shape(k), mask=_ragged(dcs),
              heads=[(0, g) for g in range(4)] + [(15, g) for g in range(4)])


@pytest.mark.parametrize("retained", [[14, 9], [5, 3], [16, 0]], ids=str)
def test_narrow_rows_gqa4_tensor_core(retained):
    """G = 4 with 16- and 8-element KV slices: two or four tokens per exact-dim step."""
    w = wl.shrink(wl.llama3_8b_layer(1, 8192, 0), B=16, Hq=8, Hkv=2, L=1400, k=127)
    mask = np.ones((2, D), dtype=np.uint8)
    rng = np.random.default_rng(9)
    for g, r in enumerate(retained):
        mask[g, rng.permutation(D)[:r]] = 0
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    assert p.e_token_major == 1 and p.de_ld[0] == (16 if max(retained) > 8 else 8)
    run_small(w, mask=mask, heads=[(0, 0), (0, 1), (15, 0), (15, 1)])


@pytest.mark.parametrize("dcs", [[97, 123, 127, 108], [120, 124, 128, 127]], ids=str)
def test_mha_tensor_core(dcs):
    """G = 1 (each KV head its own query head) at k = 255: 32- and 8-element KV slices."""
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=32, Hq=4, Hkv=4, L=1400, k=255)
    mask = _ragged(dcs)
    assert fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask).e_token_major == 1
    run_small(w, mask=mask, heads=[(0, g) for g in range(4)] + [(31, g) for g in range(4)])


# Plans that are not token-major with 256 <= k <= 1023 run the middle span on the warp-MMA
# split kernel (16 query heads per CTA): group sizes, ragged exact dims, both slot counts.
@pytest.mark.parametrize("G,Hkv,k,dcs", [(8, 2, 511, None), (1, 4, 511, [37, 1, 127, 90]),
                                         (2, 4, 1023, [100, 64, 17, 128]), (4, 2, 300, [0, 96])],
                         ids=["G8_k511", "G1_k511_ragged", "G2_k1023_ragged", "G4_k300_none_all"])
def test_warp_mma_decode(G, Hkv, k, dcs):
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=3, Hq=Hkv * G, Hkv=Hkv, L=k + 96 + 333, k=k)
    mask = wl.dim_mask(w) if dcs is None else _ragged_hkv(dcs, Hkv)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    assert p.e_token_major == 0
    run_small(w, mask=mask)


def _ragged_hkv(dcs, Hkv):
    rng = np.random.default_rng(13)
    mask = np.zeros((Hkv, D), dtype=np.uint8)
    for g, dc in enumerate(dcs):
        mask[g, rng.permutation(D)[:dc]] = 1
    return mask


# Plans with 256 <= k <= 1023, G in {2, 4, 8} and per-KV-head E blocks run the middle span
# on the cluster tensor-core kernel when their 128-query-head sets are at least three
# quarters full: the coefficient slots are split over 2 (k <= 511) or 4 CTAs of a
# thread-block cluster, partial scores summed by each quadrant's owner CTA. Every case
# leaves invalid heads in its last set.
@pytest.mark.parametrize("G,Hkv,k,B,dcs,cluster", [
    (4, 2, 511, 12, [96, 64], 2),            # ragged exact dims (32 / 64 per KV head)
    (2, 4, 511, 13, [96, 64, 90, 120], 2),   # G = 2: 32 exact KV heads per CTA; 104 heads
    (8, 2, 1023, 6, [96, 100], 4),           # G = 8
    (4, 8, 1023, 6, None, 4),                # 192 query heads: a second, half-full head set
    (4, 2, 257, 12, [96, 96], 2),            # 2 F_pad = 264 slots: 192 per CTA
    (2, 4, 1023, 12, [100, 64, 96, 128], 4), # G = 2, a KV head without exact dims
], ids=["C2_G4_ragged", "C2_G2", "C4_G8", "C4_two_head_sets", "C2_192_slots", "C4_G2_ragged"])
def test_cluster_decode(G, Hkv, k, B, dcs, cluster):
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=B, Hq=Hkv * G, Hkv=Hkv, L=k + 96 + 333, k=k)
    mask = wl.dim_mask(w) if dcs is None else _ragged_hkv(dcs, Hkv)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    info = fa.fa_decode_describe(p, 1)
    assert info.split_kernel == fa.FA_SPLIT_TC_CLUSTER and info.cluster == cluster
    run_small(w, mask=mask, heads=sorted({(0, 0), (0, Hkv - 1), (B // 2, Hkv // 2),
                                          (B - 1, 0), (B - 1, Hkv - 1)}))


@pytest.mark.parametrize("B,kind", [(1, 3), (2, 3), (3, 4)])
def test_cluster_decode_needs_full_head_sets(B, kind):
    """32 or 64 query heads (a quarter or half of a 128-head set) go to the warp-MMA kernel,
    96 to the cluster kernel; both agree with the oracle."""
    w = wl.shrink(wl.LLAMA3_8B_GQA_32K, B=B, L=1800)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, wl.dim_mask(w))
    assert fa.fa_decode_describe(p, 0).split_kernel == kind
    run_small(w, heads=[(0, 0), (B - 1, w.Hkv - 1)])


@pytest.mark.parametrize("ns", [1, 5, 1000])
def test_split_counts_warp_mma(ns):
    run_small(wl.shrink(wl.LLAMA3_8B_GQA_128K, B=1, Hq=32, Hkv=8, L=3300), num_splits=ns,
              heads=[(0, 0), (0, 7)])


TC_WIDE = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=40, Hq=8, Hkv=2, L=500, k=127, mask="rand96")


def test_more_than_128_query_heads_tensor_core():
    """Three head sets of 128 query heads; the last holds 64 valid heads."""
    run_small(TC_WIDE, heads=[(0, 0), (15, 1), (16, 0), (31, 1), (32, 0), (39, 1)])


def test_k_equals_M_matches_plain_attention():
    """With k = M nothing is lost: decode is plain attention over the original cache."""
    w = wl.shrink(wl.SINGLE_HEAD_2K, L=96 + 127, k=127)
    K, V, q = wl.kv_cache(w, "K"), wl.kv_cache(w, "V"), wl.queries(w)
    p, cache, out = run_path(w, K.cuda(), V.cuda(), q.cuda(), wl.dim_mask(w))
    ref = fo.attention(q[0].double().numpy(), K[0, 0].double().numpy(), V[0, 0].double().numpy(),
                       1 / np.sqrt(D))
    close(out[0].cpu().numpy(), ref)


def test_repeat_calls_are_deterministic():
    w = wl.shrink(wl.LLAMA3_8B_GQA_32K, B=1, Hq=8, Hkv=2, L=2000)
    K, V, q = (t.cuda() for t in (wl.kv_cache(w, "K"), wl.kv_cache(w, "V"), wl.queries(w)))
    _, c1, o1 = run_path(w, K, V, q, wl.dim_mask(w))
    _, c2, o2 = run_path(w, K, V, q, wl.dim_mask(w))
    assert torch.equal(c1.C_K, c2.C_K) and torch.equal(o1, o2)


# ----------------------------------------------------------------------------- full-size workloads

def sample_pairs(w):
    """Four distinct (batch row, KV head) pairs spread over the cache: the first, the last
    (largest offsets into every buffer), and two between them."""
    cand = [(0, 0), (w.B - 1, w.Hkv - 1), (w.B // 2, w.Hkv // 2), (w.B - 1, 0),
            (0, w.Hkv - 1), ((w.B - 1) // 3, 1 % w.Hkv), (0, 1 % w.Hkv)]
    out = []
    for c in cand:
        if c not in out:
            out.append(c)
    return out[:4]


# The single-layer workloads at full size, and points of the 32-layer LLaMA-3-8B cache
# sweep: B = 8 at L = 32K (tensor-core decode), B = 64 at L = 128K (k = 1023; E offsets of
# the last batch row near 2^31 elements), B = 64 at L = 8K (k = 63, CUDA-core decode) and
# B = 1 at L = 32K (32 query heads, CUDA-core decode).
FULL = [wl.LLAMA2_7B_MHA_32K, wl.LLAMA3_8B_GQA_32K, wl.LLAMA3_8B_GQA_128K,
        wl.llama3_8b_layer(8, 32768, 3), wl.llama3_8b_layer(64, 131072, 31),
        wl.llama3_8b_layer(64, 8192, 17), wl.llama3_8b_layer(1, 32768, 9)]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled_heads(w):
    mask = wl.dim_mask(w)
    K = wl.kv_cache(w, "K", device="cuda")
    V = wl.kv_cache(w, "V", device="cuda")
    q = wl.queries(w, device="cuda")
    p, cache, out = run_path(w, K, V, q, mask)
    for b, g in sample_pairs(w):
        check_head(w, p, cache, out, K[b, g].cpu(), V[b, g].cpu(),
                   q[b, g * w.G:(g + 1) * w.G].cpu(), mask[g], b, g)
    # every output is finite and every head's F rows are exact copies
    assert torch.isfinite(out.float()).all().item()
    idx = torch.cat([torch.arange(p.S), torch.arange(w.L - p.R, w.L)]).cuda()
    assert torch.equal(cache.F("K"), K[:, :, idx]) and torch.equal(cache.F("V"), V[:, :, idx])
    del cache, K, V
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- failure detection

def test_bounded_wait_reports_and_context_survives():
    """A kernel waiting on a barrier nothing completes gives up after its bound, the host
    reads FA_ERR_DEVICE, the word is cleared, and the next compress + decode still run."""
    fa.fa_watchdog_selftest(20_000_000)
    with pytest.raises(fa.FaError) as e:
        fa.fa_device_status()
    assert e.value.code == fa.FA_ERR_DEVICE and "kernel 15" in str(e.value)
    fa.fa_device_status()  # cleared
    run_small(wl.shrink(wl.SINGLE_HEAD_2K, L=600))


# ----------------------------------------------------------------------------- determinism at scale

def test_compress_many_heads_is_deterministic():
    """160 (KV head, tile pair) units: more CTAs than SMs; repeated calls write identical bits."""
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=40, Hq=4, Hkv=4, L=2000, k=255)
    mask = wl.dim_mask(w)
    K, V = wl.kv_cache(w, "K", device="cuda"), wl.kv_cache(w, "V", device="cuda")
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    phiT = fa.basis_table(p)
    c1, c2 = fa.Cache(p), fa.Cache(p)
    fa.fa_compress(p, K, V, phiT, c1)
    fa.fa_compress(p, K, V, phiT, c2)
    fa.fa_device_status()
    assert torch.equal(c1.C_K, c2.C_K) and torch.equal(c1.C_V, c2.C_V)
    assert torch.equal(c1.E_K, c2.E_K) and torch.equal(c1.E_V, c2.E_V)


# ----------------------------------------------------------------------------- token-split compress

@pytest.mark.parametrize("shape", [
    dict(B=1, Hq=8, Hkv=2, L=20000, k=511),    # 4 units: clusters of up to 16 CTAs
    dict(B=1, Hq=4, Hkv=1, L=5000, k=255),     # 1 unit, 78 stages: clusters of up to 16
    dict(B=3, Hq=12, Hkv=3, L=3000, k=63),     # 9 units, 47 stages: clusters of 8
    dict(B=2, Hq=8, Hkv=4, L=1100, k=127),     # 8 units, 17 stages: clusters of 4
], ids=["k511_4units", "k255_1unit", "k63_9units", "k127_8units"])
def test_compress_token_split(shape):
    """Small batches split each unit's token stages over a cluster and sum the partial
    coefficients in rank order: parity with the oracle on every head, and repeated calls
    write identical bits."""
    w = wl.shrink(wl.LLAMA3_8B_GQA_128K, S=32, R=64, **shape)
    p = run_small(w)
    mask = wl.dim_mask(w)
    K, V = wl.kv_cache(w, "K", device="cuda"), wl.kv_cache(w, "V", device="cuda")
    phiT = fa.basis_table(p)
    c1, c2 = fa.Cache(p), fa.Cache(p)
    fa.fa_compress(p, K, V, phiT, c1)
    fa.fa_compress(p, K, V, phiT, c2)
    fa.fa_device_status()
    assert torch.equal(c1.C_K, c2.C_K) and torch.equal(c1.C_V, c2.C_V)
    assert torch.equal(c1.E_K, c2.E_K) and torch.equal(c1.E_V, c2.E_V)


# ----------------------------------------------------------------------------- whole-row head warps

# With Hq = 32 each head warp of the tensor-core decode serves whole token rows of one batch
# row (G = 1 and 2 with 16- or 32-element KV slices), including a last head set with one
# populated warp.
@pytest.mark.parametrize("G,B,rows,ns", [
    (1, 4, [97, 100, 123, 127] * 8, 0),    # 32-element rows, 4 chunks per lane
    (1, 5, [114, 120, 126, 124] * 8, 7),   # 16-element rows; 160 heads: last set one warp
    (2, 4, [97, 128, 108, 120] * 4, 3),    # G = 2, 32-element rows, 2 chunks per lane
    (2, 5, [126, 120, 128, 116] * 4, 0),   # G = 2, 16-element rows, ragged, 160 heads
], ids=["G1_w32", "G1_w16_partial_set", "G2_w32", "G2_w16"])
def test_whole_row_warps_tensor_core(G, B, rows, ns):
    Hq = 32
    Hkv = Hq // G
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=B, Hq=Hq, Hkv=Hkv, L=1400, k=255)
    rng = np.random.default_rng(11)
    mask = np.zeros((Hkv, D), dtype=np.uint8)
    for g in range(Hkv):
        mask[g, rng.permutation(D)[:rows[g]]] = 1
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    assert p.e_token_major == 1
    info = fa.fa_decode_describe(p, ns)
    assert info.split_kernel == fa.FA_SPLIT_TC_TOKEN_MAJOR
    run_small(w, mask=mask, num_splits=ns,
              heads=[(0, 0), (0, Hkv - 1), (B - 1, 0), (B - 1, Hkv // 2), (B - 1, Hkv - 1)])


def test_small_k_many_heads_tensor_core():
    """k G < 255 (k = 63, G = 4) runs on the tensor cores once there are 1024 query heads."""
    w = wl.shrink(wl.llama3_8b_layer(1, 8192, 0), B=128, Hq=8, Hkv=2, L=1000, R=64, k=63)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, wl.dim_mask(w))
    assert p.e_token_major == 1
    assert fa.fa_decode_describe(p, 0).split_kernel == fa.FA_SPLIT_TC_TOKEN_MAJOR
    run_small(w, heads=[(0, 0), (0, 1), (63, 1), (127, 0), (127, 1)])


def test_compress_token_split_extreme_masks():
    """Token split with a head whose dims are all compressed (no E rows) and one with none
    compressed (no coefficients: the split CTAs only pack E)."""
    w = wl.shrink(wl.LLAMA3_8B_GQA_128K, B=1, Hq=8, Hkv=2, L=5000, S=32, R=64, k=255)
    mask = np.zeros((2, D), dtype=np.uint8)
    mask[0, :] = 1
    p = run_small(w, mask=mask)
    assert p.dc[0] == 128 and p.dc[1] == 0
    K, V = wl.kv_cache(w, "K", device="cuda"), wl.kv_cache(w, "V", device="cuda")
    phiT = fa.basis_table(p)
    c1, c2 = fa.Cache(p), fa.Cache(p)
    fa.fa_compress(p, K, V, phiT, c1)
    fa.fa_compress(p, K, V, phiT, c2)
    fa.fa_device_status()
    assert torch.equal(c1.C_K, c2.C_K) and torch.equal(c1.E_V, c2.E_V)
