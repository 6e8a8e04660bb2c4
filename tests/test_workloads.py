"""Host-side checks of the seeded synthetic workloads (no GPU)."""
import numpy as np
import torch

import workloads as wl


def test_masks_follow_recipes():
    m1 = wl.dim_mask(wl.SINGLE_HEAD_2K)
    assert m1.shape == (1, 128) and m1[0, :96].all() and not m1[0, 96:].any()
    m2 = wl.dim_mask(wl.LLAMA2_7B_MHA_32K)
    assert m2.shape == (32, 128) and (m2.sum(1) == 96).all()
    assert len({bytes(r) for r in m2}) > 1  # random per head
    m3 = wl.dim_mask(wl.LLAMA3_8B_GQA_32K)
    assert set(m3.sum(1)) <= {64, 96}
    assert np.array_equal(m2, wl.dim_mask(wl.LLAMA2_7B_MHA_32K))  # seeded


def test_generators_are_seeded_and_shaped():
    w = wl.shrink(wl.LLAMA3_8B_GQA_32K, B=2, L=700)
    K1, K2 = wl.kv_cache(w, "K"), wl.kv_cache(w, "K")
    assert K1.shape == (2, 8, 700, 128) and K1.dtype == torch.bfloat16
    assert torch.equal(K1, K2)
    V = wl.kv_cache(w, "V")
    assert not torch.equal(K1, V)
    q = wl.queries(w)
    assert q.shape == (2, 32, 128)
    # the smooth trend makes neighbouring tokens strongly correlated
    x = K1.float()
    c = torch.corrcoef(torch.stack([x[0, 0, :-1].flatten(), x[0, 0, 1:].flatten()]))[0, 1]
    assert c > 0.9


def test_sweep_layer_k_is_odd():
    for L in wl.SWEEP_L:
        w = wl.llama3_8b_layer(1, L, 0)
        assert w.k == L // 128 - 1 and w.k % 2 == 1


def test_splitmix64_matches_its_published_outputs():
    """SplitMix64 from state 0: the first outputs of the reference splitmix64.c are
    0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F."""
    z = wl.splitmix64(0, 3)
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_grid_values_are_exact_in_bf16():
    v = wl.grid_values(12345, 4096)
    assert v.min() >= -2.0 and v.max() <= 127 / 64
    assert np.array_equal(torch.from_numpy(v).to(torch.bfloat16).double().numpy(), v)
    assert len(np.unique(v)) > 200  # the whole grid is reached


def _golden_module():
    import importlib.util
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "make_c_abi_gpu_case.py")
    spec = importlib.util.spec_from_file_location("make_c_abi_gpu_case", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod, path.replace("make_c_abi_gpu_case.py", "c_abi_gpu_case.txt")


def test_c_gpu_golden_file_is_the_oracle_output():
    """The stored values the plain-C GPU program checks against are what the oracle gives
    on the recipe's inputs (to the 12 significant digits stored)."""
    mod, path = _golden_module()
    out, coef = mod.compute()
    lines = [ln.split() for ln in open(path) if not ln.startswith("#")]
    i = next(n for n, ln in enumerate(lines) if ln[0] == "out")
    vals = np.array([float(x[0]) for x in lines[i + 1:i + 1 + out.size]])
    np.testing.assert_allclose(vals, out.ravel(), rtol=1e-11, atol=1e-14)
    for which in ("K", "V"):
        j = next(n for n, ln in enumerate(lines) if ln[:2] == ["coef", which])
        kk, dc = int(lines[j][4]), int(lines[j][5])
        c = np.array([float(x[0]) for x in lines[j + 1:j + 1 + kk * dc]]).reshape(kk, dc)
        np.testing.assert_allclose(c, coef[which], rtol=1e-11, atol=1e-12)
