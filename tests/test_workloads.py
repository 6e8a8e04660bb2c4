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
