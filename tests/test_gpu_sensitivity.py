"""GPU parity of the head-dimension analysis (fa_dim_sensitivity + fa_select_dims).

The oracle runs the skill page's loop (one perturbed attention per dim, values perturbed);
the library uses one attention pass over (K, noise). Scores meet the 3e-3 bound per KV
head; the mask selected from the GPU scores is a valid selection under the oracle's scores
(no compressed dim scores above a retained one by more than the bound), which makes it
the oracle's mask wherever the oracle's cut is wider than the bound.
"""
import numpy as np
import pytest
import torch

import fourier_basis_attention_b200 as fa
import workloads as wl
from oracle import fourier_oracle as fo

pytestmark = pytest.mark.gpu
TOL = 3e-3


def gpu_scores(q, K, noise):
    B, Hkv, L, _ = K.shape
    ws = torch.empty(fa.fa_dim_sensitivity_workspace_size(B, q.shape[1], Hkv, L), dtype=torch.uint8,
                     device="cuda")
    scores = torch.full((Hkv, 128), -1.0, dtype=torch.float32, device="cuda")
    fa.fa_dim_sensitivity(q, K, noise, scores, ws)
    fa.fa_device_status()
    return scores.cpu().numpy()


def check_masks_agree(sg, so, n_compressed):
    """The mask selected from the GPU scores is a valid selection under the oracle's
    scores: every dim it compresses scores (by the oracle) no higher than every dim it
    retains, up to the score tolerance. Where the oracle's scores separate the two sets
    by more than that tolerance, this forces the masks to be identical."""
    mg = fo.select_dims(sg, n_compressed)
    comp, kept = so[mg == 1], so[mg == 0]
    if comp.size and kept.size:
        assert comp.max() <= kept.min() + TOL * so.max(), (comp.max(), kept.min())
    srt = np.sort(so)
    if 0 < n_compressed < so.size and srt[n_compressed] - srt[n_compressed - 1] > TOL * so.max():
        assert np.array_equal(mg, fo.select_dims(so, n_compressed))


@pytest.mark.parametrize("G,L", [(4, 700), (1, 300), (8, 1000), (2, 1)], ids=str)
def test_sensitivity_small(G, L):
    w = wl.shrink(wl.LLAMA3_8B_GQA_32K, B=2, Hq=2 * G, Hkv=2, L=L)
    K, V, q, n = wl.kv_cache(w, "K"), wl.kv_cache(w, "V"), wl.queries(w), wl.value_noise(w)
    sg = gpu_scores(q.cuda(), K.cuda(), n.cuda())
    for g in range(w.Hkv):
        so = fo.dim_sensitivity(q[:, g * G:(g + 1) * G].double().numpy(), K[:, g].double().numpy(),
                                V[:, g].double().numpy(), n[:, g].double().numpy())
        err = np.abs(sg[g] - so).max()
        assert err <= TOL * so.max(), (g, err, so.max())
        check_masks_agree(sg[g], so, 96)
    # the library's selection is the oracle's selection of the same scores
    assert np.array_equal(fa.fa_select_dims(sg, 96),
                          np.stack([fo.select_dims(sg[g], 96) for g in range(w.Hkv)]))


def test_sensitivity_full_size_sampled_heads():
    """The LLaMA-2-7B MHA bench workload (B=8, L=32768, 32 KV heads), two KV heads checked."""
    w = wl.LLAMA2_7B_MHA_32K
    K = wl.kv_cache(w, "K", device="cuda")
    n = wl.value_noise(w, device="cuda")
    q = wl.queries(w, device="cuda")
    sg = gpu_scores(q, K, n)
    assert np.isfinite(sg).all() and (sg > 0).all()
    for g in (0, w.Hkv - 1):
        Kg = K[:, g].double().cpu().numpy()
        so = fo.dim_sensitivity(q[:, g:g + 1].double().cpu().numpy(), Kg, np.zeros_like(Kg),
                                n[:, g].double().cpu().numpy())
        assert np.abs(sg[g] - so).max() <= TOL * so.max()
        check_masks_agree(sg[g], so, 96)
