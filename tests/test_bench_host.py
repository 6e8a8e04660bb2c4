"""Host-side accounting of bench.py: the algorithmic work model, the launch count and the
append byte count, checked against independent hand counts (no GPU)."""
import numpy as np

import bench
import fourier_basis_attention_b200 as fa
import workloads as wl


def _plan(w, mask=None):
    mask = wl.dim_mask(w) if mask is None else mask
    return fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)


def test_work_model_bench_workload_by_hand():
    """LLaMA-2-7B MHA, B=8, L=32768, k=255, 96 of 128 dims compressed in every head."""
    w = wl.LLAMA2_7B_MHA_32K
    p = _plan(w)
    assert all(p.dc[g] == 96 for g in range(w.Hkv))
    M, k, SR = 32768 - 96, 255, 96
    heads = 8 * 32
    per_head_c = 2 * (2 * M * 128 + 4 * k * 96 + 2 * M * 32 + 4 * SR * 128)   # K and V
    per_head_d = 2 * (2 * SR * 128 + 2 * M * 32 + 4 * k * 96)
    wm = bench.work_model(w, p)
    assert wm["compress_bytes"] == heads * per_head_c
    assert wm["compress_flops"] == heads * 2 * 2 * k * M * 96
    assert wm["decode_bytes"] == heads * per_head_d + 2 * 2 * 8 * 32 * 128
    # the figures quoted with the bench line
    assert wm["compress_bytes"] == 5428281344 and wm["decode_bytes"] == 1133445120


def test_algorithmic_bytes_are_the_method_minimum_by_hand():
    """The method's minimum bytes (bf16 coefficients; compress reads the middle rows once
    and writes C and E; decode reads F, E and C of K and V, the queries, writes out):
    decode 4 B Hkv [(S+R) D + M De + k Dc] + q + out, compress 4 B Hkv (M D + k Dc + M De)."""
    w = wl.LLAMA2_7B_MHA_32K
    wm = bench.work_model(w, _plan(w))
    B, Hkv, D, M, k, SR = 8, 32, 128, 32768 - 96, 255, 96
    assert wm["decode_bytes_alg"] == 4 * B * Hkv * (SR * D + M * 32 + k * 96) + 2 * 2 * B * 32 * D
    assert wm["compress_bytes_alg"] == 4 * B * Hkv * (M * D + k * 96 + M * 32)
    assert wm["compress_bytes_alg"] == 5378048000 and wm["decode_bytes_alg"] == 1108377600
    # no middle span: nothing to project, decode reads only the sink / recent rows
    w0 = wl.shrink(w, B=1, Hq=2, Hkv=2, L=90)
    wm0 = bench.work_model(w0, _plan(w0))
    assert wm0["compress_flops"] == 0 and wm0["compress_bytes_alg"] == 0
    assert wm0["decode_bytes_alg"] == 4 * 2 * 90 * 128 + 2 * 2 * 2 * 128


def test_config_dict_is_shared_by_both_arms():
    """Both arms print config_dict(workload, world): the same keys and values."""
    w = wl.LLAMA3_8B_GQA_32K
    c = bench.config_dict(w, 1)
    assert c == bench.config_dict(w, 1)
    assert c["dims_compressed_per_head"] == [64, 96] and c["workload"] == w.name
    assert bench.config_dict(wl.LLAMA2_7B_MHA_32K)["dims_compressed_per_head"] == 96
    assert bench.config_dict(wl.SINGLE_HEAD_2K)["l2"].startswith("inputs fit in L2")
    assert "reference" not in c and c["parallelism"] == "replica x1"


def test_launches_per_step_each_path():
    """6 launches on every path with a middle span and sink / recent rows: basis table,
    sink / recent copy, projection; then prologue (carrying the sink / recent rows on the
    tensor-core and warp-MMA paths), split kernel (carrying them on the CUDA-core path) and
    combine. The split kernel each workload takes is the library's documented choice."""
    tc = wl.LLAMA2_7B_MHA_32K
    cl = wl.LLAMA3_8B_GQA_128K
    cc = wl.llama3_8b_layer(1, 8192, 0)
    hm = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=3, Hq=4, Hkv=4, L=2000, k=511)   # G = 1, k = 511
    kinds = {w.name + str(w.B): fa.fa_decode_describe(_plan(w), 1) for w in (tc, cl, cc, hm)}
    assert kinds[tc.name + "8"].split_kernel == 2 and _plan(tc).e_token_major == 1
    assert kinds[cl.name + "4"].split_kernel == 4 and kinds[cl.name + "4"].cluster == 4
    assert kinds[cc.name + "1"].split_kernel == 1
    assert kinds[hm.name + "3"].split_kernel == 3
    for w in (tc, cl, cc, hm):
        assert bench.launches_per_step(w, _plan(w)) == 6
    # no middle span: basis table, sink / recent copy, the split kernel with the sink /
    # recent rows, combine
    w0 = wl.shrink(tc, B=1, Hq=2, Hkv=2, L=90)
    assert fa.fa_decode_describe(_plan(w0), 1).split_kernel == 0
    assert bench.launches_per_step(w0, _plan(w0)) == 4


def test_cluster_decode_needs_three_quarter_full_head_sets():
    """The cluster kernel serves sets of 128 query heads at about the same cost however many
    are valid, so plans whose sets are less than three quarters full take the warp-MMA kernel:
    32 and 64 query heads (k = 511 and 1023, G = 4) go to warp MMA, 96 and 128 to the cluster
    kernel, 160 (1.25 sets) to warp MMA, 192 (1.5 sets) to the cluster kernel."""
    for base, cluster in ((wl.LLAMA3_8B_GQA_32K, 2), (wl.LLAMA3_8B_GQA_128K, 4)):
        for B, kind in ((1, 3), (2, 3), (3, 4), (4, 4), (5, 3), (6, 4)):
            info = fa.fa_decode_describe(_plan(wl.shrink(base, B=B)), 1)
            assert info.split_kernel == kind, (base.name, B, info.split_kernel)
            assert info.cluster == (cluster if kind == 4 else 1)


def test_append_bytes_by_hand():
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=2, Hkv=4, Hq=4, L=5000)
    mask = np.zeros((4, 128), dtype=np.uint8)
    mask[:, :96] = 1                                  # dc = 96, de = 32 in every head
    p = _plan(w, mask)
    per = 2 * 255 * 96 * 4 + 32 * 2 + 3 * 256
    assert bench.append_bytes(p) == 2 * 2 * 4 * per
