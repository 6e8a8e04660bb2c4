"""C-ABI checks that need no GPU: exports, host-side plan derivation, argument rejection.

Only host code runs here (fa_plan_init is a pure host function; the other entry points
are called with arguments the host-side validation rejects before any CUDA call).
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import fourier_basis_attention_b200 as fa
import workloads as wl
from oracle import fourier_oracle as fo

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fourier_attention.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(fa_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert set(names) == set(fa.EXPORTED), names
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(fa.LIB, n)


def test_plan_struct_matches_header_layout(tmp_path):
    """The ctypes mirrors have the C layout of the header: gcc compiles the header and
    prints sizeof and every field's offsetof, which must equal the ctypes ones."""
    structs = {"fa_shape": fa.fa_shape, "fa_plan": fa.fa_plan, "fa_cache": fa.fa_cache,
               "fa_decode_info": fa.fa_decode_info}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "fourier_attention.h"',
             "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} sizeof %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    include = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c11", "-I", include, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for line in out:
        if line.strip():
            name, field, value = line.split()
            got[(name, field)] = int(value)
    for name, cls in structs.items():
        assert got[(name, "sizeof")] == ctypes.sizeof(cls), name
        for field, _ in cls._fields_:
            assert got[(name, field)] == getattr(cls, field).offset, (name, field)


@pytest.mark.parametrize("w", wl.CONFIGS + [wl.llama3_8b_layer(64, 131072, 5)], ids=lambda w: w.name)
def test_plan_partition_and_dims_bit_exact(w):
    m = wl.dim_mask(w)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, m)
    assert (p.S, p.R, p.M) == fo.partition(w.L, w.S, w.R)
    for g in range(w.Hkv):
        cd, ed = fa.perm_lists(p, g)
        ocd, oed = fo.split_dims(m[g])
        assert np.array_equal(cd, ocd) and np.array_equal(ed, oed)
        assert p.dc[g] == len(ocd) and p.de[g] == len(oed)


def test_plan_layout_offsets():
    w = wl.LLAMA3_8B_GQA_32K
    m = wl.dim_mask(w)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, m)
    e, c = 0, 0
    for g in range(w.Hkv):
        assert p.e_off[g] == e and p.c_off[g] == c
        assert p.de_ld[g] % 8 == 0 and p.dc_ld[g] % 8 == 0
        e += p.M * p.de_ld[g]
        c += w.k * p.dc_ld[g]
    assert p.e_batch == e and p.c_batch == c
    assert p.e_elems == w.B * e and p.c_elems == w.B * c
    assert p.f_elems == w.B * w.Hkv * (w.S + w.R) * 128
    assert p.phi_ld % 8 == 0 and p.phi_ld >= p.M


@pytest.mark.parametrize("L,S,R", [(1, 32, 64), (50, 32, 64), (96, 32, 64), (97, 32, 64),
                                   (10, 0, 0), (10, 20, 0), (10, 0, 20)])
def test_plan_edge_partitions(L, S, R):
    p = fa.fa_plan_init(1, 1, 1, L, S, R, 1, np.ones((1, 128)))
    assert (p.S, p.R, p.M) == fo.partition(L, S, R)
    assert p.kk == (1 if p.M > 0 else 0)


def test_plan_rejections():
    m = np.ones((2, 128))
    with pytest.raises(fa.FaError) as e:
        fa.fa_plan_init(1, 4, 2, 100, 32, 64, 5, m)   # k=5 > M=4
    assert e.value.code == fa.FA_ERR_UNSUPPORTED
    with pytest.raises(fa.FaError) as e:
        fa.fa_plan_init(1, 3, 2, 1000, 32, 64, 5, m)  # Hq % Hkv != 0
    assert e.value.code == fa.FA_ERR_INVALID
    with pytest.raises(fa.FaError) as e:
        fa.fa_plan_init(1, 4, 2, 1000, 32, 64, 0, m)  # k = 0
    assert e.value.code == fa.FA_ERR_INVALID
    with pytest.raises(fa.FaError) as e:
        fa.fa_plan_init(1, 4, 2, 1000, 32, 64, 5, np.ones((2, 64)), D=64)
    assert e.value.code == fa.FA_ERR_UNSUPPORTED
    with pytest.raises(fa.FaError):
        fa.fa_plan_init(1, 130, 65, 1000, 32, 64, 5, np.ones((65, 128)))
    # k > M is fine when nothing is compressed
    p = fa.fa_plan_init(1, 4, 2, 100, 32, 64, 5, np.zeros((2, 128)))
    assert p.M == 4


def test_null_and_misaligned_pointers_rejected_on_host():
    p = fa.fa_plan_init(1, 4, 1, 300, 32, 64, 31, np.ones((1, 128)))
    cache = fa.fa_cache(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    lib = fa.LIB
    r = lib.fa_compress(ctypes.byref(p), None, 0x1000, 0x1000, ctypes.byref(cache), None)
    assert r == fa.FA_ERR_INVALID and "K" in fa.fa_last_error()
    r = lib.fa_compress(ctypes.byref(p), 0x1008, 0x1000, 0x1000, ctypes.byref(cache), None)
    assert r == fa.FA_ERR_INVALID and "aligned" in fa.fa_last_error()
    r = lib.fa_decode(ctypes.byref(p), 0x1000, ctypes.byref(cache), None, fa.FA_BF16, 0x1000,
                      1 << 20, 4, None)
    assert r == fa.FA_ERR_INVALID and "out" in fa.fa_last_error()
    r = lib.fa_decode(ctypes.byref(p), 0x1000, ctypes.byref(cache), 0x1000, 7, 0x1000,
                      1 << 20, 4, None)
    assert r == fa.FA_ERR_INVALID and "out_dtype" in fa.fa_last_error()
    r = lib.fa_build_basis(100, 101, fa.FA_BF16, 0, 0x1000, 104, None)
    assert r == fa.FA_ERR_INVALID
    r = lib.fa_build_basis(100, 10, fa.FA_BF16, 0, 0x1000, 100, None)  # ld not a multiple of 8
    assert r == fa.FA_ERR_INVALID
    # a corrupted plan is rejected before any launch
    bad = fa.fa_plan_init(1, 4, 1, 300, 32, 64, 31, np.ones((1, 128)))
    bad.perm[0][5] = bad.perm[0][6]
    r = lib.fa_compress(ctypes.byref(bad), 0x1000, 0x1000, 0x1000, ctypes.byref(cache), None)
    assert r == fa.FA_ERR_INVALID and "perm" in fa.fa_last_error()


def test_decode_rejects_unsupported_group_and_k():
    p = fa.fa_plan_init(1, 3, 1, 300, 32, 64, 31, np.ones((1, 128)))  # G = 3
    assert fa.fa_decode_workspace_size(p, 4) == 0
    p = fa.fa_plan_init(1, 4, 1, 5000, 32, 64, 2049, np.ones((1, 128)))
    assert fa.fa_decode_workspace_size(p, 4) == 0
    p = fa.fa_plan_init(1, 4, 1, 5000, 32, 64, 2047, np.ones((1, 128)))
    assert fa.fa_decode_workspace_size(p, 4) > 0


def test_decode_rejects_too_many_sink_recent_records():
    """S + R so large that the combine's sink/recent record weights alone fill its shared
    memory: the size query answers 0 and both decode entry points return
    FA_ERR_UNSUPPORTED with the reason (host checks only; nothing is launched)."""
    p = fa.fa_plan_init(1, 8, 1, 32 + 460000 + 2048, 32, 460000, 1023, np.ones((1, 128)))
    assert p.M == 2048
    assert fa.fa_decode_workspace_size(p, 1) == 0
    cache = fa.fa_cache(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    r = fa.LIB.fa_decode(ctypes.byref(p), 0x1000, ctypes.byref(cache), 0x1000, fa.FA_F32,
                         0x1000, 1 << 30, 1, None)
    assert r == fa.FA_ERR_UNSUPPORTED and "sink + recent" in fa.fa_last_error()
    r = fa.LIB.fa_decode_noalloc(ctypes.byref(p), 0x1000, ctypes.byref(cache), 0x1000,
                                 fa.FA_F32, 1, None)
    assert r == fa.FA_ERR_UNSUPPORTED and "sink + recent" in fa.fa_last_error()


def test_workspace_size_formula():
    w = wl.LLAMA2_7B_MHA_32K
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, wl.dim_mask(w))
    F = w.k // 2 + 1
    F_pad = (F + 3) // 4 * 4
    ns = 37
    ntiles = (p.M + 63) // 64
    per = -(-ntiles // ns)
    ns_eff = -(-ntiles // per)
    n_rec = ns_eff + 1  # one sink/recent split (S + R = 96 rows)
    bhq = w.B * w.Hq
    expect = bhq * (128 + 2 * F_pad) * 4 + n_rec * bhq * (4 + 128 + 2 * F_pad) * 4
    assert fa.fa_decode_workspace_size(p, ns) == expect


def test_gpu_test_shapes_have_valid_plans():
    """Every workload the GPU parity tests and smoke() use must pass fa_plan_init."""
    import __graft_entry__  # noqa: F401
    import test_gpu_parity as tg
    shapes = list(tg.SMALL) + list(tg.FULL)
    shapes.append(wl.shrink(wl.LLAMA3_8B_GQA_32K, B=1, Hq=8, Hkv=2, L=2000))
    shapes.append(tg.TC_BASE)
    shapes.append(tg.TC_WIDE)
    for _, k in tg.TC_RAGGED:
        shapes.append(tg._ragged_shape(k))
    for w in shapes:
        fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, wl.dim_mask(w))


# ----------------------------------------------------------------------------- E layout

@pytest.mark.parametrize("w,token_major", [
    (wl.SINGLE_HEAD_2K, False),                   # k = 63, G = 4: k G < 255
    (wl.LLAMA2_7B_MHA_32K, True),                 # k = 255, G = 1, 256 query heads
    (wl.LLAMA3_8B_GQA_32K, False),                # k = 511
    (wl.LLAMA3_8B_GQA_128K, False),               # k = 1023
    (wl.llama3_8b_layer(8, 8192, 2), False),      # k = 63
    (wl.llama3_8b_layer(8, 32768, 2), True),      # k = 255, G = 4, 256 query heads
    (wl.llama3_8b_layer(2, 32768, 2), False),     # 64 query heads
    (wl.llama3_8b_layer(8, 131072, 2), False),    # k = 1023
], ids=lambda x: getattr(x, "name", str(x)))
def test_token_major_choice(w, token_major):
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, wl.dim_mask(w))
    assert bool(p.e_token_major) == token_major
    if token_major:
        width = p.de_ld[0]
        assert width == 32 and all(p.de_ld[g] == width for g in range(w.Hkv))
        for g in range(w.Hkv):
            assert p.e_off[g] == g * width and p.e_pitch[g] == w.Hkv * width
        assert p.e_batch == p.M * w.Hkv * width
    else:
        off = 0
        for g in range(w.Hkv):
            assert p.de_ld[g] == (p.de[g] + 7) // 8 * 8 and p.e_pitch[g] == p.de_ld[g]
            assert p.e_off[g] == off
            off += p.M * p.de_ld[g]
        assert p.e_batch == off
    assert p.e_elems == w.B * p.e_batch


@pytest.mark.parametrize("retained,G,k,B,expect", [
    ([5, 1, 3, 8], 4, 127, 8, 8), ([12, 9, 16, 0], 4, 255, 8, 16),
    ([31, 17, 2, 20], 2, 255, 16, 32), ([0, 0, 0, 0], 4, 127, 8, 0),
    ([33, 1, 1, 1], 4, 255, 8, None), ([8, 8, 8, 8], 8, 63, 8, None),
    ([8, 8, 8, 8], 4, 257, 8, None), ([8, 8, 8, 8], 4, 63, 8, None),
    ([8, 8, 8, 8], 4, 127, 7, None), ([8, 8, 8, 8], 1, 255, 32, 8),
    ([8, 8, 8, 8], 2, 127, 16, None), ([8, 8, 8, 8], 4, 63, 64, 8),
    ([8, 8, 8, 8], 2, 127, 128, 8), ([8, 8, 8, 8], 4, 63, 63, None)])
def test_token_major_width(retained, G, k, B, expect):
    """Width = the smallest of 8, 16, 32 holding every KV head's retained dims; blocked
    (None) past 32 dims, for G = 8, for k > 255, for fewer than 128 query heads, and for
    k G < 255 unless there are at least 1024 query heads."""
    Hkv = 4
    mask = np.ones((Hkv, 128), dtype=np.uint8)
    for g, r in enumerate(retained):
        mask[g, :r] = 0
    p = fa.fa_plan_init(B, Hkv * G, Hkv, 1000, 32, 64, k, mask)
    if expect is None:
        assert p.e_token_major == 0
    else:
        assert p.e_token_major == 1 and all(p.de_ld[g] == expect for g in range(Hkv))
        assert [p.de[g] for g in range(Hkv)] == retained


def test_hand_edited_layout_is_rejected():
    w = wl.llama3_8b_layer(8, 32768, 2)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, wl.dim_mask(w))
    for field, value in (("e_token_major", 0), ("e_pitch", None), ("e_off", None)):
        q = fa.fa_plan.from_buffer_copy(p)
        if value is None:
            getattr(q, field)[1] += 8
        else:
            setattr(q, field, value)
        assert fa.LIB.fa_decode_workspace_size(ctypes.byref(q), 1) == 0, field
        cache = fa.fa_cache(*([0x1000] * 6))
        rc = fa.LIB.fa_compress(ctypes.byref(q), 0x1000, 0x1000, 0x1000, ctypes.byref(cache), None)
        assert rc == fa.FA_ERR_INVALID and "layout" in fa.fa_last_error(), field


# ----------------------------------------------------------------------------- append (host side)

def test_reserve_sets_period_and_sizes_e_by_capacity():
    w = wl.llama3_8b_layer(2, 4096, 3)
    m = wl.dim_mask(w)
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, m)
    assert p.P == p.M and p.recent_head == 0
    e0, c0, f0 = p.e_elems, p.c_elems, p.f_elems
    fa.fa_plan_reserve(p, w.L + 1000)
    assert p.P == p.M + 1000 and p.phi_ld == (p.P + 7) // 8 * 8
    assert p.c_elems == c0 and p.f_elems == f0          # k coefficients and S + R rows: fixed
    assert p.e_elems * p.M == e0 * p.P                  # E holds P rows per KV head
    # the layout choice does not depend on the period
    q = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, m)
    assert p.e_token_major == q.e_token_major and list(p.de_ld) == list(q.de_ld)
    assert fa.fa_decode_workspace_size(p, 4) > 0


def test_reserve_and_append_rejections():
    m = np.ones((1, 128))
    p = fa.fa_plan_init(1, 4, 1, 300, 32, 64, 31, m)
    for L_max in (299, 32 + 64 + (1 << 21)):
        with pytest.raises(fa.FaError) as e:
            fa.fa_plan_reserve(fa.fa_plan.from_buffer_copy(p), L_max)
        assert e.value.code == fa.FA_ERR_INVALID
    q = fa.fa_plan.from_buffer_copy(p)
    fa.fa_plan_reserve(q, 400)
    with pytest.raises(fa.FaError) as e:                 # reserved twice
        fa.fa_plan_reserve(q, 500)
    assert e.value.code == fa.FA_ERR_UNSUPPORTED
    with pytest.raises(fa.FaError) as e:                 # no middle span
        fa.fa_plan_reserve(fa.fa_plan_init(1, 4, 1, 90, 32, 64, 31, m), 400)
    assert e.value.code == fa.FA_ERR_UNSUPPORTED
    cache = fa.fa_cache(*([0x1000] * 6))
    lib = fa.LIB
    # no room: P == M (a plan straight from fa_plan_init); nothing is launched
    r = lib.fa_append(ctypes.byref(p), 0x1000, 0x1000, ctypes.byref(cache), None)
    assert r == fa.FA_ERR_UNSUPPORTED and "room" in fa.fa_last_error()
    assert p.M == 204 and p.shape.L == 300
    r = lib.fa_append(ctypes.byref(q), None, 0x1000, ctypes.byref(cache), None)
    assert r == fa.FA_ERR_INVALID and "k_new" in fa.fa_last_error()
    r = lib.fa_append(ctypes.byref(q), 0x1000, 0x1008, ctypes.byref(cache), None)
    assert r == fa.FA_ERR_INVALID and "aligned" in fa.fa_last_error()
    assert q.M == 204 and q.recent_head == 0            # failed calls leave the plan alone


def test_hand_edited_period_or_ring_is_rejected():
    m = np.ones((1, 128))
    p = fa.fa_plan_init(1, 4, 1, 300, 32, 64, 31, m)
    fa.fa_plan_reserve(p, 400)
    cache = fa.fa_cache(*([0x1000] * 6))
    for field, value, word in (("P", 200, "period"), ("recent_head", 64, "recent_head"),
                               ("recent_head", -1, "recent_head"), ("phi_ld", 208, "phi_ld")):
        q = fa.fa_plan.from_buffer_copy(p)
        setattr(q, field, value)
        rc = fa.LIB.fa_compress(ctypes.byref(q), 0x1000, 0x1000, 0x1000, ctypes.byref(cache), None)
        assert rc == fa.FA_ERR_INVALID and word in fa.fa_last_error(), field
        assert fa.LIB.fa_decode_workspace_size(ctypes.byref(q), 1) == 0


# ----------------------------------------------------------------------------- dim selection

def test_select_dims_matches_oracle():
    rng = np.random.default_rng(11)
    for trial in range(20):
        Hkv = int(rng.integers(1, 9))
        sc = rng.integers(0, 40, size=(Hkv, 128)).astype(np.float32)   # ties
        if trial % 5 == 0:
            sc[0, rng.integers(0, 128, 3)] = np.nan
        nc = int(rng.integers(0, 129))
        got = fa.fa_select_dims(sc, nc)
        for g in range(Hkv):
            assert np.array_equal(got[g], fo.select_dims(sc[g].astype(np.float64), nc)), (trial, g)


def test_select_dims_rejections():
    with pytest.raises(fa.FaError):
        fa.fa_select_dims(np.zeros((2, 128)), 129)
    with pytest.raises(fa.FaError):
        fa.fa_select_dims(np.zeros((65, 128)), 3)
    shape = fa.fa_shape(1, 3, 1, 128, 100, 0, 0, 1)          # G = 3: no decode kernel
    assert fa.LIB.fa_dim_sensitivity_workspace_size(ctypes.byref(shape)) == 0
    r = fa.LIB.fa_dim_sensitivity(ctypes.byref(shape), 0x1000, 0x1000, 0x1000, 0x1000, 0x1000,
                                  1 << 20, None)
    assert r == fa.FA_ERR_UNSUPPORTED


def test_c_program_uses_the_abi(tmp_path):
    """A plain C program (gcc, no C++ or torch) links the library and runs the host-only
    entry points: plan, reservation, append refusal, dim selection."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = tmp_path / "c_abi_host"
    libdir = os.path.dirname(fa.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "c_abi_host.c"), "-o", str(exe),
                    "-L", libdir, "-lfourier_attention", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr


# ----------------------------------------------------------------------------- layout properties

from hypothesis import given, settings, strategies as st


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 40), Hkv=st.sampled_from([1, 2, 4, 8]), G=st.sampled_from([1, 2, 4, 8]),
       L=st.integers(1, 3000), S=st.integers(0, 40), R=st.integers(0, 80),
       k=st.integers(1, 300), extra=st.integers(0, 500), seed=st.integers(0, 2 ** 31 - 1))
def test_plan_layout_properties(B, Hkv, G, L, S, R, k, extra, seed):
    """Every plan the host derives (with or without reserved room) has disjoint, in-bounds
    E and C blocks, the documented token-major rule, padded row widths and sorted dim lists."""
    rng = np.random.default_rng(seed)
    mask = (rng.random((Hkv, 128)) < rng.random()).astype(np.uint8)
    Hq = Hkv * G
    try:
        p = fa.fa_plan_init(B, Hq, Hkv, L, S, R, k, mask)
    except fa.FaError as e:
        assert e.code == fa.FA_ERR_UNSUPPORTED and k > L - min(S, L) - min(R, L - min(S, L))
        return
    if p.M > 0 and extra > 0:
        fa.fa_plan_reserve(p, L + extra)
    assert p.S + p.M + p.R == L and p.P >= p.M
    assert p.f_elems == B * Hkv * (p.S + p.R) * 128
    de = [p.de[g] for g in range(Hkv)]
    tm = (p.M > 0 and k <= 255 and G in (1, 2, 4) and max(de) <= 32
          and ((k * G >= 255 and B * Hq >= 128) or B * Hq >= 1024))
    assert p.e_token_major == int(tm)
    for g in range(Hkv):
        cd, ed = fa.perm_lists(p, g)
        assert list(cd) == sorted(cd) and list(ed) == sorted(ed)
        assert sorted(list(cd) + list(ed)) == list(range(128))
        assert p.dc_ld[g] % 8 == 0 and p.dc_ld[g] >= p.dc[g]
        assert p.de_ld[g] >= p.de[g] and (p.de_ld[g] == 0 or p.de_ld[g] % 8 == 0)
    # E: element intervals [start, start + de_ld) of every (b, g, t < P) row are disjoint and
    # inside e_elems; C: the [kk][dc_ld] blocks likewise inside c_elems
    rows = []
    for b in range(min(B, 3)):
        for g in range(Hkv):
            if p.de_ld[g] == 0:
                continue
            for t in {t for t in (0, 1, p.P // 2, p.P - 1) if 0 <= t < p.P}:
                start = b * p.e_batch + p.e_off[g] + t * p.e_pitch[g]
                rows.append((start, start + p.de_ld[g]))
    rows.sort()
    for (a0, a1), (b0, _) in zip(rows, rows[1:]):
        assert a1 <= b0
    if rows:
        assert rows[0][0] >= 0 and max(r[1] for r in rows) <= p.e_elems
    blocks = sorted((b * p.c_batch + p.c_off[g], b * p.c_batch + p.c_off[g] + p.kk * p.dc_ld[g])
                    for b in range(B) for g in range(Hkv) if p.kk * p.dc_ld[g] > 0)
    for (a0, a1), (b0, _) in zip(blocks, blocks[1:]):
        assert a1 <= b0
    if blocks:
        assert blocks[-1][1] <= p.c_elems


def test_cache_views_on_host_memory():
    """The Cache views follow the documented layouts (checked on CPU tensors; no kernel)."""
    import torch
    w = wl.shrink(wl.LLAMA2_7B_MHA_32K, B=2, Hq=4, Hkv=2, L=400, S=4, R=6, k=15)
    mask = np.zeros((2, 128), dtype=np.uint8)
    mask[:, ::2] = 1                                      # 64 compressed, 64 retained
    p = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    c = fa.Cache(p, device="cpu")
    # F: write each row's token index, then rotate the ring by hand
    F = c.F("K")
    for i in range(p.S + p.R):
        F[:, :, i] = i
    p.recent_head = 2
    got = c.F_tokens("K")[0, 0, :, 0].tolist()
    assert got == [0, 1, 2, 3] + [4 + (2 + a) % 6 for a in range(6)]
    # E: row t of head (b, g) at b * e_batch + e_off[g] + t * e_pitch[g]
    c.E_K.zero_()
    c.E_K[1 * p.e_batch + p.e_off[1] + 7 * p.e_pitch[1] + 3] = 5.0
    assert c.E("K", 1, 1)[7, 3].item() == 5.0 and c.E("K", 1, 1).sum().item() == 5.0
    # C: [kk][dc_ld] block of (b, g), padding columns past dc
    assert c.C("V", 0, 1).shape == (15, 64) and c.C_raw("V", 0, 1).shape == (15, p.dc_ld[1])


def test_c_gpu_program_builds():
    """The plain-C GPU program (run by the -m gpu tests) compiles and links against the
    header, the library and the CUDA runtime."""
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location(
        "gpu_c_program", os.path.join(root, "tests", "test_gpu_c_program.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "c_abi_gpu")
        mod.build_c_program(exe)
        assert os.path.getsize(exe) > 0
