"""Writes tests/golden/c_abi_gpu_case.txt: the expected results of the plain-C GPU program
tests/c_abi_gpu.c, computed by the fp64 oracle alone.

Inputs are drawn by SplitMix64 (workloads.grid_values), which the C program reimplements
from the same published definition, so neither side reads the other's numbers:
    element i of K, V or q (row-major [B][Hkv][L][128], [B][Hkv][L][128], [B][Hq][128])
    = (signed top byte of SplitMix64 output i from the tensor's seed) / 64.
Dim mask: KV head 0 compresses the dims d with d % 4 != 0 (96 dims), KV head 1 the dims
d < 64 (64 dims).

Run from the repository root:  python tests/golden/make_c_abi_gpu_case.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402
from oracle import fourier_oracle as fo  # noqa: E402

B, HQ, HKV, D, L, S, R, K = 2, 4, 2, 128, 600, 8, 40, 31
SEED_K, SEED_V, SEED_Q = 0x0123456789ABCDEF, 0x0FEDCBA987654321, 0x00C0FFEE12345678
G = HQ // HKV
C_HEAD = (1, 1)  # (b, g) whose coefficients are stored


def mask():
    m = np.zeros((HKV, D), dtype=np.uint8)
    m[0] = (np.arange(D) % 4 != 0)
    m[1] = (np.arange(D) < 64)
    return m


def compute():
    """(decode output [B][Hq][128], {"K": C_K, "V": C_V} of head C_HEAD) from the oracle."""
    Kx = wl.grid_values(SEED_K, B * HKV * L * D).reshape(B, HKV, L, D)
    Vx = wl.grid_values(SEED_V, B * HKV * L * D).reshape(B, HKV, L, D)
    q = wl.grid_values(SEED_Q, B * HQ * D).reshape(B, HQ, D)
    m = mask()
    out = np.zeros((B, HQ, D))
    coef = {}
    for b in range(B):
        for g in range(HKV):
            hk = fo.compress(Kx[b, g], m[g], S, R, K)
            hv = fo.compress(Vx[b, g], m[g], S, R, K)
            out[b, g * G:(g + 1) * G] = fo.decode(q[b, g * G:(g + 1) * G], hk, hv)
            if (b, g) == C_HEAD:
                coef = {"K": hk.C, "V": hv.C}
    return out, coef


def main():
    out, coef = compute()
    path = os.path.join(ROOT, "tests", "golden", "c_abi_gpu_case.txt")
    with open(path, "w") as fh:
        fh.write("# Expected results of tests/c_abi_gpu.c, written by tests/golden/make_c_abi_gpu_case.py\n")
        fh.write("# from the fp64 oracle (oracle/fourier_oracle.py: compress and decode) on SplitMix64\n")
        fh.write("# grid inputs; see that script for the input recipe.\n")
        fh.write(f"shape {B} {HQ} {HKV} {D} {L} {S} {R} {K}\n")
        fh.write(f"seeds {SEED_K} {SEED_V} {SEED_Q}\n")
        fh.write(f"out {out.size}\n")
        fh.write("\n".join(f"{v:.12g}" for v in out.ravel()) + "\n")
        for which in ("K", "V"):
            c = coef[which]
            fh.write(f"coef {which} {C_HEAD[0]} {C_HEAD[1]} {c.shape[0]} {c.shape[1]}\n")
            fh.write("\n".join(f"{v:.12g}" for v in c.ravel()) + "\n")
    print(path, out.size, coef["K"].shape, coef["V"].shape)


if __name__ == "__main__":
    main()
