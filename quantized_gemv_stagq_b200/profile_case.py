"""Run a few GEMV launches of one shape and precision (for profilers).

  python -m quantized_gemv_stagq_b200.profile_case --shape 14336x4096 --bits 4 \
      [--copies 5] [--launches 5] [--group 128] [--planes 2] [--density 0.005]
      [--kernel default|general|single]

Launches rotate over `copies` device copies of the encoded matrix, so with
copies x size above the L2 size every launch reads from HBM. Exits non-zero if
y is not finite.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

import quantized_gemv_stagq_b200 as Q
from quantized_gemv_stagq_b200 import synth


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--shape", default="14336x4096")
    p.add_argument("--bits", type=int, default=4)
    p.add_argument("--copies", type=int, default=5)
    p.add_argument("--launches", type=int, default=5)
    p.add_argument("--group", type=int, default=128)
    p.add_argument("--planes", type=int, default=2)
    p.add_argument("--density", type=float, default=0.005)
    p.add_argument("--kernel", default="default", choices=["default", "general", "single"])
    a = p.parse_args()
    flags = {"default": 0, "general": Q.STAGQ_KERNEL_GENERAL, "single": Q.STAGQ_KERNEL_SINGLE}[a.kernel]
    out, inp = (int(v) for v in a.shape.lower().split("x"))
    S = Q.stagq_pack(Q.stagq_encode(synth.weights(out, inp, seed=1), a.group, a.planes, a.density, "fast"))
    mats = [Q.stagq_load(S, 0) for _ in range(a.copies)]
    x = torch.from_numpy(synth.activations(1, inp, seed=2)).cuda()
    y = torch.empty(1, out, dtype=torch.float16, device="cuda")
    for i in range(a.launches):
        Q.stagq_gemv_ex(mats[i % a.copies], a.bits, x, y, flags=flags)
    torch.cuda.synchronize()
    if not np.all(np.isfinite(y.float().cpu().numpy())):
        raise SystemExit("non-finite y")
    print(f"{a.launches} launches of {out}x{inp} p{a.bits}: ok; bytes/launch {Q.stagq_bytes(mats[0], a.bits)}")


if __name__ == "__main__":
    main()
