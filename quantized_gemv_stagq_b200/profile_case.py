"""Run a few GEMV launches of one shape (or stack of shapes) and precision,
for profilers; the command lines of the ncu summaries in profiles/ run it.

  python -m quantized_gemv_stagq_b200.profile_case --shape 14336x4096[,14336x4096] --bits 4 \
      [--copies 5] [--launches 5] [--group 128] [--planes 2] [--density 0.005]
      [--kernel default|general|single] [--n 1]

Several comma-separated shapes with one `in` are loaded as one stacked handle
(stagq_load_stack), as the benchmark loads q/k/v and gate/up. Launches rotate
over `copies` device copies, so with copies x size above the L2 size every
launch reads from HBM. Exits non-zero if y is not finite.
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
    p.add_argument("--n", type=int, default=1, help="activation vectors per launch (1..4)")
    a = p.parse_args()
    flags = {"default": 0, "general": Q.STAGQ_KERNEL_GENERAL, "single": Q.STAGQ_KERNEL_SINGLE}[a.kernel]
    shapes = [tuple(int(v) for v in s.lower().split("x")) for s in a.shape.split(",")]
    if len({i for _, i in shapes}) != 1:
        raise SystemExit("stacked shapes must share `in`")
    streams = [Q.stagq_pack(Q.stagq_encode(synth.weights(o, i, seed=1 + j), a.group, a.planes, a.density, "fast"))
               for j, (o, i) in enumerate(shapes)]
    mats = [Q.stagq_load_stack(streams, 0) for _ in range(a.copies)]
    out, inp = mats[0].out, mats[0].inp
    x = torch.from_numpy(synth.activations(a.n, inp, seed=2)).cuda()
    y = torch.empty(a.n, out, dtype=torch.float16, device="cuda")
    for i in range(a.launches):
        Q.stagq_gemv_ex(mats[i % a.copies], a.bits, x, y, n=a.n, flags=flags)
    torch.cuda.synchronize()
    Q.stagq_check(mats[0])
    if not np.all(np.isfinite(y.float().cpu().numpy())):
        raise SystemExit("non-finite y")
    print(f"{a.launches} launches of {out}x{inp} p{a.bits} n{a.n}: ok; bytes/launch {Q.stagq_bytes(mats[0], a.bits, a.n)}")


if __name__ == "__main__":
    main()
