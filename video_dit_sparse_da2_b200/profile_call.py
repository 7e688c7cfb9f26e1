"""One call of the path on a named synthetic workload, for profilers.

    python -m video_dit_sparse_da2_b200.profile_call [workload] [--heads H] [--inputs iid|structured]

Runs prepare + plan + attention once (inside `forward`) and attention once more
on cuda:0, synchronizes, checks the device status word and prints "ok".  With
--heads the workload keeps its frames, budgets and seed but has H heads (a
smaller copy for captures that replay a launch many times).  Under ncu, select
kernels with -k / -s / -c as usual.
"""
import argparse
import dataclasses
import sys

import torch

from . import da2
from .inputs import BY_NAME, workload_qkv


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(prog="profile_call")
    ap.add_argument("workload", nargs="?", default="wan2.1-1.3b-480p", choices=sorted(BY_NAME))
    ap.add_argument("--heads", type=int, default=None)
    ap.add_argument("--inputs", choices=["iid", "structured"], default="iid")
    a = ap.parse_args(sys.argv[1:] if argv is None else argv)
    w = BY_NAME[a.workload]
    if a.heads is not None:
        if a.heads < 1:
            ap.error("--heads must be positive")
        w = dataclasses.replace(w, H=a.heads)
    q, k, v = (t.cuda() for t in workload_qkv(w, structured=a.inputs == "structured"))
    m = da2.DA2(w.B, w.H, w.d, w.F, w.Hv, w.Wv, w.P)
    out, prep, plan = m.forward(q, k, v, w.bp8, w.bp4, w.lam)
    m.attention(prep, plan, out)
    torch.cuda.synchronize()
    m.check_status()
    m.close()
    print("ok")


if __name__ == "__main__":
    main()
