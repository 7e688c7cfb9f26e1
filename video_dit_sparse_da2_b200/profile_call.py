"""One call of the path on a named synthetic workload, for profilers.

    python -m video_dit_sparse_da2_b200.profile_call [workload]

Runs prepare + plan + attention once (inside `forward`) and attention once more
on cuda:0, synchronizes, checks the device status word and prints "ok".  Under
ncu, select kernels with -k / -s / -c as usual.
"""
import sys

import torch

from . import da2
from .inputs import BY_NAME, workload_qkv


def main(argv=None) -> None:
    argv = sys.argv[1:] if argv is None else argv
    w = BY_NAME[argv[0] if argv else "wan2.1-1.3b-480p"]
    q, k, v = (t.cuda() for t in workload_qkv(w))
    m = da2.DA2(w.B, w.H, w.d, w.F, w.Hv, w.Wv, w.P)
    out, prep, plan = m.forward(q, k, v, w.bp8, w.bp4, w.lam)
    m.attention(prep, plan, out)
    torch.cuda.synchronize()
    m.check_status()
    m.close()
    print("ok")


if __name__ == "__main__":
    main()
