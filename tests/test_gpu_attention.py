"""GPU parity: the phased FP8 / NVFP4 attention kernel against the oracle
with the same emulated quantization.  Tolerance (stated by the task for
unit-scale inputs): relative L2 <= 2e-3 and max-abs <= 1e-2, comparing the
kernel's bf16 output with the oracle's fp64 output rounded to bf16."""
import numpy as np
import pytest

from oracle import oracle as O
from tests.gpu_common import SMALL, bf16_round, gpu_run, inputs, rel_l2

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS = 1e-2

BUDGETS = [(2500, 2500), (10000, 0), (0, 10000), (1000, 3000), (500, 500), (0, 0), (5000, 5000)]


def _compare(res, q, k, v, F, Hv, Wv, bp8, bp4, lam=0.2):
    prep, A, plan, ref = O.run(q, k, v, F, Hv, Wv, bp8, bp4, lam)
    ref16 = bf16_round(ref)
    got = res["out"]
    err = rel_l2(got, ref16)
    mx = np.abs(got - ref16).max()
    assert err <= REL_L2 and mx <= MAX_ABS, (err, mx)
    # rows with no kept key are exactly zero on both sides
    assert np.array_equal(got == 0, ref16 == 0) or np.all((ref == 0) <= (got == 0))
    return err, mx


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("bp", BUDGETS)
def test_attention_small(name, bp):
    B, H, d, F, Hv, Wv = SMALL[name]
    res = gpu_run(B, H, d, F, Hv, Wv, *bp)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    _compare(res, q, k, v, F, Hv, Wv, *bp)
