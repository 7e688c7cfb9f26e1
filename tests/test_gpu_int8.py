"""GPU parity of the INT8 QK^T path of the 8-bit phase (DraftAttention2 App.
C.1: INT8 for QK^T, FP8 for the probability-value product): the INT8 codes
and tile scales bit for bit against the oracle, and the attention within the
output tolerance, alone and together with the 16-bit tier."""
import numpy as np
import pytest

from oracle import oracle as O
from tests.gpu_common import SMALL, bf16_round, gpu_run, inputs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", list(SMALL))
def test_int8_operands_bit_exact(name):
    B, H, d, F, Hv, Wv = SMALL[name]
    res = gpu_run(B, H, d, F, Hv, Wv, 2500, 2500, int8_qk=True)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    q8i, k8i, si8 = O.prepare_int8(q, k, F, Hv, Wv)
    g = res["prep"]
    assert np.array_equal(g["q8i"], q8i) and np.array_equal(g["k8i"], k8i)
    assert np.array_equal(g["si8"].view(np.uint32), si8.view(np.uint32))


@pytest.mark.parametrize("bp", [(2500, 2500, 0), (10000, 0, 0), (1000, 3000, 0), (1500, 1500, 2000)])
@pytest.mark.parametrize("name", list(SMALL))
def test_int8_qk_attention_within_tolerance(name, bp):
    B, H, d, F, Hv, Wv = SMALL[name]
    bp8, bp4, bp16 = bp
    res = gpu_run(B, H, d, F, Hv, Wv, bp8, bp4, bp16=bp16, int8_qk=True)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    _, _, _, ref = O.run(q, k, v, F, Hv, Wv, bp8, bp4, 0.2, bp16=bp16, int8=True)
    r16 = bf16_round(ref)
    err, mx = rel_l2(res["out"], r16), np.abs(res["out"] - r16).max()
    assert err <= 2e-3 and mx <= 1e-2, (err, mx)
