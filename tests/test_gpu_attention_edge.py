"""GPU parity of the attention kernel on inputs that stress its exactness
rules: peaky score distributions (many running-max increases, weights near
the e4m3 / e2m1 saturation), integer-valued inputs (exact ties in the scores
and in the weights), and all-zero value or key tensors.  Bar: relative L2 <=
2e-3 against the oracle rounded to bf16, and max-abs <= 1e-2 times the
largest output magnitude (at least 1: outputs of a peaky softmax approach
single value entries, where one bf16 step exceeds 1e-2)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_common import bf16_round, gpu_run, inputs, rel_l2

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS = 1e-2

SHAPES = {"tiny": (1, 2, 64, 4, 16, 16), "ragged128": (2, 3, 128, 3, 9, 13)}


def _check(res, q, k, v, F, Hv, Wv, bp8, bp4):
    _, _, _, ref = O.run(q, k, v, F, Hv, Wv, bp8, bp4, 0.2)
    ref16 = bf16_round(ref)
    got = res["out"]
    err = rel_l2(got, ref16)
    mx = np.abs(got - ref16).max()
    bound = MAX_ABS * max(1.0, float(np.abs(ref16).max()))
    assert err <= REL_L2 and mx <= bound, (err, mx, bound)
    return ref16


def _bf16(x):
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("bp", [(2500, 2500), (1000, 3000), (0, 10000)])
def test_attention_peaky_scores(name, bp):
    B, H, d, F, Hv, Wv = SHAPES[name]
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    q, k = _bf16(q.float() * 4.0), _bf16(k.float() * 4.0)
    res = gpu_run(B, H, d, F, Hv, Wv, *bp, qkv=(q, k, v))
    _check(res, q, k, v, F, Hv, Wv, *bp)


@pytest.mark.parametrize("bp", [(2500, 2500), (0, 10000), (10000, 0)])
def test_attention_integer_inputs(bp):
    B, H, d, F, Hv, Wv = SHAPES["tiny"]
    q, k, v = inputs(B, H, d, F, Hv, Wv, seed=1)
    q, k, v = (_bf16(torch.clamp(torch.round(t.float()), -2, 2)) for t in (q, k, v))
    res = gpu_run(B, H, d, F, Hv, Wv, *bp, qkv=(q, k, v))
    _check(res, q, k, v, F, Hv, Wv, *bp)


def test_attention_zero_values():
    B, H, d, F, Hv, Wv = SHAPES["ragged128"]
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    v = torch.zeros_like(v)
    res = gpu_run(B, H, d, F, Hv, Wv, 2500, 2500, qkv=(q, k, v))
    assert np.all(res["out"] == 0.0)
    _check(res, q, k, v, F, Hv, Wv, 2500, 2500)


def test_attention_zero_keys_uniform_weights():
    B, H, d, F, Hv, Wv = SHAPES["tiny"]
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    k = torch.zeros_like(k)
    res = gpu_run(B, H, d, F, Hv, Wv, 2500, 2500, qkv=(q, k, v))
    _check(res, q, k, v, F, Hv, Wv, 2500, 2500)


@pytest.mark.parametrize("bp", [(10000, 0), (0, 10000), (2500, 2500)])
def test_attention_saturated_weights(bp):
    # zero keys (every p = 1) and every V tile at the head maximum: the FP8
    # weights sit at the largest e4m3 value and the NVFP4 group scales at the
    # largest ue4m3 value, with e2m1 codes 6
    B, H, d, F, Hv, Wv = SHAPES["tiny"]
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    k = torch.zeros_like(k)
    v = v.clone()
    st, na = O.slot_tokens(F, Hv, Wv)
    for a in range(len(na)):
        v[:, :, st[a * 64], 0] = 8.0
    res = gpu_run(B, H, d, F, Hv, Wv, *bp, qkv=(q, k, v))
    _check(res, q, k, v, F, Hv, Wv, *bp)
