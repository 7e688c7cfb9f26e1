"""GPU parity: the fused preparation kernel against the oracle, bit for bit
(descriptors, FP8 / NVFP4 codes, scale factors, tile scales, V maxima)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_common import SMALL, gpu_run, inputs
from video_dit_sparse_da2_b200 import da2, layouts

pytestmark = pytest.mark.gpu

FIELDS = ("desc", "q8", "k8", "v8t", "s8", "q4", "k4", "v4t", "sfq", "sfk", "sfv", "g4", "vmax")


def _check_prepared(got, ref):
    for f in FIELDS:
        a, b = got[f], getattr(ref, f)
        assert a.shape == b.shape, f
        if a.dtype.kind == "f":
            assert np.array_equal(a.view(np.uint8), np.ascontiguousarray(b).view(np.uint8)), f
        else:
            assert np.array_equal(a, b), (f, np.argwhere(a != b)[:5])


@pytest.mark.parametrize("name", list(SMALL))
def test_prepare_bit_exact_small(name):
    B, H, d, F, Hv, Wv = SMALL[name]
    res = gpu_run(B, H, d, F, Hv, Wv, 2500, 2500)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    _check_prepared(res["prep"], O.prepare(q, k, v, F, Hv, Wv))


def test_prepare_bit_exact_wan13b():
    B, H, d, F, Hv, Wv = 1, 12, 128, 21, 30, 52
    res = gpu_run(B, H, d, F, Hv, Wv, 1000, 3000)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    _check_prepared(res["prep"], O.prepare(q, k, v, F, Hv, Wv))


def test_prepare_strided_input_and_zero_tiles():
    # [B, N, H, d] storage viewed as [B, H, N, d]; one head of V is all zero,
    # so its tiles get scale 0 and zero codes.
    B, H, d, F, Hv, Wv = 1, 3, 64, 3, 9, 13
    q, k, v = inputs(B, H, d, F, Hv, Wv, 5)
    v = v.clone()
    v[:, 1] = 0
    m = da2.DA2(B, H, d, F, Hv, Wv)
    dev = [t.transpose(1, 2).contiguous().cuda().transpose(1, 2) for t in (q, k, v)]
    prep = m.alloc_prepared()
    m.prepare(*dev, prep)
    torch.cuda.synchronize()
    got = layouts.prepared_to_logical(prep.bufs, B, H, m.R, d)
    ref = O.prepare(q, k, v, F, Hv, Wv)
    _check_prepared(got, ref)
    assert not got["v8t"][0, 1].any() and not got["s8"][2, 0, 1].any()
    m.close()


def test_prepare_rejects_bad_strides():
    m = da2.DA2(1, 1, 64, 1, 8, 8)
    x = torch.zeros(1, 1, 64, 72, dtype=torch.bfloat16, device="cuda")[..., 3:67]  # misaligned rows
    prep = m.alloc_prepared()
    with pytest.raises(da2.DA2Error):
        m.prepare(x, x, x, prep)
    m.close()
