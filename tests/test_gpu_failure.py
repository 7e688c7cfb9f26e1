"""The failure path of the bounded device-side waits, exercised without a
fault or a hang: a self-test kernel waits, with a short limit, on a device
barrier that nothing arrives on.  The kernel must return by itself, the
status check must report the timeout once and then be clear again, and the
next ordinary call on the same handle (with a shortened but ample wait limit)
must still match the oracle."""
import time

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_common import bf16_round, inputs, rel_l2
from video_dit_sparse_da2_b200 import da2

pytestmark = pytest.mark.gpu


def test_wait_timeout_reported_and_context_usable():
    B, H, d, F, Hv, Wv = 1, 2, 64, 4, 16, 16
    m = da2.DA2(B, H, d, F, Hv, Wv)
    assert m.status() == da2.OK
    limit_ns = 2_000_000  # 2 ms
    t0 = time.perf_counter()
    m.selftest_wait_timeout(limit_ns)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    # the second warp's own limit is 2 s: returning well before it shows that
    # it stopped on the first warp's abort flag
    assert dt < 0.5, dt
    assert m.status() == da2.ERR_TIMEOUT
    assert m.status() == da2.OK  # the flag was cleared by the first check

    # a short limit that no legitimate wait reaches, then an ordinary call
    m.set_wait_limit(200_000_000)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    out, _, _ = m.forward(q.cuda(), k.cuda(), v.cuda(), 2500, 2500, 0.2)
    torch.cuda.synchronize()
    assert m.status() == da2.OK
    _, _, _, ref = O.run(q, k, v, F, Hv, Wv, 2500, 2500, 0.2)
    got = out.double().cpu().numpy()
    r16 = bf16_round(ref)
    assert rel_l2(got, r16) <= 2e-3 and np.abs(got - r16).max() <= 1e-2
    m.set_wait_limit(0)
    m.close()


def test_selftest_rejects_bad_limits():
    m = da2.DA2(1, 1, 64, 1, 8, 8)
    for ns in (0, 2_000_000_000):
        assert da2.lib().da2_selftest_wait_timeout(m.handle, ns, None) == da2.ERR_ARG
    m.close()
