"""The second, structured input set (seed 1): deterministic, the smooth field
on Q and K only, and a draft map far from uniform, which is what the set is for.
The oracle (not the GPU path) computes the draft map here."""
import numpy as np
import torch

from oracle import oracle as O
from video_dit_sparse_da2_b200.inputs import make_qkv, make_qkv_structured

F, HV, WV = 4, 16, 16


def test_structured_set_is_deterministic_and_v_is_the_iid_draw():
    q1, k1, v1 = make_qkv_structured(1, 2, 64, F, HV, WV)
    q2, k2, v2 = make_qkv_structured(1, 2, 64, F, HV, WV)
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    # V carries no field: it is the third tensor of the same seeded i.i.d. draw
    _, _, v0 = make_qkv(1, 2, F * HV * WV, 64, seed=1)
    assert torch.equal(v1, v0)


def test_prefix_tokens_carry_no_field():
    P = 40
    q, k, _ = make_qkv_structured(1, 2, 64, F, HV, WV, P=P)
    q0, k0, _ = make_qkv(1, 2, P + F * HV * WV, 64, seed=1)
    assert torch.equal(q[:, :, :P], q0[:, :, :P]) and torch.equal(k[:, :, :P], k0[:, :, :P])
    assert not torch.equal(q[:, :, P:], q0[:, :, P:])


def test_structured_draft_map_is_far_from_uniform():
    # rows of A sum to 1 over R keys; with the smooth field the entries spread
    # much further from 1/R than with the i.i.d. draw of the same seed
    qi, ki, vi = make_qkv(1, 2, F * HV * WV, 64, seed=1)
    qs, ks, vs = make_qkv_structured(1, 2, 64, F, HV, WV)
    Ai = O.draft(O.prepare(qi, ki, vi, F, HV, WV).desc, 0.2)
    As = O.draft(O.prepare(qs, ks, vs, F, HV, WV).desc, 0.2)
    assert np.allclose(As.sum(-1), 1.0)
    assert As.std() > 1.5 * Ai.std()
    assert As.min() < 0.6 * Ai.min()
