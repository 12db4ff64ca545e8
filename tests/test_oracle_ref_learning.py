"""Pins of the reference-query learning oracle (oracle/ref_learning.py): the
differentiable build against the C oracle's, the loss at points where the tree is
exact, the gradient against finite differences, and that descent lowers it."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import ref_learning as RL

F64 = torch.float64


def _randn(*shape, g):
    return torch.randn(*shape, generator=g, dtype=F64)


def _keys(N, d, seed, blocks=16):
    g = torch.Generator().manual_seed(seed)
    centres = _randn(N // blocks + 1, d, g=g)
    K = centres.repeat_interleave(blocks, dim=0)[:N] + 0.3 * _randn(N, d, g=g)
    return K, centres, g


@pytest.mark.parametrize("N,C,depth,R", [(256, 4, 4, 3), (300, 4, 3, 2), (200, 3, 4, 4)])
def test_build_matches_the_c_oracle(N, C, depth, R):
    d, beta = 8, 0.5
    K, _, g = _keys(N, d, N)
    refs = _randn(R, d, g=g)
    levels = RL.build_levels(K, refs, C, depth, beta)
    t = O.build_tree(K.numpy(), refs.numpy(), C, depth, beta, store=O.STORE_F64)
    for l, (key, bias) in enumerate(levels, start=1):
        ok, ob = t.level(l)
        assert key.shape[0] == t.n_nodes[l]
        np.testing.assert_allclose(key.numpy(), ok, rtol=0, atol=1e-12 * max(1.0, np.abs(ok).max(initial=0)))
        np.testing.assert_allclose(bias.numpy(), ob, rtol=0, atol=1e-12 * max(1.0, np.abs(ob).max(initial=0)))


def test_loss_is_zero_when_the_query_is_a_reference():
    # a summary is exact at its own reference and a lower bound elsewhere, so with
    # the query among the references every node scores the log-mass under it and
    # the tree splits attention exactly as the dense softmax does, at every level
    d, C, depth, beta = 8, 4, 4, 0.7
    K, centres, g = _keys(256, d, 3)
    q = centres[5] * 1.5
    refs = torch.stack([_randn(d, g=g), q, _randn(d, g=g)])
    terms = RL.split_loss(K, refs, q[None], C, depth, beta, per_level=True)
    assert terms.shape == (depth,)
    assert terms.abs().max().item() < 1e-12
    refs = refs.clone().requires_grad_(True)
    (grad,) = torch.autograd.grad(RL.split_loss(K, refs, q[None], C, depth, beta), refs)
    assert grad.abs().max().item() < 1e-9  # a minimum


def test_loss_is_a_divergence():
    d, C, depth, beta = 8, 4, 3, 0.6
    K, centres, g = _keys(200, d, 4)
    Q = centres[torch.randint(0, len(centres), (6,), generator=g)] * 2
    refs = _randn(3, d, g=g)
    terms = RL.split_loss(K, refs, Q, C, depth, beta, per_level=True)
    assert (terms >= -1e-15).all() and terms.sum().item() > 1e-3


def test_gradient_matches_finite_differences():
    d, C, depth, beta = 6, 4, 3, 0.8
    K, centres, g = _keys(128, d, 5)
    Q = centres[torch.randint(0, len(centres), (4,), generator=g)] + 0.2 * _randn(4, d, g=g)
    refs = _randn(3, d, g=g).requires_grad_(True)
    (grad,) = torch.autograd.grad(RL.split_loss(K, refs, Q, C, depth, beta), refs)
    eps = 1e-6
    with torch.no_grad():
        for r in range(3):
            for e in range(d):
                up, dn = refs.clone(), refs.clone()
                up[r, e] += eps
                dn[r, e] -= eps
                fd = (RL.split_loss(K, up, Q, C, depth, beta) - RL.split_loss(K, dn, Q, C, depth, beta)) / (2 * eps)
                assert abs(fd.item() - grad[r, e].item()) <= 1e-6 * max(1.0, abs(fd.item())), (r, e)


def test_descent_lowers_the_loss():
    # the teacher is the dense attention of queries built from block centres
    d, C, depth, beta = 8, 4, 3, 0.5
    K, centres, g = _keys(256, d, 6)
    Q = centres[torch.randint(0, len(centres), (16,), generator=g)] * 1.5
    refs0 = 0.1 * _randn(4, d, g=g)
    refs, losses = RL.learn_refs(K, refs0, Q, C, depth, beta, steps=60, lr=0.5)
    assert losses[-1] < 0.7 * losses[0], losses[::10]
    assert all(np.isfinite(losses))


@pytest.mark.parametrize("N,C,depth,R", [(256, 4, 4, 3), (300, 4, 3, 2), (200, 3, 4, 4)])
def test_written_out_gradient_equals_autograd(N, C, depth, R):
    # the explicit backward (the one a GPU version follows) against torch's autograd
    d, beta = 8, 0.6
    K, centres, g = _keys(N, d, 10 + N)
    Q = centres[torch.randint(0, len(centres), (5,), generator=g)] * 1.5 + 0.1 * _randn(5, d, g=g)
    refs = _randn(R, d, g=g).requires_grad_(True)
    loss = RL.split_loss(K, refs, Q, C, depth, beta)
    (ga,) = torch.autograd.grad(loss, refs)
    l2, g2 = RL.split_loss_and_grad(K.numpy(), refs.detach().numpy(), Q.numpy(), C, depth, beta)
    assert abs(l2 - loss.item()) <= 1e-12 * max(1.0, abs(loss.item()))
    np.testing.assert_allclose(g2, ga.numpy(), rtol=0, atol=1e-12 * max(1.0, np.abs(ga.numpy()).max()))
