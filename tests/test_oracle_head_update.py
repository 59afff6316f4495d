"""Pins of the oracle's length-head online update: l = mean_b (bhat_b - a*_b)^2 through
bhat = sigmoid(w2 . relu(W1 h + b1) + b2), then one AdamW step (Pith verdict record
load_bearing_attack for the loss; Axiom ledger: head learning rate 2e-4)."""
import math

import numpy as np
import pytest
import torch


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float64).to(torch.bfloat16)


def _state(W1m, b1m, w2m, b2m):
    z = lambda a: np.zeros_like(a)
    return dict(W1m=W1m, b1m=b1m, w2m=w2m, b2m=b2m, mW1=z(W1m), vW1=z(W1m), mb1=z(b1m),
                vb1=z(b1m), mw2=z(w2m), vw2=z(w2m), mb2=z(b2m), vb2=z(b2m))


def _case(B, H, M, seed):
    g = np.random.default_rng(seed)
    h = _bf16(g.normal(0, 1, (B, H)))
    W1m = g.normal(0, 0.3, (M, H))
    b1m = g.normal(0, 0.1, M)
    w2m = g.normal(0, 0.5, M)
    b2m = np.array([0.1])
    label = g.uniform(0, 1, B)
    return h, W1m, b1m, w2m, b2m, label


def _torch_loss(h, W1, b1, w2, b2, label):
    # an independent expression of the same loss
    pre = h.double() @ W1.T + b1
    z = torch.relu(pre) @ w2 + b2
    return torch.mean((torch.sigmoid(z) - torch.as_tensor(label)) ** 2)


def test_gradients_match_autograd(orc):
    h, W1m, b1m, w2m, b2m, label = _case(5, 16, 8, 1)
    W1, w2 = _bf16(W1m), _bf16(w2m)
    r = orc.length_head_update(h, label, W1, b1m, w2, float(b2m[0]), _state(W1m.copy(), b1m.copy(),
                               w2m.copy(), b2m.copy()), step=1)
    tW1 = W1.double().clone().requires_grad_(True)
    tb1 = torch.tensor(b1m, requires_grad=True)
    tw2 = w2.double().clone().requires_grad_(True)
    tb2 = torch.tensor(b2m[0], requires_grad=True)
    loss = _torch_loss(h, tW1, tb1, tw2, tb2, label)
    loss.backward()
    assert r["loss"] == pytest.approx(loss.item(), rel=1e-12)
    np.testing.assert_allclose(r["gW1"], tW1.grad.numpy(), rtol=1e-10, atol=1e-15)
    np.testing.assert_allclose(r["gb1"], tb1.grad.numpy(), rtol=1e-10, atol=1e-15)
    np.testing.assert_allclose(r["gw2"], tw2.grad.numpy(), rtol=1e-10, atol=1e-15)
    assert r["gb2"] == pytest.approx(tb2.grad.item(), rel=1e-10)


def test_one_unit_by_hand(orc):
    # h = 1, W1 = 0.5, b1 = 0.25, w2 = 2, b2 = -1, a* = 0.3 (all exact in bf16)
    h = _bf16([[1.0]])
    st = _state(np.array([[0.5]]), np.array([0.25]), np.array([2.0]), np.array([-1.0]))
    r = orc.length_head_update(h, [0.3], _bf16([[0.5]]), np.array([0.25]), _bf16([2.0]), -1.0, st,
                               step=1, lr=0.0, wd=0.0)
    a = 0.75
    bh = 1.0 / (1.0 + math.exp(-(2.0 * a - 1.0)))
    delta = 2.0 * (bh - 0.3) * bh * (1.0 - bh)
    assert r["bhat"][0] == pytest.approx(bh, rel=1e-15)
    assert r["loss"] == pytest.approx((bh - 0.3) ** 2, rel=1e-15)
    assert r["gb2"] == pytest.approx(delta, rel=1e-15)
    assert r["gw2"][0] == pytest.approx(delta * a, rel=1e-15)
    assert r["gb1"][0] == pytest.approx(delta * 2.0, rel=1e-15)
    assert r["gW1"][0, 0] == pytest.approx(delta * 2.0, rel=1e-15)
    # a dead unit (negative pre-activation) passes no gradient to W1 and b1
    st2 = _state(np.array([[-0.5]]), np.array([0.25]), np.array([2.0]), np.array([-1.0]))
    r2 = orc.length_head_update(h, [0.3], _bf16([[-0.5]]), np.array([0.25]), _bf16([2.0]), -1.0,
                                st2, step=1, lr=0.0, wd=0.0)
    assert r2["gW1"][0, 0] == 0.0 and r2["gb1"][0] == 0.0 and r2["gw2"][0] == 0.0


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_three_adamw_steps_match_torch(orc, wd):
    h, W1m, b1m, w2m, b2m, label = _case(6, 12, 7, 3)
    lr, betas, eps = 2e-4, (0.9, 0.999), 1e-8
    # torch: fp64 masters, forward with bf16-rounded weights, gradient applied to the masters
    P = [torch.tensor(W1m.copy(), requires_grad=True), torch.tensor(b1m.copy(), requires_grad=True),
         torch.tensor(w2m.copy(), requires_grad=True), torch.tensor(b2m.copy(), requires_grad=True)]
    opt = torch.optim.AdamW(P, lr=lr, betas=betas, eps=eps, weight_decay=wd)
    st = _state(W1m.copy(), b1m.copy(), w2m.copy(), b2m.copy())
    for step in range(1, 4):
        W1f = P[0].detach().to(torch.bfloat16)
        w2f = P[2].detach().to(torch.bfloat16)
        leaves = [W1f.double().requires_grad_(True), P[1].detach().clone().requires_grad_(True),
                  w2f.double().requires_grad_(True), P[3].detach().clone().requires_grad_(True)]
        loss = _torch_loss(h, leaves[0], leaves[1], leaves[2], leaves[3][0], label)
        loss.backward()
        for p_, l_ in zip(P, leaves):
            p_.grad = l_.grad.clone()
        opt.step()
        r = orc.length_head_update(h, label, W1f, st["b1m"].copy(), w2f, float(st["b2m"][0]), st,
                                   step=step, lr=lr, beta1=betas[0], beta2=betas[1], eps=eps, wd=wd)
        assert r["loss"] == pytest.approx(loss.item(), rel=1e-12)
        for key, p_ in zip(("W1m", "b1m", "w2m", "b2m"), P):
            np.testing.assert_allclose(st[key], p_.detach().numpy(), rtol=1e-12, atol=1e-16)
        s0 = opt.state[P[0]]
        np.testing.assert_allclose(st["mW1"], s0["exp_avg"].numpy(), rtol=1e-12, atol=1e-20)
        np.testing.assert_allclose(st["vW1"], s0["exp_avg_sq"].numpy(), rtol=1e-12, atol=1e-24)
