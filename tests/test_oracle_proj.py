"""Pins of the projection oracle (oracle/proj.py): the split order against a hand-built
example, and every gradient against torch autograd of torch.nn.functional.linear (an
independent library), so that a transposed operand, a swapped part or a wrong product fails."""
import numpy as np
import torch

from oracle import proj


def test_split_order_by_hand():
    """Rows of W_qkvg are W_q (2 rows), W_k (1), W_v (1), W_g (2): with x = identity each output
    part is the transpose of its block of rows."""
    w = np.arange(6 * 3, dtype=np.float64).reshape(6, 3)
    q, k, v, g = proj.qkvg_forward(np.eye(3), w, 2, 1)
    assert np.array_equal(q, w[0:2].T) and np.array_equal(k, w[2:3].T)
    assert np.array_equal(v, w[3:4].T) and np.array_equal(g, w[4:6].T)


def test_gradients_match_autograd():
    torch.manual_seed(0)
    T, dm, wq, wkv, din = 5, 7, 4, 2, 6
    x = torch.randn(T, dm, dtype=torch.float64, requires_grad=True)
    w = torch.randn(2 * (wq + wkv), dm, dtype=torch.float64, requires_grad=True)
    y = torch.nn.functional.linear(x, w)
    dy = torch.randn_like(y)
    y.backward(dy)
    parts = np.split(dy.numpy(), [wq, wq + wkv, wq + 2 * wkv], axis=1)
    dx, dw = proj.qkvg_backward(x.detach(), w.detach(), *parts)
    assert np.allclose(dx, x.grad.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(dw, w.grad.numpy(), rtol=0, atol=1e-12)
    fq = proj.qkvg_forward(x.detach(), w.detach(), wq, wkv)
    assert np.allclose(np.concatenate(fq, axis=1), y.detach().numpy(), rtol=0, atol=1e-12)

    a = torch.randn(T, din, dtype=torch.float64, requires_grad=True)
    wo = torch.randn(dm, din, dtype=torch.float64, requires_grad=True)
    yo = torch.nn.functional.linear(a, wo)
    dyo = torch.randn_like(yo)
    yo.backward(dyo)
    assert np.allclose(proj.out_forward(a.detach(), wo.detach()), yo.detach().numpy(), rtol=0, atol=1e-12)
    da, dwo = proj.out_backward(a.detach(), wo.detach(), dyo)
    assert np.allclose(da, a.grad.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(dwo, wo.grad.numpy(), rtol=0, atol=1e-12)


def test_flops():
    f = proj.proj_flops(10, 8, 4, 2, 6)
    assert f == {"qkvg_fwd": 2 * 10 * 8 * 12, "qkvg_bwd": 4 * 10 * 8 * 12, "out_fwd": 2 * 10 * 6 * 8,
                 "out_bwd": 4 * 10 * 6 * 8}
