"""The Python layer API refuses tensors the library would misread (shape,
dtype, device, stride) before anything reaches the C calls, which take raw
pointers.  A layer placed on the CPU device is enough: every refusal happens
on the host, before the first library call."""
import pytest
import torch

import orthogonal_equivalence_b200 as px
from orthogonal_equivalence_b200.layer import _need


def test_need_accepts_and_refuses():
    cpu = torch.device("cpu")
    _need(torch.zeros(4, 6), (4, 6), torch.float32, cpu, "x")
    with pytest.raises(ValueError, match="shape"):
        _need(torch.zeros(4, 5), (4, 6), torch.float32, cpu, "x")
    with pytest.raises(ValueError, match="dtype"):
        _need(torch.zeros(4, 6, dtype=torch.bfloat16), (4, 6), torch.float32, cpu, "x")
    with pytest.raises(ValueError, match="contiguous"):
        _need(torch.zeros(6, 4).t(), (4, 6), torch.float32, cpu, "x")
    with pytest.raises(ValueError, match="the layer is on"):
        _need(torch.zeros(4, 6), (4, 6), torch.float32, torch.device("cuda", 0), "x")
    with pytest.raises(TypeError):
        _need([[0.0] * 6] * 4, (4, 6), torch.float32, cpu, "x")


def _layer():
    return px.PoetxLinear(128, 192, 64, px.POETX_BF16, device="cpu")


def test_forward_refuses_mismatched_tensors():
    L = _layer()
    bf = torch.bfloat16
    with pytest.raises(ValueError, match="x: shape"):
        L.forward(torch.zeros(10, 127, dtype=bf))
    with pytest.raises(ValueError, match="x: dtype"):
        L.forward(torch.zeros(10, 128, dtype=torch.float32))
    with pytest.raises(ValueError, match="z: shape"):
        L.forward(torch.zeros(10, 128, dtype=bf), z=torch.zeros(10, 128, dtype=bf))
    with pytest.raises(ValueError, match="y: shape"):
        L.forward(torch.zeros(10, 128, dtype=bf), y=torch.zeros(9, 192, dtype=bf))
    with pytest.raises(ValueError, match="xg: shape"):
        L.forward(torch.zeros(10, 128, dtype=bf), save_xg=True, xg=torch.zeros(10, 192, dtype=bf))


def test_backward_refuses_mismatched_tensors():
    L = _layer()
    bf = torch.bfloat16
    x, y, dz = torch.zeros(10, 128, dtype=bf), torch.zeros(10, 192, dtype=bf), torch.zeros(10, 192, dtype=bf)
    with pytest.raises(ValueError, match="dz: shape"):
        L.backward(x, y, torch.zeros(10, 128, dtype=bf))
    with pytest.raises(ValueError, match="x: shape"):
        L.backward(torch.zeros(11, 128, dtype=bf), y, dz)
    with pytest.raises(ValueError, match="saved y: shape"):
        L.backward(x, torch.zeros(10, 128, dtype=bf), dz)
    with pytest.raises(ValueError, match="x: needed"):
        L.backward(None, y, dz)
    with pytest.raises(ValueError, match="dx: dtype"):
        L.backward(x, y, dz, dx=torch.zeros(10, 128))
    with pytest.raises(ValueError, match="dqR: shape"):
        L.backward(x, y, dz, dqR=torch.zeros(3, 2016))
    good_R = torch.zeros(2, 64, 64)
    with pytest.raises(ValueError, match="dGP: shape"):
        L.backward_dG(x, y, dz, good_R, torch.zeros(2, 64, 64))
    with pytest.raises(ValueError, match="dGR: dtype"):
        L.backward_dG(x, y, dz, good_R.to(bf), torch.zeros(3, 64, 64))


def test_load_and_group_refuse_mismatched_tensors():
    L = _layer()
    with pytest.raises(ValueError, match="W0lin: shape"):
        L.load(torch.zeros(128, 192, dtype=torch.bfloat16), torch.arange(128), torch.arange(192),
               torch.zeros(2, 2016), torch.zeros(3, 2016))
    with pytest.raises(ValueError, match="permP: shape"):
        L.load(torch.zeros(192, 128, dtype=torch.bfloat16), torch.arange(128), torch.arange(191),
               torch.zeros(2, 2016), torch.zeros(3, 2016))
    g = px.LayerGroup([L])
    q = g.flatten_params()
    with pytest.raises(ValueError, match="grad: shape"):
        g.optimizer_step(torch.zeros(q.numel() - 1), 1e-3)
    with pytest.raises(ValueError, match="dG: shape"):
        g.cnp_backward(torch.zeros(4, 64, 64), torch.zeros_like(q))
    with pytest.raises(ValueError, match="dq: dtype"):
        g.cnp_backward(g.dG_buffer(), torch.zeros_like(q, dtype=torch.float64))
