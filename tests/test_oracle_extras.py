"""Pins of the oracle's POET-XQ weight quantization and of the AdamW step on
packed triangles (POET-X write-up: section "POET-XQ", API snippet's
get_poet_optimizer)."""
import numpy as np
import torch

import oracle


def test_quantize_hand_ties_round_half_even():
    # max |row| = 127 makes the scale exactly 1, so w / scale = w: ties go to even
    W = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.49, 126.5],
                  [0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    codes, scale = oracle.quantize_rows(W)
    assert scale[0] == 1.0 and scale[1] == 0.0
    assert codes[0].tolist() == [127, 2, 4, -2, 0, 0, 126]
    assert not codes[1].any()


def test_quantize_bounds_and_reconstruction_error():
    g = np.random.Generator(np.random.PCG64(4))
    W = (g.standard_normal((64, 300)) * np.exp(g.standard_normal((64, 1)))).astype(np.float32)
    codes, scale = oracle.quantize_rows(W)
    assert codes.dtype == np.int8 and np.abs(codes.astype(int)).max() <= 127
    assert np.all(np.abs(codes.astype(int)).max(axis=1) == 127)   # the absmax element maps to +-127
    rec = oracle.dequantize_rows(codes, scale)
    # nearest-code rounding: error at most half a step (plus float32 rounding)
    assert np.all(np.abs(rec - W) <= scale[:, None] * (0.5 + 1e-5))


def test_round_to_bf16_matches_known_values():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20], dtype=np.float32)
    np.testing.assert_array_equal(oracle.round_to_bf16(v), [1.0, 1.0, 1.0 + 2 ** -6, 1.0 + 2 ** -7])


def test_adamw_matches_torch_adamw():
    g = np.random.Generator(np.random.PCG64(9))
    n = 37
    q0 = g.standard_normal(n) * 0.01
    p = torch.tensor(q0.copy(), dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([p], lr=1e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    q, m, v = q0.copy(), np.zeros(n), np.zeros(n)
    for step in range(1, 4):
        grad = g.standard_normal(n)
        p.grad = torch.tensor(grad, dtype=torch.float64)
        opt.step()
        q, m, v = oracle.adamw_step(q, grad, m, v, 1e-3, 0.9, 0.95, 1e-8, 0.1, step)
        np.testing.assert_allclose(q, p.detach().numpy(), rtol=0, atol=1e-14)
