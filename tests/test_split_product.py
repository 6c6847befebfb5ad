"""The arithmetic behind the prologue's tensor-core form, checked on the host:
an fp32 value x split into three bf16 pieces x1 = bf16(x), x2 = bf16(x - x1),
x3 = bf16(x - x1 - x2) keeps 24 significant bits, and the six cross products of
pieces whose orders sum to at most 4 (x1y1, x1y2, x2y1, x1y3, x2y2, x3y1)
reproduce a K-term fp32 dot product to well within fp32 accuracy. (bf16 rounding
is torch's round-to-nearest-even conversion, as on the device.)"""

import numpy as np
import pytest
import torch


def _split3(x):
    x = torch.as_tensor(x, dtype=torch.float32)
    pieces = []
    r = x
    for _ in range(3):
        p = r.to(torch.bfloat16).to(torch.float32)
        pieces.append(p)
        r = r - p  # exact in fp32: r and its bf16 rounding share the exponent range
    return [p.double().numpy() for p in pieces], r.double().numpy()


@pytest.mark.parametrize("K", [256, 2688, 5376])
def test_three_piece_split_keeps_24_bits(K):
    x = np.random.default_rng(K).standard_normal(K).astype(np.float32) * 3.0
    (x1, x2, x3), rest = _split3(x)
    np.testing.assert_array_equal(x1 + x2 + x3 + rest, x.astype(np.float64))
    assert np.all(np.abs(rest) <= np.abs(x.astype(np.float64)) * 2.0 ** -23)


@pytest.mark.parametrize("K", [256, 2688, 5376])
def test_six_products_match_the_fp32_dot_product(K):
    g = np.random.default_rng([K, 1])
    a = g.standard_normal((16, K)).astype(np.float32)
    w = (g.standard_normal((16, K)) * 0.02).astype(np.float32)
    (a1, a2, a3), _ = _split3(a)
    (w1, w2, w3), _ = _split3(w)
    six = a1 @ w1.T + a1 @ w2.T + a2 @ w1.T + a1 @ w3.T + a2 @ w2.T + a3 @ w1.T
    exact = a.astype(np.float64) @ w.astype(np.float64).T
    scale = np.abs(a.astype(np.float64)) @ np.abs(w.astype(np.float64)).T
    # error bounded by the dropped products: below 2^-22 of sum |a||w|
    assert np.all(np.abs(six - exact) <= scale * 2.0 ** -22)
    # a single bf16 product (the leading term alone) is not fp32-accurate
    assert np.max(np.abs(a1 @ w1.T - exact) / scale) > 2.0 ** -16
