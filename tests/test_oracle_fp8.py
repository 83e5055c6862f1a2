"""Pins of the oracle's per-block e4m3 quantisation of Q and K ("Sparse Video-Gen" summary
page, "Measured effects": FP8 quantisation on top of the sparse attention).

Checked against torch's own float8_e4m3fn cast (round to nearest, ties to even) as an
independent library routine, hand-picked codes, and the scale rule in closed form."""
import numpy as np
import pytest
import torch

import oracle


def test_codes_match_torch_float8_cast():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((300, 16)) * np.exp(rng.uniform(-12, 8, (300, 1)))
    code, e = oracle.quantize_e4m3(x, 64)
    scaled = np.ldexp(x, -np.repeat(e, 64)[:300, None])
    want = torch.from_numpy(scaled).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(code, want)


def test_scale_is_the_smallest_power_of_two():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((200, 8)) * 3.0
    x[64:128] *= 1e-6
    x[128:192] = 0.0
    code, e = oracle.quantize_e4m3(x, 64)
    for b in range(4):
        blk = x[b * 64:(b + 1) * 64]
        amax = np.abs(blk).max()
        if amax == 0:
            assert e[b] == 0 and not code[b * 64:(b + 1) * 64].any()
            continue
        assert amax <= 448.0 * 2.0 ** e[b] and amax > 448.0 * 2.0 ** (e[b] - 1)


@pytest.mark.parametrize("value,code", [(448.0, 0x7E), (1.0, 0x38), (1.0625, 0x38), (1.1875, 0x3A),
                                        (2.0 ** -9, 0x01), (2.5 * 2.0 ** -9, 0x02), (3.5 * 2.0 ** -9, 0x04),
                                        (-1.5, 0xBC), (2.0 ** -6, 0x08), (0.0, 0x00)])
def test_hand_codes(value, code):
    """Block of one row whose largest entry is 448 (so the scale is 2^0): each value's code."""
    x = np.array([[value, 448.0]])
    c, e = oracle.quantize_e4m3(x, 1)
    assert e[0] == 0
    assert int(c[0, 0]) == code
    assert oracle.e4m3_values(c[0, 0]) == (torch.tensor([value], dtype=torch.float64)
                                           .to(torch.float8_e4m3fn).to(torch.float64).item())


def test_dequantize_round_trip_error():
    """Every value is within half an e4m3 step of its code's value (relative 2^-4 for normal
    values)."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((256, 32))
    code, e = oracle.quantize_e4m3(x, 128)
    dq = oracle.dequantize_e4m3(code, e, 128)
    scale = 2.0 ** np.repeat(e, 128)[:, None]
    normal = np.abs(x) / scale >= 2.0 ** -6
    assert np.all(np.abs(dq - x)[normal] <= np.abs(x)[normal] * 2.0 ** -4)
    assert np.all(np.abs(dq - x)[~normal] <= scale.repeat(32, axis=1)[~normal] * 2.0 ** -10)
