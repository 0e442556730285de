"""Pins for the oracle's e4m3 cache storage: the code table and the rounding
against PyTorch's float8_e4m3fn (a library routine, used inside the finite
range where it does not saturate), closed forms for saturation and the row
scale, and planted mistakes that these pins must catch."""
import numpy as np
import pytest
import torch

import oracle.hca_oracle as O

RNG = np.random.default_rng(8)


def _torch_decode_all():
    codes = torch.arange(256, dtype=torch.int64).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).float().double().numpy()


def _torch_encode(y: np.ndarray) -> np.ndarray:
    return torch.from_numpy(y.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _midpoints():
    """Every value halfway between two adjacent finite positive codes (ties)."""
    vals = np.sort(np.unique(O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))))
    return ((vals[:-1] + vals[1:]) / 2).astype(np.float32)


def pin_error(decode=O.e4m3_decode, encode=O.e4m3_encode, quant=O.quantize_e4m3_rows):
    """Number of disagreements with the references (0 when all hold)."""
    bad = 0
    ref = _torch_decode_all()
    mine = decode(np.arange(256, dtype=np.uint8))
    both_nan = np.isnan(ref) & np.isnan(mine)
    bad += int((~both_nan & (ref != mine)).sum())
    y = np.concatenate([RNG.uniform(-440, 440, 4000), RNG.standard_normal(4000) * 0.01,
                        _midpoints(), -_midpoints(), [0.0, 2.0 ** -10, 2.0 ** -9, 448.0]]
                       ).astype(np.float32)
    bad += int((encode(y) != _torch_encode(y)).sum())
    # saturation: beyond the largest finite value every magnitude maps to 448
    big = np.array([448.0001, 463.9, 464.0, 500.0, 1e30, -1e30], dtype=np.float32)
    bad += int((decode(encode(big)) != np.sign(big) * 448.0).sum())
    # row scale: amax / 448 in fp32, the amax element coded as +-448, every
    # element within half a quantum of its code's value
    x = (RNG.standard_normal((16, 512)) * RNG.uniform(0.01, 100, (16, 1))).astype(np.float32)
    codes, scale = quant(x)
    amax = np.abs(x).max(-1)
    bad += int((scale != (amax / np.float32(448.0)).astype(np.float32)).sum())
    idx = np.abs(x).argmax(-1)
    bad += int((np.abs(decode(codes[np.arange(16), idx])) != 448.0).sum())
    deq = O.dequantize_e4m3_rows(codes, scale) if decode is O.e4m3_decode else \
        decode(codes) * scale.astype(np.float64)[:, None]
    y = x.astype(np.float64) / scale[:, None]
    _, ex = np.frexp(np.maximum(np.abs(y), 2.0 ** -6))
    half_q = 2.0 ** (ex - 1 - 4) * scale[:, None]
    bad += int((np.abs(deq - x) > half_q * (1 + 1e-6)).sum())
    zc, zs = quant(np.zeros((2, 512), dtype=np.float32))
    bad += int(zc.any()) + int((zs != 1.0).any())
    return bad


def test_fp8_storage_pins():
    assert pin_error() == 0


def _truncating_encode(y):
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), 448.0)
    _, ex = np.frexp(np.maximum(a, 2.0 ** -6))
    q = 2.0 ** (ex - 4)
    return O.e4m3_encode(np.sign(y) * np.floor(a / q) * q)


def _no_saturation_encode(y):
    c = O.e4m3_encode(y)
    return np.where(np.abs(np.asarray(y)) > 448.0, np.uint8(0x7F), c).astype(np.uint8)


def _bias_8_decode(codes):
    return O.e4m3_decode(codes) / 2.0


def _scale_from_mean(x):
    x32 = np.asarray(x, dtype=np.float32)
    scale = (np.abs(x32).mean(-1) / np.float32(448.0)).astype(np.float32)
    return O.e4m3_encode(x32 / scale[:, None]), scale


@pytest.mark.parametrize("kw", [{"encode": _truncating_encode}, {"encode": _no_saturation_encode},
                                {"decode": _bias_8_decode}, {"quant": _scale_from_mean}],
                         ids=["truncate", "no_saturation", "bias_8", "scale_from_mean"])
def test_fp8_pins_catch_planted_mistakes(kw):
    try:
        bad = pin_error(**kw)
    except Exception:   # a crash also counts as caught
        bad = 1
    assert bad > 0
