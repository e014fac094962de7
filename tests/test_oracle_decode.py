"""Pins of the oracle's number-format decoding (bf16, OCP FP8 E4M3)."""
import numpy as np
import pytest
import torch

from oracle import decode_bf16, decode_e4m3, dequantize


def test_bf16_hand_values():
    codes = np.array([0x3F80, 0xC000, 0x3FC0, 0x0001, 0x0080, 0x7F7F, 0x8000, 0x0000, 0x4049],
                     np.uint16)
    want = [1.0, -2.0, 1.5, 2.0 ** -133, 2.0 ** -126, (2 - 2 ** -7) * 2.0 ** 127, -0.0, 0.0,
            (1 + 73 / 128) * 2.0]
    got = decode_bf16(codes)
    assert got.tolist() == want
    assert np.signbit(got[6]) and not np.signbit(got[7])


def test_bf16_all_finite_codes_match_library():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    e = (codes.astype(np.int64) >> 7) & 0xFF
    codes = codes[e != 0xFF]
    lib = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(decode_bf16(codes), lib)


def test_bf16_rejects_nonfinite():
    with pytest.raises(ValueError):
        decode_bf16(np.array([0x7F80], np.uint16))


def test_e4m3_hand_values():
    codes = np.array([0x38, 0x7E, 0x01, 0x08, 0x80, 0xC0, 0x3C, 0x07, 0xFE], np.uint8)
    want = [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, -0.0, -2.0, 1.5, 7 / 8 * 2.0 ** -6, -448.0]
    assert decode_e4m3(codes).tolist() == want


def test_e4m3_all_codes_match_library():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(decode_e4m3(codes), lib)


def test_e4m3_rejects_nan():
    with pytest.raises(ValueError):
        decode_e4m3(np.array([0x7F], np.uint8))


def test_fp8_scale_is_per_token():
    codes = np.array([[0x38, 0x40], [0x38, 0x40]], np.uint8)    # [[1, 2], [1, 2]]
    v = dequantize(codes, np.array([0.5, 3.0], np.float32), "fp8")
    assert v.tolist() == [[0.5, 1.0], [3.0, 6.0]]
