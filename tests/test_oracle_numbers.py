"""Pins for the oracle's number formats: binary16 decode, E4M3 decode/encode.

Each check compares against something other than the oracle's own formulas:
numpy's float16 conversion, torch's float8_e4m3fn dtype, and an independent
table-driven nearest-code search written here from the OCP E4M3 definition
(256 codes, round to nearest, ties to the even code, saturate to 448).
"""
import numpy as np
import pytest
import torch

import oracle


def test_f16_decode_all_bit_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.f16_to_double(bits.view(np.float16))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_all_codes_match_torch():
    ref = _torch_e4m3_values()
    got = oracle.e4m3_to_double(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert nan.sum() == 2            # S.1111.111 only
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0xFE] == -448.0
    assert got[0x01] == 2.0 ** -9


def _table_encoder(x: np.ndarray) -> np.ndarray:
    """Independent E4M3 encoder: nearest of the 254 finite codes, ties to even code."""
    vals = _torch_e4m3_values()
    finite = np.where(~np.isnan(vals))[0]
    pos = finite[(vals[finite] >= 0) & ~((vals[finite] == 0) & (finite >= 128))]  # +0 .. 448
    pos = pos[np.argsort(vals[pos])]
    pv = vals[pos]
    out = np.empty(x.shape, np.uint8)
    for i, xv in enumerate(x.astype(np.float64)):
        if np.isnan(xv):
            out[i] = 0x7F | (0x80 if np.signbit(xv) else 0)
            continue
        a = min(abs(xv), 448.0)
        j = np.searchsorted(pv, a)
        cands = [k for k in (j - 1, j) if 0 <= k < len(pv)]
        d = [abs(pv[k] - a) for k in cands]
        best = [cands[k] for k in range(len(cands)) if d[k] == min(d)]
        code = pos[best[0]] if len(best) == 1 else [pos[k] for k in best if pos[k] % 2 == 0][0]
        out[i] = code | (0x80 if np.signbit(xv) else 0)
    return out


@pytest.mark.parametrize("scale", [1.0, 0.5, 0.01398576982319355, 3.0])
def test_e4m3_encode_all_f16_inputs_against_table_encoder(scale):
    x16 = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    x16 = x16[np.isfinite(x16)]   # every finite fp16 input
    x = (x16.astype(np.float32) / np.float32(scale)).astype(np.float32)
    # the table encoder is slow; cover every input near code boundaries plus a stride sample
    got = oracle.e4m3_from_float(x)
    sample = np.unique(np.concatenate([np.arange(0, x.size, 7), np.arange(x.size - 2000, x.size)]))
    ref = _table_encoder(x[sample])
    assert np.array_equal(got[sample], ref)


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000).astype(np.float32) * 50,
                        rng.standard_normal(20000).astype(np.float32) * 1e-2,
                        np.float32([0.0, -0.0, 448.0, -448.0, 2 ** -9, 2 ** -10, 1.5 * 2 ** -10])])
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_from_float(x), ref)


def test_e4m3_round_trip_and_special_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_to_double(codes)
    ok = ~np.isnan(vals)
    assert np.array_equal(oracle.e4m3_from_float(vals[ok].astype(np.float32)), codes[ok])
    enc = oracle.e4m3_from_float(np.float32([448, 449, 463.9, 464, 1e30, np.inf, -np.inf, -500,
                                             2 ** -10, 1.5 * 2 ** -10, 2 ** -11, np.nan]))
    assert list(enc[:8]) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert list(enc[8:11]) == [0x00, 0x01, 0x00]       # 2^-10 ties to even (0); 1.5*2^-10 -> 2^-9
    assert enc[11] & 0x7F == 0x7F
