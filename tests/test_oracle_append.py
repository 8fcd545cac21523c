"""Pins for the oracle's cache append (e4m3 encoding, per-token key quantisation, paged
row placement).  CPU only.

The encoder is pinned to torch's float8_e4m3fn cast (a library routine that rounds to
nearest even) inside the finite range, to the format's own code table (every finite code
round-trips), to the saturation and NaN rules of the reading, and to closed forms of the
quantiser (the largest element lands on +-448, the scale is amax / 448)."""

import numpy as np
import pytest
import torch

from oracle import dsa_ref as R

FINITE_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def torch_e4m3(x):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# ---------------------------------------------------------------- pins, written against
# an encoder argument so the mutation test below can hand them planted mistakes

def pin_matches_torch(enc):
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.uniform(-448, 448, 20000),
        rng.uniform(-2.0 ** -5, 2.0 ** -5, 20000),  # subnormals and the smallest normals
    ]).astype(np.float32)
    # every midpoint between neighbouring positive codes: ties must go to the even code
    vals = R.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids]).astype(np.float32)
    assert np.array_equal(enc(x), torch_e4m3(x))


def pin_roundtrip(enc):
    v = R.decode_e4m3(FINITE_CODES).astype(np.float32)
    assert np.array_equal(enc(v), FINITE_CODES)


def pin_saturation(enc):
    big = np.array([448.0, 448.5, 465.0, 1e6, 3.0e38], dtype=np.float32)
    assert np.all(enc(big) == 0x7E)
    assert np.all(enc(-big) == 0xFE)
    assert enc(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


PINS = [pin_matches_torch, pin_roundtrip, pin_saturation]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_encoder_pin(pin):
    pin(R.encode_e4m3)


# planted mistakes: each must fail at least one pin
def m_truncate(v):  # round toward zero
    v = np.asarray(v, np.float32).astype(np.float64)
    table = R.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    a = np.minimum(np.abs(np.nan_to_num(v)), 448.0)
    code = np.clip(np.searchsorted(table, a, side="right") - 1, 0, 0x7E).astype(np.uint8)
    return code | np.where(np.signbit(v), np.uint8(0x80), np.uint8(0))


def m_ties_up(v):  # ties away from zero
    v = np.asarray(v, np.float32).astype(np.float64)
    table = R.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    a = np.minimum(np.abs(np.nan_to_num(v)), 448.0)
    hi = np.clip(np.searchsorted(table, a, side="left"), 0, 0x7E)
    lo = np.maximum(hi - 1, 0)
    code = np.where(table[hi] - a <= a - table[lo], hi, lo).astype(np.uint8)
    return code | np.where(np.signbit(v), np.uint8(0x80), np.uint8(0))


def m_no_saturation(v):  # beyond the range -> NaN, as a plain cast does
    v = np.asarray(v, np.float32)
    out = R.encode_e4m3(v)
    return np.where(np.abs(v) > 464, np.uint8(0x7F) | (out & 0x80), out).astype(np.uint8)


def m_lost_sign(v):
    return R.encode_e4m3(np.abs(np.asarray(v, np.float32)))


@pytest.mark.parametrize("mutant", [m_truncate, m_ties_up, m_no_saturation, m_lost_sign],
                         ids=lambda m: m.__name__)
def test_encoder_pins_catch_mutations(mutant):
    caught = 0
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin catches {mutant.__name__}"


# ---------------------------------------------------------------- quantiser

def test_quantize_key_closed_forms():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(128).astype(np.float32)
    codes, scale = R.quantize_key(x)
    amax = np.float32(np.abs(x).max())
    assert scale == np.float32(amax / np.float32(448.0))
    j = int(np.abs(x).argmax())
    assert codes[j] == (0xFE if x[j] < 0 else 0x7E)  # the largest element is +-448 exactly
    # every decoded value is within half an e4m3 step of x / scale
    y = (x / scale).astype(np.float64)
    got = R.decode_e4m3(codes)
    step = np.where(np.abs(y) >= 2.0 ** -6, np.exp2(np.floor(np.log2(np.abs(y) + 1e-300)) - 3),
                    2.0 ** -9)
    assert np.all(np.abs(got - y) <= step / 2 + 1e-12)


def test_quantize_key_zero_and_scale_invariance():
    codes, scale = R.quantize_key(np.zeros(64, np.float32))
    assert scale == np.float32(1.0) and not codes.any()
    # scaling a key by a power of two changes the scale, not the codes
    x = np.random.default_rng(2).standard_normal(64).astype(np.float32)
    c1, s1 = R.quantize_key(x)
    c2, s2 = R.quantize_key(x * np.float32(8.0))
    assert np.array_equal(c1, c2) and s2 == np.float32(8.0) * s1


# ---------------------------------------------------------------- paged placement

def test_cache_append_places_rows():
    rng = np.random.default_rng(9)
    page, nb, D, Dkv = 64, 6, 32, 16
    k8 = np.full((nb * page, D), 0xAA, np.uint8)
    ks = np.full(nb * page, -7.0, np.float32)
    kv = np.full((nb * page, Dkv), 0x1234, np.uint16)
    bt = np.array([[4, 1, 3], [0, 5, 2]], np.int32)
    tok_seq = np.array([0, 1, 0, 1, 1, 7], np.int32)
    tok_pos = np.array([65, 0, 191, 130, 500, 3], np.int32)  # last two: bad position / sequence
    k_in = rng.standard_normal((6, D)).astype(np.float32)
    kv_in = rng.integers(0, 65535, (6, Dkv), dtype=np.uint16)
    n8, ns, nkv, ok = R.cache_append(k8, ks, kv, bt, tok_seq, tok_pos, k_in, kv_in, page)
    assert ok.tolist() == [True, True, True, True, False, False]
    rows = {0: 1 * page + 1, 1: 0 * page + 0, 2: 3 * page + 63, 3: 2 * page + 2}
    touched = np.zeros(nb * page, bool)
    for i, row in rows.items():
        c, s = R.quantize_key(k_in[i])
        assert np.array_equal(n8[row], c) and ns[row] == s
        assert np.array_equal(nkv[row], kv_in[i])
        touched[row] = True
    assert np.all(n8[~touched] == 0xAA) and np.all(ns[~touched] == -7.0)
    assert np.all(nkv[~touched] == 0x1234)
