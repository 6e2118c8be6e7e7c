"""Pins of the low-precision V oracle (oracle/lowprec_oracle.py) against facts
fixed outside it: the E4M3 format definition worked by hand, torch's
float8_e4m3fn cast (an independent implementation of the same rounding),
structural facts of the format, the quantizer's error bound, and closed forms
of attention. [FVAttn §3.4: V is quantized on the GPU; the format is a reading.]"""

import math
import pathlib

import numpy as np
import pytest
import torch

import oracle as O
from oracle import lowprec_oracle as Lp

GOLDEN = pathlib.Path(__file__).parent / "golden" / "e4m3_quant.txt"


def _golden():
    sec, data = None, {"v": [], "codes": [], "scale": []}
    for line in GOLDEN.read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line in data:
            sec = line
            continue
        if sec == "codes":
            data[sec].append([int(t, 16) for t in line.split()])
        else:
            data[sec].append([float(t) for t in line.split()])
    return (np.array(data["v"], np.float32), np.array(data["codes"], np.uint8),
            np.array(data["scale"][0]))


def test_golden_worked_example():
    v, codes, scale = _golden()
    got_codes, got_scale = Lp.quantize_v(v[None, None], v.shape[0])
    assert np.array_equal(got_codes[0, 0], codes)
    assert np.allclose(got_scale[0, 0], scale, rtol=1e-7, atol=0)


def test_table_structure():
    t = Lp.e4m3_table()
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.isnan(t).sum() == 2
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)                       # codes 0..0x7E increase strictly
    assert pos[0] == 0.0 and pos[1] == 2.0 ** -9          # smallest subnormal
    assert t[0x08] == 2.0 ** -6                           # smallest normal
    assert t[0x38] == 1.0 and t[0x7E] == 448.0
    assert np.array_equal(t[0x80:0xFF], -pos)             # sign-magnitude
    # spacing: subnormals 2^-9 apart, then 8 values per binade
    assert np.all(np.diff(pos[:9]) == 2.0 ** -9)
    for e in range(1, 15):
        b = pos[8 * e: 8 * e + 8]
        assert np.all(np.diff(b) == 2.0 ** (e - 10))


def test_encode_matches_torch_cast():
    rng = np.random.default_rng(0)
    t = Lp.e4m3_table()[:0x7F]
    mids = (t[1:] + t[:-1]) / 2                           # every tie
    x = np.concatenate([
        t, -t, mids, -mids,
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.6, 20000),
        rng.uniform(-464, 464, 20000),
    ]).astype(np.float32)
    x = x[np.abs(x) <= 464]                              # torch turns larger values into NaN
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = Lp.e4m3_encode(x)
    assert np.array_equal(got, want), np.nonzero(got != want)[0][:5]


def test_encode_saturates_and_round_trips():
    assert np.array_equal(Lp.e4m3_encode(np.array([464.0, 500.0, 1e30, -1e30])),
                          np.array([0x7E, 0x7E, 0x7E, 0xFE], np.uint8))
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(Lp.e4m3_encode(Lp.e4m3_decode(codes)), codes)
    assert Lp.e4m3_encode(np.array([-0.0]))[0] == 0x80


def test_encode_error_bound():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(50000) * 10.0 ** rng.uniform(-5, 2.6, 50000)).astype(np.float32)
    x = x[np.abs(x) <= 448]
    err = np.abs(Lp.e4m3_decode(Lp.e4m3_encode(x)) - x.astype(np.float64))
    normal = np.abs(x) >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]))   # half an ulp of 3 mantissa bits
    assert np.all(err[~normal] <= 2.0 ** -10)                    # half the subnormal step


def _v(B=1, H=2, N=300, npad=384, d=8, seed=3):
    rng = np.random.default_rng(seed)
    v = torch.from_numpy(rng.standard_normal((B, H, npad, d)) * rng.uniform(0.1, 5, (B, H, 1, d)))
    v = v.to(torch.bfloat16).float().numpy()
    v[:, :, N:] = 0.0
    return v


def test_quantize_v_amax_maps_to_448_and_error_bound():
    N = 300
    v = _v(N=N)
    codes, scale = Lp.quantize_v(v, N)
    vh = Lp.dequantize_v(codes, scale)
    amax = np.abs(v[:, :, :N]).max(axis=2)
    assert np.allclose(scale, amax / 448.0, rtol=2 ** -23)
    # the largest magnitude of each channel encodes as +-448
    idx = np.abs(v[:, :, :N]).argmax(axis=2)
    for b, h, c in np.ndindex(*amax.shape):
        assert Lp.e4m3_decode(codes[b, h, idx[b, h, c], c]) in (448.0, -448.0)
    err = np.abs(vh - v)
    bound = (2.0 ** -4 * np.abs(v) + 2.0 ** -10 * scale[:, :, None, :]) * (1 + 1e-6)
    assert np.all(err <= bound)
    assert np.all(codes[:, :, N:] == 0)


def test_quantize_v_channels_are_independent_and_zero_channel():
    N = 300
    v = _v(N=N)
    v[0, 1, :, 3] = 0.0
    codes, scale = Lp.quantize_v(v, N)
    assert scale[0, 1, 3] == 0.0 and np.all(codes[0, 1, :, 3] == 0)
    w = v.copy()
    w[0, 0, :N, 5] *= 7.0                                # another channel's range changes
    codes2, scale2 = Lp.quantize_v(w, N)
    keep = np.ones(v.shape[-1], bool)
    keep[5] = False
    assert np.array_equal(codes2[0, 0][:, keep], codes[0, 0][:, keep])
    assert np.array_equal(scale2[0, 0][keep], scale[0, 0][keep])
    # pad rows never count towards amax
    w = v.copy()
    w[:, :, N:] = 1e4
    codes3, scale3 = Lp.quantize_v(w, N)
    assert np.array_equal(scale3, scale) and np.all(codes3[:, :, N:] == 0)


def test_attention_with_exact_codes_equals_attention_on_v():
    # every channel holds E4M3 values with amax exactly 448: scale 1, V^ = V
    rng = np.random.default_rng(4)
    B, H, N, bs, d = 1, 2, 200, 64, 16
    nb = O.num_blocks(N, bs)
    npad = nb * bs
    t = Lp.e4m3_table()[:0x7F]
    v = rng.choice(np.concatenate([t, -t]), size=(B, H, npad, d))
    v[:, :, 0, :] = 448.0
    v[:, :, N:] = 0.0
    codes, scale = Lp.quantize_v(v.astype(np.float32), N)
    assert np.all(scale == 1.0)
    q = rng.standard_normal((B, H, npad, d))
    k = rng.standard_normal((B, H, npad, d))
    mask = rng.random((B, H, nb, nb)) < 0.6
    mask[..., 0] = True
    sm = 1 / math.sqrt(d)
    assert np.allclose(Lp.masked_attention_qv(q, k, codes, scale, mask, N, bs, sm),
                       O.masked_attention(q, k, v, mask, N, bs, sm), rtol=0, atol=1e-12)


def test_attention_zero_q_is_mean_of_dequantized_v():
    N, bs = 150, 64
    v = _v(N=N, npad=192, d=8)
    codes, scale = Lp.quantize_v(v, N)
    vh = Lp.dequantize_v(codes, scale)
    nb = O.num_blocks(N, bs)
    mask = np.zeros((1, 2, nb, nb), bool)
    mask[:, :, :, 0] = True
    mask[:, :, 1, 2] = True
    q = np.zeros_like(v)
    out = Lp.masked_attention_qv(q, np.ones_like(v), codes, scale, mask, N, bs, 0.5)
    for h in range(2):
        assert np.allclose(out[0, h, 0:64], vh[0, h, 0:64].mean(axis=0), atol=1e-12)
        sel = np.concatenate([np.arange(0, 64), np.arange(128, N)])
        assert np.allclose(out[0, h, 64:128], vh[0, h, sel].mean(axis=0), atol=1e-12)


def test_softmax_weights_rows_sum_to_one_and_reproduce_attention():
    rng = np.random.default_rng(6)
    N, bs, d = 170, 64, 8
    nb = O.num_blocks(N, bs)
    q = rng.standard_normal((nb * bs, d))
    k = rng.standard_normal((nb * bs, d))
    v = rng.standard_normal((nb * bs, d))
    mrow = np.array([True, False, True])
    for i in range(nb):
        cols, w = Lp.masked_softmax_weights(q, k, mrow, N, bs, 0.3, i)
        assert np.allclose(w.sum(-1), 1.0)
        assert set(cols.tolist()) == set(range(0, 64)) | set(range(128, N))
        assert np.allclose(w @ v[cols], O.masked_attention_rows(q, k, v, mrow, N, bs, 0.3, i), atol=1e-12)


# ---------------------------------------------------------------- planted mistakes
# Modified copies of oracle steps; each must fail one of the checks that pin the oracle.

def _encode_ties_away(x):
    x = np.asarray(x, np.float64)
    pos = Lp.e4m3_table()[:0x7F]
    a = np.minimum(np.abs(x), 448.0)
    hi = np.minimum(np.searchsorted(pos, a, side="left"), len(pos) - 1)
    lo = np.maximum(hi - 1, 0)
    pick_hi = (pos[hi] - a) <= (a - pos[lo])                # ties away from zero
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return code | (np.signbit(x).astype(np.uint8) << 7)


def _encode_truncating(x):
    x = np.asarray(x, np.float64)
    pos = Lp.e4m3_table()[:0x7F]
    a = np.minimum(np.abs(x), 448.0)
    code = (np.searchsorted(pos, a, side="right") - 1).astype(np.uint8)   # rounds toward zero
    return code | (np.signbit(x).astype(np.uint8) << 7)


def _quantize_amax_with_pad(v, N):
    v32 = np.asarray(v, np.float32)
    amax = np.abs(v32).max(axis=2)                            # pad rows counted
    inv = (np.float32(448) / np.where(amax > 0, amax, 1)).astype(np.float32)
    codes = Lp.e4m3_encode((v32 * inv[:, :, None, :]).astype(np.float32))
    codes[:, :, N:, :] = 0
    return codes, (amax / np.float32(448)).astype(np.float32)


def _quantize_scale_inverted(v, N):
    codes, scale = Lp.quantize_v(v, N)
    return codes, np.where(scale > 0, np.float32(1) / np.where(scale > 0, scale, 1), 0).astype(np.float32)


def _quantize_per_token(v, N):
    v32 = np.asarray(v, np.float32)
    amax = np.abs(v32).max(axis=3, keepdims=True)             # one scale per row, not per channel
    inv = (np.float32(448) / np.where(amax > 0, amax, 1)).astype(np.float32)
    codes = Lp.e4m3_encode((v32 * inv).astype(np.float32))
    codes[:, :, N:, :] = 0
    return codes, (amax[..., 0].max(axis=2) / np.float32(448)).astype(np.float32)


def _encode_pin_holds(encode):
    t = Lp.e4m3_table()[:0x7F]
    mids = ((t[1:] + t[:-1]) / 2).astype(np.float32)
    x = np.concatenate([mids, -mids, np.linspace(-460, 460, 4001, dtype=np.float32)])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return np.array_equal(encode(x), want)


def _quantize_pins_hold(quantize):
    v, codes, scale = _golden()
    got_codes, got_scale = quantize(v[None, None], v.shape[0])
    if not (np.array_equal(got_codes[0, 0], codes) and np.allclose(got_scale[0, 0], scale, rtol=1e-7, atol=0)):
        return False
    w = _v(N=300)
    w[:, :, 300:] = 1e4
    c1, s1 = quantize(w, 300)
    c2, s2 = Lp.quantize_v(w, 300)
    return np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_pins_accept_the_oracle():
    assert _encode_pin_holds(Lp.e4m3_encode)
    assert _quantize_pins_hold(Lp.quantize_v)


@pytest.mark.parametrize("bad", [_encode_ties_away, _encode_truncating])
def test_planted_encoding_mistakes_are_caught(bad):
    assert not _encode_pin_holds(bad)


@pytest.mark.parametrize("bad", [_quantize_amax_with_pad, _quantize_scale_inverted, _quantize_per_token])
def test_planted_quantization_mistakes_are_caught(bad):
    assert not _quantize_pins_hold(bad)
