"""Pins for the oracle's FP8 (e4m3) KV cache: the code table against torch's
float8_e4m3fn decoding (a library routine), encoding against torch's
round-to-nearest-even conversion and a hand-worked table in tests/golden, the
quantizing write against the bf16 write, and FP8 attention against the
pinned bf16 attention on exactly representable values."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_table_matches_library():
    codes = np.arange(256, dtype=np.uint8)
    mine, ref = oracle.e4m3_decode(codes), _torch_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(ref[~nan]))


def test_encode_golden():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_examples.json")))
    for e in g["encode"]:
        assert int(oracle.e4m3_encode([e["x"]])[0]) == e["code"], e


def test_encode_matches_library_rounding_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * rng.choice([1e-3, 0.1, 1, 30, 200], 200000),
                        rng.uniform(-448, 448, 50000)])
    x = x.astype(np.float32).astype(np.float64)
    x = x[np.abs(x) <= 448]  # beyond, the library gives NaN where the write saturates (pinned separately)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def test_encode_decode_round_trip_and_saturation():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)
    assert oracle.e4m3_encode([5e4, -5e4, np.inf, -np.inf]).tolist() == [0x7E, 0xFE, 0x7E, 0xFE]
    assert oracle.e4m3_encode([np.nan])[0] == 0x7F


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16)


def test_write_quantizes_into_the_bf16_layout():
    """Each written row holds encode(fp32(x) * fp32(1/scale)); the rows are the
    ones the bf16 write fills, the rest stay as they were."""
    rng = np.random.default_rng(1)
    NB, Hkv, bs, d, T = 10, 3, 16, 32, 9
    kc8 = rng.integers(0, 256, (NB, Hkv, bs, d)).astype(np.uint8)
    vc8 = rng.integers(0, 256, (NB, Hkv, bs, d)).astype(np.uint8)
    k = _bf16(rng.standard_normal((T, Hkv, d)) * 3)
    v = _bf16(rng.standard_normal((T, Hkv, d)))
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[2] = -1
    ks = np.array([0.02, 0.5, 3.0], np.float32)
    vs = np.array([0.01, 1.0, 0.25], np.float32)
    k2, v2 = oracle.kv_write_fp8(kc8, vc8, k, v, slots, ks, vs)
    kf = k.float().numpy() * (np.float32(1) / ks)[None, :, None]
    vf = v.float().numpy() * (np.float32(1) / vs)[None, :, None]
    written = np.zeros((NB, bs), bool)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        b, o = divmod(int(sl), bs)
        written[b, o] = True
        assert np.array_equal(k2[b, :, o], oracle.e4m3_encode(kf[t].astype(np.float64)))
        assert np.array_equal(v2[b, :, o], oracle.e4m3_encode(vf[t].astype(np.float64)))
    untouched = ~written
    assert np.array_equal(k2.transpose(0, 2, 1, 3)[untouched], kc8.transpose(0, 2, 1, 3)[untouched])


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)])
def test_attention_equals_bf16_attention_on_exact_values(Hq, Hkv):
    """With power-of-two scales every dequantized value is exact in bf16, so
    FP8 attention must equal the bf16 oracle on those values."""
    rng = np.random.default_rng(2)
    NB, bs, d, B = 12, 16, 64, 3
    kc8 = rng.integers(0, 256, (NB, Hkv, bs, d)).astype(np.uint8)
    vc8 = rng.integers(0, 256, (NB, Hkv, bs, d)).astype(np.uint8)
    kc8[(kc8 & 0x7F) == 0x7F] = 0x00  # no NaN codes
    vc8[(vc8 & 0x7F) == 0x7F] = 0x00
    ks = np.array([2.0 ** -6, 0.5, 1.0, 2.0][:Hkv], np.float32)
    vs = np.array([0.25, 2.0 ** -3, 1.0, 4.0][:Hkv], np.float32)
    tables = np.stack([rng.permutation(NB)[:4] for _ in range(B)]).astype(np.int32)
    ctx = np.array([1, 37, 64], np.int32)
    q = _bf16(rng.standard_normal((B, Hq, d)))
    out8 = oracle.paged_attention_fp8(q, kc8, vc8, ks, vs, tables, ctx, 0.125)
    kd = oracle.e4m3_decode(kc8) * ks[None, :, None, None]
    vd = oracle.e4m3_decode(vc8) * vs[None, :, None, None]
    out = oracle.paged_attention(q, _bf16(kd), _bf16(vd), tables, ctx, 0.125)
    assert np.allclose(out8, out, rtol=0, atol=1e-12)
