"""Pins for the FP8 (e4m3) KV-cache oracle and its input generator (no GPU).

The oracle decodes every stored byte exactly (oracle/fp8.py); the generator
quantises the bf16 cache to e4m3 (synth.f64_to_e4m3_bits).  Both are checked
against hand-decoded bytes in tests/golden/fp8_e4m3_cases.json, the decoder
also exhaustively against a second, table-free reading of the format, and the
FP8 decode attention against the bf16 oracle on the dequantised values."""
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import attention as A
from oracle import fp8

GOLD = os.path.join(os.path.dirname(__file__), "golden", "fp8_e4m3_cases.json")


def _gold():
    with open(GOLD) as f:
        return json.load(f)


def test_decode_matches_hand_decoded_bytes():
    for c in _gold()["decode"]:
        got = float(fp8.e4m3_to_f64(np.asarray([int(c["bits"], 16)], dtype=np.uint8))[0])
        if c["value"] == "nan":
            assert math.isnan(got), c
        else:
            assert got == c["value"] and math.copysign(1.0, got) == math.copysign(1.0, c["value"]), c


def test_decode_all_256_codes_by_brute_force():
    """Every byte against a reading written with plain integer arithmetic: value = sign * M * 2^E
    with M = 8 + m, E = e - 10 for normals and M = m, E = -9 for subnormals."""
    got = fp8.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    for b in range(256):
        s, e, m = b >> 7, (b >> 3) & 15, b & 7
        if e == 15 and m == 7:
            assert math.isnan(got[b])
            continue
        M, E = (m, -9) if e == 0 else (8 + m, e - 10)
        want = (-1.0 if s else 1.0) * M * 2.0 ** E
        assert got[b] == want, (hex(b), got[b], want)
    finite = got[~np.isnan(got)]
    assert finite.max() == 448.0 and finite.min() == -448.0


def test_quantiser_matches_hand_worked_roundings():
    for c in _gold()["quantise"]:
        got = int(synth.f64_to_e4m3_bits(np.asarray([c["value"]]))[0])
        assert got == int(c["bits"], 16), (c, hex(got))


def test_quantiser_is_nearest_and_round_trips():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(20000) * 40
    q = synth.f64_to_e4m3_bits(x)
    v = fp8.e4m3_to_f64(q)
    codes = fp8.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    codes = codes[~np.isnan(codes)]
    best = np.min(np.abs(codes[None, :] - np.clip(x, -448, 448)[:, None]), axis=1)
    assert np.array_equal(np.abs(v - np.clip(x, -448, 448)), best)
    # every finite code decodes and re-encodes to itself (-0 and +0 apart)
    allb = np.arange(256, dtype=np.uint8)
    ok = ~np.isnan(fp8.e4m3_to_f64(allb))
    assert np.array_equal(synth.f64_to_e4m3_bits(fp8.e4m3_to_f64(allb[ok])), allb[ok])


@pytest.mark.parametrize("mistake", ["bias8", "no_subnormal", "mantissa4"])
def test_planted_decode_mistakes_fail_the_goldens(mistake):
    bits = np.asarray([int(c["bits"], 16) for c in _gold()["decode"] if c["value"] != "nan"], dtype=np.uint8)
    want = np.asarray([c["value"] for c in _gold()["decode"] if c["value"] != "nan"])
    b = bits.astype(np.int64)
    e, m = (b >> 3) & 15, b & 7
    sign = np.where(b >> 7, -1.0, 1.0)
    if mistake == "bias8":
        got = sign * np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1 + m / 8.0, e - 8))
    elif mistake == "no_subnormal":
        got = sign * np.ldexp(1 + m / 8.0, e - 7)
    else:
        got = sign * np.where(e == 0, np.ldexp(m / 16.0, -6), np.ldexp(1 + m / 16.0, e - 7))
    assert not np.array_equal(got, want)


def test_fp8_cache_of_a_batch():
    b = synth.make_batch(synth.tiny())
    c = synth.fp8_cache(b)
    assert c.k_pool.dtype == np.uint8 and c.k_pool.shape == b.k_pool.shape
    assert c.k_scale.dtype == np.float32 and c.k_scale.shape == (b.workload.num_kv_heads,)
    # poison keeps its place: +448 in K, -448 in V (a live value reaches 448 only at its head's amax)
    kf = synth.bf16_bits_to_f32(b.k_pool)
    vf = synth.bf16_bits_to_f32(b.v_pool)
    assert (c.k_pool[kf == synth.POISON_K] == synth.POISON_E4M3_K).all()
    assert (c.v_pool[vf == synth.POISON_V] == synth.POISON_E4M3_V).all()
    assert (c.k_pool[kf != synth.POISON_K] == synth.POISON_E4M3_K).sum() <= b.workload.num_kv_heads
    # dequantised values are within half a quantum (3 mantissa bits: <= 1/16 relative) of the bf16 ones
    deq = fp8.dequant_pool(c.k_pool, c.k_scale)
    live = kf != synth.POISON_K
    rel = np.abs(deq[live] - kf[live]) / np.maximum(np.abs(kf[live]), 2.0 ** -6 * float(c.k_scale.max()))
    assert rel.max() <= 1.0 / 16 + 1e-12


def test_fp8_decode_is_the_bf16_oracle_on_dequantised_values():
    """Scales fold out exactly: V scaled by 2 doubles the output; K scaled by c equals the
    softmax scale times c."""
    b = synth.make_batch(synth.tiny())
    c = synth.fp8_cache(b)
    w = b.workload
    K = fp8.dequant_pool(c.k_pool, c.k_scale)
    V = fp8.dequant_pool(c.v_pool, c.v_scale)
    base = A.attend_decode(b.q_decode, K, V, b.block_table, b.kv_lens, b.scale, w.num_kv_heads)
    v2 = A.attend_decode(b.q_decode, K, fp8.dequant_pool(c.v_pool, c.v_scale * 2), b.block_table, b.kv_lens,
                         b.scale, w.num_kv_heads)
    np.testing.assert_allclose(v2, 2 * base, rtol=1e-13, atol=1e-13)
    k2 = A.attend_decode(b.q_decode, fp8.dequant_pool(c.k_pool, c.k_scale * 2), V, b.block_table, b.kv_lens,
                         b.scale / 2, w.num_kv_heads)
    np.testing.assert_allclose(k2, base, rtol=1e-12, atol=1e-12)
