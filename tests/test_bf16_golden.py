"""Pins for the bf16 conversions every oracle call and every input depends on
(no GPU): the oracle's exact bf16 -> float64 upcast and the generator's
float32 -> bf16 round-to-nearest-even, each against hand-worked bit patterns
in tests/golden/bf16_cases.json.  A shift, byte-order or rounding mistake in
either function fails here, and the planted mistakes below show that it would."""
import json
import os

import numpy as np
import pytest

from oracle import attention as A
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "bf16_cases.json")


def _gold():
    with open(GOLD) as f:
        return json.load(f)


def _decode_cases():
    c = _gold()["decode"]["cases"]
    return np.asarray([int(x["bits"], 16) for x in c], dtype=np.uint16), np.asarray([x["value"] for x in c])


def _rne_cases():
    c = _gold()["round_to_nearest_even"]["cases"]
    f32 = np.asarray([int(x["f32_bits"], 16) for x in c], dtype=np.uint32).view(np.float32)
    return f32, np.asarray([int(x["bf16_bits"], 16) for x in c], dtype=np.uint16)


def _same_f64(got, want):
    # bit-exact, so that -0.0 and subnormals are checked too
    return np.array_equal(np.asarray(got, dtype=np.float64).view(np.uint64), np.asarray(want).view(np.uint64))


def test_oracle_upcast_matches_hand_decoded_bits():
    bits, want = _decode_cases()
    got = A._as_f64(bits)
    assert got.dtype == np.float64
    assert _same_f64(got, want)
    # the same bits laid out as a paged pool go through the same upcast in gather_tokens
    pool = bits.reshape(1, 1, len(bits), 1)
    pool = np.concatenate([pool, np.zeros((1, 1, 16 - len(bits), 1), dtype=np.uint16)], axis=2)
    g = A.gather_tokens(pool, np.asarray([0]), len(bits), 0)[:, 0]
    assert _same_f64(g, want)


def test_synth_decoder_matches_hand_decoded_bits():
    bits, want = _decode_cases()
    assert _same_f64(synth.bf16_bits_to_f64(bits), want)


def test_round_to_nearest_even_matches_hand_worked_ties():
    f32, want = _rne_cases()
    got = synth.f32_to_bf16_bits(f32)
    assert got.dtype == np.uint16
    assert np.array_equal(got, want), [hex(x) for x in got]


def test_rounding_is_nearest_on_random_values():
    """Away from ties the rounded value is the nearer of the two bf16 neighbours
    (checked in float64 against both candidates, not through the bit trick)."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(50)
    b = synth.f32_to_bf16_bits(x)
    up = synth.bf16_bits_to_f64(b)
    lo_bits = (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    cand = np.stack([synth.bf16_bits_to_f64(lo_bits), synth.bf16_bits_to_f64(lo_bits + np.uint16(1))])
    err = np.abs(cand - x.astype(np.float64)[None])
    best = np.min(err, axis=0)
    assert np.array_equal(np.abs(up - x.astype(np.float64)), best)


@pytest.mark.parametrize("mistake", ["shift15", "byteswap", "truncate"])
def test_planted_conversion_mistakes_fail_the_goldens(mistake):
    bits, want = _decode_cases()
    f32, want_rne = _rne_cases()
    if mistake == "shift15":
        got = (bits.astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)
        assert not _same_f64(got, want)
    elif mistake == "byteswap":
        got = (bits.byteswap().astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
        assert not _same_f64(got, want)
    else:
        got = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)   # round toward zero
        assert not np.array_equal(got, want_rne)
