"""Pins for the CPU oracle (no GPU).  Each test ties the oracle to something
other than itself: hand-derived closed forms (tests/golden/), pure-Python brute
force, and invariants of softmax attention, so that a dropped term, a wrong
sign or index, or a transposed operand anywhere in the oracle fails one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention as A
import synth
from tests.paging import paged

GOLD = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


def _gold():
    with open(GOLD) as f:
        return json.load(f)


def _one_request(keys, values, rng=None):
    k = np.asarray(keys, dtype=np.float64)[:, None, :]
    v = np.asarray(values, dtype=np.float64)[:, None, :]
    return paged([k], [v], 1, rng)


# ---------------------------------------------------------------- closed forms

def test_golden_two_key_decode():
    g = _gold()["two_key_decode"]
    kp, vp, bt, lens = _one_request(g["keys"], g["values"])
    # decode request r lives in block-table row 1 + r: prepend an empty row 0
    bt2 = np.vstack([bt, bt])
    lens2 = np.asarray([0, lens[0]], dtype=np.int32)
    q = np.asarray(g["q"], dtype=np.float64)[None, None, :]
    out = A.attend_decode(q, kp, vp, bt2, lens2, g["scale"], 1)
    np.testing.assert_allclose(out[0, 0], g["expected"], rtol=0, atol=1e-12)


def test_golden_three_key_causal_prefill():
    g = _gold()["three_key_causal_prefill"]
    kp, vp, bt, lens = _one_request(g["keys"], g["values"])
    q = np.asarray(g["q"], dtype=np.float64)[:, None, :]
    out = A.attend_prefill(q, kp, vp, bt, g["prior_ctx"], g["scale"], 1)
    np.testing.assert_allclose(out[:, 0], g["expected"], rtol=0, atol=1e-12)


def test_golden_gqa():
    g = _gold()["gqa_two_heads_one_kv_head"]
    kp, vp, bt, lens = _one_request(g["keys"], g["values"])
    bt2 = np.vstack([bt, bt])
    lens2 = np.asarray([0, lens[0]], dtype=np.int32)
    q = np.asarray(g["q"], dtype=np.float64)[None]
    out = A.attend_decode(q, kp, vp, bt2, lens2, g["scale"], 1)
    np.testing.assert_allclose(out[0], g["expected"], rtol=0, atol=1e-12)


def test_golden_split_merge():
    g = _gold()["two_split_merge"]
    q = np.asarray(g["q"])[None]
    K = np.asarray(g["keys"])
    V = np.asarray(g["values"])
    parts = [A.attend_partial(q, K, V, g["scale"], a, b) for a, b in g["splits"]]
    for (o, lse), exp in zip(parts, g["expected_partials"]):
        np.testing.assert_allclose(o[0], exp["o"], atol=1e-12)
        assert abs(lse[0] - exp["lse"]) < 1e-12
    np.testing.assert_allclose(A.lse_merge(parts)[0], g["expected"], atol=1e-12)


def test_single_key_returns_value():
    rng = np.random.default_rng(7)
    V = rng.standard_normal((1, 1, 8))
    K = rng.standard_normal((1, 1, 8))
    kp, vp, bt, lens = paged([K], [V], 1, rng)
    bt2 = np.vstack([bt, bt])
    q = rng.standard_normal((1, 3, 8)) * 5.0
    out = A.attend_decode(q, kp, vp, bt2, np.asarray([0, 1], dtype=np.int32), 0.3, 1)
    for h in range(3):
        np.testing.assert_allclose(out[0, h], V[0, 0], atol=1e-14)
    # prefill with no prior context: chunk row 0 sees exactly key 0
    qp = rng.standard_normal((1, 1, 8))
    outp = A.attend_prefill(qp, kp, vp, bt, 0, 0.3, 1)
    np.testing.assert_allclose(outp[0, 0], V[0, 0], atol=1e-14)


def test_zero_query_and_identical_keys_give_mean():
    rng = np.random.default_rng(8)
    L, d = 37, 16
    K = rng.standard_normal((L, 1, d))
    V = rng.standard_normal((L, 1, d))
    kp, vp, bt, lens = paged([K], [V], 1, rng)
    bt2 = np.vstack([bt, bt])
    lens2 = np.asarray([0, L], dtype=np.int32)
    out = A.attend_decode(np.zeros((1, 1, d)), kp, vp, bt2, lens2, 0.25, 1)
    np.testing.assert_allclose(out[0, 0], V[:, 0].mean(axis=0), atol=1e-13)
    Ksame = np.repeat(K[:1], L, axis=0)
    kp2, vp2, bt3, _ = paged([Ksame], [V], 1, rng)
    out2 = A.attend_decode(rng.standard_normal((1, 1, d)), kp2, vp2, np.vstack([bt3, bt3]), lens2, 0.25, 1)
    np.testing.assert_allclose(out2[0, 0], V[:, 0].mean(axis=0), atol=1e-13)


def test_rows_sum_to_one_via_constant_values():
    """With V = 1 everywhere the output is exactly the sum of the weights."""
    rng = np.random.default_rng(9)
    L, d = 50, 8
    K = rng.standard_normal((L, 2, d)) * 3
    V = np.ones((L, 2, d))
    kp, vp, bt, _ = paged([K], [V], 2, rng)
    q = rng.standard_normal((11, 4, d)) * 3
    out = A.attend_prefill(q, kp, vp, bt, L - 11, 0.7, 2)
    np.testing.assert_allclose(out, 1.0, atol=1e-13)


# ------------------------------------------------------------------ brute force

@pytest.mark.parametrize("seed", [0, 1])
def test_oracle_matches_brute_force(seed):
    w = synth.custom("brute", 4, 2, 16, 5, 19, [1, 7, 16, 17, 33], seed, 0.31)
    b = synth.make_batch(w)
    od = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    bd = A.attend_brute_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    np.testing.assert_allclose(od, bd, atol=1e-12)
    op = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    bp = A.attend_brute_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    np.testing.assert_allclose(op, bp, atol=1e-12)


def test_tiny_config_matches_brute_force_sampled():
    b = synth.make_batch(synth.tiny())
    od = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    bd = A.attend_brute_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    np.testing.assert_allclose(od, bd, atol=1e-12)
    rows = [0, 31, 63]
    op = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2, rows=rows)
    full = A.attend_brute_prefill(b.q_prefill[[0]], b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    np.testing.assert_allclose(op[0], full[0], atol=1e-12)


# ------------------------------------------------------------------- invariants

def test_split_merge_equals_unsplit():
    rng = np.random.default_rng(11)
    L, d = 301, 32
    q = rng.standard_normal((4, d)) * 2
    K = rng.standard_normal((L, d)) * 2
    V = rng.standard_normal((L, d))
    full = A.attend_rows(q, K, V, 0.2, [L] * 4)
    for cuts in ([0, 100, 301], [0, 1, 2, 300, 301], [0, 16, 48, 160, 256, 301]):
        parts = [A.attend_partial(q, K, V, 0.2, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
        np.testing.assert_allclose(A.lse_merge(parts), full, atol=1e-12)


def test_gqa_equals_repeated_kv_heads():
    w = synth.custom("gqa", 8, 2, 16, 9, 30, [5, 40], 3, 0.25)
    b = synth.make_batch(w)
    g = 4
    kp_rep = np.repeat(b.k_pool, g, axis=1)   # kv head h -> heads h*g .. h*g+g-1
    vp_rep = np.repeat(b.v_pool, g, axis=1)
    od = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    od_rep = A.attend_decode(b.q_decode, kp_rep, vp_rep, b.block_table, b.kv_lens, b.scale, 8)
    np.testing.assert_allclose(od, od_rep, atol=1e-13)
    op = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    op_rep = A.attend_prefill(b.q_prefill, kp_rep, vp_rep, b.block_table, b.prefill_ctx, b.scale, 8)
    np.testing.assert_allclose(op, op_rep, atol=1e-13)


@pytest.mark.parametrize("C", [0, 13, 32])
def test_causal_row_equals_decode_over_prefix(C):
    """Chunk row i (absolute position C+i) equals a decode query over the first C+i+1 tokens."""
    rng = np.random.default_rng(12 + C)
    P, d, Hkv, g = 20, 16, 2, 2
    K = rng.standard_normal((C + P, Hkv, d))
    V = rng.standard_normal((C + P, Hkv, d))
    kp, vp, bt, _ = paged([K], [V], Hkv, rng)
    q = rng.standard_normal((P, Hkv * g, d))
    op = A.attend_prefill(q, kp, vp, bt, C, 0.4, Hkv)
    for i in (0, 7, P - 1):
        bt2 = np.vstack([bt, bt])
        lens = np.asarray([0, C + i + 1], dtype=np.int32)
        od = A.attend_decode(q[i:i + 1], kp, vp, bt2, lens, 0.4, Hkv)
        np.testing.assert_allclose(op[i], od[0], atol=1e-13)


def test_paging_permutation_invariance():
    rng = np.random.default_rng(13)
    d, Hkv = 16, 2
    ks = [rng.standard_normal((L, Hkv, d)) for L in (3, 16, 50)]
    vs = [rng.standard_normal((L, Hkv, d)) for L in (3, 16, 50)]
    q = rng.standard_normal((2, 4, d))
    res = []
    for r in (None, np.random.default_rng(1), np.random.default_rng(2)):
        kp, vp, bt, lens = paged(ks, vs, Hkv, r)
        res.append(A.attend_decode(q, kp, vp, bt, lens, 0.5, Hkv))
    np.testing.assert_allclose(res[0], res[1], atol=1e-14)
    np.testing.assert_allclose(res[0], res[2], atol=1e-14)


def test_poison_slots_are_ignored():
    """Values in unused slots of a request's last page never reach the output."""
    b = synth.make_batch(synth.tiny())
    kp = b.k_pool.copy()
    vp = b.v_pool.copy()
    out0 = A.attend_decode(b.q_decode, kp, vp, b.block_table, b.kv_lens, b.scale, 2)
    L = int(b.kv_lens[2])        # 100 tokens: last page has 4 used slots
    blk = int(b.block_table[2, (L - 1) // 16])
    kp[blk, :, L % 16:, :] = synth.f32_to_bf16_bits(np.float32(-1000.0)).item()
    vp[blk, :, L % 16:, :] = synth.f32_to_bf16_bits(np.float32(1000.0)).item()
    out1 = A.attend_decode(b.q_decode, kp, vp, b.block_table, b.kv_lens, b.scale, 2)
    np.testing.assert_array_equal(out0, out1)


# ------------------------------------------------- planted mistakes are caught

def _mutants(orig):
    def no_scale(q, K, V, scale, limits):
        return orig(q, K, V, 1.0, limits)

    def off_by_one(q, K, V, scale, limits):
        return orig(q, K, V, scale, [max(1, x - 1) for x in limits])

    def swapped_kv(q, K, V, scale, limits):
        return orig(q, V, K, scale, limits)

    def no_max(q, K, V, scale, limits):
        s = (q @ K.T) * scale
        mask = np.arange(K.shape[0])[None, :] >= np.asarray(limits)[:, None]
        p = np.where(mask, 0.0, np.exp(s))
        return (p @ V) / (p.sum(axis=1, keepdims=True) + 1e-3)

    return {"no_scale": no_scale, "off_by_one": off_by_one, "swapped_kv": swapped_kv, "bad_norm": no_max}


@pytest.mark.parametrize("name", ["no_scale", "off_by_one", "swapped_kv", "bad_norm"])
def test_planted_mistake_fails_brute_force(monkeypatch, name):
    """A mistake planted in the oracle (CPU only) is caught by the brute-force pin."""
    monkeypatch.setattr(A, "attend_rows", _mutants(A.attend_rows)[name])
    w = synth.custom("brute", 4, 2, 16, 5, 19, [1, 7, 16, 17, 33], 0, 0.31)
    b = synth.make_batch(w)
    od = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    bd = A.attend_brute_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    op = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    bp = A.attend_brute_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    err = max(np.abs(od - bd).max(), np.abs(op - bp).max())
    assert err > 1e-3, f"mutant {name} not caught (err {err})"


def test_planted_gqa_mapping_mistake_is_caught(monkeypatch):
    """q head h -> kv head h % Hkv (instead of h // g) fails the GQA pin."""
    w = synth.custom("gqa", 8, 2, 16, 0, 0, [5, 40], 3, 0.25)
    b = synth.make_batch(w)
    kp_rep = np.repeat(b.k_pool, 4, axis=1)
    vp_rep = np.repeat(b.v_pool, 4, axis=1)
    q = A._as_f64(b.q_decode)
    wrong = np.empty_like(q)
    kp, vp = A._as_f64(b.k_pool), A._as_f64(b.v_pool)
    for r in range(2):
        L = int(b.kv_lens[1 + r])
        for h in range(8):
            K = A.gather_tokens(kp, b.block_table[1 + r], L, h % 2)
            V = A.gather_tokens(vp, b.block_table[1 + r], L, h % 2)
            wrong[r, h] = A.attend_rows(q[r, h:h + 1], K, V, b.scale, [L])[0]
    ref = A.attend_decode(b.q_decode, kp_rep, vp_rep, b.block_table, b.kv_lens, b.scale, 8)
    assert np.abs(wrong - ref).max() > 1e-3


# ----------------------------------------------- several prefill requests (batched)

def _tiny_batched(seed):
    w = synth.custom_batched("tiny_batched", 4, 2, 8, [(5, 3), (1, 0), (0, 0), (7, 9)], [6, 17, 1], seed,
                             scale=0.35)
    return synth.make_batch(w)


@pytest.mark.parametrize("seed", [41, 42])
def test_batched_oracle_matches_brute_force(seed):
    """Each prefill request reads its own block-table row and its own prior
    context; decodes start after the prefill rows (brute-force loops)."""
    b = _tiny_batched(seed)
    Hkv = b.workload.num_kv_heads
    got = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_qo_lens,
                                   b.prefill_kv_lens, b.scale, Hkv)
    parts, start = [], 0
    for i, (P, K) in enumerate(zip(b.prefill_qo_lens, b.prefill_kv_lens)):
        if P:
            parts.append(A.attend_brute_prefill(b.q_prefill[start:start + P], b.k_pool, b.v_pool, b.block_table,
                                                K - P, b.scale, Hkv, bt_row=i))
        start += P
    np.testing.assert_allclose(got, np.concatenate(parts), rtol=0, atol=1e-12)
    gd = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, Hkv,
                         first_row=b.num_prefill)
    bd = A.attend_brute_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, Hkv,
                               first_row=b.num_prefill)
    np.testing.assert_allclose(gd, bd, rtol=0, atol=1e-12)


def test_batched_request_order_invariance():
    """Reordering the prefill requests (their block-table rows, lengths and Q
    rows together) reorders the outputs and changes nothing else."""
    b = _tiny_batched(43)
    Hkv = b.workload.num_kv_heads
    qo, kv = b.prefill_qo_lens, b.prefill_kv_lens
    ref = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, qo, kv, b.scale, Hkv)
    starts = np.concatenate([[0], np.cumsum(qo)])
    perm = [3, 0, 2, 1]
    q_perm = np.concatenate([b.q_prefill[starts[i]:starts[i + 1]] for i in perm])
    bt = b.block_table.copy()
    bt[:len(qo)] = b.block_table[perm]
    got = A.attend_prefill_batched(q_perm, b.k_pool, b.v_pool, bt, [qo[i] for i in perm], [kv[i] for i in perm],
                                   b.scale, Hkv)
    want = np.concatenate([ref[starts[i]:starts[i + 1]] for i in perm])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_planted_batched_row_mistake_is_caught(monkeypatch):
    """A planted mistake -- every prefill request reading block-table row 0 --
    fails the brute-force pin above."""
    b = _tiny_batched(44)
    Hkv = b.workload.num_kv_heads
    orig = A.attend_prefill

    def always_row0(*args, **kw):
        kw["bt_row"] = 0
        return orig(*args, **kw)

    monkeypatch.setattr(A, "attend_prefill", always_row0)
    got = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_qo_lens,
                                   b.prefill_kv_lens, b.scale, Hkv)
    monkeypatch.undo()
    parts, start = [], 0
    for i, (P, K) in enumerate(zip(b.prefill_qo_lens, b.prefill_kv_lens)):
        if P:
            parts.append(A.attend_brute_prefill(b.q_prefill[start:start + P], b.k_pool, b.v_pool, b.block_table,
                                                K - P, b.scale, Hkv, bt_row=i))
        start += P
    assert np.abs(got - np.concatenate(parts)).max() > 1e-3
