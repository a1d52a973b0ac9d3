"""Invariant pins for the plan rule (oracle/plan_ref.py), no GPU.

The pages fix no formula for the split or the ratio, so these check what any
valid plan must satisfy: every (decode request, kv head, key) and every
(prefill row, query head) is covered exactly once, the split cap holds, the
ordering is longest-first, and degenerate batches plan as expected."""
import numpy as np
import pytest

import synth
from oracle.plan_ref import plan_ref, plan_ref_batched, PlanError, PAGE

SMS = 148


def _lens(w):
    b_lens = synth._draw_lengths(np.random.default_rng(w.seed), w)
    return [int(x) for x in b_lens]


CONFIGS = [synth.tiny(), synth.llama3_8b_mix(), synth.long_context_mix(), synth.decode_heavy_mix()] + synth.sweep_points()


def _plan(w, **kw):
    P, C = w.prefill_len, w.prefill_ctx
    return plan_ref(w.num_q_heads, w.num_kv_heads, w.head_dim, SMS, P, C + P, _lens(w), **kw)


def check_plan(pl, Hq, Hkv, P, C, lens, sms=SMS, waves=2, minc=16, dwarps=6):
    # prefill coverage: each (tile, head) once, kv_end = C + tile end
    T = -(-P // 128)
    seen = set()
    for q0, h, kv_end, req in pl.prefill_items.tolist():
        assert q0 % 128 == 0 and 0 <= h < Hq and req == 0
        assert kv_end == C + min(q0 + 128, P)
        assert (q0, h) not in seen
        seen.add((q0, h))
    assert len(seen) == T * Hq
    # prefill order: longest (highest tile) first
    q0s = pl.prefill_items[:, 0].tolist()
    assert q0s == sorted(q0s, reverse=True)
    # decode coverage: every key of every (r, kvh) exactly once, page-aligned splits
    cover = {}
    merges = pl.merge_items.tolist()
    for r, kvh, k0, k1, part, midx, nsplit, c in pl.decode_items.tolist():
        assert c == 0
        if part < 0:
            assert midx == -1 and nsplit == 1
        else:
            assert merges[midx][:2] == [r, kvh] and merges[midx][3] == nsplit
            assert merges[midx][2] <= part < merges[midx][2] + nsplit
        assert 0 <= r < len(lens) and 0 <= kvh < Hkv
        assert k0 % PAGE == 0 and k0 < k1 <= lens[r]
        assert (k1 - k0) <= pl.chunk_pages * PAGE or part == -1
        cover.setdefault((r, kvh), []).append((k0, k1, part))
    for r, L in enumerate(lens):
        for kvh in range(Hkv):
            segs = sorted(cover[(r, kvh)])
            assert segs[0][0] == 0 and segs[-1][1] == L
            for (a0, a1, _), (b0, b1, _) in zip(segs[:-1], segs[1:]):
                assert a1 == b0
            if len(segs) == 1:
                assert segs[0][2] == -1
            else:
                assert all(s[2] >= 0 for s in segs)
    # ordering: non-increasing page count
    pages = [-(-(k1 - k0) // PAGE) for _, _, k0, k1, *_ in pl.decode_items.tolist()]
    assert pages == sorted(pages, reverse=True)
    # cap: at most max_waves * decode warps items unless nothing splits
    cap = waves * sms * pl.ctas_per_sm * dwarps
    if pl.num_partials > 0:
        assert len(pl.decode_items) <= cap
    # merge items: contiguous partial ranges covering all partials once
    parts = []
    for r, kvh, first, S in pl.merge_items.tolist():
        assert S >= 2
        parts.extend(range(first, first + S))
        mine = sorted(p for (_, _, p) in cover[(r, kvh)])
        assert mine == list(range(first, first + S))
    assert sorted(parts) == list(range(pl.num_partials))
    assert pl.chunk_pages >= minc


@pytest.mark.parametrize("w", CONFIGS, ids=lambda w: w.name)
def test_plan_invariants_configs(w):
    pl = _plan(w)
    check_plan(pl, w.num_q_heads, w.num_kv_heads, w.prefill_len, w.prefill_ctx, _lens(w))


def test_plan_invariants_random():
    rng = np.random.default_rng(99)
    for _ in range(60):
        Hkv = int(rng.choice([1, 2, 8]))
        g = int(rng.choice([1, 2, 4, 8]))
        P = int(rng.choice([0, 1, 127, 128, 129, 700]))
        C = int(rng.integers(0, 3000)) if P else 0
        B = int(rng.integers(0 if P else 1, 40))
        lens = [int(x) for x in rng.integers(1, 5000, size=B)]
        sms = int(rng.integers(1, 149))
        k = int(rng.choice([0, 1, 2]))
        waves = int(rng.choice([0, 1, 2, 3]))
        dw = int(rng.choice([4, 6]))
        pl = plan_ref(Hkv * g, Hkv, 128, sms, P, C + P, lens, ctas_per_sm=k, max_waves=waves, decode_warps=dw)
        check_plan(pl, Hkv * g, Hkv, P, C, lens, sms, waves or 2, dwarps=dw)


def test_split_cap_counts_decode_warps():
    """Six decode warps per CTA allow 1.5x the items of four: the cap of four warps at 3 waves."""
    w = synth.decode_heavy_mix()
    six = _plan(w)
    four = _plan(w, decode_warps=4)
    four_w3 = _plan(w, decode_warps=4, max_waves=3)
    assert len(six.decode_items) > len(four.decode_items)
    np.testing.assert_array_equal(six.decode_items, four_w3.decode_items)
    with pytest.raises(PlanError):
        _plan(w, decode_warps=5)


def test_ratio_rules():
    w = synth.llama3_8b_mix()
    assert (_plan(w).ratio_p, _plan(w).ratio_d) == (1, 1)
    pl = _plan(w, ratio_p=2, ratio_d=6)
    assert (pl.ratio_p, pl.ratio_d) == (1, 3)
    assert (_plan(w, ratio_p=0, ratio_d=5).ratio_p, _plan(w, ratio_p=0, ratio_d=5).ratio_d) == (0, 1)
    po = plan_ref(32, 8, 128, SMS, 1024, 5120, [])
    assert (po.ratio_p, po.ratio_d) == (1, 0) and len(po.decode_items) == 0
    do = plan_ref(32, 8, 128, SMS, 0, 0, [4096] * 8)
    assert (do.ratio_p, do.ratio_d) == (0, 1) and len(do.prefill_items) == 0
    one = _plan(w, ctas_per_sm=1)
    assert (one.ratio_p, one.ratio_d) == (1, 0)


def test_decode_heavy_splits_long_tail():
    w = synth.decode_heavy_mix()
    pl = _plan(w)
    longest = max(k1 - k0 for _, _, k0, k1, *_ in pl.decode_items.tolist())
    assert longest <= pl.chunk_pages * PAGE
    assert pl.num_partials > 0 and len(pl.merge_items) > 0


@pytest.mark.parametrize("bad", [
    dict(num_q_heads=30, num_kv_heads=8),
    dict(num_q_heads=32, num_kv_heads=2),      # g = 16 unsupported
    dict(head_dim=96),
    dict(page_size=32),
    dict(num_sms=0),
    dict(ctas_per_sm=4),
    dict(prefill_len=10, prefill_kv_len=5),
    dict(decode_lens=[0]),
    dict(decode_lens=[-3]),
    dict(ratio_p=-1),
])
def test_plan_rejects(bad):
    args = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, num_sms=SMS, prefill_len=64,
                prefill_kv_len=128, decode_lens=[100, 200])
    kw = {}
    for k, v in bad.items():
        if k in ("page_size", "ctas_per_sm", "ratio_p"):
            kw[k] = v
        else:
            args[k] = v
    with pytest.raises(PlanError):
        plan_ref(**args, **kw)


def check_prefill_batched(pl, Hq, qo, kv):
    """Every (request, tile, head) once with its own kv_end, longest first,
    and a request table of consecutive q_prefill rows."""
    seen = set()
    for q0, h, kv_end, req in pl.prefill_items.tolist():
        P, C = qo[req], kv[req] - qo[req]
        assert 0 <= req < len(qo) and P > 0
        assert q0 % 128 == 0 and q0 < P and 0 <= h < Hq
        assert kv_end == C + min(q0 + 128, P)
        assert (req, q0, h) not in seen
        seen.add((req, q0, h))
    assert len(seen) == sum(-(-P // 128) for P in qo) * Hq
    ends = pl.prefill_items[:, 2].tolist()
    assert ends == sorted(ends, reverse=True)
    start = 0
    for i, (q_start, P, C, z) in enumerate(pl.prefill_requests.tolist()):
        assert (q_start, P, z) == (start, qo[i], 0)
        assert C == (kv[i] - qo[i] if qo[i] > 0 else 0)
        start += P


BATCHED = [
    ([300, 50, 129], [900, 50, 129], [100, 2000, 17]),
    ([512, 512, 1024], [4608, 1024, 5120], list(range(300, 6000, 300))),
    ([0, 200, 0, 7], [10, 300, 0, 7], [64]),
    ([1536], [1536], []),
    ([128] * 9, [128 * (i + 1) for i in range(9)], [4096] * 4),
]


@pytest.mark.parametrize("case", BATCHED, ids=lambda c: f"np{len(c[0])}_b{len(c[2])}")
def test_batched_plan_invariants(case):
    qo, kv, lens = case
    pl = plan_ref_batched(8, 2, 128, SMS, qo, kv, lens)
    check_prefill_batched(pl, 8, qo, kv)
    # the decode side is planned exactly as with one prefill request of the same work
    one = plan_ref(8, 2, 128, SMS, 0, 0, lens)
    assert np.array_equal(pl.decode_items, one.decode_items)
    assert np.array_equal(pl.merge_items, one.merge_items)


def test_batched_one_request_is_the_single_form():
    a = plan_ref(32, 8, 128, SMS, 512, 4608, [1000, 2500, 4096])
    b = plan_ref_batched(32, 8, 128, SMS, [512], [4608], [1000, 2500, 4096])
    for f in ("prefill_items", "decode_items", "merge_items", "prefill_requests"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    assert (a.ratio_p, a.ratio_d, a.chunk_pages) == (b.ratio_p, b.ratio_d, b.chunk_pages)


def test_batched_ratio_counts_every_request():
    # many prefill requests make the batch prefill-heavy; the same work in one request plans the same ratio
    many = plan_ref_batched(32, 8, 128, SMS, [512] * 8, [4608] * 8, [2048] * 4, ctas_per_sm=1)
    assert (many.ratio_p, many.ratio_d) == (1, 0)
    mixed = plan_ref_batched(32, 8, 128, SMS, [512, 512], [4608, 4608], [2048] * 64)
    assert (mixed.ratio_p, mixed.ratio_d) == (1, 1)


@pytest.mark.parametrize("qo,kv", [([-1], [5]), ([10], [5]), ([10, 5], [10]), ([1 << 24, 1], [1 << 24, 1])])
def test_batched_rejects(qo, kv):
    with pytest.raises(PlanError):
        plan_ref_batched(8, 2, 128, SMS, qo, kv, [100])


def test_plan_rejects_too_many_heads_and_overflowing_work():
    """More than 4096 query heads, or work counts past int64, are rejected before anything is built."""
    with pytest.raises(PlanError):
        plan_ref(4104, 513, 128, SMS, 64, 128, [100])
    big = 1 << 24   # 4 d Hq * (about P^2 / 2) keys seen = 2^21 * 2^47 > 2^63
    with pytest.raises(PlanError):
        plan_ref_batched(4096, 512, 128, SMS, [big], [big], [100])
    pl = plan_ref_batched(4096, 512, 128, SMS, [128], [1 << 20], [100])
    assert len(pl.prefill_items) == 4096 and (pl.prefill_items[:, 2] == 1 << 20).all()
