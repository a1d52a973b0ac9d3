"""Invariant pins for the plan rule (oracle/plan_ref.py), no GPU.

The pages fix no formula for the split or the ratio, so these check what any
valid plan must satisfy: every (decode request, kv head, key) and every
(prefill row, query head) is covered exactly once, the split cap holds, the
ordering is longest-first, and degenerate batches plan as expected."""
import dataclasses

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


def check_prefill_pieces(pl, Hq, qo, kv):
    """Every (request, tile, head) once, cut into contiguous KV pieces that cover
    its key tiles [0, ceil(kv_end / 64)) exactly once; split items carry
    consecutive partials and one merge entry; pieces are ordered longest first."""
    pieces = {}
    for q0, h, kv_end, req, j0, j1, part, midx in pl.prefill_items.tolist():
        P, C = qo[req], kv[req] - qo[req]
        assert 0 <= req < len(qo) and P > 0
        assert q0 % 128 == 0 and q0 < P and 0 <= h < Hq
        assert kv_end == C + min(q0 + 128, P)
        assert 0 <= j0 < j1 <= -(-kv_end // 64)
        pieces.setdefault((req, q0, h), []).append((j0, j1, part, midx))
    assert len(pieces) == sum(-(-P // 128) for P in qo) * Hq
    merges = pl.prefill_merge_items.tolist()
    used_parts = []
    for (req, q0, h), ps in pieces.items():
        ps.sort()
        kv_end = kv[req] - qo[req] + min(q0 + 128, qo[req])
        assert ps[0][0] == 0 and ps[-1][1] == -(-kv_end // 64)
        for a, b in zip(ps[:-1], ps[1:]):
            assert a[1] == b[0]
        if len(ps) == 1:
            assert ps[0][2:] == (-1, -1)
        else:
            midx = ps[0][3]
            assert all(x[3] == midx for x in ps)
            first, S, z0, z1 = merges[midx]
            assert (S, z0, z1) == (len(ps), 0, 0)
            assert [x[2] for x in ps] == list(range(first, first + S))
            used_parts.extend(range(first, first + S))
            # every piece spans at least 8 tiles, and every row of the tile sees a key of every piece
            for j0, j1, _, _ in ps:
                assert j1 - j0 >= 8 and 64 * j0 <= kv[req] - qo[req] + q0
    assert sorted(used_parts) == list(range(pl.num_prefill_partials))
    assert len(merges) == sum(1 for ps in pieces.values() if len(ps) > 1)
    keys = [min(64 * j1, kv_end) - 64 * j0 for _, _, kv_end, _, j0, j1, _, _ in pl.prefill_items.tolist()]
    assert keys == sorted(keys, reverse=True)


def check_plan(pl, Hq, Hkv, P, C, lens, sms=SMS, waves=2, minc=16, dwarps=6):
    # prefill coverage: each (tile, head) once, cut into KV pieces
    check_prefill_pieces(pl, Hq, [P], [C + P])
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


def check_split_minimal(pl, Hkv, lens, sms=SMS, waves=2, minc=16, dwarps=6):
    """The split size is the SMALLEST page count the rule allows, and each row is cut evenly.

    The rule takes c = max(min_chunk, ceil(N / cap)) and grows it one page at a
    time while c < the longest request's pages and the item count breaks the
    cap.  So whenever c is above that lower bound, c - 1 pages must break the
    cap (else the rule would have stopped there), and c itself must meet it
    unless no request can be cut any further (c = the longest request)."""
    cap = waves * sms * pl.ctas_per_sm * dwarps
    pages = [-(-L // PAGE) for L in lens]
    if not pages:
        return

    def items(c):
        return Hkv * sum(-(-p // c) for p in pages)

    lo = max(minc, -(-Hkv * sum(pages) // cap))
    c = pl.chunk_pages
    assert c >= lo
    if c > lo:
        assert items(c - 1) > cap, f"c = {c} is not minimal: {c - 1} pages also meet the cap"
    assert items(c) <= cap or c >= max(pages)
    assert len(pl.decode_items) == items(c)
    # even partition: the splits of one (request, kv head) differ by at most one page
    per_row = {}
    for r, kvh, k0, k1, *_ in pl.decode_items.tolist():
        per_row.setdefault((r, kvh), []).append(-(-k1 // PAGE) - k0 // PAGE)
    for (r, kvh), sizes in per_row.items():
        assert max(sizes) - min(sizes) <= 1, (r, kvh, sizes)
        assert sum(sizes) == pages[r] and len(sizes) == -(-pages[r] // c)


@pytest.mark.parametrize("w", CONFIGS, ids=lambda w: w.name)
def test_split_size_is_minimal_configs(w):
    check_split_minimal(_plan(w), w.num_kv_heads, _lens(w))


def test_split_size_is_minimal_random():
    rng = np.random.default_rng(123)
    for _ in range(200):
        Hkv = int(rng.choice([1, 2, 8]))
        B = int(rng.integers(1, 80))
        kind = rng.integers(0, 3)
        if kind == 0:
            lens = [int(x) for x in rng.integers(1, 5000, size=B)]
        elif kind == 1:
            lens = [int(x) for x in np.clip(np.rint(np.exp(np.log(2048) + rng.standard_normal(B))), 16, 32768)]
        else:
            lens = [int(rng.integers(1, 40000))] + [int(x) for x in rng.integers(1, 300, size=B - 1)]
        sms = int(rng.integers(1, 149))
        k = int(rng.choice([1, 2]))
        waves = int(rng.choice([1, 2, 3]))
        minc = int(rng.choice([1, 4, 16]))
        dw = int(rng.choice([4, 6]))
        pl = plan_ref(Hkv * 4, Hkv, 128, sms, 0, 0, lens, ctas_per_sm=k, max_waves=waves,
                      min_chunk_pages=minc, decode_warps=dw)
        check_split_minimal(pl, Hkv, lens, sms, waves, minc, dw)


def test_planted_non_minimal_split_is_caught():
    """A rule that stopped one page late would pass every coverage invariant; the minimality check catches it."""
    w = synth.llama3_8b_mix()
    pl = _plan(w)
    lens = _lens(w)
    late = plan_ref(w.num_q_heads, w.num_kv_heads, w.head_dim, SMS, 0, 0, lens,
                    min_chunk_pages=pl.chunk_pages + 1)
    check_plan(late, w.num_q_heads, w.num_kv_heads, 0, 0, lens, minc=pl.chunk_pages + 1)
    assert late.chunk_pages == pl.chunk_pages + 1
    with pytest.raises(AssertionError):
        check_split_minimal(late, w.num_kv_heads, lens)   # checked against the default minimum of 16 pages


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
    check_prefill_pieces(pl, Hq, qo, kv)
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


# ------------------------------------------------------------- prefill KV split

def _pieces(pl):
    return [tuple(x) for x in pl.prefill_items[:, 4:6].tolist()]


def test_prefill_split_hand_worked():
    """One 64-row tile over 1600 earlier tokens: kv_end = 1664 keys = 26 tiles, no decodes (never limited).
    One SM x 2 CTAs = 2 slots: tau = max(8, ceil(26 / 2)) = 13, S = 26 // 13 = 2 -> tiles [0,13), [13,26).
    Four SMs = 8 slots: tau = max(8, ceil(26 / 8)) = 8, S = 26 // 8 = 3 -> [0,8), [8,17), [17,26)."""
    two = plan_ref(1, 1, 128, 1, 64, 1664, [])
    assert sorted(_pieces(two)) == [(0, 13), (13, 26)]
    assert two.prefill_merge_items.tolist() == [[0, 2, 0, 0]] and two.num_prefill_partials == 2
    three = plan_ref(1, 1, 128, 4, 64, 1664, [])
    assert sorted(_pieces(three)) == [(0, 8), (8, 17), (17, 26)]
    # longest piece first: [8,17) and [17,26) hold 9 tiles (the last one 576 keys, kv_end is tile-aligned)
    assert _pieces(three) == [(8, 17), (17, 26), (0, 8)]
    assert three.prefill_items[:, 6].tolist() == [1, 2, 0]


def test_prefill_split_limited_by_colocated_decode_ctas():
    """A short prefill (<= 1536 tokens) next to decode work fills only its prefill-home CTAs (FlashInfer PR
    "Limit kv split when prefill tokens <= 1536"): on the Llama-3-8B mix the 128 base items already fill
    the 148 prefill-home CTAs (ratio 1:1, two CTAs per SM), so nothing is split; without the limit the
    296 slots give each item 2 pieces."""
    w = synth.llama3_8b_mix()
    lim = _plan(w)
    unl = _plan(w, split_unlimited=True)
    assert (lim.ratio_p, lim.ratio_d) == (1, 1)
    assert len(lim.prefill_items) == 128 and lim.num_prefill_partials == 0
    assert len(unl.prefill_items) == 256 and unl.num_prefill_partials == 256
    # each base item of n tiles is cut at n // 2
    for q0, h, kv_end, req, j0, j1, part, midx in unl.prefill_items.tolist():
        n = -(-kv_end // 64)
        assert (j0, j1) in ((0, n // 2), (n // 2, n))
    check_prefill_pieces(unl, 32, [512], [4608])


def test_prefill_split_limit_applies_only_to_short_prefills_with_decode():
    lens = [4096] * 8
    # no decode: the limit never applies, the flag changes nothing
    a = plan_ref(32, 8, 128, SMS, 512, 4608, [])
    b = plan_ref(32, 8, 128, SMS, 512, 4608, [], split_unlimited=True)
    assert np.array_equal(a.prefill_items, b.prefill_items) and len(a.prefill_items) == 256
    # more than 1536 prefill tokens: not limited either
    c = plan_ref_batched(8, 2, 128, SMS, [1024, 1024], [2048, 2048], lens)
    d = plan_ref_batched(8, 2, 128, SMS, [1024, 1024], [2048, 2048], lens, split_unlimited=True)
    assert np.array_equal(c.prefill_items, d.prefill_items) and c.num_prefill_partials > 0
    # 1536 tokens exactly: limited (prefill-home CTAs only) -> fewer pieces than without the limit
    e = plan_ref_batched(8, 2, 128, SMS, [1024, 512], [2048, 1024], lens)
    f = plan_ref_batched(8, 2, 128, SMS, [1024, 512], [2048, 1024], lens, split_unlimited=True)
    assert len(e.prefill_items) < len(f.prefill_items)


def test_prefill_split_knob_and_caps():
    # one 128-row tile over 16384 earlier tokens, 8 heads, no decode: 8 base items of 258 tiles, 296 slots
    base = plan_ref(8, 8, 128, SMS, 128, 16512, [])
    assert base.num_prefill_partials == 8 * 16          # tau = 8 -> 258 // 8 = 32 pieces, capped at 16
    two = plan_ref(8, 8, 128, SMS, 128, 16512, [], prefill_splits=2)
    assert two.num_prefill_partials == 16 and len(two.prefill_merge_items) == 8
    off = plan_ref(8, 8, 128, SMS, 128, 16512, [], prefill_splits=1)
    assert off.num_prefill_partials == 0 and len(off.prefill_items) == 8
    # base items that already fill every slot are never split (long-context mix: 256 items >= 148 slots)
    w = synth.long_context_mix()
    assert _plan(w).num_prefill_partials == 0 and _plan(w, split_unlimited=True).num_prefill_partials == 0
    # short items (< 16 tiles) are never cut below 8 tiles
    short = plan_ref(4, 4, 128, SMS, 64, 960, [])     # 15 tiles: 15 // 8 = 1 piece
    assert short.num_prefill_partials == 0
    with pytest.raises(PlanError):
        plan_ref(8, 8, 128, SMS, 128, 16512, [], prefill_splits=17)


def test_planted_split_mistakes_fail_the_piece_invariants():
    """Pieces that overlap, leave a gap, or carry a wrong partial index break check_prefill_pieces."""
    pl = plan_ref(1, 1, 128, 4, 64, 1664, [])
    for col, delta in ((5, 1), (4, -1), (6, 1)):
        bad = dataclasses.replace(pl, prefill_items=pl.prefill_items.copy())
        bad.prefill_items[0, col] += delta
        with pytest.raises(AssertionError):
            check_prefill_pieces(bad, 1, [64], [1664])


def test_prefill_split_limited_counts_one_slot_per_sm():
    """With every CTA prefill-home (ratio 1:0) a short prefill beside decode work still counts one prefill
    slot per SM: the Llama-3-8B mix's 128 items are not cut (a second prefill CTA on an SM would only queue
    behind the first); without the limit they are cut for all 296 CTA slots."""
    w = synth.llama3_8b_mix()
    forced = _plan(w, ratio_p=1, ratio_d=0)
    assert (forced.ratio_p, forced.ratio_d) == (1, 0) and forced.num_prefill_partials == 0
    assert _plan(w, ratio_p=1, ratio_d=0, split_unlimited=True).num_prefill_partials == 256
    one = _plan(w, ctas_per_sm=1, split_unlimited=True)      # one CTA per SM: 148 slots either way
    assert one.num_prefill_partials == _plan(w, ctas_per_sm=1).num_prefill_partials == 0
