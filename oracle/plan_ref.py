"""The scheduling plan rule, restated in plain Python (test oracle; see package doc).

The pages describe the knobs but give no formula for them (POD-Attention
explainer, "How POD-Attention overlaps prefill and decode": 2 or 4 CTAs per SM,
split-KV capped at two full waves, CTAs allocated in proportion to the batch's
prefill:decode mix; FlashInfer POD PR "Limit kv split when prefill tokens <=
1536": the split count accounts for co-located decode CTAs).  This module is
the written rule that the C planner must reproduce bit for bit.  Parity of the
plan is therefore unpinned by the sources; tests pin it by invariants.

Rule
  Validation: Hq % Hkv == 0, Hq <= 4096; g = Hq/Hkv in 1..8; d in {64, 128}; page == 16;
    1 <= num_sms <= 512; ctas_per_sm in {0 (auto = 2), 1, 2}; ratios >= 0;
    max_waves >= 0 (0 = 2); min_chunk_pages >= 0 (0 = 16); 0 <= prefill_splits <= 16
    (0 = the rule below, 1 = never split the prefill); P >= 0;
    if P > 0: P <= prefill_kv_len <= 2^24; 0 <= B <= 65536; 1 <= L_r <= 2^24;
    sum_r L_r <= 2^31 - 1; every work count reported (4 d Hq sum of keys seen
    over prefill rows, 4 d Hq sum L_r, 4 d Hkv K/V tokens, 4 d Hq Q/O rows)
    fits int64.
  Prefill requests i = 0 .. NP-1 (chunk P_i over C_i = kv_i - P_i earlier
    tokens; the one-prefill form is NP = 1, P_0 = P).  Base prefill items (one
    128-row query tile of one query head each): for i, for t = T_i-1 .. 0
    (T_i = ceil(P_i/128)), for h = 0 .. Hq-1: (q0 = 128 t, h,
    kv_end = C_i + min(128 (t+1), P_i), request i), n = ceil(kv_end / 64)
    key tiles.  Prefill request table (q_start_i = P_0 + .. + P_{i-1}, P_i,
    C_i, 0).
  Prefill KV split (after the ratio below; FlashInfer PR "Limit kv split when
    prefill tokens <= 1536": the prefill's split count leaves room for the
    decode CTAs co-located on the same SMs while the prefill is short):
    limited = (B > 0 and sum_i P_i <= 1536 and the unlimited ablation is
    off); slots = num_sms if limited (one prefill slot per SM: the SM's
    other CTA, decode-home or a second prefill-home one, stays for decode)
    else num_sms * k;
    n0 = number of base items.  If prefill_splits == 1, or n0 == 0, or
    n0 >= slots: every item has S = 1 piece.  Otherwise W = sum of n over the
    base items, tau = max(8, ceil(W / slots)) and an item of n tiles gets
    S = min(smax, max(1, floor(n / tau))) pieces, smax = prefill_splits if
    >= 2 else 16.  Piece s covers key tiles [floor(s n / S), floor((s+1) n / S)),
    i.e. keys [64 j0, min(64 j1, kv_end)); every piece is at least 8 tiles
    long, so every row of the tile sees at least one key of every piece.
    Prefill items (q0, h, kv_end, request, j0, j1, partial, merge): partial =
    running index over the pieces of split items in base-item order, else
    -1; merge = index of the item's prefill merge entry, else -1.  Prefill
    merge entries (first partial, S, 0, 0), one per split base item, in
    base-item order.  All pieces are then stably sorted by their key count,
    longest first.
  Decode split: W = num_sms * ctas_per_sm * decode warps per CTA (6, or 4 in
    the four-warp ablation); cap = max_waves * W;
    pages_r = ceil(L_r / 16); N = Hkv * sum pages_r; maxp = max pages_r;
    c = max(min_chunk_pages, ceil(N / cap)); then c += 1 while c < maxp and
    Hkv * sum ceil(pages_r / c) > cap.  Decode request r (block-table row
    NP + r) is cut into
    S_r = ceil(pages_r / c) splits; split s covers pages
    [floor(s pages_r / S_r), floor((s+1) pages_r / S_r)), i.e. tokens
    [16 p0, min(16 p1, L_r)).
  Decode items (r, kv_head, k0, k1, partial, merge, S_r, 0): partial = running
    index over (r, kv_head, s) of rows with S_r > 1, else -1; merge = index of
    the row's merge item, else -1; sorted by (-pages, r, kv_head, s).
  Merge items (r, kv_head, first_partial, S_r) for every (r, kv_head) with S_r > 1,
    in (r, kv_head) order.
  Ratio p:d of per-SM tickets (ticket t -> prefill iff t mod (p+d) < p):
    explicit (ratio_p, ratio_d) reduced by gcd (a zero side gives 1:0 or 0:1);
    proportional (both 0): no prefill -> 0:1; no decode -> 1:0; otherwise
    cost_pre = 4 d sum over every prefill request's rows of keys seen, times Hq (FLOPs);
    cost_dec = 248 * 4 d Hkv sum_r L_r (bytes x 248, the measured B200
    tensor-FLOP/s per HBM-byte/s); k = ctas_per_sm;
    n_p = floor((2 k cost_pre + tot) / (2 tot)), tot = cost_pre + cost_dec,
    clamped to [1, k-1] when k >= 2 and n_p = 1 when k = 1; but n_p = k when
    2 cost_pre >= tot (the prefill side dominates: every CTA starts prefill-first
    and decode fills in as CTAs run out of prefill items; measured on B200, this
    beats 1:1 by ~16% exactly on the sweep points where it applies and loses
    where decode holds more than half the roofline cost); (p, d) = (n_p, k - n_p)
    reduced by gcd (k = 1 gives 1:0).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Sequence

import numpy as np

PAGE = 16
BM = 128
BN = 64                     # keys per prefill key tile
SPLIT_LIMIT_TOKENS = 1536   # prefill tokens up to which the split leaves room for co-located decode CTAs
MIN_SPLIT_TILES = 8         # shortest prefill piece, in key tiles
MAX_PREFILL_SPLITS = 16
DECODE_WARPS = 6            # per CTA: every warp decodes (4 in the four-warp ablation)
COST_RATIO = 248
MAX_SMS = 512
MAX_PREFILL_REQUESTS = 4096
MAX_HEADS = 4096
INT64_MAX = (1 << 63) - 1


class PlanError(ValueError):
    pass


@dataclasses.dataclass
class PlanRef:
    prefill_items: np.ndarray   # int32 [n, 8]: q0, q head, kv_end, request, j0, j1, partial, merge
    decode_items: np.ndarray    # int32 [n, 8]
    merge_items: np.ndarray     # int32 [n, 4]
    ctas_per_sm: int
    ratio_p: int
    ratio_d: int
    chunk_pages: int
    num_partials: int
    prefill_requests: np.ndarray = None   # int32 [NP, 4]: q_start, P, C, 0
    prefill_merge_items: np.ndarray = None   # int32 [n, 4]: first partial, pieces, 0, 0
    num_prefill_partials: int = 0


def _ceil(a: int, b: int) -> int:
    return -(-a // b)


def plan_ref(num_q_heads: int, num_kv_heads: int, head_dim: int, num_sms: int,
             prefill_len: int, prefill_kv_len: int, decode_lens: Sequence[int], **knobs) -> PlanRef:
    """One prefill request (block-table row 0, P = 0 for none) and B decodes (rows 1..B)."""
    return plan_ref_batched(num_q_heads, num_kv_heads, head_dim, num_sms, [prefill_len], [prefill_kv_len],
                            decode_lens, **knobs)


def plan_ref_batched(num_q_heads: int, num_kv_heads: int, head_dim: int, num_sms: int,
                     prefill_qo_lens: Sequence[int], prefill_kv_lens: Sequence[int], decode_lens: Sequence[int], *,
                     page_size: int = 16, ctas_per_sm: int = 0, ratio_p: int = 0, ratio_d: int = 0,
                     max_waves: int = 0, min_chunk_pages: int = 0, decode_warps: int = DECODE_WARPS,
                     prefill_splits: int = 0, split_unlimited: bool = False) -> PlanRef:
    """NP prefill requests (block-table rows 0..NP-1) and B decodes (rows NP..NP+B-1)."""
    Hq, Hkv, d = int(num_q_heads), int(num_kv_heads), int(head_dim)
    pre_qo = [int(x) for x in prefill_qo_lens]
    pre_kv = [int(x) for x in prefill_kv_lens]
    lens = [int(x) for x in decode_lens]
    B = len(lens)
    if Hq <= 0 or Hkv <= 0 or Hq % Hkv or Hq > MAX_HEADS:
        raise PlanError("invalid head counts")
    g = Hq // Hkv
    if g > 8 or d not in (64, 128) or page_size != PAGE:
        raise PlanError("unsupported")
    if not (1 <= num_sms <= MAX_SMS) or ctas_per_sm not in (0, 1, 2):
        raise PlanError("invalid launch knobs")
    if ratio_p < 0 or ratio_d < 0 or max_waves < 0 or min_chunk_pages < 0 or not (0 <= prefill_splits <= MAX_PREFILL_SPLITS):
        raise PlanError("invalid knobs")
    if len(pre_qo) != len(pre_kv) or len(pre_qo) > MAX_PREFILL_REQUESTS:
        raise PlanError("invalid prefill requests")
    for P, KVp in zip(pre_qo, pre_kv):
        if P < 0 or (P > 0 and not (P <= KVp <= (1 << 24))):
            raise PlanError("invalid prefill lengths")
    if sum(pre_qo) > (1 << 24):
        raise PlanError("invalid prefill lengths")
    if B > 65536 or any(not (1 <= L <= (1 << 24)) for L in lens) or sum(lens) > (1 << 31) - 1:
        raise PlanError("invalid decode lengths")
    k = 2 if ctas_per_sm == 0 else ctas_per_sm
    waves = 2 if max_waves == 0 else max_waves
    minc = 16 if min_chunk_pages == 0 else min_chunk_pages
    ctx = [KVp - P if P > 0 else 0 for P, KVp in zip(pre_qo, pre_kv)]
    # the work counts a plan reports (prefill FLOPs, decode FLOPs, K/V bytes, Q/O bytes) must fit int64
    rows_keys = sum(P * (C + 1) + P * (P - 1) // 2 for P, C in zip(pre_qo, ctx))
    pre_kv_tokens = sum(C + P for P, C in zip(pre_qo, ctx) if P > 0)
    if max(4 * d * Hq * rows_keys, 4 * d * Hq * sum(lens), 4 * d * Hkv * (pre_kv_tokens + sum(lens)),
           4 * d * Hq * (sum(pre_qo) + B)) > INT64_MAX:
        raise PlanError("work counts overflow")

    # prefill items per request, last tile first; then all requests' items longest first
    pre = []
    for i, (P, C) in enumerate(zip(pre_qo, ctx)):
        for t in range(_ceil(P, BM) - 1, -1, -1):
            for h in range(Hq):
                pre.append((BM * t, h, C + min(BM * (t + 1), P), i))
    preq, q_start = [], 0
    for P, C in zip(pre_qo, ctx):
        preq.append((q_start, P, C, 0))
        q_start += P

    # decode split
    if decode_warps not in (4, 6):
        raise PlanError("decode warps per CTA must be 4 or 6")
    W = num_sms * k * decode_warps
    cap = waves * W
    pages = [_ceil(L, PAGE) for L in lens]
    N = Hkv * sum(pages)
    maxp = max(pages) if pages else 0
    c = max(minc, _ceil(N, cap))
    while c < maxp and Hkv * sum(_ceil(p, c) for p in pages) > cap:
        c += 1
    dec = []
    merge = []
    npart = 0
    for r in range(B):
        S = _ceil(pages[r], c) if pages[r] > 0 else 1
        for kvh in range(Hkv):
            first = npart
            midx = len(merge) if S > 1 else -1
            for s in range(S):
                p0 = (s * pages[r]) // S
                p1 = ((s + 1) * pages[r]) // S
                part = -1
                if S > 1:
                    part = npart
                    npart += 1
                dec.append((p1 - p0, r, kvh, s, (r, kvh, PAGE * p0, min(PAGE * p1, lens[r]), part, midx, S, 0)))
            if S > 1:
                merge.append((r, kvh, first, S))
    dec.sort(key=lambda e: (-e[0], e[1], e[2], e[3]))

    # ticket ratio
    n_pre, n_dec = len(pre), len(dec)
    if ratio_p or ratio_d:
        if ratio_p == 0:
            p_, d_ = 0, 1
        elif ratio_d == 0:
            p_, d_ = 1, 0
        else:
            gg = math.gcd(ratio_p, ratio_d)
            p_, d_ = ratio_p // gg, ratio_d // gg
    elif n_pre == 0:
        p_, d_ = 0, 1
    elif n_dec == 0:
        p_, d_ = 1, 0
    else:
        rows_keys = 0
        for P, C in zip(pre_qo, ctx):
            for t in range(_ceil(P, BM)):
                q0 = BM * t
                n = min(BM, P - q0)
                rows_keys += n * (C + 1) + n * q0 + n * (n - 1) // 2
        cost_pre = 4 * d * Hq * rows_keys
        cost_dec = COST_RATIO * 4 * d * Hkv * sum(lens)
        tot = cost_pre + cost_dec
        n_p = (2 * k * cost_pre + tot) // (2 * tot)
        if k >= 2:
            n_p = min(max(n_p, 1), k - 1)
        else:
            n_p = 1
        if 2 * cost_pre >= tot:
            n_p = k
        p_, d_ = n_p, k - n_p
        if d_ == 0:
            p_ = 1
        else:
            gg = math.gcd(p_, d_)
            p_, d_ = p_ // gg, d_ // gg

    # prefill KV split
    limited = B > 0 and sum(pre_qo) <= SPLIT_LIMIT_TOKENS and not split_unlimited
    slots = num_sms if limited else num_sms * k
    tiles = [_ceil(kv_end, BN) for (_, _, kv_end, _) in pre]
    n0 = len(pre)
    if prefill_splits == 1 or n0 == 0 or n0 >= slots:
        nsplit = [1] * n0
    else:
        tau = max(MIN_SPLIT_TILES, _ceil(sum(tiles), slots))
        smax = prefill_splits if prefill_splits >= 2 else MAX_PREFILL_SPLITS
        nsplit = [min(smax, max(1, n // tau)) for n in tiles]
    pieces, pmerge, nppart = [], [], 0
    for (q0, h, kv_end, i), n, S in zip(pre, tiles, nsplit):
        midx = len(pmerge) if S > 1 else -1
        if S > 1:
            pmerge.append((nppart, S, 0, 0))
        for sp in range(S):
            j0, j1 = (sp * n) // S, ((sp + 1) * n) // S
            part = -1
            if S > 1:
                part = nppart
                nppart += 1
            pieces.append((q0, h, kv_end, i, j0, j1, part, midx))
    # longest piece first; stable, so equal lengths keep (request, tile, head, piece) order
    pieces.sort(key=lambda e: -(min(BN * e[5], e[2]) - BN * e[4]))

    def arr(rows, w):
        a = np.asarray(rows, dtype=np.int32)
        return a.reshape(len(rows), w)

    return PlanRef(arr(pieces, 8), arr([e[4] for e in dec], 8), arr(merge, 4), k, p_, d_, c, npart, arr(preq, 4),
                   arr(pmerge, 4), nppart)
