// Host planner: turns one hybrid batch's lengths into the persistent kernel's
// work tables, the split-KV partition and the prefill:decode ticket ratio.
//
// The knobs come from the POD-Attention explainer ("How POD-Attention overlaps
// prefill and decode"): CTAs per SM, split-KV capped at two waves, CTAs
// allocated in proportion to the prefill:decode mix; the prefill's KV split
// leaves room for co-located decode CTAs while the prefill is short (FlashInfer
// PR "Limit kv split when prefill tokens <= 1536").  The pages give no formula,
// so the rule is this library's own; it is written out in include/pod_attn.h
// (above pod_attn_plan).  Integer arithmetic only.
#include <algorithm>
#include <cstring>
#include <new>
#include <numeric>

#include "pod_plan.h"

namespace {

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

constexpr int kMaxHeads = 4096;   // query heads per plan
constexpr int32_t kSplitLimitTokens = 1536;   // prefill tokens up to which the split counts co-located decode CTAs
constexpr int32_t kMinSplitTiles = 8;         // shortest prefill piece, in 64-key tiles
constexpr int kDecodeWarpsAll = 6;  // decode warps per CTA when every warp decodes (the kernel's 192 threads)

struct DecEntry {
  int32_t pages, r, kvh, s;
  int32_t item[pod::kDecodeItemInts];
};

}  // namespace

int pod_plan_build(const pod_attn_config* cfg, int num_sms, int32_t NP, const int32_t* pre_qo,
                   const int32_t* pre_kv, int32_t B, const int32_t* lens, pod_attn_plan_t** out) {
  using namespace pod;
  if (!cfg || !out) return POD_ERR_INVALID_ARG;
  const int32_t Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, d = cfg->head_dim;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || Hq > kMaxHeads) return POD_ERR_INVALID_ARG;
  const int32_t g = Hq / Hkv;
  if (g > 8 || (d != 64 && d != 128) || cfg->page_size != kPage) return POD_ERR_UNSUPPORTED;
  if (num_sms < 1 || num_sms > kMaxSms) return POD_ERR_INVALID_ARG;
  if (cfg->ctas_per_sm < 0 || cfg->ctas_per_sm > 2) return POD_ERR_INVALID_ARG;
  if (cfg->ratio_prefill < 0 || cfg->ratio_decode < 0 || cfg->max_waves < 0 || cfg->min_chunk_pages < 0 ||
      cfg->max_prefill_splits < 0 || cfg->max_prefill_splits > kMaxPrefillPieces)
    return POD_ERR_INVALID_ARG;
  if (NP < 0 || NP > kMaxPrefillRequests || (NP > 0 && (!pre_qo || !pre_kv))) return POD_ERR_INVALID_ARG;
  int64_t sumP = 0;
  for (int32_t i = 0; i < NP; ++i) {
    const int32_t P = pre_qo[i];
    if (P < 0 || (P > 0 && (pre_kv[i] < P || pre_kv[i] > (1 << 24)))) return POD_ERR_INVALID_ARG;
    sumP += P;
  }
  if (sumP > (1 << 24)) return POD_ERR_INVALID_ARG;
  if (B < 0 || B > 65536 || (B > 0 && !lens)) return POD_ERR_INVALID_ARG;
  int64_t sumL = 0;
  for (int32_t r = 0; r < B; ++r) {
    if (lens[r] < 1 || lens[r] > (1 << 24)) return POD_ERR_INVALID_ARG;
    sumL += lens[r];
  }
  if (sumL > INT32_MAX) return POD_ERR_INVALID_ARG;

  // ---- algorithmic work (roofline numerators); checked before anything is built
  int64_t rows_keys = 0, pre_kv_tokens = 0;
  for (int32_t i = 0; i < NP; ++i) {
    const int64_t P = pre_qo[i], C = P > 0 ? pre_kv[i] - P : 0;
    for (int64_t q0 = 0; q0 < P; q0 += kBM) {
      const int64_t n = std::min<int64_t>(kBM, P - q0);
      rows_keys += n * (C + 1) + n * q0 + n * (n - 1) / 2;
    }
    if (P > 0) pre_kv_tokens += C + P;
  }
  {
    // the work counts must fit the int64 fields they are reported in
    const __int128 lim = (__int128)INT64_MAX;
    const __int128 pf = (__int128)4 * d * Hq * rows_keys, df = (__int128)4 * d * Hq * sumL;
    const __int128 kb = (__int128)4 * d * Hkv * (pre_kv_tokens + sumL), qb = (__int128)4 * d * Hq * (sumP + B);
    if (pf > lim || df > lim || kb > lim || qb > lim) return POD_ERR_INVALID_ARG;
  }

  pod_attn_plan_t* pl = new (std::nothrow) pod_attn_plan_t();
  if (!pl) return POD_ERR_INVALID_ARG;
  pl->cfg = *cfg;
  const int32_t k = cfg->ctas_per_sm == 0 ? 2 : cfg->ctas_per_sm;
  const int32_t waves = cfg->max_waves == 0 ? 2 : cfg->max_waves;
  const int32_t minc = cfg->min_chunk_pages == 0 ? 16 : cfg->min_chunk_pages;
  std::vector<int32_t> ctx(NP);
  for (int32_t i = 0; i < NP; ++i) ctx[i] = pre_qo[i] > 0 ? pre_kv[i] - pre_qo[i] : 0;
  pl->NP = NP;
  pl->P = (int32_t)sumP;
  pl->B = B;
  pl->g = g;
  pl->ctas = k;
  pl->num_sms = num_sms;
  pl->grid = num_sms * k;
  pl->decode_lens.assign(lens, lens + B);

  // ---- base prefill items: one 128-row query tile of one query head, per request last
  // tile first (they are cut into KV pieces and ordered once the ratio is known)
  struct BaseItem {
    int32_t q0, h, kv_end, req;
  };
  std::vector<BaseItem> base;
  for (int32_t i = 0; i < NP; ++i) {
    const int32_t P = pre_qo[i], C = ctx[i];
    for (int32_t t = (int32_t)ceil_div(P, kBM) - 1; t >= 0; --t)
      for (int32_t h = 0; h < Hq; ++h) base.push_back(BaseItem{kBM * t, h, C + std::min(kBM * (t + 1), P), i});
  }
  int32_t q_start = 0;
  for (int32_t i = 0; i < NP; ++i) {
    const int32_t rq[kPrefillReqInts] = {q_start, pre_qo[i], ctx[i], 0};
    pl->preq.insert(pl->preq.end(), rq, rq + kPrefillReqInts);
    q_start += pre_qo[i];
  }

  // ---- decode split: chunk c pages, at most waves x decode warps items
  // decode warps: every warp of the CTA, or warps 0-3 with POD_FLAG_DECODE_FOUR_WARPS
  const int32_t dwarps = (cfg->flags & POD_FLAG_DECODE_FOUR_WARPS) ? kWarpsPerCta : kDecodeWarpsAll;
  const int64_t W = (int64_t)num_sms * k * dwarps;
  const int64_t cap = (int64_t)waves * W;
  std::vector<int32_t> pages(B);
  int64_t N = 0;
  int32_t maxp = 0;
  for (int32_t r = 0; r < B; ++r) {
    pages[r] = (int32_t)ceil_div(lens[r], kPage);
    N += pages[r];
    maxp = std::max(maxp, pages[r]);
  }
  N *= Hkv;
  int64_t c = std::max<int64_t>(minc, ceil_div(N, cap));
  while (c < maxp) {
    int64_t items = 0;
    for (int32_t r = 0; r < B; ++r) items += ceil_div(pages[r], c);
    if ((int64_t)Hkv * items <= cap) break;
    ++c;
  }
  pl->chunk_pages = (int32_t)c;

  std::vector<DecEntry> ents;
  int32_t npart = 0;
  for (int32_t r = 0; r < B; ++r) {
    const int32_t S = (int32_t)ceil_div(pages[r], c);
    for (int32_t kvh = 0; kvh < Hkv; ++kvh) {
      const int32_t first = npart;
      const int32_t midx = S > 1 ? (int32_t)(pl->merge.size() / kMergeItemInts) : -1;
      for (int32_t s = 0; s < S; ++s) {
        const int32_t p0 = (int32_t)(((int64_t)s * pages[r]) / S);
        const int32_t p1 = (int32_t)(((int64_t)(s + 1) * pages[r]) / S);
        int32_t part = -1;
        if (S > 1) part = npart++;
        DecEntry e{p1 - p0, r, kvh, s, {r, kvh, kPage * p0, std::min(kPage * p1, lens[r]), part, midx, S, 0}};
        ents.push_back(e);
      }
      if (S > 1) {
        int32_t m[kMergeItemInts] = {r, kvh, first, S};
        pl->merge.insert(pl->merge.end(), m, m + kMergeItemInts);
      }
    }
  }
  std::stable_sort(ents.begin(), ents.end(), [](const DecEntry& a, const DecEntry& b) {
    if (a.pages != b.pages) return a.pages > b.pages;
    if (a.r != b.r) return a.r < b.r;
    if (a.kvh != b.kvh) return a.kvh < b.kvh;
    return a.s < b.s;
  });
  for (const DecEntry& e : ents) pl->dec.insert(pl->dec.end(), e.item, e.item + kDecodeItemInts);
  pl->n_dec = (int32_t)ents.size();
  pl->n_merge = (int32_t)(pl->merge.size() / kMergeItemInts);
  pl->n_part = npart;

  pl->prefill_flops = 4LL * d * Hq * rows_keys;
  pl->decode_flops = 4LL * d * Hq * sumL;
  pl->kv_bytes = 4LL * d * Hkv * (pre_kv_tokens + sumL);
  pl->qo_bytes = 4LL * d * Hq * (sumP + B);

  // ---- ticket ratio p:d
  int32_t rp, rd;
  if (cfg->ratio_prefill || cfg->ratio_decode) {
    if (cfg->ratio_prefill == 0) {
      rp = 0; rd = 1;
    } else if (cfg->ratio_decode == 0) {
      rp = 1; rd = 0;
    } else {
      const int32_t gg = std::gcd(cfg->ratio_prefill, cfg->ratio_decode);
      rp = cfg->ratio_prefill / gg;
      rd = cfg->ratio_decode / gg;
    }
  } else if (base.empty()) {
    rp = 0; rd = 1;
  } else if (pl->n_dec == 0) {
    rp = 1; rd = 0;
  } else {
    const __int128 cost_pre = (__int128)pl->prefill_flops;
    const __int128 cost_dec = (__int128)kCostRatio * 4 * d * Hkv * sumL;
    const __int128 tot = cost_pre + cost_dec;
    int64_t n_p = (int64_t)((2 * (__int128)k * cost_pre + tot) / (2 * tot));
    if (k >= 2) n_p = std::min<int64_t>(std::max<int64_t>(n_p, 1), k - 1);
    else n_p = 1;
    if (2 * cost_pre >= tot) n_p = k;   // prefill dominates: every CTA prefill-first, decode fills in
    rp = (int32_t)n_p;
    rd = k - rp;
    if (rd == 0) {
      rp = 1;
    } else {
      const int32_t gg = std::gcd(rp, rd);
      rp /= gg;
      rd /= gg;
    }
  }
  pl->ratio_p = rp;
  pl->ratio_d = rd;

  // ---- prefill KV split: fill the prefill CTA slots when the base items leave some empty;
  // a short prefill (<= 1536 tokens) next to decode work counts one slot per SM (the SM's
  // other CTA stays for decode)
  {
    const bool limited = B > 0 && sumP <= kSplitLimitTokens && !(cfg->flags & POD_FLAG_PREFILL_SPLIT_UNLIMITED);
    const int64_t slots = limited ? (int64_t)num_sms : (int64_t)num_sms * k;
    const int64_t n0 = (int64_t)base.size();
    std::vector<int32_t> nsplit(base.size(), 1);
    if (cfg->max_prefill_splits != 1 && n0 > 0 && n0 < slots) {
      int64_t tiles = 0;
      for (const BaseItem& b : base) tiles += ceil_div(b.kv_end, kBN);
      const int64_t tau = std::max<int64_t>(kMinSplitTiles, ceil_div(tiles, slots));
      const int32_t smax = cfg->max_prefill_splits >= 2 ? cfg->max_prefill_splits : kMaxPrefillPieces;
      for (size_t i = 0; i < base.size(); ++i)
        nsplit[i] = (int32_t)std::min<int64_t>(smax, std::max<int64_t>(1, ceil_div(base[i].kv_end, kBN) / tau));
    }
    struct PreEntry {
      int32_t keys;
      int32_t item[kPrefillItemInts];
    };
    std::vector<PreEntry> pents;
    int32_t nppart = 0;
    for (size_t i = 0; i < base.size(); ++i) {
      const BaseItem& b = base[i];
      const int32_t n = (int32_t)ceil_div(b.kv_end, kBN), S = nsplit[i];
      const int32_t midx = S > 1 ? (int32_t)(pl->pmerge.size() / kPrefillMergeInts) : -1;
      if (S > 1) {
        const int32_t m[kPrefillMergeInts] = {nppart, S, 0, 0};
        pl->pmerge.insert(pl->pmerge.end(), m, m + kPrefillMergeInts);
      }
      for (int32_t sp = 0; sp < S; ++sp) {
        const int32_t j0 = (int32_t)(((int64_t)sp * n) / S), j1 = (int32_t)(((int64_t)(sp + 1) * n) / S);
        const int32_t part = S > 1 ? nppart++ : -1;
        pents.push_back(PreEntry{std::min(kBN * j1, b.kv_end) - kBN * j0,
                                 {b.q0, b.h, b.kv_end, b.req, j0, j1, part, midx}});
      }
    }
    // longest piece first; stable, so equal lengths keep (request, tile, head, piece) order
    std::stable_sort(pents.begin(), pents.end(), [](const PreEntry& a, const PreEntry& b) { return a.keys > b.keys; });
    for (const PreEntry& e : pents) pl->pre.insert(pl->pre.end(), e.item, e.item + kPrefillItemInts);
    pl->n_pre = (int32_t)pents.size();
    pl->n_ppart = nppart;
    pl->n_pmerge = (int32_t)(pl->pmerge.size() / kPrefillMergeInts);
  }

  // ---- workspace layout and the host image of the tables
  pl->off_merge_cnt = kCountersBytes;
  pl->off_pmerge_cnt = pl->off_merge_cnt + 4LL * pl->n_merge;
  pl->off_pre = align_up(pl->off_pmerge_cnt + 4LL * kWarpsPerCta * pl->n_pmerge, 256);
  pl->off_dec = align_up(pl->off_pre + 4LL * kPrefillItemInts * pl->n_pre, 256);
  pl->off_merge = align_up(pl->off_dec + 4LL * kDecodeItemInts * pl->n_dec, 256);
  pl->off_preq = align_up(pl->off_merge + 4LL * kMergeItemInts * pl->n_merge, 256);
  pl->off_pmerge = align_up(pl->off_preq + 4LL * kPrefillReqInts * NP, 256);
  pl->off_part_o = align_up(pl->off_pmerge + 4LL * kPrefillMergeInts * pl->n_pmerge, 256);
  pl->off_part_lse = align_up(pl->off_part_o + 4LL * g * d * npart, 256);
  pl->off_ppart_o = align_up(pl->off_part_lse + 4LL * g * npart, 256);
  pl->off_ppart_lse = align_up(pl->off_ppart_o + 4LL * kBM * d * pl->n_ppart, 256);
  pl->ws_bytes = align_up(pl->off_ppart_lse + 4LL * kBM * pl->n_ppart, 256);
  pl->image.assign((size_t)(pl->off_part_o - kCountersBytes), 0);
  auto put = [&](int64_t off, const std::vector<int32_t>& v) {
    if (!v.empty()) std::memcpy(pl->image.data() + (off - kCountersBytes), v.data(), v.size() * 4);
  };
  put(pl->off_pre, pl->pre);
  put(pl->off_dec, pl->dec);
  put(pl->off_merge, pl->merge);
  put(pl->off_preq, pl->preq);
  put(pl->off_pmerge, pl->pmerge);
  *out = pl;
  return POD_OK;
}
