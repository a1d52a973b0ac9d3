// Host planner: turns one hybrid batch's lengths into the persistent kernel's
// work tables, the split-KV partition and the prefill:decode ticket ratio.
//
// The knobs come from the POD-Attention explainer ("How POD-Attention overlaps
// prefill and decode"): CTAs per SM, split-KV capped at two waves, CTAs
// allocated in proportion to the prefill:decode mix.  The pages give no
// formula, so the rule here is this library's own, written out in prose in
// oracle/plan_ref.py's docstring (the test oracle restates it in Python and the
// tests compare the two bit for bit).  Integer arithmetic only.
#include <algorithm>
#include <cstring>
#include <new>
#include <numeric>

#include "pod_plan.h"

namespace {

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

constexpr int kMaxHeads = 4096;   // query heads per plan
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
  if (cfg->ratio_prefill < 0 || cfg->ratio_decode < 0 || cfg->max_waves < 0 || cfg->min_chunk_pages < 0)
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

  // ---- prefill items: one 128-row query tile of one query head, per request last
  // tile first, then all requests' items longest (largest kv_end) first, stably
  struct PreEntry {
    int32_t item[kPrefillItemInts];
  };
  std::vector<PreEntry> pents;
  for (int32_t i = 0; i < NP; ++i) {
    const int32_t P = pre_qo[i], C = ctx[i];
    for (int32_t t = (int32_t)ceil_div(P, kBM) - 1; t >= 0; --t)
      for (int32_t h = 0; h < Hq; ++h) pents.push_back(PreEntry{{kBM * t, h, C + std::min(kBM * (t + 1), P), i}});
  }
  std::stable_sort(pents.begin(), pents.end(),
                   [](const PreEntry& a, const PreEntry& b) { return a.item[2] > b.item[2]; });
  for (const PreEntry& e : pents) pl->pre.insert(pl->pre.end(), e.item, e.item + kPrefillItemInts);
  pl->n_pre = (int32_t)pents.size();
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
  } else if (pl->n_pre == 0) {
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

  // ---- workspace layout and the host image of the tables
  pl->off_merge_cnt = kCountersBytes;
  pl->off_pre = align_up(pl->off_merge_cnt + 4LL * pl->n_merge, 256);
  pl->off_dec = align_up(pl->off_pre + 4LL * kPrefillItemInts * pl->n_pre, 256);
  pl->off_merge = align_up(pl->off_dec + 4LL * kDecodeItemInts * pl->n_dec, 256);
  pl->off_preq = align_up(pl->off_merge + 4LL * kMergeItemInts * pl->n_merge, 256);
  pl->off_part_o = align_up(pl->off_preq + 4LL * kPrefillReqInts * NP, 256);
  pl->off_part_lse = align_up(pl->off_part_o + 4LL * g * d * npart, 256);
  pl->ws_bytes = align_up(pl->off_part_lse + 4LL * g * npart, 256);
  pl->image.assign((size_t)(pl->off_part_o - kCountersBytes), 0);
  if (!pl->pre.empty())
    std::memcpy(pl->image.data() + (pl->off_pre - kCountersBytes), pl->pre.data(), pl->pre.size() * 4);
  if (!pl->dec.empty())
    std::memcpy(pl->image.data() + (pl->off_dec - kCountersBytes), pl->dec.data(), pl->dec.size() * 4);
  if (!pl->merge.empty())
    std::memcpy(pl->image.data() + (pl->off_merge - kCountersBytes), pl->merge.data(), pl->merge.size() * 4);
  if (!pl->preq.empty())
    std::memcpy(pl->image.data() + (pl->off_preq - kCountersBytes), pl->preq.data(), pl->preq.size() * 4);
  *out = pl;
  return POD_OK;
}
