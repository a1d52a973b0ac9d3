// Internal definitions shared by the host planner (plan.cpp) and the launcher
// (pod_attn.cu).  Not part of the public ABI.
#pragma once

#include <cstdint>
#include <vector>

#include "pod_attn.h"

namespace pod {

constexpr int kPage = 16;            // tokens per KV page
constexpr int kBM = 128;             // prefill query-tile rows (= TMEM lanes)
constexpr int kBN = 64;              // prefill key-tile columns
constexpr int kWarpsPerCta = 4;      // softmax / single-warp decode warps per CTA (plus the MMA and TMA warps)
constexpr int kMaxSms = 512;         // ticket slots (smid is folded modulo this)
constexpr int kCostRatio = 248;      // B200 tensor FLOP/s per HBM byte/s (1624.7e12 / 6539.5e9)

// Workspace layout (bytes).  Counters first, then one completion counter per
// decode merge item and per split prefill item (zero whenever a launch starts:
// pod_attn_upload zeroes them, a two-kernel or traced run zeroes them before
// its launches, and a fused launch leaves them at zero when it ends); the
// tables follow in the order prefill items | decode items | merge items |
// prefill requests | prefill merge items; then the decode split partials
// (O [n, g, d] and LSE [n, g], fp32) and the prefill piece partials
// (O [n, 128, d] and LSE [n, 128], fp32).
constexpr int64_t kCountersBytes = 4096;
constexpr int kTicketBase = 0;       // int32 [kMaxSms]
constexpr int kNextPrefill = 512;    // int32
constexpr int kNextDecode = 513;     // int32
constexpr int kErrorWord = 514;      // int32 (first error code recorded)
constexpr int kErrorInfo = 515;      // int32 (item or block that caused it)
constexpr int kRescaleCount = 516;   // int32: prefill softmax warps that rescaled O (counted with POD_FLAG_TRACE)
constexpr int kExitCount = 517;      // int32: CTAs of a fused launch that have finished
constexpr int kRunError = 518;       // int32: first error code of the fused launch in flight
constexpr int kRunErrorInfo = 519;   // int32: item or block that caused it
constexpr int kPrefillItemInts = 8;  // q0 (within the request), q_head, kv_end, prefill request,
                                     // first and end key tile (64 keys each), partial (-1 = unsplit), merge
constexpr int kPrefillMergeInts = 4; // first partial, pieces, 0, 0
constexpr int kMaxPrefillPieces = 16; // KV pieces per prefill item at most
constexpr int kPrefillReqInts = 4;   // q_start (row of q_prefill), P, C, 0
constexpr int kMaxPrefillRequests = 4096;
constexpr int kDecodeItemInts = 8;   // r, kv_head, k0, k1, partial, merge item, splits, 0
constexpr int kMergeItemInts = 4;    // r, kv_head, first_partial, num_splits

inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

}  // namespace pod

struct pod_attn_plan {
  pod_attn_config cfg;      // as given, with defaults resolved
  int32_t NP = 0, P = 0, B = 0, g = 1;   // prefill requests, their query rows in total, decodes
  int32_t n_pre = 0, n_dec = 0, n_merge = 0, n_part = 0;
  int32_t n_ppart = 0, n_pmerge = 0;       // prefill partials and split prefill items
  int32_t ctas = 2, ratio_p = 1, ratio_d = 1, chunk_pages = 16, num_sms = 148, grid = 0;
  int64_t off_merge_cnt = 0;   // int32 per decode merge item: splits finished (zeroed every run)
  int64_t off_pmerge_cnt = 0;  // int32 per split prefill item and softmax warp: pieces finished (zeroed every run)
  int64_t off_pre = 0, off_dec = 0, off_merge = 0, off_preq = 0, off_pmerge = 0;
  int64_t off_part_o = 0, off_part_lse = 0, off_ppart_o = 0, off_ppart_lse = 0, ws_bytes = 0;
  int64_t prefill_flops = 0, decode_flops = 0, kv_bytes = 0, qo_bytes = 0;
  std::vector<int32_t> decode_lens;
  std::vector<int32_t> pre, dec, merge, preq, pmerge;   // host tables
  std::vector<uint8_t> image;                // host image of workspace [kCountersBytes, off_part_o)
  void* ev_start = nullptr;
  void* ev_stop = nullptr;
};

// Implemented in plan.cpp (pure host code, no CUDA calls).
// Request rows of the block table and kv_lens: prefill requests 0..NP-1, then
// decode requests NP..NP+B-1.
int pod_plan_build(const pod_attn_config* cfg, int num_sms, int32_t NP, const int32_t* prefill_qo_lens,
                   const int32_t* prefill_kv_lens, int32_t B, const int32_t* lens, pod_attn_plan_t** out);
