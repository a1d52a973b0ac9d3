// Fused hybrid-batch attention for B200 (sm_100a): one persistent kernel runs
// causal chunked-prefill tiles on the tcgen05 tensor cores and paged-KV decode
// attention on the load/store path, side by side on every SM.
//
// Method: "POD-Attention: Unlocking Full Prefill-Decode Overlap for Faster LLM
// Inference" (explainer page, "How POD-Attention overlaps prefill and decode"):
//   * one kernel holds both kinds of work ("Fuse prefill and decode attention
//     into one kernel");
//   * a CTA's leader reads %smid and takes a ticket from an SM-local counter;
//     the ticket picks the CTA's role at the plan's p:d ratio ("Self-assign
//     roles per SM in software");
//   * decode runs in single-warp virtual blocks ("Balance shared memory and
//     threadblock count") with small tensor-core tiles ("Shrink decode tiles");
//   * KV is split for decode parallelism, and for the prefill when its items
//     leave CTA slots empty, capped by the plan ("Cap prefill splitting"; the
//     FlashInfer PR "Limit kv split when prefill tokens <= 1536" keeps room
//     for co-located decode CTAs); splits are merged by log-sum-exp (PAT
//     record) by whoever finishes a row's last split.
// B200 re-design (prior art, not the blueprint): CTAs are persistent -- the
// ticket fixes a CTA's home role, the CTA drains that role's queue and then
// steals from the other, so no CTA ever waits on another.  Prefill tiles are
// 128 x 64 tcgen05 MMAs: S = Q K^T with Q held in TMEM, O += P V with P staged
// in shared memory, both accumulated in TMEM; K and V arrive by TMA with
// 128-byte swizzle straight from the 16-token pages.  Decode warps stage pages
// with TMA into a per-warp ring and use m16n8k16 MMAs with keys as rows, on
// bf16 pages or on e4m3 pages converted to f16 in registers (the FP8 cache of
// the blog post "Prefill vs. Decode GPU Utilization Imbalance").
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "pod_plan.h"
#include "pod_ptx.cuh"

namespace pod {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: a healthy wait takes microseconds
constexpr uint32_t kTmemCols = 256;   // S (64 fp32 columns) at 0, Q (d/2 columns of bf16 pairs) at 64, O (d) at 128
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemQ = 64;
constexpr uint32_t kTmemO = 128;

enum Mode : int32_t { kFused = 0, kPrefillOnly = 1, kDecodeOnly = 2 };
enum Role : int32_t { kRolePrefill = 0, kRoleDecode = 1 };

struct alignas(64) PodParams {
  CUtensorMap tm_k;    // K cache viewed as 2D [num_blocks*Hkv*16 rows, d], box {64, 16}, 128B swizzle
  CUtensorMap tm_kp;   // K cache as 3D [d/64 halves][rows][64]: one box {64, 16, d/64} = one whole page
  CUtensorMap tm_vp;   // V cache, same view
  CUtensorMap tm_k8;   // e4m3 K cache of the decode requests, 2D [rows, d] bytes, box {d, 16} (unused for bf16)
  CUtensorMap tm_v8;   // e4m3 V cache, same view
  const __nv_bfloat16* q_pre;
  const __nv_bfloat16* q_dec;
  __nv_bfloat16* o_pre;
  __nv_bfloat16* o_dec;
  const int32_t* block_table;
  const int32_t* kv_lens;
  int32_t* counters;
  const int4* pre_items;   // two int4 per item: q0, q head, kv_end, request | j0, j1, partial, merge
  const int4* dec_items;   // two int4 per item
  const int4* merge_items; // r, kvh, first_partial, num_splits
  const int4* pre_reqs;    // per prefill request: first row in q_pre / o_pre, P, C, 0
  const int4* pmerge_items; // per split prefill item: first partial, pieces, 0, 0
  int32_t* merge_cnt;      // splits finished per decode merge item (zero at launch)
  int32_t* pmerge_cnt;     // pieces finished per split prefill item and softmax warp (zero at launch)
  float* part_o;
  float* part_lse;
  float* ppart_o;          // prefill piece partials: O [n, 128, d] (normalised) and LSE [n, 128], log2 domain
  float* ppart_lse;
  int32_t* trace;
  int32_t bt_stride;
  int32_t kv_rows;         // num_blocks * Hkv * 16 (rows of the K/V tensor maps)
  int32_t num_blocks;
  int32_t kv_rows8;        // the same for the e4m3 cache of the decode requests
  int32_t num_blocks8;
  int32_t n_pre, n_dec;
  int32_t Hq, Hkv, g, NP, B;   // NP prefill requests own block-table rows 0..NP-1
  int32_t ratio_p, ratio_d;
  int32_t mode;
  int32_t use_tmem;
  int32_t merge_in_kernel; // 1: the warp finishing a row's last split merges the row
  int32_t selftest_timeout; // 1: CTA 0 exercises the expired-wait path once
  int32_t partition_sms;   // > 0: roles by SM id instead of per-SM tickets (ablation)
  int32_t decode_warps;    // warps of a CTA that run decode items: 4, or 6 (the MMA and TMA warps too)
  int32_t self_reset;      // 1 (a fused launch): errors go to the launch's own slot and the last CTA
                           // out publishes them and returns every counter to zero
  int32_t n_ppart;         // prefill piece partials of the plan (0: no prefill item is split)
  int32_t n_merge_cnt;     // ints of merge_cnt / pmerge_cnt (cleared by the last CTA after an error)
  int32_t n_pmerge_cnt;
  float scale_log2;        // softmax scale * log2(e)
  const float* k_scale8;   // e4m3 caches: per kv head, dequantised value = scale * stored value
  const float* v_scale8;
};

constexpr int kThreads = 192;        // warps 0-3: softmax (prefill) / decode units; warp 4: MMA; warp 5: TMA
                                     // (in decode, warps 4 and 5 decode too, or idle with decode_warps == 4)
constexpr int kMmaWarp = 4;
constexpr int kTmaWarp = 5;
constexpr int kAllWarps = kThreads / 32;

// mbarrier slots in the CTA control block
enum : int {
  kBarQ = 0,        // Q rows of the item stored into TMEM                      count 4 (softmax warps)
  kBarKFull = 1,    // [3] K tile landed (TMA)                                  count 1 + tx
  kBarSFull = 4,    // [3] S_t ready in TMEM, [t % 3] (commit); K slot t % 3   count 1
                    //     is free again (one commit serves both: ~200 cycles each)
  kBarVFull = 7,    // [2] V tile landed (TMA)                                  count 1 + tx
  // 9: unused
  kBarSFree = 10,   // softmax has read S out of TMEM                           count 4 (softmax warps)
  kBarPFull = 11,   // [2] P tile t stored in shared-memory buffer t&1          count 4 (softmax warps)
  kBarODone = 13,   // [2] P.V MMA of tile t finished: P buffer and V slot t&1  count 1
                    //     are free again (commit)
  kBarOFinal = 15,  // last P.V MMA of an item finished (commit)                count 1
  kBarDecode = 16,  // [decode warps * ring depth] decode page rings            count 1 + tx
};
// Parity waits are only sound when the waiter for completion k of a barrier
// knows that completion k + 1 cannot have happened yet.  For key tile t
// (counted over the CTA's lifetime): s_full[t % 3] completes once per three
// tiles; the softmax waits on it for S_t, and S_{t+3} needs the softmax to have
// read S_{t+2} (s_free); the TMA warp waits on it before K_{t+3} goes into slot
// t % 3, and S_{t+3} needs that K tile; P_t goes into buffer t&1 only after P.V_{t-2} finished and
// P.V_t needs P_t, so p_full is at most one phase ahead per buffer; o_done[t&1]
// is waited on by the TMA warp (before V_{t+2} goes into slot t&1) and by the
// softmax (tiles t+1 and t+2, before it rescales O or reuses the P buffer),
// and P.V_{t+2} needs both; q and o_final complete once per item.

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;                      // 128-byte swizzle atoms along d
  static constexpr int kKTile = kBN * D * 2;                  // 64 keys of K (or V)
  static constexpr int kKSlots = 3;                           // K ring: two tiles of lead
  static constexpr int kVSlots = 2;                           // V ring: two tiles of lead
  static constexpr int kPBytes = kBM * kBN * 2;               // P tile, bf16, K-major 128B-swizzled
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKSlots * kKTile;
  static constexpr int kOffP = kOffV + kVSlots * kKTile;      // [2] P buffers
  static constexpr int kPrefillSmem = kOffP + 2 * kPBytes;
  static constexpr int kPageBytes = kPage * D * 2;            // one 16-token page of one kv head
  static constexpr int kDecStage = 2 * kPageBytes;            // K page + V page
  static constexpr int kNS = (kPrefillSmem / kWarpsPerCta) / kDecStage;   // decode ring depth per warp
  static constexpr int kNSAll = (kPrefillSmem / kAllWarps) / kDecStage;    // ... when all warps decode
  static constexpr int kPageBytes8 = kPage * D;               // the same page in e4m3
  static constexpr int kDecStage8 = 2 * kPageBytes8;
  static constexpr int kNS8 = (kPrefillSmem / kWarpsPerCta) / kDecStage8;
  static constexpr int kNSAll8 = (kPrefillSmem / kAllWarps) / kDecStage8;
  static constexpr int kSmem = kPrefillSmem;
  static constexpr int cmax(int a, int b) { return a > b ? a : b; }
  static constexpr int kNumBars = kBarDecode + cmax(cmax(kWarpsPerCta * kNS, kAllWarps * kNSAll),
                                                    cmax(kWarpsPerCta * kNS8, kAllWarps * kNSAll8));
  static constexpr int kCtrlBytes = 512;                      // barriers, TMEM address, broadcast slots
  static_assert((kNumBars + 1) * 8 + 32 <= kCtrlBytes, "control block too small");   // + the self-test barrier
  // at least 80 KB so that no more than two CTAs (2 x 256 TMEM columns) can share an SM
  static constexpr int kSmemAlloc = (kSmem + kCtrlBytes) > 80 * 1024 ? (kSmem + kCtrlBytes) : 80 * 1024;
};
static_assert(Cfg<128>::kNS >= 3 && Cfg<64>::kNS >= 3, "decode ring too shallow");
static_assert(Cfg<128>::kNSAll >= 2 && Cfg<64>::kNSAll >= 2, "decode ring too shallow");
static_assert(kAllWarps * Cfg<128>::kNSAll * Cfg<128>::kDecStage <= Cfg<128>::kPrefillSmem &&
                  kAllWarps * Cfg<64>::kNSAll * Cfg<64>::kDecStage <= Cfg<64>::kPrefillSmem,
              "decode rings exceed the shared-memory union");
static_assert(kAllWarps * Cfg<128>::kNSAll8 * Cfg<128>::kDecStage8 <= Cfg<128>::kPrefillSmem &&
                  kWarpsPerCta * Cfg<64>::kNS8 * Cfg<64>::kDecStage8 <= Cfg<64>::kPrefillSmem &&
                  Cfg<128>::kDecStage8 % 1024 == 0,
              "e4m3 decode rings exceed the shared-memory union or break the swizzle alignment");

static_assert(kErrorInfo == kErrorWord + 1 && kRunErrorInfo == kRunError + 1, "error code and info are adjacent");

// The first error of a launch wins.  A fused launch records into its own slot, which its last CTA
// copies into the error word (so the word always tells about the last completed launch).
__device__ __forceinline__ void record_error(const PodParams& p, int code, int info) {
  const int w = p.self_reset ? kRunError : kErrorWord;
  if (atomicCAS(&p.counters[w], 0, code) == 0) atomicExch(&p.counters[w + 1], info);
}

// Row of the K/V tensor maps holding page `blk`, kv head `kvh`; an
// out-of-range block id is recorded and mapped past the end (TMA reads zeros).
__device__ __forceinline__ int kv_row(const PodParams& p, int blk, int kvh) {
  if (blk < 0 || blk >= p.num_blocks) {
    record_error(p, POD_ERR_BOUNDS, blk);
    return p.kv_rows;
  }
  return (blk * p.Hkv + kvh) * kPage;
}
// ... of the e4m3 cache (decode requests of pod_attn_run_fp8kv)
__device__ __forceinline__ int kv_row8(const PodParams& p, int blk, int kvh) {
  if (blk < 0 || blk >= p.num_blocks8) {
    record_error(p, POD_ERR_BOUNDS, blk);
    return p.kv_rows8;
  }
  return (blk * p.Hkv + kvh) * kPage;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int D>
struct PrefillSmem {
  uint8_t* base;
  __device__ uint8_t* k(uint32_t t) const { return base + Cfg<D>::kOffK + (t % Cfg<D>::kKSlots) * Cfg<D>::kKTile; }
  __device__ uint8_t* v(uint32_t t) const { return base + Cfg<D>::kOffV + (t % Cfg<D>::kVSlots) * Cfg<D>::kKTile; }
  __device__ uint8_t* pbuf(uint32_t t) const { return base + Cfg<D>::kOffP + (t & 1u) * Cfg<D>::kPBytes; }
};

// One prefill work item: query rows q0 .. q0+127 of `req` for query head qh,
// key tiles j0 .. j1-1 (64 keys each, absolute within the request) of a causal
// range that ends at kv_end.  part < 0: the item covers every key tile and
// writes bf16 O; otherwise it is one KV piece of a split item and writes a
// partial, and the last piece to finish merges them (prefill merge item midx).
struct PreItem {
  int q0, qh, kv_end, req, j0, j1, part, midx;
};

__device__ __forceinline__ PreItem load_pre_item(const PodParams& p, int i) {
  const int4 a = __ldg(&p.pre_items[2 * i]), b = __ldg(&p.pre_items[2 * i + 1]);
  return PreItem{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
}

// Block ids of the prefill request's pages, read 32 at a time (one per lane) a
// window ahead of use: `cur` holds pages [32 w, 32 w + 32) (key tiles 8w ..
// 8w + 7), `nxt` the next 32.
struct PageWindows {
  int cur, nxt, w;
};

__device__ __forceinline__ int load_page_window(const PodParams& p, const int* bt_row, int w, int kv_end, int lane) {
  const int gp = 32 * w + lane;
  return gp * kPage < kv_end ? __ldg(&bt_row[gp]) : 0;
}

// Tensor-map row of page `lane & 3` of key tile kb (kb in window w or w + 1);
// pages past kv_end map past the tensor's end, where TMA reads zeros.
__device__ __forceinline__ int tile_page_row(const PodParams& p, const PageWindows& pw, int kb, int kvh, int kv_end,
                                             int lane) {
  const int src = (kb >> 3) == pw.w ? pw.cur : pw.nxt;
  const int blk = __shfl_sync(0xffffffffu, src, ((kb & 7) << 2) + (lane & 3));
  const int gp = kb * (kBN / kPage) + (lane & 3);
  return gp * kPage < kv_end ? kv_row(p, blk, kvh) : p.kv_rows;
}

template <int D>
__device__ __forceinline__ void issue_tile(const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int row_lane,
                                           int lane) {
  using CF = Cfg<D>;
  // lanes 0-3 each issue the boxes of one page (row_lane of lane l is page l & 3)
  if (lane == 0) mbar_arrive_expect_tx(bar, CF::kKTile);
  __syncwarp();
  if (lane < kBN / kPage) {
#pragma unroll
    for (int h = 0; h < CF::kHalves; ++h)
      tma_load_2d(dst + h * (kBN * 128) + lane * (kPage * 128), map, bar, h * 64, row_lane);
  }
}

// V tile of 4 pages as one page box each ([page][d/64 halves][16 rows][128 B]);
// a P.V MMA step of 16 keys reads exactly one page, so the page-major layout
// only changes the B descriptor's strides.
template <int D>
__device__ __forceinline__ void issue_vtile(const PodParams& p, uint8_t* dst, uint64_t* bar, int row_lane, int lane) {
  using CF = Cfg<D>;
  if (lane == 0) mbar_arrive_expect_tx(bar, CF::kKTile);
  __syncwarp();
  if (lane < kBN / kPage) tma_load_3d(dst + lane * CF::kPageBytes, &p.tm_vp, bar, 0, row_lane, 0);
}

// TMA warp of one prefill item: K into a 3-deep ring and V into a 2-deep
// ring; K_{t+3} goes into slot t%3 once S_t finished, V_{t+2} into slot t&1
// once P.V_t finished.  `t0` = key tiles this CTA processed before this item
// (it indexes every ring and mbarrier phase); the item's tiles are j0 .. j1-1.
template <int D>
__device__ bool prefill_tma(const PodParams& p, const PreItem& it, uint8_t* smem, uint64_t* bars, uint32_t t0) {
  using CF = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const int kv_end = it.kv_end, j0 = it.j0;
  const int kvh = it.qh / p.g;
  const int nkb = it.j1 - it.j0;
  const PrefillSmem<D> sm{smem};
  const int* bt_row = p.block_table + (size_t)it.req * p.bt_stride;
  if (lane == 0 && p.kv_lens && __ldg(&p.kv_lens[it.req]) < kv_end) record_error(p, POD_ERR_PLAN_MISMATCH, it.req);
  const int w0 = j0 >> 3;   // 32-page windows hold 8 key tiles
  PageWindows pw{load_page_window(p, bt_row, w0, kv_end, lane), load_page_window(p, bt_row, w0 + 1, kv_end, lane),
                 w0};
  for (int j = 0; j < nkb && j < CF::kKSlots; ++j) {
    const uint32_t t = t0 + j;
    const int r = tile_page_row(p, pw, j0 + j, kvh, kv_end, lane);
    issue_tile<D>(&p.tm_k, sm.k(t), &bars[kBarKFull + t % 3], r, lane);
    if (j < CF::kVSlots) issue_vtile<D>(p, sm.v(t), &bars[kBarVFull + (t & 1u)], r, lane);
  }
  for (int j = 0; j + CF::kVSlots < nkb; ++j) {
    const uint32_t t = t0 + j;
    if (((j0 + j + CF::kVSlots) >> 3) > pw.w) {   // tile j+2 enters the next window; fetch the one after it
      ++pw.w;
      pw.cur = pw.nxt;
      pw.nxt = load_page_window(p, bt_row, pw.w + 1, kv_end, lane);
    }
    const bool more_k = j + CF::kKSlots < nkb;
    const int rk = more_k ? tile_page_row(p, pw, j0 + j + CF::kKSlots, kvh, kv_end, lane) : 0;
    const int rv = tile_page_row(p, pw, j0 + j + CF::kVSlots, kvh, kv_end, lane);
    if (more_k) {                // K first: S_{t+3} is issued well before P.V_{t+2}
      if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull + t % 3], (t / 3) & 1u, kWaitLimitNs))) return false;
      issue_tile<D>(&p.tm_k, sm.k(t + CF::kKSlots), &bars[kBarKFull + t % 3], rk, lane);
    }
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarODone + (t & 1u)], (t >> 1) & 1u, kWaitLimitNs))) return false;
    issue_vtile<D>(p, sm.v(t + CF::kVSlots), &bars[kBarVFull + (t & 1u)], rv, lane);
  }
  return true;
}

// MMA warp of one prefill item (lane 0 issues): S_t = Q K_t^T into TMEM with Q
// read from TMEM (stored there by the softmax warps), issued as soon as the
// softmax has read S_{t-1} out; O += P_t V_t with P_t read from shared memory.
// One commit after S_t (s_full: S ready, K slot free) and one after P.V_t
// (o_done: V slot and P buffer free); a commit holds the issuing thread ~200
// cycles, so each serves every consumer it can.
template <int D>
__device__ bool prefill_mma(const PodParams& p, const PreItem& it, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                            uint32_t t0, uint32_t nq) {
  using CF = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const int kv_end = it.kv_end;
  const int nkb = it.j1 - it.j0;
  const PrefillSmem<D> sm{smem};
  constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false, false);
  constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, false, true);
  // descriptors of the slot bases; a byte offset b within a slot adds b >> 4
  const uint64_t dk0 = sdesc_sw128(smem_u32(smem + CF::kOffK), 16, 1024);
  // V: MN-major, halves of d 16*128 bytes apart inside a page, 8-key groups 1024 apart
  const uint64_t dv0 = sdesc_sw128(smem_u32(smem + CF::kOffV), kPage * 128, 1024);
  const uint64_t dp0 = sdesc_sw128(smem_u32(smem + CF::kOffP), 16, 1024);

  auto issue_s = [&](uint32_t t) {
    const uint64_t dk = dk0 + (uint64_t)(((t % CF::kKSlots) * CF::kKTile) >> 4);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t boff = ((kk >> 2) * (kBN * 128) + (kk & 3) * 32) >> 4;
      umma_bf16_tmem_a(tmem + kTmemS, tmem + kTmemQ + kk * 8, dk + boff, idesc_s, kk > 0 ? 1u : 0u);
    }
    umma_commit(&bars[kBarSFull + t % 3]);
  };

  {                              // S of the first tile, once Q is in TMEM
    const bool ok = mbar_wait(&bars[kBarQ], nq & 1u, kWaitLimitNs) &&
                    mbar_wait(&bars[kBarKFull + t0 % 3], (t0 / 3) & 1u, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) return false;
    if (lane == 0) {
      tc_fence_after();
      issue_s(t0);
    }
    __syncwarp();
  }
  for (int j = 0; j < nkb; ++j) {
    const uint32_t t = t0 + j;
    if (j + 1 < nkb) {           // S_{t+1} once the softmax has read S_t out of TMEM
      const uint32_t tn = t + 1;
      const bool ws = mbar_wait(&bars[kBarSFree], t & 1u, kWaitLimitNs) &&
                      mbar_wait(&bars[kBarKFull + tn % 3], (tn / 3) & 1u, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ws)) return false;
      if (lane == 0) {
        tc_fence_after();
        issue_s(tn);
      }
      __syncwarp();
    }
    const bool wp = mbar_wait(&bars[kBarVFull + (t & 1u)], (t >> 1) & 1u, kWaitLimitNs) &&
                    mbar_wait(&bars[kBarPFull + (t & 1u)], (t >> 1) & 1u, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, wp)) return false;
    const int valid = kv_end - (it.j0 + j) * kBN;
    if (valid < kBN) {           // V rows past the request's end may hold anything: zero them
      uint8_t* vt = sm.v(t);
      for (int i = lane; i < (kBN - valid) * CF::kHalves * 8; i += 32) {
        const int chunk = i & 7, rh = i >> 3;
        const int key = valid + rh % (kBN - valid), h = rh / (kBN - valid);
        *reinterpret_cast<uint4*>(vt + (key / kPage) * CF::kPageBytes + h * (kPage * 128) + (key % kPage) * 128 +
                                  chunk * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      __syncwarp();
    }
    if (lane == 0) {
      tc_fence_after();
      const uint64_t dv = dv0 + (uint64_t)(((t & 1u) * CF::kKTile) >> 4);
      const uint64_t dp = dp0 + (uint64_t)(((t & 1u) * CF::kPBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        umma_bf16(tmem + kTmemO, dp + (uint64_t)((kk * 32) >> 4), dv + (uint64_t)((kk * CF::kPageBytes) >> 4), idesc_o,
                  (j > 0 || kk > 0) ? 1u : 0u);
      umma_commit(&bars[kBarODone + (t & 1u)]);
      if (j == nkb - 1) umma_commit(&bars[kBarOFinal]);
    }
    __syncwarp();
  }
  return true;
}

// Softmax warps of one prefill item (threads 0..127, thread = tile row = TMEM
// lane).  First the thread's Q row goes into TMEM (the A operand of S = Q K^T).
// Per key tile: read S_t from TMEM (and hand the buffer back to the MMA warp
// at once), mask (bottom-right causal), online softmax in the exp2 domain with
// a lazily updated row max (O in TMEM is rescaled only when the max grows by
// more than 2^8), write P_t as bf16 into shared-memory buffer t&1 in the
// K-major 128B-swizzled layout.  Epilogue: O / l -> bf16 -> global, or, for
// one KV piece of a split item, the piece's partial rows (O / l in fp32) into
// shared memory and their log-sum-exps into the workspace; the CTA finishes
// the piece after the item's barrier (prefill_piece_end).
template <int D>
__device__ bool prefill_softmax(const PodParams& p, const PreItem& it, int item, uint8_t* smem, uint64_t* bars,
                                uint32_t tmem, uint32_t t0, uint32_t nq) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = it.q0, qh = it.qh, kv_end = it.kv_end, j0 = it.j0;
  const int4 rq = __ldg(&p.pre_reqs[it.req]);     // first row in q_pre / o_pre, P, C
  const int q_first = rq.x, P = rq.y, C = rq.z;
  const int nkb = it.j1 - it.j0;
  const int row = tid;
  const int row_limit = min(C + q0 + row + 1, kv_end);
  const int full_tiles = (C + q0 + 1) / kBN;     // tiles visible to every row of this item
  const uint32_t t_lane = (uint32_t)(warp * 32) << 16;
  const float sl2 = p.scale_log2;
  {
    // Q row (bf16 pairs along d) into TMEM lane `row`; rows past the chunk are zero
    const int q = q0 + row;
    const uint4* src = reinterpret_cast<const uint4*>(p.q_pre + ((size_t)(q_first + q) * p.Hq + qh) * D);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = q < P ? __ldg(src + c * 8 + i) : make_uint4(0u, 0u, 0u, 0u);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
      tmem_st32_u(tmem + t_lane + kTmemQ + c * 32, w);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarQ]);
  }
  float m = -INFINITY, l = 0.f;
  for (int jj = 0; jj < nkb; ++jj) {
    const int j = j0 + jj;       // absolute key tile
    const uint32_t t = t0 + jj;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull + t % 3], (t / 3) & 1u, kWaitLimitNs))) return false;
    tc_fence_after();
    float s[kBN];
    tmem_ld32(tmem + t_lane + kTmemS, s);
    tmem_ld32(tmem + t_lane + kTmemS + 32, s + 32);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarSFree]);   // S_{t+1} may overwrite the buffer now
    // P.V of tile t-2 read P buffer t&1; tiles of an earlier item finished with it
    bool pbuf_free = jj < 2;
    float mx = -INFINITY;        // row max of the raw scores; m below is in scaled (log2) units
    if (j >= full_tiles) {
      const int lim = row_limit - j * kBN;
#pragma unroll
      for (int k = 0; k < kBN; ++k) s[k] = k < lim ? s[k] : -INFINITY;
    }
#pragma unroll
    for (int k = 0; k < kBN / 2; ++k) mx = fmax3(mx, s[2 * k], s[2 * k + 1]);
    mx *= sl2;
    if (jj == 0) {
      m = mx;                    // every row sees at least one key of a piece's first tile
    } else {
      const bool need = mx > m + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        if (p.trace && lane == 0) atomicAdd(&p.counters[kRescaleCount], 1);
        // O holds the P.V sums of the earlier tiles: wait for the last one, then rescale
        const uint32_t tp = t - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarODone + (tp & 1u)], (tp >> 1) & 1u, kWaitLimitNs)))
          return false;
        pbuf_free = true;        // P.V MMAs finish in issue order
        tc_fence_after();
        const float m_new = need ? mx : m;
        const float alpha = ex2(m - m_new);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tmem + t_lane + kTmemO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(tmem + t_lane + kTmemO + c * 32, o);
        }
        tmem_wait_st();
        l *= alpha;
        m = m_new;
      }
    }
    // exponent arguments and row sums two at a time (packed fp32 pairs)
    const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m, -m);
    uint64_t rs2 = f2_pack(0.f, 0.f);
    uint32_t pk[kBN / 2];
#pragma unroll
    for (int k = 0; k < kBN / 2; ++k) {
      float a0, a1;
      f2_unpack(f2_fma(f2_pack(s[2 * k], s[2 * k + 1]), scale2, negm2), a0, a1);
      const float e0 = ex2(a0), e1 = ex2(a1);
      rs2 = f2_add(rs2, f2_pack(e0, e1));
      pk[k] = pack_bf16(e0, e1);
    }
    float r0, r1;
    f2_unpack(rs2, r0, r1);
    l += r0 + r1;
    // P_t into shared P buffer t&1 (the A operand of P.V_t) once P.V_{t-2} has read it
    if (!pbuf_free) {
      const uint32_t tp = t - 2;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarODone + (tp & 1u)], (tp >> 1) & 1u, kWaitLimitNs)))
        return false;
    }
    uint8_t* prow = smem + Cfg<D>::kOffP + (t & 1u) * Cfg<D>::kPBytes + row * 128;   // 128 B, swizzled
#pragma unroll
    for (int c = 0; c < kBN / 8; ++c)
      *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) =
          make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    fence_proxy_async_smem();   // generic-proxy stores -> visible to the tensor core's reads
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarPFull + (t & 1u)]);
  }
  // epilogue: O / l, one row per thread
  if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarOFinal], nq & 1u, kWaitLimitNs))) return false;
  tc_fence_after();
  const int q = q0 + row;
  const float inv = 1.f / l;
  __nv_bfloat16* orow = p.o_pre + ((size_t)(q_first + q) * p.Hq + qh) * D;
  // the piece fields are read again here rather than kept live through the tile loop
  const int4 piece = ld_nc_v4(&p.pre_items[2 * item + 1]);   // j0, j1, partial, merge
  const int part = piece.z;
  if (part < 0) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      tmem_ld32(tmem + t_lane + kTmemO + c * 32, o);
      tmem_wait_ld();
      if (q < P) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 v;
          v.x = pack_bf16(o[k * 8 + 0] * inv, o[k * 8 + 1] * inv);
          v.y = pack_bf16(o[k * 8 + 2] * inv, o[k * 8 + 3] * inv);
          v.z = pack_bf16(o[k * 8 + 4] * inv, o[k * 8 + 5] * inv);
          v.w = pack_bf16(o[k * 8 + 6] * inv, o[k * 8 + 7] * inv);
          dst[k] = v;
        }
      }
    }
    return true;
  }
  // One KV piece of a split item: each thread's row (O / l, fp32) goes to shared memory (the K and V rings,
  // free once the item's last P.V MMA finished), row-major as the workspace holds it, and the row's log-sum-exp
  // (log2 domain) to the workspace; after the item's barrier the CTA sends the tile out in one bulk copy
  // and merges it if it was the last piece (prefill_piece_end).
  float4* stg = reinterpret_cast<float4*>(smem + Cfg<D>::kOffK) + row * (D / 4);
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    float o[32];
    tmem_ld32(tmem + t_lane + kTmemO + c * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k)
      stg[c * 8 + k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv, o[4 * k + 3] * inv);
  }
  if (q < P) p.ppart_lse[(size_t)part * kBM + row] = m + __log2f(l);
  fence_proxy_async_smem();   // the row is read by the bulk copy (async proxy) ...
  __threadfence();            // ... and the log-sum-exp by other CTAs once the piece is counted
  return true;
}

// ------------------------------------------------------------------ decode
// One warp = one virtual decode block.  Item (r, kvh, k0, k1): the g query
// heads of kv head kvh of decode request r against keys k0..k1-1.
// Per 16-token page: S^T[16 keys x 8 heads] = K_page . Q^T (m16n8k16, keys as
// rows so only the head dimension is padded), online softmax per head across
// lanes, P^T moved into the B-operand layout with movmatrix, then
// O^T[d x 8] += V_page^T . P^T.  Pages arrive by TMA into a kNS-deep ring.
// The block ids of an item's pages are read 32 at a time, one per lane, a
// window ahead of use, so refilling a ring slot never waits on a global load.
// Called by the whole warp: lane 0 expects the stage's bytes, then lanes 0 and 1
// issue the K and the V box of the page in one TMA instruction (a TMA
// instruction holds its warp ~130 cycles plus ~50 per box, so one instruction of
// two boxes costs less than two of one).
template <int D, int NS, bool KV8>
__device__ __forceinline__ void decode_issue_page(const PodParams& p, uint8_t* ring, uint64_t* wbars, uint32_t seq,
                                                  int blk, int kvh, int lane) {
  using CF = Cfg<D>;
  constexpr int kStage = KV8 ? CF::kDecStage8 : CF::kDecStage;
  constexpr int kPageB = KV8 ? CF::kPageBytes8 : CF::kPageBytes;
  const int s = seq % NS;
  uint8_t* dst = ring + s * kStage + (lane == 1 ? kPageB : 0);
  uint64_t* bar = &wbars[s];
  if (lane == 0) mbar_arrive_expect_tx(bar, kStage);
  if (lane < 2) {
    const int row = KV8 ? kv_row8(p, blk, kvh) : kv_row(p, blk, kvh);
    if constexpr (KV8) {
      // one box per e4m3 page of K (lane 0) and of V (lane 1): 16 rows of d bytes
      // (128-byte swizzle at d = 128)
      tma_load_2d(dst, lane == 0 ? &p.tm_k8 : &p.tm_v8, bar, 0, row);
    } else {
      // one box per page of K (lane 0) and of V (lane 1): both 64-element halves of
      // 16 rows land as [half][16 rows][128 B], the layout two 2D boxes would give
      tma_load_3d(dst, lane == 0 ? &p.tm_kp : &p.tm_vp, bar, 0, row, 0);
    }
  }
}

__device__ __forceinline__ uint32_t swz(int row, int col_elem) {
  // byte offset of (row, col) inside a [rows][64 bf16] 128-byte-swizzled atom column
  return (uint32_t)(row * 128 + ((((col_elem >> 3) ^ row) & 7) << 4));
}

// One warp merges the split partials of merge item `midx` into bf16 outputs:
// O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M), M = max_s lse_s (log2 domain).
// Lane l owns d elements [4l, 4l + 4) (and +128 ... for larger d) of every head.
// The per-head maxima come from one lane-parallel pass over the S*G
// log-sum-exps (contiguous, [S][G]); the weighted sum then loads U splits of
// all G heads per round trip (16 independent 16-byte loads per lane), so a
// row costs about 1 + S/U memory latencies.  The partials were written by
// other warps of this launch: read them through L2.
template <int D, int G>
__device__ void merge_row_g(const PodParams& p, int r, int kvh, int first, int S) {
  constexpr int kV = D / 128 > 0 ? D / 128 : 1;   // float4 chunks per lane and head
  constexpr int U = 16 / G > 0 ? 16 / G : 1;       // splits per round trip
  const int lane = threadIdx.x & 31;
  const bool active = (lane * 4) < D;
  const float* lse = p.part_lse + (size_t)first * G;
  const int n = S * G;
  float M[G];
#pragma unroll
  for (int h = 0; h < G; ++h) M[h] = -INFINITY;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const float v = i < n ? __ldcg(lse + i) : -INFINITY;
    const int hi = i % G;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float x = hi == h ? v : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
      M[h] = fmaxf(M[h], x);
    }
  }
  float den[G];
  float4 acc[G][kV];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    den[h] = 0.f;
#pragma unroll
    for (int v = 0; v < kV; ++v) acc[h][v] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int s0 = 0; s0 < S; s0 += U) {
    float4 x[U][G][kV];
    float l[U][G];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool in = s0 + u < S;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const size_t e = (size_t)(first + s0 + u) * G + h;
        l[u][h] = in ? __ldcg(p.part_lse + e) : -INFINITY;
        const float4* po = reinterpret_cast<const float4*>(p.part_o + e * D);
#pragma unroll
        for (int v = 0; v < kV; ++v)
          x[u][h][v] = (in && active) ? __ldcg(&po[lane + 32 * v]) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float w = s0 + u < S ? ex2(l[u][h] - M[h]) : 0.f;
        den[h] += w;
#pragma unroll
        for (int v = 0; v < kV; ++v) {
          acc[h][v].x += w * x[u][h][v].x;
          acc[h][v].y += w * x[u][h][v].y;
          acc[h][v].z += w * x[u][h][v].z;
          acc[h][v].w += w * x[u][h][v].w;
        }
      }
    }
  }
  if (!active) return;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float inv = 1.f / den[h];
    __nv_bfloat16* ob = p.o_dec + ((size_t)r * p.Hq + kvh * G + h) * D;
#pragma unroll
    for (int v = 0; v < kV; ++v) {
      uint2 o;
      o.x = pack_bf16(acc[h][v].x * inv, acc[h][v].y * inv);
      o.y = pack_bf16(acc[h][v].z * inv, acc[h][v].w * inv);
      *reinterpret_cast<uint2*>(ob + 4 * (lane + 32 * v)) = o;
    }
  }
}

template <int D>
__device__ void merge_row_warp(const PodParams& p, int midx) {
  const int4 mi = __ldg(&p.merge_items[midx]);
  switch (p.g) {
    case 1: merge_row_g<D, 1>(p, mi.x, mi.y, mi.z, mi.w); break;
    case 2: merge_row_g<D, 2>(p, mi.x, mi.y, mi.z, mi.w); break;
    case 3: merge_row_g<D, 3>(p, mi.x, mi.y, mi.z, mi.w); break;
    case 4: merge_row_g<D, 4>(p, mi.x, mi.y, mi.z, mi.w); break;
    case 5: merge_row_g<D, 5>(p, mi.x, mi.y, mi.z, mi.w); break;
    case 6: merge_row_g<D, 6>(p, mi.x, mi.y, mi.z, mi.w); break;
    case 7: merge_row_g<D, 7>(p, mi.x, mi.y, mi.z, mi.w); break;
    default: merge_row_g<D, 8>(p, mi.x, mi.y, mi.z, mi.w); break;
  }
}

// Score rows of the e4m3 decode page math.  Both m16n8k16 MMAs of a page
// contract over a permuted order (a dot product does not depend on the order
// of its terms, only on both operands using the same one):
//  * d: in the S^T = K Q^T MMA, k-step ks = 4h + j (16 wide) gives lane q of a
//    quad the four d values 64h + 16q + 4j .. +3, so one 16-byte shared load of
//    a key row feeds four k-steps and the query fragment is read the same way;
//  * keys: score row r of the 16-row tile is key sigma(r) of the page, chosen so
//    that after the movmatrix transpose the P^T fragment of lane (n, q) holds
//    keys sigma(2q), sigma(2q+1), sigma(2q+8), sigma(2q+9) = the 4q..4q+3 block,
//    so the lane reads exactly four key rows of V;
//  * in O^T = V^T P^T, lane (g, q) owns the d/8 consecutive d values starting at
//    (d/8) g: M-tile mt holds d = (d/8) g + 2 mt (rows g) and + 1 (rows g + 8),
//    so one 16-byte (8-byte at d = 64) load per key row feeds every M-tile, and
//    each head's outputs of a lane are contiguous.
// sigma(r) = 4 q' + e + 2 (hi ^ (q' >> 1)) with q' = (r & 7) >> 1, e = r & 1,
// hi = r >> 3: the 2-key blocks of lanes q >= 2 are swapped, which spreads the
// four key rows one V load instruction touches over distinct swizzle phases.
__device__ __forceinline__ int sigma_key(int r) {
  const int qp = (r & 7) >> 1, e = r & 1, hi = r >> 3;
  return 4 * qp + e + 2 * (hi ^ (qp >> 1));
}

// Byte offset of (row, byte b) of an e4m3 page in shared memory: rows of d
// bytes, 16-byte chunks XOR-swizzled by the row at d = 128 (the tensor map's
// 128-byte swizzle), plain at d = 64.
template <int D>
__device__ __forceinline__ uint32_t page8_off(int row, int b) {
  if constexpr (D == 128) return (uint32_t)(row * 128 + ((((b >> 4) ^ row) & 7) << 4) + (b & 15));
  else return (uint32_t)(row * D + b);
}

template <int D, int NS, bool KV8>
__device__ bool decode_warp(const PodParams& p, uint8_t* ring, uint64_t* wbars, uint32_t& seq,
                            volatile int* abort_flag, int home_role) {
  using CF = Cfg<D>;
  constexpr int kStage = KV8 ? CF::kDecStage8 : CF::kDecStage;
  constexpr int kPageB = KV8 ? CF::kPageBytes8 : CF::kPageBytes;
  const int lane = threadIdx.x & 31;
  const int g = p.g;
  const int gq = lane >> 2, q4 = lane & 3;   // quad row / lane within the quad
  while (true) {
    if (*abort_flag) return false;
    int item = 0;
    if (lane == 0) item = atomicAdd(&p.counters[kNextDecode], 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    if (item >= p.n_dec) return true;
    const int4 a = __ldg(&p.dec_items[2 * item]);
    const int4 b = __ldg(&p.dec_items[2 * item + 1]);
    const int r = a.x, kvh = a.y, k0 = a.z, k1 = a.w, part = b.x, midx = b.y, nsplit = b.z;
    const int p0 = k0 / kPage;
    const int np = (k1 - k0 + kPage - 1) / kPage;
    // block ids: bt_cur holds pages [32 win, 32 win + 32) of the item, bt_nxt the next window;
    // the request's length is read in the same round trip and checked once the pages are under way
    const int* bt_item = p.block_table + (size_t)(p.NP + r) * p.bt_stride + p0;
    int bt_cur = lane < np ? __ldg(bt_item + lane) : 0;
    int bt_nxt = 32 + lane < np ? __ldg(bt_item + 32 + lane) : 0;
    const int len_now = (lane == 0 && p.kv_lens) ? __ldg(&p.kv_lens[p.NP + r]) : k1;
    int win = 0;
    {
      const int pre = np < NS ? np : NS;
      for (int j = 0; j < pre; ++j) {
        const int blk = __shfl_sync(0xffffffffu, bt_cur, j);
        decode_issue_page<D, NS, KV8>(p, ring, wbars, seq + j, blk, kvh, lane);
      }
    }
    if (lane == 0) {
      if (len_now < k1) record_error(p, POD_ERR_PLAN_MISMATCH, item);
      if (p.trace) {
        int32_t* e = p.trace + 4 * (p.n_pre + item);
        e[0] = (int32_t)smid();
        e[1] = blockIdx.x;
        e[2] = home_role;
        atomicAdd(&e[3], 1);
      }
    }
    // Q^T as the B operand: lane holds head n = lane/4; bf16 pairs of d (lane%4)*2 (+8) per 16-wide
    // step, or, for e4m3 pages, f16 pairs of d 64h + 16(lane%4) + 4j (+2) for step 4h + j
    uint32_t qf[D / 16][2];
    const float sl2 = KV8 ? p.scale_log2 * __ldg(&p.k_scale8[kvh]) : p.scale_log2;
    {
      const int n = gq;
      if (n < g) {
        const __nv_bfloat16* qp = p.q_dec + ((size_t)r * p.Hq + kvh * g + n) * D;
        if constexpr (KV8) {
#pragma unroll
          for (int h = 0; h < D / 64; ++h) {
            const uint4* src = reinterpret_cast<const uint4*>(qp + 64 * h + 16 * q4);
            const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
              qf[4 * h + (i >> 1)][i & 1] = pack_f16(f.x, f.y);
            }
          }
        } else {
          const int dc = q4 * 2;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            qf[ks][0] = __ldg(reinterpret_cast<const uint32_t*>(qp + ks * 16 + dc));
            qf[ks][1] = __ldg(reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8 + dc));
          }
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) qf[ks][0] = qf[ks][1] = 0u;
      }
    }
    float acc[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    // score rows held by this lane: keys key_lo and key_hi of the page
    const int key_lo = KV8 ? sigma_key(gq) : gq;
    const int key_hi = KV8 ? sigma_key(gq + 8) : gq + 8;
    // ldmatrix lane roles (bf16 pages)
    const int a_row = lane & 15, a_colh = (lane >> 4) * 8;                  // K as A (non-trans)
    const int v_key = (lane & 7) + ((lane >> 4) << 3), v_colh = ((lane >> 3) & 1) * 8;  // V^T as A (trans)
    bool ok = true;
    int jfail = 0;
    for (int j = 0; j < np; ++j) {
      const uint32_t sq = seq + j;
      const int s = sq % NS;
      const bool w = mbar_wait(&wbars[s], (sq / NS) & 1u, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        jfail = j;
        break;
      }
      uint8_t* kbuf = ring + s * kStage;
      uint8_t* vbuf = kbuf + kPageB;
      const int valid = min(kPage, k1 - (p0 + j) * kPage);
      if (valid < kPage) {
        // clear V rows past the end of the request: they may hold anything
        if constexpr (KV8) {
          for (int i = lane; i < (kPage - valid) * (D / 16); i += 32)
            *reinterpret_cast<uint4*>(vbuf + (valid + i / (D / 16)) * D + (i % (D / 16)) * 16) = make_uint4(0, 0, 0, 0);
        } else {
          for (int i = lane; i < (kPage - valid) * CF::kHalves * 8; i += 32) {
            const int chunk = i & 7, rh = i >> 3;
            const int key = valid + rh % (kPage - valid), h = rh / (kPage - valid);
            *reinterpret_cast<uint4*>(vbuf + h * (kPage * 128) + key * 128 + chunk * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      const uint32_t kb_u = smem_u32(kbuf), vb_u = smem_u32(vbuf);
      // S^T = K Q^T over d in two independent accumulator chains (even and odd
      // 16-wide d slices), so the page's score latency is half a dependent chain
      float c[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (KV8) {
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          const uint4 ka = lds_u128(kb_u + page8_off<D>(key_lo, 64 * h + 16 * q4));
          const uint4 kb = lds_u128(kb_u + page8_off<D>(key_hi, 64 * h + 16 * q4));
          const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w}, wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int ks = 4 * h + jj;
            mma_16816_f16((ks & 1) ? c2 : c, lo16_e4m3_to_f16x2(wa[jj]), lo16_e4m3_to_f16x2(wb[jj]),
                          hi16_e4m3_to_f16x2(wa[jj]), hi16_e4m3_to_f16x2(wb[jj]), qf[ks][0], qf[ks][1]);
          }
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int col = ks * 16 + a_colh;
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kb_u + (col >> 6) * (kPage * 128) + swz(a_row, col & 63), a0, a1, a2, a3);
          mma_16816((ks & 1) ? c2 : c, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) c[i] += c2[i];
      // mask, scale, online softmax per head (columns (lane%4)*2 and +1)
      const float s0 = key_lo < valid ? c[0] * sl2 : -INFINITY;
      const float s1 = key_lo < valid ? c[1] * sl2 : -INFINITY;
      const float s2 = key_hi < valid ? c[2] * sl2 : -INFINITY;
      const float s3 = key_hi < valid ? c[3] * sl2 : -INFINITY;
      float tA = fmaxf(s0, s2), tB = fmaxf(s1, s3);
      // the running max is kept stale until a score beats it by more than 2^8 (any base gives the same
      // softmax; exponentials stay <= 2^8): only then reduce the page max across lanes and rescale
      if (__any_sync(0xffffffffu, tA > mA + 8.f || tB > mB + 8.f)) {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          tA = fmaxf(tA, __shfl_xor_sync(0xffffffffu, tA, o));
          tB = fmaxf(tB, __shfl_xor_sync(0xffffffffu, tB, o));
        }
        const float nA = fmaxf(mA, tA), nB = fmaxf(mB, tB);
        const float alA = ex2(mA - nA), alB = ex2(mB - nB);
        mA = nA;
        mB = nB;
        lA *= alA;
        lB *= alB;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          acc[mt][0] *= alA;
          acc[mt][1] *= alB;
          acc[mt][2] *= alA;
          acc[mt][3] *= alB;
        }
      }
      const float e0 = ex2(s0 - mA), e1 = ex2(s1 - mB), e2 = ex2(s2 - mA), e3 = ex2(s3 - mB);
      lA += e0 + e2;
      lB += e1 + e3;
      if constexpr (KV8) {
        const uint32_t pb0 = movmatrix_t(pack_f16(e0, e1));   // score rows 0..7
        const uint32_t pb1 = movmatrix_t(pack_f16(e2, e3));   // score rows 8..15
        // this lane's V key rows sigma(2q), sigma(2q+1), sigma(2q+8), sigma(2q+9)
        const int rot = 2 * (q4 >> 1);
        const int ra = 4 * q4 + rot, rb = ra + 1, rc = 4 * q4 + (rot ^ 2), rd = rc + 1;
        // lane (gq, q) owns d = (D/8) gq .. +D/8-1: M-tile mt holds d = (D/8) gq + 2 mt (rows gq) and +1
        constexpr int W = D / 32;                  // 32-bit words of a lane's d range per key row
        uint32_t wa[W], wb[W], wc[W], wd[W];
        {
          const int col = (D / 8) * gq;
          if constexpr (W == 4) {
            const uint4 a4 = lds_u128(vb_u + page8_off<D>(ra, col)), b4 = lds_u128(vb_u + page8_off<D>(rb, col));
            const uint4 c4 = lds_u128(vb_u + page8_off<D>(rc, col)), d4 = lds_u128(vb_u + page8_off<D>(rd, col));
            wa[0] = a4.x; wa[1] = a4.y; wa[2] = a4.z; wa[3] = a4.w;
            wb[0] = b4.x; wb[1] = b4.y; wb[2] = b4.z; wb[3] = b4.w;
            wc[0] = c4.x; wc[1] = c4.y; wc[2] = c4.z; wc[3] = c4.w;
            wd[0] = d4.x; wd[1] = d4.y; wd[2] = d4.z; wd[3] = d4.w;
          } else {
            const uint2 a2 = lds_u64(vb_u + page8_off<D>(ra, col)), b2 = lds_u64(vb_u + page8_off<D>(rb, col));
            const uint2 c2v = lds_u64(vb_u + page8_off<D>(rc, col)), d2 = lds_u64(vb_u + page8_off<D>(rd, col));
            wa[0] = a2.x; wa[1] = a2.y; wb[0] = b2.x; wb[1] = b2.y;
            wc[0] = c2v.x; wc[1] = c2v.y; wd[0] = d2.x; wd[1] = d2.y;
          }
        }
#pragma unroll
        for (int w = 0; w < W; ++w) {
          // byte pairs (key a, key b) for d = 4w + 0/1 (M-tile 2w) and 4w + 2/3 (M-tile 2w + 1)
          const uint32_t ab01 = __byte_perm(wa[w], wb[w], 0x5140), ab23 = __byte_perm(wa[w], wb[w], 0x7362);
          const uint32_t cd01 = __byte_perm(wc[w], wd[w], 0x5140), cd23 = __byte_perm(wc[w], wd[w], 0x7362);
          mma_16816_f16(acc[2 * w], lo16_e4m3_to_f16x2(ab01), hi16_e4m3_to_f16x2(ab01), lo16_e4m3_to_f16x2(cd01),
                        hi16_e4m3_to_f16x2(cd01), pb0, pb1);
          mma_16816_f16(acc[2 * w + 1], lo16_e4m3_to_f16x2(ab23), hi16_e4m3_to_f16x2(ab23),
                        lo16_e4m3_to_f16x2(cd23), hi16_e4m3_to_f16x2(cd23), pb0, pb1);
        }
      } else {
        const uint32_t pb0 = movmatrix_t(pack_bf16(e0, e1));   // keys 0..7
        const uint32_t pb1 = movmatrix_t(pack_bf16(e2, e3));   // keys 8..15
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int col = mt * 16 + v_colh;
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vb_u + (col >> 6) * (kPage * 128) + swz(v_key, col & 63), a0, a1, a2, a3);
          mma_16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
        }
      }
      const int jn = j + NS;
      if (jn < np) {
        if ((jn >> 5) > win) {     // next window; fetch the one after it
          ++win;
          bt_cur = bt_nxt;
          const int pg = 32 * (win + 1) + lane;
          bt_nxt = pg < np ? __ldg(bt_item + pg) : 0;
        }
        const int blk = __shfl_sync(0xffffffffu, bt_cur, jn & 31);
        __syncwarp();
        decode_issue_page<D, NS, KV8>(p, ring, wbars, sq + NS, blk, kvh, lane);
      }
    }
    if (!ok) {
      // drain copies still in flight into this warp's ring before giving up
      if (lane == 0) {
        record_error(p, POD_ERR_TIMEOUT, 3);
        const int jend = min(np, jfail + NS);
        for (int j = jfail + 1; j < jend; ++j) {
          const uint32_t sq = seq + (uint32_t)j;
          mbar_wait(&wbars[sq % NS], (sq / NS) & 1u, kWaitLimitNs / 4);
        }
      }
      *abort_flag = 1;
      return false;
    }
    seq += (uint32_t)np;
    // finalize: full row sums across the 8 lanes that share a head pair
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lA += __shfl_xor_sync(0xffffffffu, lA, o);
      lB += __shfl_xor_sync(0xffffffffu, lB, o);
    }
    const int hA = q4 * 2, hB = hA + 1;
    const float vsc = KV8 ? __ldg(&p.v_scale8[kvh]) : 1.f;
    const float iA = vsc / lA, iB = vsc / lB;
    if (part < 0) {
      __nv_bfloat16* ob = p.o_dec + ((size_t)r * p.Hq + kvh * g) * D;
      if constexpr (KV8) {
        // M-tile mt holds d = (D/8) gq + 2 mt (+1 in rows gq + 8): D/8 consecutive d per head
#pragma unroll
        for (int v = 0; v < D / 64; ++v) {
          const int dd = (D / 8) * gq + 8 * v;
          const int m0 = 4 * v;
          if (hA < g)
            *reinterpret_cast<uint4*>(ob + hA * D + dd) =
                make_uint4(pack_bf16(acc[m0][0] * iA, acc[m0][2] * iA), pack_bf16(acc[m0 + 1][0] * iA, acc[m0 + 1][2] * iA),
                           pack_bf16(acc[m0 + 2][0] * iA, acc[m0 + 2][2] * iA), pack_bf16(acc[m0 + 3][0] * iA, acc[m0 + 3][2] * iA));
          if (hB < g)
            *reinterpret_cast<uint4*>(ob + hB * D + dd) =
                make_uint4(pack_bf16(acc[m0][1] * iB, acc[m0][3] * iB), pack_bf16(acc[m0 + 1][1] * iB, acc[m0 + 1][3] * iB),
                           pack_bf16(acc[m0 + 2][1] * iB, acc[m0 + 2][3] * iB), pack_bf16(acc[m0 + 3][1] * iB, acc[m0 + 3][3] * iB));
        }
      } else {
        const int d_lo = gq;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int dd = mt * 16 + d_lo;
          if (hA < g) {
            ob[hA * D + dd] = __float2bfloat16_rn(acc[mt][0] * iA);
            ob[hA * D + dd + 8] = __float2bfloat16_rn(acc[mt][2] * iA);
          }
          if (hB < g) {
            ob[hB * D + dd] = __float2bfloat16_rn(acc[mt][1] * iB);
            ob[hB * D + dd + 8] = __float2bfloat16_rn(acc[mt][3] * iB);
          }
        }
      }
    } else {
      float* po = p.part_o + (size_t)part * g * D;
      if constexpr (KV8) {
#pragma unroll
        for (int v = 0; v < D / 32; ++v) {
          const int dd = (D / 8) * gq + 4 * v;
          const int m0 = 2 * v;
          if (hA < g)
            *reinterpret_cast<float4*>(po + hA * D + dd) =
                make_float4(acc[m0][0] * iA, acc[m0][2] * iA, acc[m0 + 1][0] * iA, acc[m0 + 1][2] * iA);
          if (hB < g)
            *reinterpret_cast<float4*>(po + hB * D + dd) =
                make_float4(acc[m0][1] * iB, acc[m0][3] * iB, acc[m0 + 1][1] * iB, acc[m0 + 1][3] * iB);
        }
      } else {
        const int d_lo = gq;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int dd = mt * 16 + d_lo;
          if (hA < g) {
            po[hA * D + dd] = acc[mt][0] * iA;
            po[hA * D + dd + 8] = acc[mt][2] * iA;
          }
          if (hB < g) {
            po[hB * D + dd] = acc[mt][1] * iB;
            po[hB * D + dd + 8] = acc[mt][3] * iB;
          }
        }
      }
      if (gq == 0) {
        if (hA < g) p.part_lse[(size_t)part * g + hA] = mA + __log2f(lA);
        if (hB < g) p.part_lse[(size_t)part * g + hB] = mB + __log2f(lB);
      }
      if (p.merge_in_kernel) {
        // the warp that finishes a row's last split merges it (no waiting on other warps)
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          last = atomicAdd(&p.merge_cnt[midx], 1) == nsplit - 1;
          if (last) p.merge_cnt[midx] = 0;   // every split has counted: ready for the next launch
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          merge_row_warp<D>(p, midx);
        }
      }
    }
  }
}

// The end of one KV piece of a split prefill item, by the whole CTA after the item's barrier (the
// softmax threads have put the tile's 128 partial rows, O / l in fp32, row-major into the K and V rings and
// their log-sum-exps into the workspace).  One thread sends the tile out in one bulk copy (the rows are
// contiguous there as here) and counts the piece; the CTA that counts the item's last piece merges the
// pieces: O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M), M = max_s lse_s (log2 domain).  Each of
// threads 0..127 turns its row's log-sum-exps into normalised weights (in the P buffers, free as well);
// then the six warps walk the rows with lanes along d, this piece's partial from shared memory and every
// other piece's with one coalesced load per row (written by other CTAs of this launch: read through L2),
// eight rows per lane in flight, and write the bf16 result as whole rows.  No CTA waits for another.
template <int D>
__device__ void prefill_piece_end(const PodParams& p, int item, uint8_t* smem, volatile uint32_t* flag) {
  constexpr int kF4 = D / 4;            // float4 per row
  constexpr int kRowsPer = 32 / kF4;    // rows per warp-wide access (1 at d = 128, 2 at d = 64)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.n_ppart == 0) return;
  // the piece fields are read again rather than kept live through the item
  const int4 pc = ld_nc_v4(&p.pre_items[2 * item + 1]);   // j0, j1, partial, merge
  const int part = pc.z, midx = pc.w;
  if (part < 0) return;
  const float4* stg = reinterpret_cast<const float4*>(smem + Cfg<D>::kOffK);
  if (tid == 0) {
    bulk_store_s2g(p.ppart_o + (size_t)part * kBM * D, stg, (uint32_t)(kBM * D * 4));
    bulk_commit();
    bulk_wait_all();              // the rows are in global memory (and the rings may be reused) ...
    fence_proxy_async_global();   // ... ordered before the count
    __threadfence();
    const int4 pm = ld_nc_v4(&p.pmerge_items[midx]);   // first partial, pieces
    const bool last = atomicAdd(&p.pmerge_cnt[kWarpsPerCta * midx], 1) == pm.y - 1;
    if (last) p.pmerge_cnt[kWarpsPerCta * midx] = 0;   // every piece has counted: ready for the next launch
    *flag = last ? 1u : 0u;
  }
  __syncthreads();
  if (*flag == 0u) return;
  __threadfence();
  const int4 pm = ld_nc_v4(&p.pmerge_items[midx]);
  const int first = pm.x, S = pm.y, own = part - first;
  const int4 ia = ld_nc_v4(&p.pre_items[2 * item]);      // q0, q head, kv_end, request
  const int4 rq = __ldg(&p.pre_reqs[ia.w]);               // first row in q_pre / o_pre, P, C
  const int rows_left = rq.y - ia.x;                      // tile rows r < rows_left are inside the chunk
  float* wtab = reinterpret_cast<float*>(smem + Cfg<D>::kOffP);   // [piece][128 rows]
  if (tid < kBM) {
    const float* lse = p.ppart_lse + (size_t)first * kBM + tid;
    float M = -INFINITY;
#pragma unroll 4
    for (int sp = 0; sp < S; ++sp) {
      const float x = __ldcg(lse + (size_t)sp * kBM);
      wtab[sp * kBM + tid] = x;
      M = fmaxf(M, x);
    }
    float den = 0.f;
    for (int sp = 0; sp < S; ++sp) {
      const float e = ex2(wtab[sp * kBM + tid] - M);
      wtab[sp * kBM + tid] = e;
      den += e;
    }
    const float dinv = 1.f / den;   // rows past the chunk (never written) give garbage weights, never used
    for (int sp = 0; sp < S; ++sp) wtab[sp * kBM + tid] *= dinv;
  }
  __syncthreads();
  constexpr int kBatch = 8;                       // rows per lane in flight
  constexpr int kSteps = kBM / kRowsPer;          // warp-wide row steps of the tile
  const int sub = lane / kF4, f4 = lane % kF4;
  const float4* part0 = reinterpret_cast<const float4*>(p.ppart_o) + ((size_t)first * kBM + sub) * kF4 + f4;
  const size_t ostride = (size_t)p.Hq * D;
  __nv_bfloat16* out0 = p.o_pre + ((size_t)(rq.x + ia.x + sub) * p.Hq + ia.y) * D + 4 * f4;
  for (int s0 = warp; s0 < kSteps; s0 += kAllWarps * kBatch) {
    // this warp's row steps s0, s0 + 6, ..., s0 + 6 (kBatch - 1): row r = step * kRowsPer + sub
    float4 acc[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int st = s0 + u * kAllWarps;
      const int r = (st < kSteps ? st : 0) * kRowsPer + sub;
      const float w = wtab[own * kBM + r];
      const float4 v = stg[r * kF4 + f4];
      acc[u] = make_float4(w * v.x, w * v.y, w * v.z, w * v.w);
    }
    for (int sp = 0; sp < S; ++sp) {
      if (sp == own) continue;
      float4 va[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int st = s0 + u * kAllWarps;
        va[u] = __ldcg(part0 + ((size_t)sp * kBM + (st < kSteps ? st : 0) * kRowsPer) * kF4);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int st = s0 + u * kAllWarps;
        const float w = wtab[sp * kBM + (st < kSteps ? st : 0) * kRowsPer + sub];
        acc[u].x += w * va[u].x;
        acc[u].y += w * va[u].y;
        acc[u].z += w * va[u].z;
        acc[u].w += w * va[u].w;
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int st = s0 + u * kAllWarps;
      const int r = st * kRowsPer + sub;
      if (st < kSteps && r < rows_left) {
        uint2 v;
        v.x = pack_bf16(acc[u].x, acc[u].y);
        v.y = pack_bf16(acc[u].z, acc[u].w);
        *reinterpret_cast<uint2*>(out0 + (size_t)st * kRowsPer * ostride) = v;
      }
    }
  }
  fence_proxy_async_smem();   // the next item's TMA loads reuse the rings and the P buffers
}

// --------------------------------------------------------- persistent kernel
// Grid = SMs x CTAs/SM.  Each CTA takes one ticket from its SM's counter; the
// ticket fixes its home role (prefill iff t mod (p+d) < p).  The CTA drains
// its home queue, then the other one; no CTA ever waits for another.
template <int D, bool KV8>
__global__ void __launch_bounds__(kThreads, 2) pod_attn_kernel(const __grid_constant__ PodParams p) {
  using CF = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + CF::kSmem);
  // TMEM address, home role, item, abort
  uint32_t* ctrl = reinterpret_cast<uint32_t*>(bars + CF::kNumBars + 1);
  volatile int* sh_abort = reinterpret_cast<volatile int*>(ctrl + 3);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (smem_u32(smem) & 1023u) {   // the swizzled tiles need 1024-byte alignment
    if (tid == 0) {
      griddep_wait();
      record_error(p, POD_ERR_UNSUPPORTED, 1024);
    }
    return;
  }
  if (tid == 0) {
    for (int i = 0; i <= CF::kNumBars; ++i) {   // [kNumBars]: self-test barrier, never arrived at
      uint32_t count = 1;
      if (i == kBarQ || i == kBarSFree || i == kBarPFull || i == kBarPFull + 1) count = kWarpsPerCta;
      mbar_init(&bars[i], count);
    }
    fence_mbar_init();
    *sh_abort = 0;
    if (!KV8 || p.n_pre > 0) {   // with an e4m3 cache and no prefill the bf16 maps are not encoded
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_kp);
      tma_prefetch_desc(&p.tm_vp);
    }
    if (KV8) {
      tma_prefetch_desc(&p.tm_k8);
      tma_prefetch_desc(&p.tm_v8);
    }
    // everything above touched only shared memory and the kernel parameters; the counters, the tables
    // and the inputs may still be written by the grid this launch follows (programmatic dependent launch)
    griddep_wait();
    // and a dependent launch may be scheduled once every CTA of this grid got here (its CTAs take SMs
    // only as this grid's CTAs leave them, and wait for this grid to complete before they start)
    griddep_launch_dependents();
    int home = p.mode == kDecodeOnly ? kRoleDecode : kRolePrefill;
    if (p.mode == kFused && p.partition_sms > 0) {
      // ablation: whole SMs start on one role (the first partition_sms SM ids prefill-first)
      home = (int)smid() < p.partition_sms ? kRolePrefill : kRoleDecode;
    } else if (p.mode == kFused) {
      const uint32_t sm = smid();
      const int t = atomicAdd(&p.counters[kTicketBase + (int)(sm % kMaxSms)], 1);
      const int span = p.ratio_p + p.ratio_d;
      home = (span > 0 && (t % span) < p.ratio_p) ? kRolePrefill : kRoleDecode;
    }
    ctrl[1] = (uint32_t)home;
  }
  __syncwarp();
  if (warp == 0) {
    if (p.use_tmem) tmem_alloc(&ctrl[0], kTmemCols);
    // every CTA gives up its TMEM allocation permit at once, whether it allocated
    // or not: a resident CTA still holding the permit keeps the SM from taking
    // the second CTA of this kernel
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = p.use_tmem ? ctrl[0] : 0u;
  const int home = (int)ctrl[1];
  if (p.selftest_timeout && blockIdx.x == 0 && tid == 0) {
    // nothing ever arrives at this barrier: the bounded wait must expire and report
    if (!mbar_wait(&bars[CF::kNumBars], 0u, 1000000ull)) record_error(p, POD_ERR_TIMEOUT, -1);
  }

  uint32_t tiles_done = 0, items_done = 0, seq = 0;
  // decode page rings: warp w < decode_warps owns ring w (ns stages) and its ns barriers
  const bool all_decode = p.decode_warps == kAllWarps;
  const int dwarps = all_decode ? kAllWarps : kWarpsPerCta;
  const int ns = KV8 ? (all_decode ? CF::kNSAll8 : CF::kNS8) : (all_decode ? CF::kNSAll : CF::kNS);
  uint8_t* ring = smem + (warp < dwarps ? warp : 0) * ns * (KV8 ? CF::kDecStage8 : CF::kDecStage);
  uint64_t* wbars = &bars[kBarDecode + (warp < dwarps ? warp : 0) * ns];

  for (int phase = 0; phase < 2; ++phase) {
    const int role = phase == 0 ? home : 1 - home;
    if (p.mode == kPrefillOnly && role != kRolePrefill) continue;
    if (p.mode == kDecodeOnly && role != kRoleDecode) continue;
    if (role == kRolePrefill) {
      while (true) {
        if (tid == 0) ctrl[2] = (uint32_t)(*sh_abort ? p.n_pre : atomicAdd(&p.counters[kNextPrefill], 1));
        __syncthreads();
        const int item = (int)ctrl[2];
        if (item >= p.n_pre) break;
        if (tid == 0 && p.trace) {
          int32_t* e = p.trace + 4 * item;
          e[0] = (int32_t)smid();
          e[1] = blockIdx.x;
          e[2] = home;
          atomicAdd(&e[3], 1);
        }
        const PreItem it = load_pre_item(p, item);
        bool ok;
        if (warp == kMmaWarp) ok = prefill_mma<D>(p, it, smem, bars, tmem, tiles_done, items_done);
        else if (warp == kTmaWarp) ok = prefill_tma<D>(p, it, smem, bars, tiles_done);
        else ok = prefill_softmax<D>(p, it, item, smem, bars, tmem, tiles_done, items_done);
        tc_fence_before();
        const int fail = __syncthreads_or(!ok);
        tc_fence_after();
        if (fail) {
          if (tid == 0) {
            record_error(p, POD_ERR_TIMEOUT, 2);
            *sh_abort = 1;
          }
          __syncthreads();
          break;
        }
        prefill_piece_end<D>(p, item, smem, ctrl + 4);
        tiles_done += (uint32_t)(it.j1 - it.j0);
        items_done += 1;
      }
    } else {
      if (all_decode) decode_warp<D, KV8 ? CF::kNSAll8 : CF::kNSAll, KV8>(p, ring, wbars, seq, sh_abort, home);
      else if (warp < kWarpsPerCta) decode_warp<D, KV8 ? CF::kNS8 : CF::kNS, KV8>(p, ring, wbars, seq, sh_abort, home);
      __syncthreads();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (p.use_tmem && warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (p.self_reset) {
    // The last CTA out returns the launch's counters to zero for the next launch on this workspace (the
    // warp that completes a merge has already reset that merge's count) and publishes the launch's
    // first error, or none, in the error word.  No CTA of this launch touches the counters afterwards.
    if (tid == 0) {
      __threadfence();
      ctrl[2] = atomicAdd(&p.counters[kExitCount], 1) == (int)gridDim.x - 1 ? 1u : 0u;
    }
    __syncthreads();
    if (ctrl[2]) {
      __threadfence();
      volatile int32_t* c = p.counters;
      const int err = c[kRunError];
      for (int i = tid; i < kMaxSms; i += kThreads) c[kTicketBase + i] = 0;
      if (err != 0) {   // an aborted launch can leave merges uncounted
        for (int i = tid; i < p.n_merge_cnt; i += kThreads) p.merge_cnt[i] = 0;
        for (int i = tid; i < p.n_pmerge_cnt; i += kThreads) p.pmerge_cnt[i] = 0;
      }
      if (tid == 0) {
        c[kErrorInfo] = c[kRunErrorInfo];
        c[kErrorWord] = err;
        c[kRunError] = 0;
        c[kRunErrorInfo] = 0;
        c[kNextPrefill] = 0;
        c[kNextDecode] = 0;
        c[kExitCount] = 0;
      }
    }
  }
}

// --------------------------------------------------------------- LSE merge
struct MergeParams {
  const int4* items;       // r, kvh, first_partial, num_splits
  const float* part_o;     // [n_part, g, D]
  const float* part_lse;   // [n_part, g], log2 domain
  __nv_bfloat16* o_dec;
  int32_t n_merge, Hq, g;
};

// One CTA per (request, kv head) row with splits: O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M).
template <int D>
__global__ void __launch_bounds__(128) pod_merge_kernel(const MergeParams mp) {
  const int4 it = __ldg(&mp.items[blockIdx.x]);
  const int r = it.x, kvh = it.y, first = it.z, S = it.w;
  const int g = mp.g;
  for (int idx = threadIdx.x; idx < g * D; idx += blockDim.x) {
    const int h = idx / D, dd = idx % D;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, __ldg(&mp.part_lse[(size_t)(first + s) * g + h]));
    float num = 0.f, den = 0.f;
    for (int s = 0; s < S; ++s) {
      const float w = ex2(__ldg(&mp.part_lse[(size_t)(first + s) * g + h]) - M);
      num += w * __ldg(&mp.part_o[((size_t)(first + s) * g + h) * D + dd]);
      den += w;
    }
    mp.o_dec[((size_t)r * mp.Hq + kvh * g + h) * D + dd] = __float2bfloat16_rn(num / den);
  }
}

}  // namespace pod

// =========================================================== host side (ABI)
#include <atomic>

using namespace pod;

namespace {

thread_local int g_last_cuda = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda = (int)e;
  return POD_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int D, bool KV8>
int configure_kernels() {
  static std::atomic<bool> done[64];   // per device and instantiation; setting the attributes twice is harmless
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 64 && done[dev].load(std::memory_order_acquire)) return POD_OK;
  e = cudaFuncSetAttribute(pod_attn_kernel<D, KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cfg<D>::kSmemAlloc);
  if (e != cudaSuccess) return cuda_fail(e);
  // two CTAs of ~113 KB need the whole 228 KB shared-memory carveout on every launch
  e = cudaFuncSetAttribute(pod_attn_kernel<D, KV8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 64) done[dev].store(true, std::memory_order_release);
  return POD_OK;
}

// Library-owned side stream and fork/join events for the two-stream ablation,
// one set per device, made on first use; `lock` serialises the enqueue order.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex lock;
};

int side_stream(SideStream** out) {
  static SideStream sides[64];
  static std::mutex make;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev >= 64) return POD_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(make);
  SideStream& s = sides[dev];
  if (!s.stream) {
    // publish the set only when all three objects exist; release what a failed attempt made
    cudaStream_t st = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      if (join) cudaEventDestroy(join);
      if (fork) cudaEventDestroy(fork);
      if (st) cudaStreamDestroy(st);
      return cuda_fail(e);
    }
    s.fork = fork;
    s.join = join;
    s.stream = st;
  }
  *out = &s;
  return POD_OK;
}

template <int D, bool KV8>
int launch(const pod_attn_plan_t* pl, PodParams& prm, const MergeParams& mp, cudaStream_t st) {
  int rc = configure_kernels<D, KV8>();
  if (rc != POD_OK) return rc;
  const size_t smem = Cfg<D>::kSmemAlloc;
  if (pl->ev_start) cudaEventRecord(static_cast<cudaEvent_t>(pl->ev_start), st);
  if (pl->cfg.flags & POD_FLAG_SEQUENTIAL) {
    if (pl->n_pre > 0) {
      prm.mode = kPrefillOnly;
      prm.use_tmem = 1;
      const int grid = pl->n_pre < pl->grid ? pl->n_pre : pl->grid;
      pod_attn_kernel<D, KV8><<<grid, kThreads, smem, st>>>(prm);
    }
    if (pl->n_dec > 0) {
      prm.mode = kDecodeOnly;
      prm.use_tmem = 0;
      pod_attn_kernel<D, KV8><<<pl->grid, kThreads, smem, st>>>(prm);
    }
  } else if ((pl->cfg.flags & POD_FLAG_TWO_STREAMS) && pl->n_pre > 0 && pl->n_dec > 0) {
    SideStream* side = nullptr;
    rc = side_stream(&side);
    if (rc != POD_OK) return rc;
    std::lock_guard<std::mutex> g(side->lock);
    cudaError_t e = cudaEventRecord(side->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
    if (e != cudaSuccess) return cuda_fail(e);
    prm.mode = kPrefillOnly;
    prm.use_tmem = 1;
    const int grid = pl->n_pre < pl->grid ? pl->n_pre : pl->grid;
    pod_attn_kernel<D, KV8><<<grid, kThreads, smem, st>>>(prm);
    prm.mode = kDecodeOnly;
    prm.use_tmem = 0;
    pod_attn_kernel<D, KV8><<<pl->grid, kThreads, smem, side->stream>>>(prm);
    e = cudaEventRecord(side->join, side->stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, side->join, 0);
    if (e != cudaSuccess) return cuda_fail(e);
  } else if (pl->n_pre > 0 || pl->n_dec > 0) {
    prm.mode = kFused;
    prm.use_tmem = pl->n_pre > 0 ? 1 : 0;
    // programmatic dependent launch: this grid's CTAs may be scheduled while the previous kernel on the
    // stream finishes; they wait for it (griddep_wait) before touching global memory
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)pl->grid);
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    lc.attrs = attr;
    lc.numAttrs = 1;
    const cudaError_t le = cudaLaunchKernelEx(&lc, pod_attn_kernel<D, KV8>, prm);
    if (le != cudaSuccess) return cuda_fail(le);
  }
  if (pl->ev_stop) cudaEventRecord(static_cast<cudaEvent_t>(pl->ev_stop), st);
  if (pl->n_merge > 0 && (pl->cfg.flags & POD_FLAG_MERGE_KERNEL))
    pod_merge_kernel<D><<<pl->n_merge, 128, 0, st>>>(mp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return POD_OK;
}

}  // namespace

extern "C" {

const char* pod_attn_status_string(int s) {
  switch (s) {
    case POD_OK: return "ok";
    case POD_ERR_INVALID_ARG: return "invalid argument";
    case POD_ERR_UNSUPPORTED: return "unsupported shape (head_dim 64/128, group <= 8, page 16)";
    case POD_ERR_WORKSPACE: return "workspace too small";
    case POD_ERR_CUDA: return "CUDA runtime error";
    case POD_ERR_BOUNDS: return "block id out of range";
    case POD_ERR_TIMEOUT: return "device wait timed out";
    case POD_ERR_PLAN_MISMATCH: return "kv lengths disagree with the plan";
    default: return "unknown status";
  }
}

int pod_attn_last_cuda_error(void) { return g_last_cuda; }

int pod_attn_plan_batched(const pod_attn_config* cfg, int32_t num_prefill, const int32_t* prefill_qo_lens,
                          const int32_t* prefill_kv_lens, int32_t num_decode, const int32_t* decode_kv_lens,
                          pod_attn_plan_t** plan_out, size_t* workspace_bytes_out) {
  if (!cfg || !plan_out) return POD_ERR_INVALID_ARG;
  *plan_out = nullptr;
  int sms = cfg->num_sms;
  if (sms == 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  pod_attn_plan_t* pl = nullptr;
  const int rc = pod_plan_build(cfg, sms, num_prefill, prefill_qo_lens, prefill_kv_lens, num_decode, decode_kv_lens,
                                &pl);
  if (rc != POD_OK) return rc;
  pl->cfg.num_sms = sms;
  *plan_out = pl;
  if (workspace_bytes_out) *workspace_bytes_out = (size_t)pl->ws_bytes;
  return POD_OK;
}

int pod_attn_plan(const pod_attn_config* cfg, int32_t prefill_qo_len, int32_t prefill_kv_len,
                  int32_t num_decode, const int32_t* decode_kv_lens,
                  pod_attn_plan_t** plan_out, size_t* workspace_bytes_out) {
  return pod_attn_plan_batched(cfg, 1, &prefill_qo_len, &prefill_kv_len, num_decode, decode_kv_lens, plan_out,
                               workspace_bytes_out);
}

int pod_attn_plan_get_info(const pod_attn_plan_t* pl, pod_attn_plan_info* info) {
  if (!pl || !info) return POD_ERR_INVALID_ARG;
  info->num_prefill_items = pl->n_pre;
  info->num_decode_items = pl->n_dec;
  info->num_merge_items = pl->n_merge;
  info->num_partials = pl->n_part;
  info->ctas_per_sm = pl->ctas;
  info->ratio_prefill = pl->ratio_p;
  info->ratio_decode = pl->ratio_d;
  info->chunk_pages = pl->chunk_pages;
  info->num_sms = pl->num_sms;
  info->grid = pl->grid;
  info->workspace_bytes = pl->ws_bytes;
  info->error_offset = 4LL * kErrorWord;
  info->prefill_flops = pl->prefill_flops;
  info->decode_flops = pl->decode_flops;
  info->kv_bytes = pl->kv_bytes;
  info->qo_bytes = pl->qo_bytes;
  info->table_bytes = (int64_t)pl->image.size();
  info->num_prefill_requests = pl->NP;
  info->num_prefill_rows = pl->P;
  info->num_prefill_partials = pl->n_ppart;
  info->num_prefill_merge_items = pl->n_pmerge;
  info->rescale_count_offset = 4LL * kRescaleCount;
  return POD_OK;
}

int pod_attn_plan_prefill_requests(const pod_attn_plan_t* pl, int32_t* out) {
  if (!pl) return POD_ERR_INVALID_ARG;
  if (out && !pl->preq.empty()) std::memcpy(out, pl->preq.data(), pl->preq.size() * 4);
  return POD_OK;
}

int pod_attn_plan_prefill_merges(const pod_attn_plan_t* pl, int32_t* out) {
  if (!pl) return POD_ERR_INVALID_ARG;
  if (out && !pl->pmerge.empty()) std::memcpy(out, pl->pmerge.data(), pl->pmerge.size() * 4);
  return POD_OK;
}

int pod_attn_plan_tables(const pod_attn_plan_t* pl, int32_t* pre, int32_t* dec, int32_t* merge) {
  if (!pl) return POD_ERR_INVALID_ARG;
  if (pre && !pl->pre.empty()) std::memcpy(pre, pl->pre.data(), pl->pre.size() * 4);
  if (dec && !pl->dec.empty()) std::memcpy(dec, pl->dec.data(), pl->dec.size() * 4);
  if (merge && !pl->merge.empty()) std::memcpy(merge, pl->merge.data(), pl->merge.size() * 4);
  return POD_OK;
}

int pod_attn_upload(const pod_attn_plan_t* pl, void* ws, size_t ws_bytes, void* stream) {
  if (!pl || !ws) return POD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return POD_ERR_INVALID_ARG;
  if ((int64_t)ws_bytes < pl->ws_bytes) return POD_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)pl->off_pre, st);
  if (e == cudaSuccess && !pl->image.empty())
    e = cudaMemcpyAsync(static_cast<uint8_t*>(ws) + kCountersBytes, pl->image.data(), pl->image.size(),
                        cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return POD_OK;
}

}  // extern "C"

namespace {

// The e4m3 cache of the decode requests (pod_attn_run_fp8kv).
struct Fp8Args {
  const void* k8;
  const void* v8;
  int64_t num_blocks8;
  const float* k_scale;
  const float* v_scale;
};

int run_impl(const pod_attn_plan_t* pl, const void* q_prefill, const void* q_decode, const void* k_cache,
             const void* v_cache, int64_t num_blocks, const int32_t* block_table, int32_t block_table_stride,
             const int32_t* kv_lens, float scale, void* o_prefill, void* o_decode, void* ws, size_t ws_bytes,
             int32_t* trace, void* stream, const Fp8Args* f8) {
  if (!pl || !ws) return POD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return POD_ERR_INVALID_ARG;
  if ((int64_t)ws_bytes < pl->ws_bytes) return POD_ERR_WORKSPACE;
  const int D = pl->cfg.head_dim, Hq = pl->cfg.num_q_heads, Hkv = pl->cfg.num_kv_heads;
  const bool has_pre = pl->n_pre > 0, has_dec = pl->n_dec > 0;
  if (has_pre && (!q_prefill || !o_prefill || !aligned16(q_prefill) || !aligned16(o_prefill)))
    return POD_ERR_INVALID_ARG;
  if (has_dec && (!q_decode || !o_decode || !aligned16(q_decode) || !aligned16(o_decode)))
    return POD_ERR_INVALID_ARG;
  // the bf16 pools serve the prefill requests, and the decodes too unless an e4m3 cache is given
  const bool need16 = has_pre || (has_dec && !f8);
  if (need16 && (!k_cache || !v_cache || !aligned16(k_cache) || !aligned16(v_cache) || num_blocks < 1))
    return POD_ERR_INVALID_ARG;
  if ((has_pre || has_dec) && !block_table) return POD_ERR_INVALID_ARG;
  if (f8 && has_dec &&
      (!f8->k8 || !f8->v8 || !aligned16(f8->k8) || !aligned16(f8->v8) || f8->num_blocks8 < 1 || !f8->k_scale ||
       !f8->v_scale))
    return POD_ERR_INVALID_ARG;
  if (f8 && f8->num_blocks8 * Hkv * kPage >= (int64_t)INT32_MAX) return POD_ERR_UNSUPPORTED;
  if (block_table_stride < 1 || !(scale > 0.f) || scale != scale) return POD_ERR_INVALID_ARG;
  if (num_blocks * Hkv * kPage >= (int64_t)INT32_MAX) return POD_ERR_UNSUPPORTED;
  if ((pl->cfg.flags & POD_FLAG_TRACE) && !trace) return POD_ERR_INVALID_ARG;
  if (!(has_pre || has_dec)) return POD_OK;

  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return cuda_fail(cudaErrorNotSupported);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  PodParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (need16) {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)num_blocks * Hkv * kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kPage};
    const cuuint32_t es[2] = {1, 1};
    CUresult r1 = enc(&prm.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k_cache), dims, strides, box,
                      es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r1 != CUDA_SUCCESS) return POD_ERR_INVALID_ARG;
    // page view: x = element within a 64-element half, y = row, z = half (row stride 2d bytes, half stride 128 B)
    const cuuint64_t pdims[3] = {64, (cuuint64_t)num_blocks * Hkv * kPage, (cuuint64_t)(D / 64)};
    const cuuint64_t pstrides[2] = {(cuuint64_t)D * 2, 128};
    const cuuint32_t pbox[3] = {64, (cuuint32_t)kPage, (cuuint32_t)(D / 64)};
    const cuuint32_t pes[3] = {1, 1, 1};
    CUresult r3 = enc(&prm.tm_kp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k_cache), pdims, pstrides, pbox,
                      pes, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    CUresult r4 = enc(&prm.tm_vp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(v_cache), pdims, pstrides, pbox,
                      pes, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r3 != CUDA_SUCCESS || r4 != CUDA_SUCCESS) return POD_ERR_INVALID_ARG;
  }
  if (f8 && has_dec) {
    // e4m3 pages: rows of d bytes, one box {d, 16} per page (128-byte swizzle at d = 128)
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)f8->num_blocks8 * Hkv * kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)D};
    const cuuint32_t box[2] = {(cuuint32_t)D, (cuuint32_t)kPage};
    const cuuint32_t es[2] = {1, 1};
    const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r1 = enc(&prm.tm_k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(f8->k8), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    CUresult r2 = enc(&prm.tm_v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(f8->v8), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r1 != CUDA_SUCCESS || r2 != CUDA_SUCCESS) return POD_ERR_INVALID_ARG;
    prm.k_scale8 = f8->k_scale;
    prm.v_scale8 = f8->v_scale;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  prm.q_pre = static_cast<const __nv_bfloat16*>(q_prefill);
  prm.q_dec = static_cast<const __nv_bfloat16*>(q_decode);
  prm.o_pre = static_cast<__nv_bfloat16*>(o_prefill);
  prm.o_dec = static_cast<__nv_bfloat16*>(o_decode);
  prm.block_table = block_table;
  prm.kv_lens = kv_lens;
  prm.counters = reinterpret_cast<int32_t*>(w);
  prm.pre_items = reinterpret_cast<const int4*>(w + pl->off_pre);
  prm.dec_items = reinterpret_cast<const int4*>(w + pl->off_dec);
  prm.merge_items = reinterpret_cast<const int4*>(w + pl->off_merge);
  prm.pre_reqs = reinterpret_cast<const int4*>(w + pl->off_preq);
  prm.merge_cnt = reinterpret_cast<int32_t*>(w + pl->off_merge_cnt);
  prm.pmerge_items = reinterpret_cast<const int4*>(w + pl->off_pmerge);
  prm.pmerge_cnt = reinterpret_cast<int32_t*>(w + pl->off_pmerge_cnt);
  prm.ppart_o = reinterpret_cast<float*>(w + pl->off_ppart_o);
  prm.ppart_lse = reinterpret_cast<float*>(w + pl->off_ppart_lse);
  prm.merge_in_kernel = (pl->cfg.flags & POD_FLAG_MERGE_KERNEL) ? 0 : 1;
  prm.selftest_timeout = (pl->cfg.flags & POD_FLAG_SELFTEST_TIMEOUT) ? 1 : 0;
  prm.decode_warps = (pl->cfg.flags & POD_FLAG_DECODE_FOUR_WARPS) ? kWarpsPerCta : kAllWarps;
  if ((pl->cfg.flags & POD_FLAG_SM_PARTITION) && pl->n_pre > 0 && pl->n_dec > 0) {
    // as many SMs as the prefill items fill with every CTA of the SM, at least one, at most all
    const int64_t want = ((int64_t)pl->n_pre + pl->ctas - 1) / pl->ctas;
    prm.partition_sms = (int32_t)(want < 1 ? 1 : (want > pl->num_sms ? pl->num_sms : want));
  }
  prm.part_o = reinterpret_cast<float*>(w + pl->off_part_o);
  prm.part_lse = reinterpret_cast<float*>(w + pl->off_part_lse);
  prm.trace = (pl->cfg.flags & POD_FLAG_TRACE) ? trace : nullptr;
  prm.bt_stride = block_table_stride;
  prm.kv_rows = (int32_t)(num_blocks * Hkv * kPage);
  prm.num_blocks = (int32_t)num_blocks;
  if (f8 && has_dec) {
    prm.kv_rows8 = (int32_t)(f8->num_blocks8 * Hkv * kPage);
    prm.num_blocks8 = (int32_t)f8->num_blocks8;
  }
  prm.n_pre = pl->n_pre;
  prm.n_dec = pl->n_dec;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.g = pl->g;
  prm.NP = pl->NP;
  prm.B = pl->B;
  prm.ratio_p = pl->ratio_p;
  prm.ratio_d = pl->ratio_d;
  prm.scale_log2 = scale * 1.4426950408889634f;

  MergeParams mp;
  mp.items = reinterpret_cast<const int4*>(w + pl->off_merge);
  mp.part_o = prm.part_o;
  mp.part_lse = prm.part_lse;
  mp.o_dec = prm.o_dec;
  mp.n_merge = pl->n_merge;
  mp.Hq = Hq;
  mp.g = pl->g;

  prm.n_ppart = pl->n_ppart;
  prm.n_merge_cnt = pl->n_merge;
  prm.n_pmerge_cnt = kWarpsPerCta * pl->n_pmerge;
  // Counters (tickets, queue heads, error word, merge completions) are zero when a launch starts.  A
  // fused launch leaves them at zero itself (its last CTA), so only the two-kernel paths, the traced
  // path (its rescale count) and an empty batch (no launch, fresh error word) clear them here.
  const uint32_t fl = pl->cfg.flags;
  const bool two_kernels = (fl & POD_FLAG_SEQUENTIAL) || ((fl & POD_FLAG_TWO_STREAMS) && pl->n_pre > 0 && pl->n_dec > 0);
  prm.self_reset = (pl->n_pre > 0 || pl->n_dec > 0) && !two_kernels && !(fl & POD_FLAG_TRACE) ? 1 : 0;
  if (!prm.self_reset) {
    const cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)pl->off_pre, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (f8 && has_dec) return D == 128 ? launch<128, true>(pl, prm, mp, st) : launch<64, true>(pl, prm, mp, st);
  return D == 128 ? launch<128, false>(pl, prm, mp, st) : launch<64, false>(pl, prm, mp, st);
}

}  // namespace

extern "C" {

int pod_attn_run(const pod_attn_plan_t* pl, const void* q_prefill, const void* q_decode, const void* k_cache,
                 const void* v_cache, int64_t num_blocks, const int32_t* block_table, int32_t block_table_stride,
                 const int32_t* kv_lens, float scale, void* o_prefill, void* o_decode, void* ws, size_t ws_bytes,
                 int32_t* trace, void* stream) {
  return run_impl(pl, q_prefill, q_decode, k_cache, v_cache, num_blocks, block_table, block_table_stride, kv_lens,
                  scale, o_prefill, o_decode, ws, ws_bytes, trace, stream, nullptr);
}

int pod_attn_run_fp8kv(const pod_attn_plan_t* pl, const void* q_prefill, const void* q_decode, const void* k_cache,
                       const void* v_cache, int64_t num_blocks, const void* k_cache_fp8, const void* v_cache_fp8,
                       int64_t num_blocks_fp8, const float* k_scale, const float* v_scale,
                       const int32_t* block_table, int32_t block_table_stride, const int32_t* kv_lens, float scale,
                       void* o_prefill, void* o_decode, void* ws, size_t ws_bytes, int32_t* trace, void* stream) {
  const Fp8Args f8{k_cache_fp8, v_cache_fp8, num_blocks_fp8, k_scale, v_scale};
  return run_impl(pl, q_prefill, q_decode, k_cache, v_cache, num_blocks, block_table, block_table_stride, kv_lens,
                  scale, o_prefill, o_decode, ws, ws_bytes, trace, stream, &f8);
}

int pod_attn_plan_set_events(pod_attn_plan_t* pl, void* ev_start, void* ev_stop) {
  if (!pl) return POD_ERR_INVALID_ARG;
  pl->ev_start = ev_start;
  pl->ev_stop = ev_stop;
  return POD_OK;
}

int pod_attn_event_create(void** ev_out) {
  if (!ev_out) return POD_ERR_INVALID_ARG;
  cudaEvent_t ev;
  cudaError_t e = cudaEventCreate(&ev);
  if (e != cudaSuccess) return cuda_fail(e);
  *ev_out = ev;
  return POD_OK;
}

int pod_attn_event_destroy(void* ev) {
  if (!ev) return POD_OK;
  cudaError_t e = cudaEventDestroy(static_cast<cudaEvent_t>(ev));
  return e == cudaSuccess ? POD_OK : cuda_fail(e);
}

int pod_attn_event_elapsed_ms(void* a, void* b, float* ms) {
  if (!a || !b || !ms) return POD_ERR_INVALID_ARG;
  cudaError_t e = cudaEventElapsedTime(ms, static_cast<cudaEvent_t>(a), static_cast<cudaEvent_t>(b));
  return e == cudaSuccess ? POD_OK : cuda_fail(e);
}

void pod_attn_plan_destroy(pod_attn_plan_t* pl) { delete pl; }

}  // extern "C"
