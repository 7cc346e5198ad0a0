// pod_plan.h -- work-unit plan shared by the host planner and the kernels.
//
// The planner splits a hybrid batch into independent work units (POD-Attention
// §4 "POD-Attention": prefill and decode CTAs are remapped onto the device
// functions of the two phases; §4.2.3 caps chunked-prefill splits at two full
// waves; the persistent-thread form of §4.4 pulls units from queues):
//   prefill unit = (request, query head, 128-row query tile, KV split)
//   decode unit  = (request, KV head, KV split of `dec_split_len` keys)
// Units whose KV range is split write fp32 partial results and are merged by
// log-sum-exp in split order, so results never depend on which CTA ran what.
#pragma once
#include <cuda.h>
#include <stdint.h>

namespace pod {

constexpr int kMaxPrefillReqs = 16;
constexpr int kQTile = 128;           // prefill query rows per unit (= UMMA M)
constexpr int kKVTile = 128;          // prefill keys per KV tile (= UMMA N of S)
constexpr int kPrefillStages = 2;     // K/V smem ring depth in the prefill role
constexpr int kDecTile = 16;          // decode keys per mma block (= mma M)
// Keys per decode stage: one 16-key block at d = 128, two at d = 64, so a
// stage moves the same bytes (8 KB) and its fixed per-stage work (waits, row
// maxima, exponentials, transposes) is spread over as many bytes.
constexpr int dec_stage_blocks(int D) { return D == 64 ? 2 : 1; }
constexpr int dec_stage_keys(int D) { return kDecTile * dec_stage_blocks(D); }
constexpr int kRoleWarps = 10;        // 8 softmax (2 query tiles) + MMA issuer + TMA producer;
                                      // all of them run decode units in a decode turn
constexpr int kSideDecWarps = 2;      // warps that stream decode units for the CTA's whole life,
                                      // beside whatever role the other warps have
constexpr int kFusedWarps = kRoleWarps + kSideDecWarps;
constexpr int kFusedThreads = kFusedWarps * 32;
constexpr int kSoftmaxWarps = 8;
constexpr int kFusedDecWarps = kRoleWarps;  // decode runners of a decode turn
constexpr int kFusedSlotsPerSm = 1;   // persistent CTAs per SM (the CTA owns all TMEM)
static_assert(kRoleWarps == kSoftmaxWarps + 2, "softmax warps + MMA issuer + producer");
constexpr int kFusedDecStages = 2;    // per-warp decode ring depth in the fused kernel
constexpr int kDecodeWarps = 6;       // warps (virtual decode units) per decode-only CTA
constexpr int kDecodeStages = 2;      // per-warp ring depth in the decode-only kernel
constexpr int kMaxGroup = 8;          // query heads per KV head (mma N = 8)
constexpr int kTmemCols = 512;        // TMEM columns per CTA (all of an SM's tensor memory)
constexpr int kMaxSmid = 256;         // per-SM ticket slots (indexed by %smid)
constexpr long long kDefaultWaitBudget = 2000000000LL;  // cycles (~1 s at 2 GHz)
// Plan::flags bits set by the library itself (the low byte carries the
// POD_FLAG_* bits of the context's configuration).
constexpr int kFlagGlobalTicket = 0x100;    // one ticket counter instead of one per SM
constexpr int kFlagFrontPolicy = 0x200;     // each SM's first ticket takes prefill
constexpr int kFlagBalancedPolicy = 0x400;  // a fixed set of CTAs takes prefill first
constexpr int kFlagPoisonOnStatus = 0x800;  // merge writes NaN when the status word is set

struct PrefillReq {
  int prior, chunk, q_row0, n_qtiles;
  int kv_len, bt_row, n_split, pair_heads;  // n_split: largest split count of its units;
                                            // pair_heads: see PrefillUnit
};

// Two query tiles: heads (head, head + 1) at token tile qtile when the
// request's pair_heads is set, else token tiles (qtile, qtile + 1) of head.
// The unit covers KV split `split` of `n_split` of the pair's key range. A
// split pair (n_split > 1) owns merge groups group0 (tile 0) and group0 + 1
// (tile 1) and partial slots slot0 + i * n_split + s for tile i, split s.
struct PrefillUnit {
  int req, head, qtile, split;
  int n_split, group0, slot0, work;  // work: KV tiles of this split (planner's sort key)
};

struct DecodeReq {
  const uint16_t* k;  // contiguous caches (null when paged)
  const uint16_t* v;
  int len, n_split, unit0, slot0;   // slot0: first partial slot (split requests)
  int group0, bt_row, pad0, pad1;
};

// Kernel parameters (by value). Pointers refer to the device workspace or to
// the caller's tensors.
struct Plan {
  int H, Hk, G, D;
  float scale_log2;              // log2(e) / sqrt(d)
  int n_prefill_units, n_decode_units, n_prefill_reqs, n_decode_reqs;
  int dec_split_len;
  int rho_num, rho_den;          // prefill share of claims (per-SM Bresenham)
  int paged;
  int bt_stride_p, bt_stride_d;
  int flags;
  int pool_blocks;               // paged: blocks in the pool (bounds every block id)
  int dec_turn;                  // decode units per warp per fused decode turn
  int p_cap;                     // balanced policy: CTAs 0..p_cap-1 take prefill first
  long long wait_budget;         // cycles a bounded wait may spin
  const PrefillReq* preq;
  const PrefillUnit* punits;
  const DecodeReq* dreq;         // unit0 ascending: a unit's request is found by search
  const uint16_t* q_p; uint16_t* o_p; float* lse_p;
  const uint16_t* q_d; uint16_t* o_d; float* lse_d;
  const int* bt_p; const int* bt_d;
  const uint16_t* k_pool; const uint16_t* v_pool;
  float* ppart_o; float* ppart_lse;   // prefill partials [slot][128][d], [slot][128]
  float* dpart_o; float* dpart_lse;   // decode partials  [slot][8][d],   [slot][8]
  int* ctl;                           // [0] prefill queue head, [1] decode queue head
  int* sm_ticket;                     // [kMaxSmid]
  int* pgroup_ctr;                    // arrivals per prefill merge group
  int* dgroup_ctr;                    // arrivals per decode merge group
  int* stats;                         // [kMaxSmid][2] claims per role (POD_FLAG_STATS)
  int* status;                        // sticky status word (not reset per call)
  const int* never_set;               // test-only flag that nothing writes
};

// Tensor maps for TMA, passed as a __grid_constant__ kernel parameter.
// Contiguous layout: k[p] / v[p] map request p's [len, Hk, d] cache with a
// 128-key box. Paged layout: k[0] / v[0] map the pool as [blocks*16, Hk, d]
// with a 16-key (one page) box.
struct TmaDescs {
  CUtensorMap q;
  CUtensorMap k[kMaxPrefillReqs];
  CUtensorMap v[kMaxPrefillReqs];
};

}  // namespace pod
