// pod_kernels.cu -- sm_100a kernels of the hybrid prefill + decode attention.
//
// Roles (POD-Attention §4 "POD-Attention"; the paper's FlashAttention device
// functions for A100 are prior art here, rebuilt for Blackwell):
//  * prefill unit (pod_prefill.cuh): two 128-row query tiles that share K/V
//    against a range of 128-key KV tiles. A TMA producer warp stages Q and
//    K/V (128-byte swizzle), one thread issues tcgen05.mma (S_i = Q_i K^T into
//    a TMEM S buffer the two tiles take in turn, O_i += P_i V with P_i read
//    from its own TMEM columns), and two groups of four softmax warps (one
//    thread per query row = TMEM lane) run the online softmax of the two
//    tiles while the tensor pipe works on the other tile's MMAs.
//  * decode unit: one warp (a "virtual decode CTA", paper §4.2.3) streams the
//    K/V rows of (request, KV head, key split) with 16-byte cp.async copies
//    into a padded smem ring and runs S^T = K Q^T and O^T += V^T P^T on the
//    legacy m16n8k16 tensor-core path with the G query heads of the group as
//    N = 8 (the paper's small decode tile, §4.2.1). A claimed unit finds its
//    request by a search of the requests' first-unit indices.
//  * merge: log-sum-exp combination of split partials, in split order.
//  * fused kernel: one persistent 12-warp CTA per SM (the CTA-pair kernel
//    further down runs the same roles on clusters of two). Its ten role warps
//    read %smid, take a ticket from that SM's counter and pick prefill or decode
//    work (§4.1 SM-aware scheduling, §4.4 persistent threads, §5.4.2 role
//    allocation); its two side warps stream decode units for the CTA's whole
//    life, beside a prefill unit. The last CTA (or warp) to finish a split
//    group merges it, so no CTA ever waits for another (the digest's
//    deadlock-free merge requirement).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "pod_exp2.cuh"
#include "pod_plan.h"
#include "pod_ptx.cuh"

namespace pod {

// Share of the prefill softmax's exponentials evaluated by exp2_poly on the
// FMA pipe instead of MUFU (pairs out of 8), and the bf16 packing used for P.
// Measured on B200 (long-context prefill, 64/8 heads, d 128, two query tiles
// per CTA): 0 pairs is fastest; 1 and 2 pairs cost 1.17x and 1.28x, since the
// polynomial takes more FMA-pipe time per element than ex2 takes on MUFU.
// cvt packing (round to nearest even) is 3 % faster than the integer
// round-half-away one.
#ifndef POD_SOFT_EXP2_PAIRS
#define POD_SOFT_EXP2_PAIRS 0
#endif
constexpr int kSoftPairs = POD_SOFT_EXP2_PAIRS;
#if defined(POD_RHA_PACK)
#define POD_PACK(a, b) pack_bf16_rha(a, b)
#elif defined(POD_INT_PACK)
#define POD_PACK(a, b) pack_bf16_int(a, b)
#else
#define POD_PACK(a, b) pack_bf16(a, b)
#endif

// Softmax form of the one-SM prefill tile: 0 = one warp per query row and tile
// (warps 0-3 tile 0, 4-7 tile 1); 1 = two warps per row splitting its keys,
// all eight warps serving both tiles in turn.
#ifndef POD_SOFTMAX_SPLIT
#define POD_SOFTMAX_SPLIT 0
#endif
// TMEM use of the one-SM prefill tile. 1 (default): one S buffer that the two
// query tiles take in turn and a separate P_i per tile, so the next S is
// issued as soon as the softmax has loaded the last one. 0: S_i per query
// tile, P_i written over S_i (the next S_i waits for P_i V to complete).
// Measured on B200, long-context batch (64 / 8 heads, d 128): the shared S
// takes about 13 % fewer SM cycles per KV step, but the board's power limit
// lowers the clock with it, so the call is 1-2 % faster.
#ifndef POD_SHARED_S
#define POD_SHARED_S 1
#endif

// L2 cache-policy hints: the decode K/V copies are evict-first (read once), so
// the decode stream of a fused launch does not push the prefill's K/V tiles
// (re-read by several query tiles) out of L2; the CTA-pair tile's K/V loads
// are also marked evict-last (on the one-SM tile that measured no gain).
#ifndef POD_L2_HINTS
#define POD_L2_HINTS 1
#endif

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kStatusTimeout = -5;
constexpr int kStatusUnsupported = -2;

POD_DEV void set_status(const Plan& P, int code) { atomicCAS(P.status, 0, code); }

// Bounded mbarrier wait. On timeout records POD_ETIMEOUT, raises the CTA's
// abort flag and returns false; once the flag is up every later wait returns
// false at once, so all roles reach the end of the CTA.
POD_DEV bool wait_bar(uint32_t bar, uint32_t parity, const Plan& P, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > P.wait_budget) {
      set_status(P, kStatusTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}
// Warp-collective form: every lane gets the same answer, so warp-collective
// instructions after it (tcgen05.ld, shuffles, ldmatrix) stay convergent.
POD_DEV bool wait_bar_warp(uint32_t bar, uint32_t parity, const Plan& P,
                           volatile int* abort_flag) {
  const bool ok = wait_bar(bar, parity, P, abort_flag);
  return __all_sync(0xffffffffu, ok);
}
// Drain wait used only after an abort: waits for an async copy or MMA this
// thread issued itself, bounded, ignoring the abort flag.
POD_DEV void drain_bar(uint32_t bar, uint32_t parity, long long budget) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > budget) return;
  }
}

// ============================================================= smem layout
template <int D>
struct FusedLayout {
  static constexpr int QB = kQTile * D * 2;   // one Q tile
  static constexpr int KT = kKVTile * D * 2;  // one K (or V) tile of 128 keys
  static constexpr int Q_OFF = 0;                               // Q0, Q1
  static constexpr int K_OFF = Q_OFF + 2 * QB;                  // K ring
  static constexpr int V_OFF = K_OFF + kPrefillStages * KT;     // V ring
  static constexpr int PREFILL_END = V_OFF + kPrefillStages * KT;
  static constexpr int DEC_ROW = D * 2 + 16;  // padded row: conflict-free ldmatrix
  static constexpr int DEC_STAGE = 2 * dec_stage_keys(D) * DEC_ROW;
  static constexpr int DEC_WARP = kFusedDecStages * DEC_STAGE;
  static constexpr int DEC_END = kFusedDecWarps * DEC_WARP;  // decode turns overlay prefill
  static constexpr int SIDE_OFF = PREFILL_END > DEC_END ? PREFILL_END : DEC_END;
  static constexpr int DATA_END = SIDE_OFF + kSideDecWarps * DEC_WARP;  // side decode rings
  // The key-split softmax exchanges, per query row, four floats (two tiles x two
  // key halves) through the 16-byte padding that ends every row of the side
  // decode rings (the decode copies and ldmatrix reads stay in the row's first
  // 2 D bytes); one row of padding per query row.
  static constexpr int XCH_OFF = SIDE_OFF + D * 2;
  static constexpr int XCH_STRIDE = DEC_ROW;
  static_assert(kSideDecWarps * DEC_WARP / DEC_ROW >= kQTile, "one padded ring row per query row");
  static constexpr int BAR_OFF = (DATA_END + 127) & ~127;
  // barrier indices
  static constexpr int B_Q = 0;                         // Q0 and Q1 landed
  static constexpr int B_KF = 1;                        // K tile landed
  static constexpr int B_KE = B_KF + kPrefillStages;    // K tile read by both S MMAs
  static constexpr int B_VF = B_KE + kPrefillStages;    // V tile landed
  static constexpr int B_VE = B_VF + kPrefillStages;    // V tile read by both PV MMAs
  static constexpr int B_SF = B_VE + kPrefillStages;    // S_i in TMEM [2]
  static constexpr int B_SE = B_SF + 2;                 // S_i free (its P read by PV_i) [2];
                                                        // shared S: [0] the S buffer loaded
  static constexpr int B_PF = B_SE + 2;                 // P_i in TMEM, one arrival per warp [2]
  static constexpr int B_PE = B_PF + 2;                 // shared S: P_i read by PV_i [2]
  static constexpr int B_OR = B_PE + 2;                 // O_i final for the unit [2]
  static constexpr int N_BARS = B_OR + 2;
  static constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
  static constexpr int TOTAL = MISC_OFF + 64;
  static_assert(TOTAL <= 227 * 1024, "fused CTA exceeds the shared memory of an SM");
  // The dynamic shared memory window of a CTA without static shared memory
  // starts 1024-byte aligned; the kernel checks it and refuses to run (status)
  // otherwise. At least 116 KB are requested so that two CTAs never share an
  // SM (2 x 117 KB > 228 KB): each CTA holds all 512 TMEM columns for its life.
  static constexpr int SMEM_BYTES = TOTAL > 116 * 1024 ? TOTAL : 116 * 1024;
};

template <int D>
struct DecodeLayout {
  static constexpr int ROW = D * 2 + 16;
  static constexpr int STAGE = 2 * dec_stage_keys(D) * ROW;
  static constexpr int WARP = kDecodeStages * STAGE;
  static constexpr int FLAG_OFF = kDecodeWarps * WARP;  // one abort flag per warp
  static constexpr int SMEM_BYTES = FLAG_OFF + kDecodeWarps * 4;
};

// ============================================================= LSE merge
POD_DEV float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
POD_DEV float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// One warp merges rows i0 .. i0+RB-1 (those < nrows) of n split partials:
// M = max_s lse_s, w_s = exp(lse_s - M), O = sum_s w_s O_s / sum_s w_s,
// LSE = M + ln sum_s w_s. Lanes hold the splits' LSE values (32 at a time) and
// the partial-O loads of all RB rows of a split are issued together, so the
// merge costs a few L2 round trips per split chunk rather than per split.
// Every output element accumulates w_s O_s in split order 0..n-1, whoever
// calls this and with whatever RB, so all merge paths agree bitwise.
// Partials written by other CTAs are read with ld.global.cg (L2, not L1).
template <int D, int RB>
POD_DEV void merge_rows_warp(const float* po, long long po_split, long long po_row,
                             const float* pl, long long pl_split, long long pl_row, int n, int i0,
                             int nrows, uint16_t* out, long long out_row, float* lse_out,
                             long long lse_row, int lane) {
  constexpr int PER = D / 32;
  float M[RB], W[RB], acc[RB][PER];
#pragma unroll
  for (int rb = 0; rb < RB; ++rb) {
    M[rb] = -INFINITY;
    W[rb] = 0.f;
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[rb][k] = 0.f;
  }
  for (int s0 = 0; s0 < n; s0 += 32) {
    const int s = s0 + lane;
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
      const float v = (s < n && i0 + rb < nrows) ? __ldcg(pl + s * pl_split + (i0 + rb) * pl_row)
                                                 : -INFINITY;
      M[rb] = fmaxf(M[rb], v);
    }
  }
#pragma unroll
  for (int rb = 0; rb < RB; ++rb) M[rb] = warp_max(M[rb]);
  for (int s0 = 0; s0 < n; s0 += 32) {
    const int s = s0 + lane;
    float w[RB];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
      const float v = (s < n && i0 + rb < nrows) ? __ldcg(pl + s * pl_split + (i0 + rb) * pl_row)
                                                 : -INFINITY;
      w[rb] = (v == -INFINITY) ? 0.f : ex2((v - M[rb]) * kLog2e);
      W[rb] += w[rb];
    }
    const int cnt = min(32, n - s0);
    // loads of several splits in flight: the merge is L2-latency bound
#pragma unroll(RB == 1 ? 8 : 2)
    for (int t = 0; t < cnt; ++t) {
      const float* src = po + (long long)(s0 + t) * po_split + lane * PER;
      float x[RB][PER];
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        if (i0 + rb < nrows) {
          if constexpr (PER == 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (i0 + rb) * po_row));
            x[rb][0] = v.x; x[rb][1] = v.y; x[rb][2] = v.z; x[rb][3] = v.w;
          } else {
            const float2 v = __ldcg(reinterpret_cast<const float2*>(src + (i0 + rb) * po_row));
            x[rb][0] = v.x; x[rb][1] = v.y;
          }
        } else {
#pragma unroll
          for (int k = 0; k < PER; ++k) x[rb][k] = 0.f;
        }
      }
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const float wt = __shfl_sync(0xffffffffu, w[rb], t);
#pragma unroll
        for (int k = 0; k < PER; ++k) acc[rb][k] = fmaf(wt, x[rb][k], acc[rb][k]);
      }
    }
  }
#pragma unroll
  for (int rb = 0; rb < RB; ++rb) {
    W[rb] = warp_sum(W[rb]);
    if (i0 + rb >= nrows) continue;
    const float inv = 1.f / W[rb];
    uint16_t* o = out + (i0 + rb) * out_row + lane * PER;
    if constexpr (PER == 4) {
      uint2 v;
      v.x = pack_bf16(acc[rb][0] * inv, acc[rb][1] * inv);
      v.y = pack_bf16(acc[rb][2] * inv, acc[rb][3] * inv);
      *reinterpret_cast<uint2*>(o) = v;
    } else {
      *reinterpret_cast<uint32_t*>(o) = pack_bf16(acc[rb][0] * inv, acc[rb][1] * inv);
    }
    if (lane == 0) lse_out[(i0 + rb) * lse_row] = M[rb] + logf(W[rb]);
  }
}

// All G rows of decode merge group (request r, KV head g); one warp.
template <int D>
POD_DEV void merge_decode_group(const Plan& P, const DecodeReq& R, int r, int g, int lane) {
  const int slot0 = R.slot0 + g;
  for (int i0 = 0; i0 < P.G; i0 += 4)
    merge_rows_warp<D, 4>(P.dpart_o + (size_t)slot0 * kMaxGroup * D, (long long)P.Hk * kMaxGroup * D,
                          D, P.dpart_lse + (size_t)slot0 * kMaxGroup, (long long)P.Hk * kMaxGroup, 1,
                          R.n_split, i0, P.G, P.o_d + ((size_t)r * P.H + (size_t)g * P.G) * D, D,
                          P.lse_d + (size_t)r * P.H + (size_t)g * P.G, 1, lane);
}

// The request of decode unit u: the last request whose first unit is <= u.
// Requests own consecutive unit ranges (n_split x Hk units each, never empty)
// in request order, so the per-request table replaces a per-unit one and the
// plan a call copies grows with its requests, not with its units.
POD_DEV int decode_unit_request(const Plan& P, int u) {
  int lo = 0, hi = P.n_decode_reqs - 1;  // dreq[lo].unit0 <= u throughout
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(&P.dreq[mid].unit0) <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// ============================================================= decode unit
// One warp, one unit (request r, KV head g, keys [kbeg, kend)). The ring of
// `NST` stages lives at `wsm` (each stage: 16 K rows then 16 V rows, padded).
// `ring` counts tiles this warp has staged so far (the stage slot rotates
// across units).
//
// Staging: every lane copies 16-byte pieces with cp.async (one commit group
// per stage), so a warp instruction moves two whole 256-byte rows (d = 128)
// and a stage takes D / 8 instructions per lane. A row of one KV head is the
// only contiguous run of a (token, head)-major cache, and 256-byte bulk
// (TMA) copies, one per lane, took far longer to issue than the stage's
// arithmetic; plain asynchronous copies issue at the load/store rate and need
// no mbarrier and no proxy fence between a stage's reads and its refill.
template <int D, int NST>
POD_DEV bool decode_unit_warp(const Plan& P, int u, uint8_t* wsm, uint32_t& ring, int lane,
                              bool inline_merge, volatile int* abort_flag) {
  static_assert(NST >= 1 && NST <= 8, "cp.async.wait_group counts at most 7 pending groups");
  constexpr int ROW = D * 2 + 16;
  constexpr int NB = dec_stage_blocks(D);  // 16-key mma blocks per stage
  constexpr int KPS = kDecTile * NB;       // keys per stage
  constexpr int STAGE = 2 * KPS * ROW;     // K rows 0..KPS-1, then V rows
  constexpr int KS = D / 16;
  constexpr int CH = D * 2 / 16;  // 16-byte pieces per row
  constexpr int RPI = 32 / CH;    // rows per warp instruction
  static_assert(kDecTile % RPI == 0, "a block is a whole number of warp instructions");
  const int r = decode_unit_request(P, u);
  const DecodeReq R = P.dreq[r];
  const int Hk = P.Hk, G = P.G;
  const int local = u - R.unit0;
  const int s = local / Hk;
  const int g = local - s * Hk;
  const int kbeg = s * P.dec_split_len;
  const int kend = min(R.len, kbeg + P.dec_split_len);
  const int n_tiles = (kend - kbeg + KPS - 1) / KPS;  // stages
  const int q4 = lane & 3;
  const int hrow = lane >> 2;  // query head within the group (B column / C row of S^T)

  // Q^T as the B operand of S^T = K Q^T: lane holds Q[head lane/4][16kk + 2q4 (+1, +8, +9)].
  uint32_t qb[KS][2];
  {
    const uint16_t* qrow = P.q_d + ((size_t)r * P.H + (size_t)g * G + hrow) * D;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      if (hrow < G) {
        qb[kk][0] = __ldg(reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * q4));
        qb[kk][1] = __ldg(reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * q4 + 8));
      } else {
        qb[kk][0] = 0u;
        qb[kk][1] = 0u;
      }
    }
  }
  const size_t row_elems = (size_t)Hk * D;
  const uint16_t* kbase = P.paged ? P.k_pool : R.k;
  const uint16_t* vbase = P.paged ? P.v_pool : R.v;
  const uint32_t wsm_a = smem_u32(wsm);
#if POD_L2_HINTS
  const uint64_t once = l2_evict_first();  // decode K/V is read once
#endif
  const int col = lane % CH, rsub = lane / CH;  // this lane's piece and row phase

  // Stage t: keys kbeg + KPS t .. +KPS-1, in 16-key blocks (a ragged tail
  // re-reads the last valid row; those keys are masked below). Split lengths
  // are multiples of KPS, so a block never crosses a 16-token page: one
  // block-table entry per block.
  auto issue = [&](int t) {
    const uint32_t st = (ring + t) % NST;
#if POD_L2_HINTS
#define POD_DEC_COPY(d, s) cp_async16_hint(d, s, once)
#else
#define POD_DEC_COPY(d, s) cp_async16(d, s)
#endif
#pragma unroll
    for (int bk = 0; bk < NB; ++bk) {
      // a block wholly past the end re-reads the last valid row as well
      const int key0 = min(kbeg + t * KPS + bk * kDecTile, kend - 1) & ~(kDecTile - 1);
      size_t base_off;
      if (P.paged) {
        int phys = __ldg(P.bt_d + (size_t)R.bt_row * P.bt_stride_d + (key0 >> 4));
        phys = min(max(phys, 0), P.pool_blocks - 1);  // never read outside the pool
        base_off = (size_t)phys * kDecTile * row_elems + (size_t)g * D;
      } else {
        base_off = (size_t)key0 * row_elems + (size_t)g * D;
      }
      const int last = kend - 1 - key0;  // last valid key of the block (>= 0)
      // this lane's piece of key rows rsub, rsub + RPI, ... of K (then V)
      const uint32_t dk = wsm_a + st * STAGE + (bk * kDecTile + rsub) * ROW + col * 16;
      const uint16_t* sk = kbase + base_off + col * 8;
      const uint16_t* sv = vbase + base_off + col * 8;
      if (last >= kDecTile - 1) {  // a full block: rows advance by RPI rows of the cache
        const size_t step = (size_t)RPI * row_elems;
        sk += (size_t)rsub * row_elems;
        sv += (size_t)rsub * row_elems;
#pragma unroll
        for (int i = 0; i < kDecTile / RPI; ++i, sk += step, sv += step) {
          POD_DEC_COPY(dk + i * RPI * ROW, sk);
          POD_DEC_COPY(dk + (KPS + i * RPI) * ROW, sv);
        }
      } else {  // the ragged tail re-reads the last valid row (masked in the softmax)
#pragma unroll
        for (int i = 0; i < kDecTile / RPI; ++i) {
          const size_t k = (size_t)min(i * RPI + rsub, last) * row_elems;
          POD_DEC_COPY(dk + i * RPI * ROW, sk + k);
          POD_DEC_COPY(dk + (KPS + i * RPI) * ROW, sv + k);
        }
      }
    }
#undef POD_DEC_COPY
    cp_async_commit();
  };

  int issued = min(NST, n_tiles);  // tiles [0, issued) have been issued
  for (int t = 0; t < issued; ++t) issue(t);

  float o[KS][4];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sc = P.scale_log2;
  bool ok = true;

  for (int t = 0; t < n_tiles; ++t) {
    const uint32_t st = (ring + t) % NST;
    // stage t landed: the groups issued after it may still be in flight
    cp_async_wait_pending(issued - 1 - t);
    __syncwarp();  // every lane's pieces visible to the whole warp
    if (__any_sync(0xffffffffu, *abort_flag != 0)) {
      ok = false;
      break;
    }
    const uint32_t kb0 = wsm_a + st * STAGE;
    const uint32_t vb0 = kb0 + KPS * ROW;
    // S^T[16 keys x 8 heads] per block; the G query heads of the KV group
    // are the mma N dimension. Lane: keys hrow and hrow + 8 of each block,
    // heads 2 q4 and 2 q4 + 1.
    float sv[NB][4];
#pragma unroll
    for (int bk = 0; bk < NB; ++bk) {
      const uint32_t kb = kb0 + bk * kDecTile * ROW;
      // two independent accumulator chains halve the dependent mma latency
      float c[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < KS; kk += 2) {
        uint32_t a[4], a2[4];
        ldsm_x4(kb + (lane & 15) * ROW + (kk * 16 + 8 * (lane >> 4)) * 2, a);
        ldsm_x4(kb + (lane & 15) * ROW + ((kk + 1) * 16 + 8 * (lane >> 4)) * 2, a2);
        mma_16816(c, a, qb[kk][0], qb[kk][1]);
        mma_16816(c2, a2, qb[kk + 1][0], qb[kk + 1][1]);
      }
      const int key_a = kbeg + t * KPS + bk * kDecTile + hrow;
      sv[bk][0] = (key_a < kend) ? (c[0] + c2[0]) * sc : -INFINITY;
      sv[bk][1] = (key_a < kend) ? (c[1] + c2[1]) * sc : -INFINITY;
      sv[bk][2] = (key_a + 8 < kend) ? (c[2] + c2[2]) * sc : -INFINITY;
      sv[bk][3] = (key_a + 8 < kend) ? (c[3] + c2[3]) * sc : -INFINITY;
    }
    float mx0 = fmaxf(sv[0][0], sv[0][2]), mx1 = fmaxf(sv[0][1], sv[0][3]);
#pragma unroll
    for (int bk = 1; bk < NB; ++bk) {
      mx0 = max3(mx0, sv[bk][0], sv[bk][2]);
      mx1 = max3(mx1, sv[bk][1], sv[bk][3]);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    // Lazy rescaling (as in the prefill tile): a head's reference max moves
    // only when the stage max exceeds it by more than 8 (log2 units), so every
    // weight is <= 2^8 and O and l are rescaled only then. Every stage has a
    // valid key, so the first stage always sets the reference (alpha = 0).
    const bool up0 = mx0 > m0 + 8.f, up1 = mx1 > m1 + 8.f;
    if (__any_sync(0xffffffffu, up0 || up1)) {
      float a0 = 1.f, a1 = 1.f;
      if (up0) {
        a0 = ex2(m0 - mx0);
        m0 = mx0;
      }
      if (up1) {
        a1 = ex2(m1 - mx1);
        m1 = mx1;
      }
      l0 *= a0;
      l1 *= a1;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        o[mt][0] *= a0;
        o[mt][1] *= a1;
        o[mt][2] *= a0;
        o[mt][3] *= a1;
      }
    }
#pragma unroll
    for (int bk = 0; bk < NB; ++bk) {
      const float p0 = ex2(sv[bk][0] - m0), p1 = ex2(sv[bk][1] - m1);
      const float p2 = ex2(sv[bk][2] - m0), p3 = ex2(sv[bk][3] - m1);
      // The normaliser sums the unrounded fp32 weights: summing the
      // bf16-rounded ones would put their rounding (2^-9 relative) straight
      // into the LSE.
      l0 += p0 + p2;
      l1 += p1 + p3;
      // P^T as the B operand: transpose each 8x8 (key x head) block.
      const uint32_t b0 = movmatrix_t(pack_bf16(p0, p1));  // key hrow
      const uint32_t b1 = movmatrix_t(pack_bf16(p2, p3));  // key hrow + 8
      const uint32_t vb = vb0 + bk * kDecTile * ROW;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        uint32_t a[4];
        ldsm_x4_t(vb + ((lane & 7) + 8 * (lane >> 4)) * ROW + (mt * 16 + 8 * ((lane >> 3) & 1)) * 2,
                  a);
        mma_16816(o[mt], a, b0, b1);
      }
    }
    __syncwarp();  // every lane's reads of this stage are done before its refill
    if (t + NST < n_tiles) {
      issue(t + NST);
      issued = t + NST + 1;
    }
  }
  // All copies landed (on an abort too, so none lands after the CTA exits).
  // The ring may next hold a prefill tile written by TMA: order this warp's
  // generic-proxy accesses before any later async-proxy write.
  cp_async_wait_pending(0);
  fence_proxy_async_smem();
  ring += n_tiles;
  if (!ok) return false;

  // l: sum of lane partials over the 8 lanes sharing q4.
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  const int h0 = 2 * q4, h1 = 2 * q4 + 1;  // heads of c0/c2 and c1/c3
  if (R.n_split <= 1) {
    const float i0 = 1.f / l0, i1 = 1.f / l1;
    uint16_t* ob = P.o_d + ((size_t)r * P.H + (size_t)g * G) * D;
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      const int d0 = mt * 16 + hrow;
      if (h0 < G) {
        ob[(size_t)h0 * D + d0] = (uint16_t)(pack_bf16(o[mt][0] * i0, 0.f) & 0xFFFF);
        ob[(size_t)h0 * D + d0 + 8] = (uint16_t)(pack_bf16(o[mt][2] * i0, 0.f) & 0xFFFF);
      }
      if (h1 < G) {
        ob[(size_t)h1 * D + d0] = (uint16_t)(pack_bf16(o[mt][1] * i1, 0.f) & 0xFFFF);
        ob[(size_t)h1 * D + d0 + 8] = (uint16_t)(pack_bf16(o[mt][3] * i1, 0.f) & 0xFFFF);
      }
    }
    if (hrow == 0) {
      float* lb = P.lse_d + (size_t)r * P.H + (size_t)g * G;
      if (h0 < G) lb[h0] = (m0 + log2f(l0)) * kLn2;
      if (h1 < G) lb[h1] = (m1 + log2f(l1)) * kLn2;
    }
    return true;
  }
  // split: fp32 partial (normalised) + partial LSE
  const int slot = R.slot0 + s * Hk + g;
  float* po = P.dpart_o + (size_t)slot * kMaxGroup * D;
  {
    const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      const int d0 = mt * 16 + hrow;
      if (h0 < G) {
        po[h0 * D + d0] = o[mt][0] * i0;
        po[h0 * D + d0 + 8] = o[mt][2] * i0;
      }
      if (h1 < G) {
        po[h1 * D + d0] = o[mt][1] * i1;
        po[h1 * D + d0 + 8] = o[mt][3] * i1;
      }
    }
    if (hrow == 0) {
      float* pl = P.dpart_lse + (size_t)slot * kMaxGroup;
      if (h0 < G) pl[h0] = (m0 + log2f(l0)) * kLn2;
      if (h1 < G) pl[h1] = (m1 + log2f(l1)) * kLn2;
    }
  }
  if (!inline_merge) return true;
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = (atomicAdd(P.dgroup_ctr + R.group0 + g, 1) == R.n_split - 1);
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return true;
  __threadfence();
  merge_decode_group<D>(P, R, r, g, lane);
  return true;
}

// ============================================================= prefill unit
#include "pod_prefill.cuh"

// ============================================================= fused kernel
// Roles: PREFILL = 1, DECODE = 2. allow_prefill / allow_decode restrict the
// queues (prefill-only launch = allow_decode 0).
template <int D>
__global__ void __launch_bounds__(kFusedThreads, kFusedSlotsPerSm)
    pod_fused_kernel(const __grid_constant__ Plan P, const __grid_constant__ TmaDescs T,
                     int allow_prefill, int allow_decode) {
  using L = FusedLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  const int tid = threadIdx.x;
  if (smem_u32(sm) & 1023u) {  // 128-byte swizzle atoms need 1024-byte alignment
    if (tid == 0) set_status(P, kStatusUnsupported);
    return;
  }
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t bars = smem_u32(sm) + L::BAR_OFF;
  int* misc = reinterpret_cast<int*>(sm + L::MISC_OFF);
  // misc[0] tmem addr, [1] role, [2] unit, [3] abort flag, [5] prefill queue
  // empty, [6] decode queue empty, [7..8] merge flags of the two query tiles
  volatile int* abort_flag = misc + 3;

  if (tid == 0) {
    for (int i = 0; i < L::N_BARS; ++i) {
      uint32_t cnt = 1;
      if (i == L::B_PF || i == L::B_PF + 1)  // one arrival per softmax warp of the tile
        cnt = POD_SOFTMAX_SPLIT ? kSoftmaxWarps : kSoftmaxWarps / 2;
      if (POD_SHARED_S && i == L::B_SE)  // one arrival per warp that loads a part of S
        cnt = POD_SOFTMAX_SPLIT ? kSoftmaxWarps : kSoftmaxWarps / 2;
      mbar_init(bars + i * 8, cnt);
    }
    fence_mbar_init();
    misc[3] = 0;
    misc[5] = allow_prefill ? 0 : 1;
    misc[6] = allow_decode ? 0 : 1;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(misc), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);

  // Test hook: one thread waits on a flag nothing sets, with a short budget,
  // then records the timeout and carries on.
  if ((P.flags & 0x2) && blockIdx.x == 0 && tid == 0) {
    const long long t0 = clock64();
    while (*reinterpret_cast<volatile const int*>(P.never_set) == 0) {
      if (clock64() - t0 > 2000000LL) {
        set_status(P, kStatusTimeout);
        break;
      }
    }
  }

  const uint32_t my_sm = smid() & (kMaxSmid - 1);
  PipeState ps = {0u, 0u, 0u, 0u, 0u};
  uint32_t dec_ring = 0;
  uint32_t last_commit_bar = 0, last_commit_par = 0;
  bool issued_mma = false;

  // The role warps (softmax, MMA issuer, producer) loop over claims and sync
  // among themselves on named barrier 1; the side warps stream decode units
  // from the same queue for the CTA's whole life, so an SM keeps reading
  // decode K/V while its tensor cores run a prefill unit.
  auto role_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kRoleWarps * 32) : "memory"); };
  if (warp < kRoleWarps) {
    while (true) {
      if (tid == 0) {
        int role = 0, unit = -1;
        if (!*abort_flag) {
          // per-SM ticket (SM-aware), or one global counter when that is switched off
          const int t = atomicAdd(P.sm_ticket + ((P.flags & kFlagGlobalTicket) ? 0 : my_sm), 1);
          const long long num = P.rho_num, den = P.rho_den > 0 ? P.rho_den : 1;
          bool want_p = ((long long)(t + 1) * num) / den > ((long long)t * num) / den;
          // front-loaded: each SM's first ticket (one per resident CTA) takes
          // prefill work, so the long prefill units start first
          if ((P.flags & kFlagFrontPolicy) && t < kFusedSlotsPerSm) want_p = true;
          // balanced: a fixed set of CTAs (one per SM) serves prefill first and
          // the rest serve decode first, sized so both finish together
          if (P.flags & kFlagBalancedPolicy) want_p = (int)blockIdx.x < P.p_cap;
          for (int attempt = 0; attempt < 2 && role == 0; ++attempt, want_p = !want_p) {
            if (want_p && !misc[5]) {
              const int u = atomicAdd(P.ctl + 0, 1);
              if (u < P.n_prefill_units) {
                role = 1;
                unit = u;
              } else {
                misc[5] = 1;
              }
            } else if (!want_p && !misc[6]) {
              role = 2;  // a decode turn: the warps claim their own units
              unit = 0;
            }
          }
          if (role && (P.flags & 0x1)) atomicAdd(P.stats + my_sm * 2 + (role - 1), 1);
        }
        misc[1] = role;
        misc[2] = unit;
      }
      role_sync();
      const int role = misc[1];
      const int unit = misc[2];
      if (role == 0) break;
      if (role == 1) {
        const PrefillRange pr = prefill_range(P, unit);
        if (warp < kSoftmaxWarps) {
#if POD_SOFTMAX_SPLIT
          prefill_softmax_split<D>(P, pr, sm, tmem, ps, tid, abort_flag, misc + 7);
#else
          prefill_softmax<D>(P, pr, sm, tmem, ps, tid, abort_flag, misc + 7);
#endif
        } else if (warp == kSoftmaxWarps) {
          if (lane == 0) {
            issued_mma = true;
            prefill_mma<D>(P, pr, sm, tmem, ps, last_commit_bar, last_commit_par, abort_flag);
          }
          __syncwarp();
        } else if (warp == kSoftmaxWarps + 1) {
          if (lane == 0) prefill_producer<D>(P, T, pr, sm, ps, abort_flag);
          __syncwarp();
        }
        // warps past the producer have no prefill role; they run decode turns
      } else {
        // decode turn: every warp is a virtual decode unit runner and claims up
        // to dec_turn units one at a time; once every prefill unit has been
        // claimed there is nothing to regroup for, so the warp keeps claiming
        // until the decode queue is empty. An empty queue ends the turn.
        for (int k = 0;; ++k) {
          // balanced: a decode-first CTA stays on decode until the queue is
          // empty (regrouping after every unit would idle its warps at the
          // role barrier while the slowest unit finishes)
          if (k >= P.dec_turn && !(P.flags & kFlagBalancedPolicy) &&
              *reinterpret_cast<volatile const int*>(P.ctl + 0) < P.n_prefill_units)
            break;
          int u = 0;
          if (lane == 0) u = atomicAdd(P.ctl + 1, 1);
          u = __shfl_sync(0xffffffffu, u, 0);
          if (u >= P.n_decode_units) {
            if (lane == 0) misc[6] = 1;
            break;
          }
          if (!decode_unit_warp<D, kFusedDecStages>(P, u, sm + warp * L::DEC_WARP, dec_ring, lane,
                                                    true, abort_flag))
            break;
        }
      }
      // The loop ends only through the role thread 0 posts (0 once the CTA
      // has aborted): the abort flag can change at any moment (side warps, the
      // peer CTA), so testing it here could split the warps at bar.sync 1.
      role_sync();
    }
  } else if (allow_decode) {
    const int sw = warp - kRoleWarps;
    uint32_t side_ring = 0;
    while (!*abort_flag) {
      int u = 0;
      if (lane == 0) u = atomicAdd(P.ctl + 1, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u >= P.n_decode_units) {
        if (lane == 0) misc[6] = 1;
        break;
      }
      if (!decode_unit_warp<D, kFusedDecStages>(P, u, sm + L::SIDE_OFF + sw * L::DEC_WARP,
                                                side_ring, lane, true, abort_flag))
        break;
    }
  }
  // Teardown. After an abort, wait (bounded) for this CTA's own async work.
  if (*abort_flag) {
    if (warp == kSoftmaxWarps + 1 && lane == 0) prefill_producer_drain<D>(P, sm, ps);
    if (warp == kSoftmaxWarps && lane == 0 && issued_mma && last_commit_bar)
      drain_bar(last_commit_bar, last_commit_par, P.wait_budget);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ============================================================= CTA-pair fused kernel
#include "pod_prefill2.cuh"

// One persistent cluster of two 12-warp CTAs per SM pair. The leader CTA's
// thread 0 takes the tickets (from its SM's counter) and claims prefill units
// for the pair; it posts each decision to the peer through a mailbox in the
// peer's shared memory (a remote store plus a remote barrier arrival) and
// waits for the peer's acknowledgement before posting the next one. A prefill
// unit runs on both CTAs (pair_*); a decode turn runs on each CTA's role warps
// independently. Warps 10-11 of both CTAs stream decode units throughout.
template <int D>
__global__ void __launch_bounds__(kFusedThreads, 1)
    pod_fused_pair_kernel(const __grid_constant__ Plan P, const __grid_constant__ TmaDescs T,
                          int allow_prefill, int allow_decode) {
  using L = PairLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  const int tid = threadIdx.x;
  // Both CTAs of the pair have the same layout, so both take this branch or
  // neither does.
  if (smem_u32(sm) & 1023u) {  // 128-byte swizzle atoms need 1024-byte alignment
    if (tid == 0) set_status(P, kStatusUnsupported);
    return;
  }
  const int warp = tid >> 5, lane = tid & 31;
  const int rank = (int)cluster_ctarank();
  const uint32_t bars = smem_u32(sm) + L::BAR_OFF;
  int* misc = reinterpret_cast<int*>(sm + L::MISC_OFF);
  const uint32_t peer = (uint32_t)(rank ^ 1);
  const PairAbort pa{reinterpret_cast<volatile int*>(misc + kMiscAbort),
                     mapa_shared(smem_u32(misc + kMiscAbort), peer)};
  volatile int* abort_flag = pa.flag;

  if (tid == 0) {
    for (int i = 0; i < L::N_BARS; ++i) {
      uint32_t cnt = 1;
      if (i == L::B_SE || i == L::B_SE + 1 || i == L::B_PF || i == L::B_PF + 1)
        cnt = 2 * kTileOwners;  // the tile's owner warps in both CTAs
      mbar_init(bars + i * 8, cnt);
    }
    fence_mbar_init();
    for (int i = 0; i < 16; ++i) misc[i] = 0;
    misc[kMiscPEmpty] = allow_prefill ? 0 : 1;
    misc[kMiscDEmpty] = allow_decode ? 0 : 1;
  }
  // barrier initialisation visible to the peer before any remote arrival
  cluster_sync_all();
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(misc + kMiscTmem), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[kMiscTmem]);

  // Test hook: one thread waits on a flag nothing sets, with a short budget,
  // then records the timeout and carries on.
  if ((P.flags & 0x2) && blockIdx.x == 0 && tid == 0) {
    const long long t0 = clock64();
    while (*reinterpret_cast<volatile const int*>(P.never_set) == 0) {
      if (clock64() - t0 > 2000000LL) {
        set_status(P, kStatusTimeout);
        break;
      }
    }
  }

  const uint32_t my_sm = smid() & (kMaxSmid - 1);
  PairPipe ps = {0u, 0u, 0u, 0u, 0u};
  uint32_t dec_ring = 0;
  uint32_t last_commit_bar = 0, last_commit_par = 0;
  bool issued_mma = false;
  const uint32_t peer_misc = mapa_shared(smem_u32(misc), peer);
  const uint32_t peer_bars = mapa_shared(bars, peer);

  auto role_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kRoleWarps * 32) : "memory"); };
  if (warp < kRoleWarps) {
    uint32_t posts = 0;  // mailbox posts sent (leader) or read (peer)
    while (true) {
      if (tid == 0) {
        int role = 0, unit = -1;
        if (rank == 0) {
          if (!*abort_flag) {
            const int t = atomicAdd(P.sm_ticket + ((P.flags & kFlagGlobalTicket) ? 0 : my_sm), 1);
            const long long num = P.rho_num, den = P.rho_den > 0 ? P.rho_den : 1;
            bool want_p = ((long long)(t + 1) * num) / den > ((long long)t * num) / den;
            if ((P.flags & kFlagFrontPolicy) && t < kFusedSlotsPerSm) want_p = true;
            if (P.flags & kFlagBalancedPolicy) want_p = (int)(blockIdx.x >> 1) < P.p_cap;
            for (int attempt = 0; attempt < 2 && role == 0; ++attempt, want_p = !want_p) {
              if (want_p && !misc[kMiscPEmpty]) {
                const int u = atomicAdd(P.ctl + 0, 1);
                if (u < P.n_prefill_units) {
                  role = 1;
                  unit = u;
                } else {
                  misc[kMiscPEmpty] = 1;
                }
              } else if (!want_p && !misc[kMiscDEmpty]) {
                role = 2;
                unit = 0;
              }
            }
            if (role && (P.flags & 0x1)) atomicAdd(P.stats + my_sm * 2 + (role - 1), 1);
          }
          // the peer must have read the previous post before it is overwritten
          if (posts > 0 && !pwait_c(bars + L::B_ACK * 8, (posts - 1) & 1, P, pa)) role = 0;
          st_cluster_u32(peer_misc + 4 * kMiscPending, 1u);
          st_cluster_u32(peer_misc + 4 * kMiscMbRole, (uint32_t)role);
          st_cluster_u32(peer_misc + 4 * kMiscMbUnit, (uint32_t)unit);
          mbar_arrive_cluster(peer_bars + L::B_MB * 8);
        } else {
          if (pwait_c(bars + L::B_MB * 8, posts & 1, P, pa)) {
            role = *reinterpret_cast<volatile int*>(misc + kMiscMbRole);
            unit = *reinterpret_cast<volatile int*>(misc + kMiscMbUnit);
            *reinterpret_cast<volatile int*>(misc + kMiscPending) = 0;
            mbar_arrive_cluster(mapa_shared(bars + L::B_ACK * 8, 0));
          }
        }
        ++posts;
        misc[kMiscRole] = role;
        misc[kMiscUnit] = unit;
      }
      role_sync();
      const int role = misc[kMiscRole];
      const int unit = misc[kMiscUnit];
      if (role == 0) break;
      if (role == 1) {
        const PrefillRange pr = prefill_range(P, unit);
        if (warp < kSoftmaxWarps) {
          pair_softmax<D>(P, pr, rank, sm, tmem, ps, tid, pa, misc + kMiscMerge);
        } else if (warp == kSoftmaxWarps) {
          if (lane == 0 && rank == 0) {
            issued_mma = true;
            pair_mma<D>(P, pr, sm, tmem, ps, last_commit_bar, last_commit_par, pa);
          }
          __syncwarp();
        } else if (warp == kSoftmaxWarps + 1) {
          if (lane == 0) pair_producer<D>(P, T, pr, rank, sm, ps, pa);
          __syncwarp();
        }
      } else if (warp < L::TURN_WARPS) {
        // decode turn: each turn warp claims up to dec_turn units; once every
        // prefill unit has been claimed it keeps claiming until the decode
        // queue is empty. The peer also ends its turn when the leader has
        // posted a new decision (the pair is wanted for a prefill unit).
        for (int k = 0;; ++k) {
          if (k >= P.dec_turn && !(P.flags & kFlagBalancedPolicy) &&
              *reinterpret_cast<volatile const int*>(P.ctl + 0) < P.n_prefill_units)
            break;
          if (rank == 1 && *reinterpret_cast<volatile int*>(misc + kMiscPending)) break;
          int u = 0;
          if (lane == 0) u = atomicAdd(P.ctl + 1, 1);
          u = __shfl_sync(0xffffffffu, u, 0);
          if (u >= P.n_decode_units) {
            if (lane == 0) misc[kMiscDEmpty] = 1;
            break;
          }
          if (!decode_unit_warp<D, L::ROLE_DEC_ST>(P, u, sm + warp * L::ROLE_DEC_WARP, dec_ring,
                                                  lane, true, abort_flag))
            break;
        }
      }
      // The loop ends only through the role thread 0 posts (0 once the CTA
      // has aborted): the abort flag can change at any moment (side warps, the
      // peer CTA), so testing it here could split the warps at bar.sync 1.
      role_sync();
    }
  } else if (allow_decode) {
    const int sw = warp - kRoleWarps;
    uint32_t side_ring = 0;
    while (!*abort_flag) {
      int u = 0;
      if (lane == 0) u = atomicAdd(P.ctl + 1, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u >= P.n_decode_units) {
        if (lane == 0) misc[kMiscDEmpty] = 1;
        break;
      }
      if (!decode_unit_warp<D, L::SIDE_DEC_ST>(P, u, sm + L::SIDE_OFF + sw * L::SIDE_DEC_WARP,
                                               side_ring, lane, true, abort_flag))
        break;
    }
  }
  // Teardown. After an abort, wait (bounded) for this CTA's own async work:
  // the MMAs the leader issued, and the loads the producers issued (a peer's
  // loads complete on the leader's barriers, so the peer gives them a short
  // grace period).
  if (*abort_flag) {
    if (warp == kSoftmaxWarps && lane == 0 && issued_mma && last_commit_bar)
      drain_bar(last_commit_bar, last_commit_par, P.wait_budget);
    if (warp == kSoftmaxWarps + 1 && lane == 0) {
      if (rank == 0) {
        if (ps.q > 0) drain_bar(bars + L::B_QF * 8, (ps.q - 1) & 1, P.wait_budget);
        for (uint32_t k = 0; k < (uint32_t)L::KS && k < ps.kissued; ++k) {
          const uint32_t it = ps.kissued - 1 - k;
          drain_bar(bars + (L::B_KF + it % L::KS) * 8, (it / L::KS) & 1, P.wait_budget);
        }
        for (uint32_t k = 0; k < (uint32_t)L::VS && k < ps.vissued; ++k) {
          const uint32_t it = ps.vissued - 1 - k;
          drain_bar(bars + (L::B_VF + it % L::VS) * 8, (it / L::VS) & 1, P.wait_budget);
        }
      } else {
        const long long t0 = clock64();
        while (clock64() - t0 < 4000000LL) {
        }
      }
    }
  }
  tc_fence_before();
  // neither CTA leaves (or frees TMEM) while the other may still touch its
  // shared memory or the pair's tensor memory
  cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ============================================================= decode-only kernels
// Persistent: every warp is a virtual decode unit runner that claims the next
// unit from the decode queue until it is empty.
template <int D>
__global__ void __launch_bounds__(kDecodeWarps * 32)
    pod_decode_kernel(const __grid_constant__ Plan P) {
  using L = DecodeLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::FLAG_OFF) + warp;
  if (lane == 0) *abort_flag = 0;
  __syncwarp();
  uint32_t ring = 0;
  while (true) {
    int u = 0;
    if (lane == 0) u = atomicAdd(P.ctl + 1, 1);
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u >= P.n_decode_units) break;
    if (!decode_unit_warp<D, kDecodeStages>(P, u, sm + warp * L::WARP, ring, lane, false,
                                            abort_flag))
      break;
  }
}

// One warp per decode query row (request r, query head h) whose KV range was
// split: its KV head's partials are merged for that row alone, so the launch
// has H x requests warps in flight instead of Hk x requests. The per-row
// arithmetic is that of the fused kernel's last-arriver merge (which merges
// all G rows of a group in one warp), so both give the same bits.
// With kFlagPoisonOnStatus set, a non-zero status word (a decode warp gave up
// on a bounded wait) makes every row write NaN instead, so a call whose
// partial results are incomplete cannot be mistaken for a result.
template <int D>
__global__ void __launch_bounds__(128) pod_merge_kernel(const __grid_constant__ Plan P) {
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= P.n_decode_reqs * P.H) return;
  const int r = gw / P.H, h = gw - r * P.H;
  const int g = h / P.G, i = h - g * P.G;
  if ((P.flags & kFlagPoisonOnStatus) && *reinterpret_cast<volatile const int*>(P.status) != 0) {
    uint16_t* o = P.o_d + ((size_t)r * P.H + h) * D;
    for (int k = lane; k < D; k += 32) o[k] = 0x7FC0u;  // bf16 quiet NaN
    if (lane == 0) P.lse_d[(size_t)r * P.H + h] = __int_as_float(0x7FC00000);
    return;
  }
  const DecodeReq R = P.dreq[r];
  if (R.n_split <= 1) return;
  const int slot0 = R.slot0 + g;
  merge_rows_warp<D, 1>(P.dpart_o + (size_t)slot0 * kMaxGroup * D, (long long)P.Hk * kMaxGroup * D,
                        D, P.dpart_lse + (size_t)slot0 * kMaxGroup, (long long)P.Hk * kMaxGroup, 1,
                        R.n_split, i, P.G, P.o_d + ((size_t)r * P.H + (size_t)g * P.G) * D, D,
                        P.lse_d + (size_t)r * P.H + (size_t)g * P.G, 1, lane);
}

// ============================================================= host-side launchers
template <int D>
static cudaError_t set_attrs() {
  cudaError_t e = cudaFuncSetAttribute(pod_fused_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FusedLayout<D>::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(pod_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              DecodeLayout<D>::SMEM_BYTES);
}

cudaError_t kernels_init(int D) {
  if (D == 128) {
    cudaError_t e = set_attrs<128>();
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(pod_fused_pair_kernel<128>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                PairLayout<128>::SMEM_BYTES);
  }
  return set_attrs<64>();
}

static cudaLaunchConfig_t pair_config(int grid, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kFusedThreads, 1, 1);
  cfg.dynamicSmemBytes = PairLayout<128>::SMEM_BYTES;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Clusters of two pair CTAs that fit on the device at once (0: none).
cudaError_t pair_max_clusters(int* clusters) {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_config(2, nullptr, attr);
  return cudaOccupancyMaxActiveClusters(clusters, pod_fused_pair_kernel<128>, &cfg);
}

// grid = 2 x clusters (head_dim 128 only).
cudaError_t launch_fused_pair(const Plan& P, const TmaDescs& T, int grid, int allow_prefill,
                              int allow_decode, cudaStream_t s) {
  if (P.D != 128 || grid < 2 || (grid & 1)) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_config(grid, s, attr);
  return cudaLaunchKernelEx(&cfg, pod_fused_pair_kernel<128>, P, T, allow_prefill, allow_decode);
}

int fused_smem_bytes(int D) {
  return D == 128 ? FusedLayout<128>::SMEM_BYTES : FusedLayout<64>::SMEM_BYTES;
}
int decode_smem_bytes(int D) {
  return D == 128 ? DecodeLayout<128>::SMEM_BYTES : DecodeLayout<64>::SMEM_BYTES;
}

cudaError_t launch_fused(const Plan& P, const TmaDescs& T, int grid, int allow_prefill,
                         int allow_decode, cudaStream_t s) {
  if (P.D == 128)
    pod_fused_kernel<128><<<grid, kFusedThreads, FusedLayout<128>::SMEM_BYTES, s>>>(
        P, T, allow_prefill, allow_decode);
  else
    pod_fused_kernel<64><<<grid, kFusedThreads, FusedLayout<64>::SMEM_BYTES, s>>>(
        P, T, allow_prefill, allow_decode);
  return cudaGetLastError();
}

cudaError_t decode_occupancy(int D, int* blocks_per_sm) {
  if (D == 128)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pod_decode_kernel<128>,
                                                         kDecodeWarps * 32,
                                                         DecodeLayout<128>::SMEM_BYTES);
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pod_decode_kernel<64>,
                                                       kDecodeWarps * 32,
                                                       DecodeLayout<64>::SMEM_BYTES);
}

cudaError_t launch_decode(const Plan& P, int max_grid, cudaStream_t s) {
  const int need = (P.n_decode_units + kDecodeWarps - 1) / kDecodeWarps;
  const int grid = need < max_grid ? need : max_grid;
  if (grid == 0) return cudaSuccess;
  if (P.D == 128)
    pod_decode_kernel<128><<<grid, kDecodeWarps * 32, DecodeLayout<128>::SMEM_BYTES, s>>>(P);
  else
    pod_decode_kernel<64><<<grid, kDecodeWarps * 32, DecodeLayout<64>::SMEM_BYTES, s>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_merge(const Plan& P, cudaStream_t s) {
  const int rows = P.n_decode_reqs * P.H;  // one warp per query row, four per block
  const int grid = (rows + 3) / 4;
  if (grid == 0) return cudaSuccess;
  if (P.D == 128)
    pod_merge_kernel<128><<<grid, 128, 0, s>>>(P);
  else
    pod_merge_kernel<64><<<grid, 128, 0, s>>>(P);
  return cudaGetLastError();
}

}  // namespace pod
