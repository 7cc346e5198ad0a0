// pod_prefill2.cuh -- the prefill unit on a CTA pair (two SMs), sm_100a.
//
// A prefill unit is two 128-row query tiles that read the same K/V (two heads
// of one KV-head group at one token tile, or two consecutive token tiles of
// one head when the group size is odd). Here the two tiles run on the two
// CTAs of a cluster, one tile per SM, as ONE M = 256 tensor-core tile: the
// leader CTA issues tcgen05.mma.cta_group::2, each CTA holds its own query
// tile and HALF of every K and V tile (K: 64 of the 128 keys; V: 64 of the
// head_dim columns), so each SM moves half of every K/V tile through its
// shared memory and the pair reads K/V from L2 once per 256 query rows.
//
// TMEM of each CTA (512 columns, allocated for the pair):
//   O  [0, 128)    output accumulator of this CTA's 128 rows
//   P0 [128, 192)  P of even KV tiles (bf16 pairs), the A operand of P V
//   P1 [192, 256)  P of odd KV tiles
//   S0 [256, 384)  S of even KV tiles
//   S1 [384, 512)  S of odd KV tiles
// With S and P double-buffered and apart from each other, S of KV tile j + 2
// is issued as soon as the softmax of tile j has read S_j, so the tensor pipe
// computes S_{j+2} and P_j V_j while the softmax works on tile j + 1: the
// per-tile chain softmax -> P V -> next S of a one-SM tile whose P overwrites
// its S is gone.
//
// Warps of each CTA (12):
//   0-7   softmax: warp w serves TMEM lanes 32 (w % 4) .. +31 (its rows) on
//         the KV tiles t with t % 2 == w / 4, all 128 keys of each; the lazily
//         raised reference max passes from the owner of tile t to the owner of
//         tile t + 1 through shared memory. Each warp rescales all of O when
//         its rows' reference moves, and writes O columns 64 (w / 4) .. +63 in
//         the epilogue
//   8     leader CTA: one thread issues the pair MMAs; peer CTA: idle
//   9     TMA producer: this CTA's query tile, K halves, V halves
//   10-11 stream decode units for the CTA's whole life
// This is the FlashAttention-style tile of the POD-Attention summary (§1,
// §A.1) rebuilt for Blackwell's two-SM tensor-core tiles; the pair plays the
// role of the paper's larger prefill tile (§4.2.2).
#pragma once
// Included by pod_kernels.cu inside namespace pod, after the one-SM prefill.

template <int D>
struct PairLayout {
  static_assert(D == 128, "the CTA-pair prefill tile is built for head_dim 128");
  static constexpr int QB = kQTile * D * 2;              // this CTA's query tile (32 KB)
  static constexpr int KH = (kKVTile / 2) * D * 2;       // K half: 64 keys x d (16 KB)
  static constexpr int VH = kKVTile * (D / 2) * 2;       // V half: 128 keys x d/2 (16 KB)
  static constexpr int KS = 3;                           // K ring depth
  static constexpr int VS = 3;                           // V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + QB;
  static constexpr int V_OFF = K_OFF + KS * KH;
  static constexpr int PREFILL_END = V_OFF + VS * VH;
  static constexpr int DEC_ROW = D * 2 + 16;             // padded row: conflict-free ldmatrix
  static constexpr int DEC_STAGE = 2 * kDecTile * DEC_ROW;
  // Decode turns run on the 8 softmax warps (the MMA and producer warps sit
  // them out); their 2-stage rings overlay the prefill rings. The side
  // warps' deeper rings lie beyond both, so every SM keeps 80 KB of decode
  // K/V loads in flight beside a prefill unit.
  static constexpr int TURN_WARPS = kSoftmaxWarps;
  static constexpr int ROLE_DEC_ST = 2;                  // ring depth of a decode-turn warp
  static constexpr int SIDE_DEC_ST = 5;                  // ring depth of a side decode warp
  static constexpr int ROLE_DEC_WARP = ROLE_DEC_ST * DEC_STAGE;
  static constexpr int SIDE_DEC_WARP = SIDE_DEC_ST * DEC_STAGE;
  static constexpr int DEC_END = TURN_WARPS * ROLE_DEC_WARP;  // decode turns overlay prefill
  static constexpr int SIDE_OFF = PREFILL_END > DEC_END ? PREFILL_END : DEC_END;
  static constexpr int XCH_OFF = SIDE_OFF + kSideDecWarps * SIDE_DEC_WARP;
  // the handed-on reference max [2][128], then the final references and
  // row-sum shares [2][128] + [2][128]
  static constexpr int XCH_BYTES = 6 * kQTile * 4;
  static constexpr int BAR_OFF = (XCH_OFF + XCH_BYTES + 127) & ~127;
  // barrier indices
  static constexpr int B_QF = 0;                  // both query tiles landed (leader)
  static constexpr int B_QE = 1;                  // query tiles read by the unit's last S
  static constexpr int B_KF = 2;                  // K tile (both halves) landed (leader) [KS]
  static constexpr int B_KE = B_KF + KS;          // K stage read by its S MMA [KS]
  static constexpr int B_VF = B_KE + KS;          // V tile landed (leader) [VS]
  static constexpr int B_VE = B_VF + VS;          // V stage read by its P V MMA [VS]
  static constexpr int B_SF = B_VE + VS;          // S_b in TMEM [2]
  static constexpr int B_SE = B_SF + 2;           // S_b read by its 8 owner warps (leader) [2]
  static constexpr int B_PF = B_SE + 2;           // P_b written by its 8 owner warps (leader) [2]
  static constexpr int B_PE = B_PF + 2;           // P_b V done: P_b free, O current [2]
  static constexpr int B_OR = B_PE + 2;           // O final for the unit
  static constexpr int B_MB = B_OR + 1;           // peer: the leader posted a claim
  static constexpr int B_ACK = B_MB + 1;          // leader: the peer read the claim
  static constexpr int N_BARS = B_ACK + 1;
  static constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
  static constexpr int TOTAL = MISC_OFF + 64;
  static_assert(TOTAL <= 227 * 1024, "pair CTA exceeds the shared memory of an SM");
  static_assert(TOTAL > 116 * 1024, "a pair CTA must own its SM (it holds all TMEM)");
  static constexpr int SMEM_BYTES = TOTAL;
  // TMEM columns
  static constexpr uint32_t T_O = 0, T_P = 128, T_S = 256;
};

// Pairs (of every 8) of the pair softmax's exponentials evaluated by
// exp2_poly2 on the FMA pipe instead of ex2 on MUFU, on tiles without masked
// keys. Per SM and KV tile the MMAs take 1024 tensor-core cycles and the
// 16384 exponentials 1024 MUFU cycles (16 per clock per SM), so moving a
// share off MUFU keeps it from setting the pace.
#ifndef POD_PAIR_POLY_PAIRS
#define POD_PAIR_POLY_PAIRS 0
#endif
constexpr int kPairPolyPairs = POD_PAIR_POLY_PAIRS;

// The softmax warps' hand-offs to the leader's MMA thread (S read, P
// written) are tensor-memory hand-offs ordered by tcgen05 fences around the
// barrier: by default a plain remote arrival and wait, as for shared-memory
// stages; POD_PAIR_ACQREL_CLUSTER=1 makes them cluster-scope release /
// acquire (measured slower, kept for comparison).
#ifndef POD_PAIR_ACQREL_CLUSTER
#define POD_PAIR_ACQREL_CLUSTER 0
#endif

// How the pair softmax rounds P to bf16 pairs: 0 cvt.rn.bf16x2 (the XU pipe,
// which the exponentials also use), 1 round half away from zero with integer
// adds (P >= 0; differs from nearest-even only on exact ties), 2 nearest even
// with integer ops.
#ifndef POD_PAIR_PACK
#define POD_PAIR_PACK 1
#endif
POD_DEV uint32_t pair_pack(float lo, float hi) {
#if POD_PAIR_PACK == 0
  return pack_bf16(lo, hi);
#elif POD_PAIR_PACK == 1
  return pack_bf16_rha(lo, hi);
#else
  return pack_bf16_int(lo, hi);
#endif
}

// K tiles the pair producer issues ahead of V tiles (0: K_j, V_j, K_j+1, ...).
#ifndef POD_PAIR_K_LEAD
#define POD_PAIR_K_LEAD 2
#endif
constexpr int kKLead = POD_PAIR_K_LEAD;
static_assert(kKLead >= 0 && kKLead < 3, "the lead must leave a K stage for the next tile");

// Named barriers of the pair kernel: 1 the role warps; per lane quarter q,
// kBarHandoff0 + 2 q + h carries the reference max from the owner of tiles of
// parity h to the other warp (one-way: arrive, then sync), kBarFinal0 + q the
// two warps' final exchange; kBarSoftmaxAll all eight softmax warps.
constexpr int kBarHandoff0 = 2;    // 2 .. 9
constexpr int kBarFinal0 = 10;     // 10 .. 13
constexpr int kBarSoftmaxAll = 14;
// softmax warps that read each S tile and write each P tile (per CTA)
constexpr int kTileOwners = kSoftmaxWarps / 2;

// misc[] words of the pair kernel
constexpr int kMiscTmem = 0, kMiscRole = 1, kMiscUnit = 2, kMiscAbort = 3, kMiscPEmpty = 5,
              kMiscDEmpty = 6, kMiscPending = 7, kMiscMerge = 8, kMiscMbRole = 10,
              kMiscMbUnit = 11;

// Abort state of a CTA of the pair: its own flag, and the peer's flag (a
// cluster address) so that a wait that runs out stops both CTAs.
struct PairAbort {
  volatile int* flag;
  uint32_t peer_flag;
};

POD_DEV void pair_raise_abort(const Plan& P, const PairAbort& pa) {
  set_status(P, kStatusTimeout);
  *pa.flag = 1;
  st_cluster_u32(pa.peer_flag, 1u);
}

// Bounded wait for a TMA / MMA-commit barrier of this CTA: one try inline,
// the spinning slow path out of line (it keeps the hot loops' registers free).
__device__ __noinline__ bool pwait_slow(uint32_t bar, uint32_t parity, const Plan& P,
                                        volatile int* flag, uint32_t peer_flag) {
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*flag) return false;
    if (clock64() - t0 > P.wait_budget) {
      pair_raise_abort(P, PairAbort{flag, peer_flag});
      return false;
    }
  }
}
POD_DEV bool pwait(uint32_t bar, uint32_t parity, const Plan& P, const PairAbort& pa) {
  if (mbar_try_wait(bar, parity)) return true;
  return pwait_slow(bar, parity, P, pa.flag, pa.peer_flag);
}
// Bounded wait for a barrier that threads of the other CTA arrive on
// (cluster-scope acquire).
POD_DEV bool pwait_c(uint32_t bar, uint32_t parity, const Plan& P, const PairAbort& pa) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*pa.flag) return false;
    if (clock64() - t0 > P.wait_budget) {
      pair_raise_abort(P, pa);
      return false;
    }
  }
}
// The MMA thread's wait for the softmax warps' hand-offs.
POD_DEV bool pwait_handoff(uint32_t bar, uint32_t parity, const Plan& P, const PairAbort& pa) {
#if POD_PAIR_ACQREL_CLUSTER
  return pwait_c(bar, parity, P, pa);
#else
  return pwait(bar, parity, P, pa);
#endif
}
POD_DEV void handoff_arrive(uint32_t cluster_addr) {
#if POD_PAIR_ACQREL_CLUSTER
  mbar_arrive_cluster(cluster_addr);
#else
  mbar_arrive_remote(cluster_addr);
#endif
}
POD_DEV bool pwait_warp(uint32_t bar, uint32_t parity, const Plan& P, const PairAbort& pa) {
  const bool ok = pwait(bar, parity, P, pa);
  return __all_sync(0xffffffffu, ok);
}

// Per-CTA iteration counters; both CTAs of a pair run the same units, so the
// counters (and with them every barrier phase) agree between them.
struct PairPipe {
  uint32_t kv;       // KV tiles processed
  uint32_t q;        // query tiles loaded (units started)
  uint32_t units;    // units finished (O-ready phases)
  uint32_t kissued;  // producer: K tiles issued
  uint32_t vissued;  // producer: V tiles issued
};

// ---- TMA producer (one thread of each CTA): this CTA's query tile, its half
// of every K tile (keys 64 rank .. +63) and of every V tile (columns 64 rank ..
// +63). Completion is counted on the leader's barriers, which expect both
// halves.
template <int D>
POD_DEV bool pair_producer(const Plan& P, const TmaDescs& T, const PrefillRange& pr, int rank,
                           uint8_t* sm, PairPipe& ps, const PairAbort& pa) {
  using L = PairLayout<D>;
  const uint32_t base = smem_u32(sm);
  const uint32_t bars = base + L::BAR_OFF;
  const uint32_t lbars = mapa_shared(bars, 0);
  const PrefillReq R = P.preq[pr.req];
  const int g = pr.head[0] / P.G;
  constexpr int NB = D / 64;  // 64-column swizzle blocks of Q and K
  // query tile, once the previous unit's last S has read the old one
  if (ps.q > 0 && !pwait(bars + L::B_QE * 8, (ps.q - 1) & 1, P, pa)) return false;
  if (rank == 0) mbar_expect_tx(bars + L::B_QF * 8, 2 * L::QB);
  for (int b = 0; b < NB; ++b)
    tma_load_3d_pair(base + L::Q_OFF + b * (kQTile * 128), &T.q, lbars + L::B_QF * 8, 64 * b,
                     pr.head[rank], R.q_row0 + pr.qtile[rank] * kQTile);
  ps.q++;
  const CUtensorMap* km = P.paged ? &T.k[0] : &T.k[pr.req];
  const CUtensorMap* vm = P.paged ? &T.v[0] : &T.v[pr.req];
  const int last_page = (R.kv_len - 1) >> 4;
#if POD_L2_HINTS
  const uint64_t keep = l2_evict_last();  // K/V tiles are re-read by other query tiles
#define POD_PAIR_LOAD(d, m, f, x, y, z) tma_load_3d_pair_hint(d, m, f, x, y, z, keep)
#else
#define POD_PAIR_LOAD(d, m, f, x, y, z) tma_load_3d_pair(d, m, f, x, y, z)
#endif
  // K tiles are issued kKLead tiles ahead of V tiles: the MMA order needs
  // K_{j+2} (for S_{j+2}) before V_j (for P_j V_j), and a V stage is freed
  // only by a P V, which waits for the softmax.
  for (int t = 0; t < pr.n + kKLead; ++t) {
    const int j = t;  // K tile of this step
    if (j < pr.n) {  // K half: keys key0 + 64 rank .. +63, every column (two 64-column blocks)
      const uint32_t it = ps.kv + j;
      const int key0 = (pr.t0 + j) * kKVTile;
      const uint32_t st = it % L::KS, ph = (it / L::KS) & 1;
      if (it >= (uint32_t)L::KS && !pwait(bars + (L::B_KE + st) * 8, ph ^ 1, P, pa)) return false;
      const uint32_t full = lbars + (L::B_KF + st) * 8;
      if (rank == 0) mbar_expect_tx(bars + (L::B_KF + st) * 8, 2 * L::KH);
      const uint32_t dst = base + L::K_OFF + st * L::KH;
      const int k0 = key0 + 64 * rank;
      if (!P.paged) {
        for (int b = 0; b < NB; ++b) POD_PAIR_LOAD(dst + b * (64 * 128), km, full, 64 * b, g, k0);
      } else {
        for (int pg = 0; pg < 4; ++pg) {
          const int lp = min((k0 >> 4) + pg, last_page);
          const int phys = __ldg(P.bt_p + (size_t)R.bt_row * P.bt_stride_p + lp);
          for (int b = 0; b < NB; ++b)
            POD_PAIR_LOAD(dst + b * (64 * 128) + pg * 16 * 128, km, full, 64 * b, g, phys * 16);
        }
      }
      ps.kissued = it + 1;
    }
    if (t - kKLead >= 0) {  // V half: keys key0 .. +127, columns 64 rank .. +63 (one block)
      const int jv = t - kKLead;
      const uint32_t it = ps.kv + jv;
      const int key0 = (pr.t0 + jv) * kKVTile;
      const uint32_t st = it % L::VS, ph = (it / L::VS) & 1;
      if (it >= (uint32_t)L::VS && !pwait(bars + (L::B_VE + st) * 8, ph ^ 1, P, pa)) return false;
      const uint32_t full = lbars + (L::B_VF + st) * 8;
      if (rank == 0) mbar_expect_tx(bars + (L::B_VF + st) * 8, 2 * L::VH);
      const uint32_t dst = base + L::V_OFF + st * L::VH;
      if (!P.paged) {
        POD_PAIR_LOAD(dst, vm, full, 64 * rank, g, key0);
      } else {
        for (int pg = 0; pg < kKVTile / 16; ++pg) {
          const int lp = min((key0 >> 4) + pg, last_page);
          const int phys = __ldg(P.bt_p + (size_t)R.bt_row * P.bt_stride_p + lp);
          POD_PAIR_LOAD(dst + pg * 16 * 128, vm, full, 64 * rank, g, phys * 16);
        }
      }
      ps.vissued = it + 1;
    }
  }
  ps.kv += pr.n;
  return true;
#undef POD_PAIR_LOAD
}

// ---- MMA issuer (one thread of the leader CTA). Order per unit:
// S0 S1 | S2 PV0 | S3 PV1 | ... | PV(n-1): S_{j+2} goes in as soon as the
// softmax has read S_j, P_j V_j as soon as P_j is written.
template <int D>
POD_DEV bool pair_mma(const Plan& P, const PrefillRange& pr, uint8_t* sm, uint32_t tmem,
                      PairPipe& ps, uint32_t& last_commit_bar, uint32_t& last_commit_par,
                      const PairAbort& pa) {
  using L = PairLayout<D>;
  constexpr int KSTEPS = D / 16;
  constexpr uint32_t IDESC_S = umma_idesc_bf16(2 * kQTile, kKVTile, 0, 0);
  constexpr uint32_t IDESC_PV = umma_idesc_bf16(2 * kQTile, D, 0, 1);
  constexpr uint16_t kBoth = 3;  // commits arrive on both CTAs' barriers
  const uint32_t base = smem_u32(sm);
  const uint32_t bars = base + L::BAR_OFF;
  if (!pwait(bars + L::B_QF * 8, ps.q & 1, P, pa)) return false;
  ps.q++;
  tc_fence_after();
  const uint64_t dq = sw128_desc(base + L::Q_OFF, 16, 1024);
  const uint64_t dk0 = sw128_desc(base + L::K_OFF, 16, 1024);
  const uint64_t dv0 = sw128_desc(base + L::V_OFF, L::VH, 1024);
  const int n = pr.n;

  // S_b = Q K_j^T: A = this CTA's and the peer's query tiles (K-major), B =
  // the two K halves (64 keys each, K-major); D = 128 rows x 128 keys per CTA.
  auto issue_s = [&](int j) -> bool {
    const uint32_t it = ps.kv + j, b = it & 1;
    const uint32_t st = it % L::KS, ph = (it / L::KS) & 1;
    if (!pwait(bars + (L::B_KF + st) * 8, ph, P, pa)) return false;
    // S_b last held S_{it-2}: every softmax warp of both CTAs has read it
    if (it >= 2 && !pwait_handoff(bars + (L::B_SE + b) * 8, ((it - 2) >> 1) & 1, P, pa))
      return false;
    tc_fence_after();
    const uint64_t kd = dk0 + (uint64_t)(st * (L::KH >> 4));
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const uint64_t ad = dq + (uint64_t)(((kk >> 2) * (kQTile * 128) + (kk & 3) * 32) >> 4);
      const uint64_t bd = kd + (uint64_t)(((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4);
      umma_ss_pair(tmem + L::T_S + 128 * b, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
    }
    umma_commit_pair(bars + (L::B_SF + b) * 8, kBoth);
    umma_commit_pair(bars + (L::B_KE + st) * 8, kBoth);
    if (j == n - 1) umma_commit_pair(bars + L::B_QE * 8, kBoth);
    last_commit_bar = bars + (L::B_SF + b) * 8;
    last_commit_par = (it >> 1) & 1;
    return true;
  };
  // O += P_b V_j: A = P_b from each CTA's TMEM, B = the two V halves (64
  // columns each, MN-major); D = 128 rows x d per CTA.
  auto issue_pv = [&](int j) -> bool {
    const uint32_t it = ps.kv + j, b = it & 1;
    const uint32_t st = it % L::VS, ph = (it / L::VS) & 1;
    if (!pwait(bars + (L::B_VF + st) * 8, ph, P, pa)) return false;
    if (!pwait_handoff(bars + (L::B_PF + b) * 8, (it >> 1) & 1, P, pa)) return false;
    tc_fence_after();
    const uint64_t vd = dv0 + (uint64_t)(st * (L::VH >> 4));
    const uint32_t pcol = tmem + L::T_P + 64 * b;
#pragma unroll
    for (int kk = 0; kk < kKVTile / 16; ++kk) {
      const uint64_t bd = vd + (uint64_t)((kk * 16 * 128) >> 4);
      umma_ts_pair(tmem + L::T_O, pcol + kk * 8, bd, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
    }
    umma_commit_pair(bars + (L::B_PE + b) * 8, kBoth);
    umma_commit_pair(bars + (L::B_VE + st) * 8, kBoth);
    if (j == n - 1) umma_commit_pair(bars + L::B_OR * 8, kBoth);
    last_commit_bar = bars + (L::B_PE + b) * 8;
    last_commit_par = (it >> 1) & 1;
    return true;
  };

  if (!issue_s(0)) return false;
  if (n > 1 && !issue_s(1)) return false;
  for (int j = 0; j < n; ++j) {
    if (j + 2 < n && !issue_s(j + 2)) return false;
    if (!issue_pv(j)) return false;
  }
  ps.kv += n;
  return true;
}

// ---- softmax + epilogue (warps 0-7 of each CTA). Warp w serves the rows of
// its TMEM lane quarter, 32 (w % 4) .. +31, and the unit's KV tiles t with
// t % 2 == w / 4, all 128 keys of each: the two warps of a lane quarter share
// a sub-partition and work on consecutive tiles at the same time, so their
// exponentials interleave on its MUFU unit. The lazily raised reference max
// of the rows passes from the owner of tile t to the owner of tile t + 1
// through shared memory under a one-way named barrier (arrive, then sync),
// handed on before the exponentials. Every warp passes its named barriers the
// same number of times whatever happens (a failed wait only skips
// tensor-memory work), so a timeout can never leave a barrier short.
template <int D>
POD_DEV bool pair_softmax(const Plan& P, const PrefillRange& pr, int rank, uint8_t* sm,
                          uint32_t tmem, PairPipe& ps, int tid, const PairAbort& pa,
                          int* merge_flag) {
  using L = PairLayout<D>;
  const uint32_t bars = smem_u32(sm) + L::BAR_OFF;
  const uint32_t lbars = mapa_shared(bars, 0);
  const PrefillReq R = P.preq[pr.req];
  const int warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, hf = warp >> 2;  // lane quarter, tile parity
  const int row = q4 * 32 + lane;
  const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
  const int head = pr.head[rank], qtile = pr.qtile[rank];
  const bool tile_ok = (rank == 0) || pr.valid1;
  const int q_local = qtile * kQTile + row;        // token index within the chunk
  const int lim = R.prior + q_local;               // last visible key (inclusive)
  const int mask_from = R.prior + qtile * kQTile;  // KV tiles ending above this need masking
  const float sc = P.scale_log2;
  float* xref = reinterpret_cast<float*>(sm + L::XCH_OFF);  // [2 from][128] handed-on reference
  float* xfin = xref + 2 * kQTile;                          // [2][128] m, then [2][128] l
  const int hand_to = kBarHandoff0 + 2 * q4 + hf;           // this warp -> the other
  const int hand_from = kBarHandoff0 + 2 * q4 + (hf ^ 1);   // the other -> this warp
  const int n = pr.n;
  float m_ref = -INFINITY;  // reference max (log2 units) O and l_h are scaled to
  float l_h = 0.f;          // this warp's share of the row sum, relative to m_ref
  bool failed = false;      // warp-uniform

  for (int t = hf; t < n; t += 2) {
    const uint32_t it = ps.kv + t, b = it & 1;
    const int tile0 = (pr.t0 + t) * kKVTile;
    const bool masked_tile = tile0 + kKVTile - 1 > mask_from;  // uniform over the CTA
    // Straight-line body: once the CTA has aborted every wait returns at once
    // and the tensor-memory work below only moves stale values, whose results
    // are never stored (`failed`).
    failed |= !pwait_warp(bars + (L::B_SF + b) * 8, (it >> 1) & 1, P, pa);
    tc_fence_after();
    float s[128];
    {
      uint32_t r[128];
      tmem_ld128(tmem + lane_base + L::T_S + 128 * b, r);
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(r[c]);
    }
    // S_b may be overwritten once all its readers in both CTAs have it
    tc_fence_before();
    __syncwarp();
    if (lane == 0) handoff_arrive(lbars + (L::B_SE + b) * 8);
    if (masked_tile) {
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (tile0 + c > lim) s[c] = -INFINITY;
    }
    // row max: eight chains of three-input max (few live temporaries beside s)
    float mc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mc[k] = fmaxf(s[k], s[8 + k]);
#pragma unroll
    for (int c = 16; c < 128; c += 16)
#pragma unroll
      for (int k = 0; k < 8; ++k) mc[k] = max3(mc[k], s[c + k], s[c + 8 + k]);
    float mx = fmaxf(max3(mc[0], mc[1], mc[2]), max3(max3(mc[3], mc[4], mc[5]), mc[6], mc[7]));
    // the reference after tile t - 1, from its owner (none before the unit's first tile)
    if (t >= 1) {
      named_bar_sync(hand_from, 64);
      const float m_prev = xref[(hf ^ 1) * kQTile + row];
      if (m_prev > m_ref) {  // monotone: rescale this warp's share to the newer reference
        l_h = (m_ref == -INFINITY) ? 0.f : l_h * ex2(m_ref - m_prev);
        m_ref = m_prev;
      }
    }
    // Lazy rescaling: the reference is raised only when the row max exceeds it
    // by more than 8 (log2 units), so every weight is <= 2^8.
    mx *= sc;
    float alpha = 1.f;
    bool rescale = false;
    if (mx > m_ref + 8.f) {
      alpha = ex2(m_ref - mx);         // 0 when nothing was seen yet
      rescale = (m_ref != -INFINITY);  // O holds earlier tiles' sums
      l_h *= alpha;
      m_ref = mx;
    }
    // hand the reference on to the owner of tile t + 1 before the exponentials
    if (t + 1 < n) {
      xref[hf * kQTile + row] = m_ref;
      asm volatile("bar.arrive %0, 64;" ::"r"(hand_to) : "memory");
    }
    const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;  // fully masked row so far
    // P_b is free once P_{it-2} V has completed
    if (it >= 2) failed |= !pwait_warp(bars + (L::B_PE + b) * 8, ((it - 2) >> 1) & 1, P, pa);
    tc_fence_after();
    // P = 2^(s sc - m) as bf16 pairs over P_b, one 64-key half at a time (each
    // half stored as soon as it is packed), and the row sum of the unrounded
    // weights
    const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(-m_use, -m_use);
    uint64_t acc[4];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int k = 64 * hh + 2 * c;
        float x0, x1;
        f2_unpack(ffma2(f2_pack(s[k], s[k + 1]), sc2, nm2), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        const uint64_t p2 = f2_pack(p0, p1);
        pk[c] = pair_pack(p0, p1);
        acc[c & 3] = (hh == 0 && c < 4) ? p2 : fadd2(acc[c & 3], p2);
      }
      if (hh == 0)
        tmem_st32_nowait(tmem + lane_base + L::T_P + 64 * b, pk);
      else
        tmem_st32(tmem + lane_base + L::T_P + 64 * b + 32, pk);  // waits for both stores
    }
    {
      float a0, a1;
      f2_unpack(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), a0, a1);
      l_h += a0 + a1;
    }
    // O to the raised reference, after P_{it-1} V and before this tile's P V
    // (issued only after the P-ready arrival below); a rescale never happens
    // on a unit's first tile, so it - 1 belongs to this unit
    if (__any_sync(0xffffffffu, rescale)) {
      failed |= !pwait_warp(bars + (L::B_PE + ((it - 1) & 1)) * 8, ((it - 1) >> 1) & 1, P, pa);
      tc_fence_after();
      const float f = rescale ? alpha : 1.f;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t ov[32];
        const uint32_t oc = tmem + lane_base + L::T_O + 32 * cb;
        tmem_ld32(oc, ov);
#pragma unroll
        for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * f);
        tmem_st32(oc, ov);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) handoff_arrive(lbars + (L::B_PF + b) * 8);
  }
  // O complete
  if (!failed) {
    failed = !pwait_warp(bars + L::B_OR * 8, ps.units & 1, P, pa);
    if (!failed) tc_fence_after();
  }
  ps.kv += pr.n;
  ps.units++;
  // The two warps' references and row-sum shares meet: the larger reference
  // is the final one (references only grow), and each share is rescaled to it.
  xfin[hf * kQTile + row] = m_ref;
  xfin[(2 + hf) * kQTile + row] = l_h;
  named_bar_sync(kBarFinal0 + q4, 64);
  const float m_o = xfin[(hf ^ 1) * kQTile + row], l_o = xfin[(2 + (hf ^ 1)) * kQTile + row];
  const float m_run = fmaxf(m_ref, m_o);
  const float l_tot = (m_run == -INFINITY)
                          ? 0.f
                          : ((m_ref == -INFINITY) ? 0.f : l_h * ex2(m_ref - m_run)) +
                                ((m_o == -INFINITY) ? 0.f : l_o * ex2(m_o - m_run));
  const bool valid = tile_ok && (q_local < R.chunk) && !failed;
  const size_t out_row = (size_t)(R.q_row0 + q_local);
  const float lse2 = (l_tot > 0.f) ? (m_run + log2f(l_tot)) : -INFINITY;
  const uint32_t o_col = tmem + lane_base + L::T_O + 64 * hf;
  if (pr.n_split <= 1) {
    if (failed) return false;
    const float inv = 1.f / l_tot;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t ov[32];
      tmem_ld32(o_col + 32 * cb, ov);
      if (valid) {
        uint16_t* dst = P.o_p + (out_row * P.H + head) * D + 64 * hf + 32 * cb;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(ov[8 * q + 0]) * inv, __uint_as_float(ov[8 * q + 1]) * inv);
          v.y = pack_bf16(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv);
          v.z = pack_bf16(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv);
          v.w = pack_bf16(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + 8 * q) = v;
        }
      }
    }
    if (valid && hf == 0) P.lse_p[out_row * P.H + head] = lse2 * kLn2;
    return true;
  }
  // Split partial: O normalised by its own sum (fp32) and the natural-log LSE
  // of the KV range, stored [slot][d / 4][row] as float4 so a warp's accesses
  // are 512 contiguous bytes; the last split of the query tile merges.
  const int slot0 = pr.slot_base[rank];
  const float inv = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
  float4* part = reinterpret_cast<float4*>(P.ppart_o);
  {
    float4* po = part + ((size_t)(slot0 + pr.split) * (D / 4) + 16 * hf) * kQTile + row;
#pragma unroll
    for (int cb = 0; cb < 2 && !failed; ++cb) {
      uint32_t ov[32];
      tmem_ld32(o_col + 32 * cb, ov);
      if (valid) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          po[(size_t)(cb * 8 + q) * kQTile] =
              make_float4(__uint_as_float(ov[4 * q]) * inv, __uint_as_float(ov[4 * q + 1]) * inv,
                          __uint_as_float(ov[4 * q + 2]) * inv, __uint_as_float(ov[4 * q + 3]) * inv);
      }
    }
  }
  if (valid && hf == 0) P.ppart_lse[(size_t)(slot0 + pr.split) * kQTile + row] = lse2 * kLn2;
  __threadfence();
  named_bar_sync(kBarSoftmaxAll, kSoftmaxWarps * 32);
  if (tid == 0) {
    // a missing tile has no group; after a failure nobody merges
    const int old = (*pa.flag || !tile_ok) ? -1 : atomicAdd(P.pgroup_ctr + pr.group[rank], 1);
    *merge_flag = (old == pr.n_split - 1);
  }
  named_bar_sync(kBarSoftmaxAll, kSoftmaxWarps * 32);
  if (*merge_flag && !failed && valid) {
    // The last split to finish merges all of them in split order (each
    // thread: one row, its 64 columns): O = sum_s w_s O_s / sum_s w_s,
    // w_s = exp(LSE_s - max LSE).
    __threadfence();
    const int ns = pr.n_split;
    const float* pl = P.ppart_lse + (size_t)slot0 * kQTile + row;
    float m = -INFINITY;
    for (int sp = 0; sp < ns; ++sp) m = fmaxf(m, __ldcg(pl + (size_t)sp * kQTile));
    float wsum = 0.f;
    for (int sp = 0; sp < ns; ++sp) {
      const float v = __ldcg(pl + (size_t)sp * kQTile);
      wsum += (v == -INFINITY) ? 0.f : ex2((v - m) * kLog2e);
    }
    const float winv = 1.f / wsum;
    uint16_t* dst = P.o_p + (out_row * P.H + head) * D + 64 * hf;
    const float4* src = part + ((size_t)slot0 * (D / 4) + 16 * hf) * kQTile + row;
#pragma unroll 1
    for (int cb = 0; cb < 2; ++cb) {
      float acc2[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc2[c] = 0.f;
#pragma unroll 2
      for (int sp = 0; sp < ns; ++sp) {
        const float v = __ldcg(pl + (size_t)sp * kQTile);
        const float w = ((v == -INFINITY) ? 0.f : ex2((v - m) * kLog2e)) * winv;
        const float4* s4 = src + (size_t)sp * (D / 4) * kQTile + (size_t)(cb * 8) * kQTile;
        float4 x[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) x[q] = __ldcg(s4 + (size_t)q * kQTile);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          acc2[4 * q] = fmaf(w, x[q].x, acc2[4 * q]);
          acc2[4 * q + 1] = fmaf(w, x[q].y, acc2[4 * q + 1]);
          acc2[4 * q + 2] = fmaf(w, x[q].z, acc2[4 * q + 2]);
          acc2[4 * q + 3] = fmaf(w, x[q].w, acc2[4 * q + 3]);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16(acc2[8 * q + 0], acc2[8 * q + 1]);
        v.y = pack_bf16(acc2[8 * q + 2], acc2[8 * q + 3]);
        v.z = pack_bf16(acc2[8 * q + 4], acc2[8 * q + 5]);
        v.w = pack_bf16(acc2[8 * q + 6], acc2[8 * q + 7]);
        *reinterpret_cast<uint4*>(dst + cb * 32 + 8 * q) = v;
      }
    }
    if (hf == 0) P.lse_p[out_row * P.H + head] = m + logf(wsum);
  }
  return !failed;
}
