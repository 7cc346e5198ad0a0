// pod_prefill.cuh -- the prefill unit of the fused kernel (sm_100a).
//
// A unit is two 128-row query tiles that read the same K/V: two heads of one
// KV-head group at the same token tile (G even), or two consecutive token
// tiles of one head (G odd), against a range of 128-key KV tiles. One CTA per
// SM runs it with ten warps:
//   warp 9      TMA producer: Q0 and Q1 once per unit, then a K ring and a V
//               ring of two stages each (128-byte swizzle), K one tile ahead;
//   warp 8      one thread issuing tcgen05.mma: S_i = Q_i K^T into TMEM, and
//               O_i += P_i V with P_i read from TMEM as the A operand;
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1: one thread per
//               query row (= TMEM lane), 128 keys per KV tile.
// (Warps 10-11 of the CTA stream decode units meanwhile; see pod_kernels.cu.)
// TMEM (512 columns), default layout: O0 [0,128), O1 [128,256), one S buffer
// [256,384) that the two tiles take in turn, P0 [384,448), P1 [448,512) (bf16
// pairs). A softmax warp frees the S buffer as soon as it has loaded its row,
// so the next S is issued while it computes; MMA order S0 S1 | S0' PV0 |
// S1' PV1 | ... The softmax waits for the previous P_i V before it rewrites
// P_i (and rescales O_i).
// With POD_SHARED_S=0: S0 [256,384), S1 [384,512), P_i written over the first
// 64 columns of S_i, and S_i' waits for P_i V to complete (order S0 S1 | PV0
// S0' | PV1 S1').
// This is the FlashAttention-style tile of the POD-Attention summary (§1,
// §A.1) rebuilt for Blackwell; the pairing plays the role of the paper's
// larger prefill tile when fewer CTAs share an SM (§4.2.2).
#pragma once
// Included by pod_kernels.cu inside namespace pod, after the decode code.

struct PrefillRange {
  int req, split, n_split;
  int head[2], qtile[2];  // the unit's two query tiles
  int valid1;             // tile 1 exists (a token-tile pair may run past the chunk)
  int t0, n;              // first KV tile and number of KV tiles
  int group[2];           // merge group of each tile (split units)
  int slot_base[2];       // first partial slot of each tile (split units)
};

POD_DEV PrefillRange prefill_range(const Plan& P, int u) {
  const PrefillUnit U = P.punits[u];
  const PrefillReq R = P.preq[U.req];
  PrefillRange pr;
  pr.req = U.req;
  pr.split = U.split;
  pr.n_split = U.n_split;
  pr.group[0] = U.group0;
  pr.group[1] = U.group0 + 1;
  pr.slot_base[0] = U.slot0;
  pr.slot_base[1] = U.slot0 + U.n_split;
  if (R.pair_heads) {
    pr.head[0] = U.head;
    pr.head[1] = U.head + 1;
    pr.qtile[0] = pr.qtile[1] = U.qtile;
    pr.valid1 = 1;
  } else {
    pr.head[0] = pr.head[1] = U.head;
    pr.qtile[0] = U.qtile;
    pr.qtile[1] = U.qtile + 1;
    pr.valid1 = U.qtile + 1 < R.n_qtiles;
  }
  const int last_qt = pr.valid1 ? pr.qtile[1] : pr.qtile[0];
  const int kv_hi = R.prior + min(R.chunk, (last_qt + 1) * kQTile);
  const int n_all = (kv_hi + kKVTile - 1) / kKVTile;
  pr.t0 = (int)((long long)U.split * n_all / U.n_split);
  pr.n = (int)((long long)(U.split + 1) * n_all / U.n_split) - pr.t0;
  return pr;
}

// Per-CTA iteration counters that carry mbarrier phases across units.
struct PipeState {
  uint32_t kv;       // KV tiles processed
  uint32_t q;        // Q tile pairs loaded
  uint32_t units;    // prefill units finished (O-ready phases)
  uint32_t kissued;  // producer: K tiles issued (for the abort drain)
  uint32_t vissued;  // producer: V tiles issued
};

// ---- TMA producer (one thread).
template <int D>
POD_DEV bool prefill_producer(const Plan& P, const TmaDescs& T, const PrefillRange& pr,
                              uint8_t* sm, PipeState& ps, volatile int* abort_flag) {
  using L = FusedLayout<D>;
  const uint32_t base = smem_u32(sm);
  const uint32_t bars = base + L::BAR_OFF;
  const PrefillReq R = P.preq[pr.req];
  const int g = pr.head[0] / P.G;
  constexpr int NB = D / 64;  // 64-column swizzle blocks
  // Q tiles (a missing second tile is loaded anyway: its rows are never stored)
  mbar_expect_tx(bars + L::B_Q * 8, 2 * L::QB);
  for (int i = 0; i < 2; ++i)
    for (int b = 0; b < NB; ++b)
      tma_load_3d(base + L::Q_OFF + i * L::QB + b * (kQTile * 128), &T.q, bars + L::B_Q * 8,
                  64 * b, pr.head[i], R.q_row0 + pr.qtile[i] * kQTile);
  ps.q++;
  const CUtensorMap* km = P.paged ? &T.k[0] : &T.k[pr.req];
  const CUtensorMap* vm = P.paged ? &T.v[0] : &T.v[pr.req];
  const int last_page = (R.kv_len - 1) >> 4;

  // one 128-key K or V tile: per 64-column block, one 128-row box (contiguous
  // caches; rows past the cache are zero-filled) or eight 16-row pages (paged pool)
  auto load_tile = [&](const CUtensorMap* m, uint32_t dst, uint32_t full, int key0) {
    mbar_expect_tx(full, L::KT);
    if (!P.paged) {
      for (int b = 0; b < NB; ++b)
        tma_load_3d(dst + b * (kKVTile * 128), m, full, 64 * b, g, key0);
    } else {
      for (int pg = 0; pg < kKVTile / 16; ++pg) {
        const int lp = min((key0 >> 4) + pg, last_page);
        const int phys = __ldg(P.bt_p + (size_t)R.bt_row * P.bt_stride_p + lp);
        for (int b = 0; b < NB; ++b)
          tma_load_3d(dst + b * (kKVTile * 128) + pg * 16 * 128, m, full, 64 * b, g, phys * 16);
      }
    }
  };
  auto issue = [&](int j, bool is_k) -> bool {
    const uint32_t it = ps.kv + j;
    const uint32_t st = it % kPrefillStages;
    const uint32_t ph = (it / kPrefillStages) & 1;
    const int empty = is_k ? L::B_KE : L::B_VE;
    if (it >= kPrefillStages && !wait_bar(bars + (empty + st) * 8, ph ^ 1, P, abort_flag))
      return false;
    const uint32_t dst = base + (is_k ? L::K_OFF : L::V_OFF) + st * L::KT;
    load_tile(is_k ? km : vm, dst, bars + ((is_k ? L::B_KF : L::B_VF) + st) * 8,
              (pr.t0 + j) * kKVTile);
    return true;
  };
  bool ok = issue(0, true);
  if (ok) ps.kissued = ps.kv + 1;
  for (int j = 0; ok && j < pr.n; ++j) {
    if (j + 1 < pr.n) {
      ok = issue(j + 1, true);
      if (ok) ps.kissued = ps.kv + j + 2;
    }
    if (ok) {
      ok = issue(j, false);
      if (ok) ps.vissued = ps.kv + j + 1;
    }
  }
  ps.kv += pr.n;
  return ok;
}

template <int D>
POD_DEV void prefill_producer_drain(const Plan& P, uint8_t* sm, const PipeState& ps) {
  using L = FusedLayout<D>;
  const uint32_t bars = smem_u32(sm) + L::BAR_OFF;
  if (ps.q > 0) drain_bar(bars + L::B_Q * 8, (ps.q - 1) & 1, P.wait_budget);
  for (uint32_t k = 0; k < kPrefillStages && k < ps.kissued; ++k) {
    const uint32_t it = ps.kissued - 1 - k;
    drain_bar(bars + (L::B_KF + it % kPrefillStages) * 8, (it / kPrefillStages) & 1,
              P.wait_budget);
  }
  for (uint32_t k = 0; k < kPrefillStages && k < ps.vissued; ++k) {
    const uint32_t it = ps.vissued - 1 - k;
    drain_bar(bars + (L::B_VF + it % kPrefillStages) * 8, (it / kPrefillStages) & 1,
              P.wait_budget);
  }
}

// ---- MMA issuer (one thread). TMEM columns: O_i at 128 i; the shared S buffer
// at 256 and P_i at 384 + 64 i (with POD_SHARED_S=0: S_i and P_i at 256 + 128 i).
template <int D>
POD_DEV bool prefill_mma(const Plan& P, const PrefillRange& pr, uint8_t* sm, uint32_t tmem,
                         PipeState& ps, uint32_t& last_commit_bar, uint32_t& last_commit_par,
                         volatile int* abort_flag) {
  using L = FusedLayout<D>;
  constexpr int KS = D / 16;
  constexpr uint32_t IDESC_QK = umma_idesc_bf16(kQTile, kKVTile, 0, 0);
  constexpr uint32_t IDESC_PV = umma_idesc_bf16(kQTile, D, 0, 1);
  const uint32_t base = smem_u32(sm);
  const uint32_t bars = base + L::BAR_OFF;
  if (!wait_bar(bars + L::B_Q * 8, ps.q & 1, P, abort_flag)) return false;
  ps.q++;
  tc_fence_after();
  // Descriptors of the tile bases; a k step adds its byte offset / 16 to the
  // start-address field (shared-memory offsets stay below 256 KB, so the add
  // never carries out of the field).
  const uint64_t dq0 = sw128_desc(base + L::Q_OFF, 16, 1024);
  const uint64_t dq1 = sw128_desc(base + L::Q_OFF + L::QB, 16, 1024);
  const uint64_t dk0 = sw128_desc(base + L::K_OFF, 16, 1024);
  const uint64_t dv0 = sw128_desc(base + L::V_OFF, kKVTile * 128, 1024);
  constexpr uint64_t kStageStep = (uint64_t)(L::KT >> 4);

  // S_i = Q_i K_j^T (K-major A and B, 128-byte swizzle)
  auto issue_s = [&](int i, int j) -> bool {
    const uint32_t it = ps.kv + j;
    const uint32_t st = it % kPrefillStages, ph = (it / kPrefillStages) & 1;
    if (i == 0 && !wait_bar(bars + (L::B_KF + st) * 8, ph, P, abort_flag)) return false;
#if POD_SHARED_S
    // the S buffer's previous content (use m - 1) has been loaded by its softmax
    const uint32_t m = 2 * it + (uint32_t)i;
    if (m >= 1 && !wait_bar(bars + L::B_SE * 8, (m - 1) & 1, P, abort_flag)) return false;
    const uint32_t s_tm = tmem + 256;
#else
    // S_i still holds P_i of the previous tile until that PV has read it
    if (it >= 1 && !wait_bar(bars + (L::B_SE + i) * 8, (it - 1) & 1, P, abort_flag)) return false;
    const uint32_t s_tm = tmem + 256 + 128 * i;
#endif
    tc_fence_after();
    const uint64_t qd = i ? dq1 : dq0;
    const uint64_t kd = dk0 + st * kStageStep;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const uint64_t ad = qd + (uint64_t)(((kk >> 2) * (kQTile * 128) + (kk & 3) * 32) >> 4);
      const uint64_t bd = kd + (uint64_t)(((kk >> 2) * (kKVTile * 128) + (kk & 3) * 32) >> 4);
      umma_ss(s_tm, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
    }
    umma_commit(bars + (L::B_SF + i) * 8);
    if (i == 1) umma_commit(bars + (L::B_KE + st) * 8);  // both S have read K_j
    last_commit_bar = bars + (L::B_SF + i) * 8;
    last_commit_par = it & 1;
    return true;
  };
  // O_i += P_i V_j (P_i from TMEM, V MN-major in shared memory)
  auto issue_pv = [&](int i, int j) -> bool {
    const uint32_t it = ps.kv + j;
    const uint32_t st = it % kPrefillStages, ph = (it / kPrefillStages) & 1;
    if (i == 0 && !wait_bar(bars + (L::B_VF + st) * 8, ph, P, abort_flag)) return false;
    if (!wait_bar(bars + (L::B_PF + i) * 8, it & 1, P, abort_flag)) return false;
    tc_fence_after();
    const uint64_t vd = dv0 + st * kStageStep;
    const uint32_t pcol = tmem + (POD_SHARED_S ? 384 + 64 * i : 256 + 128 * i);
#pragma unroll
    for (int kk = 0; kk < kKVTile / 16; ++kk) {
      const uint64_t bd = vd + (uint64_t)((kk * 16 * 128) >> 4);
      umma_ts(tmem + 128 * i, pcol + kk * 8, bd, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
    }
    // P_i read (shared S: P_i may be rewritten; else S_i is free again)
    const uint32_t done_bar = bars + ((POD_SHARED_S ? L::B_PE : L::B_SE) + i) * 8;
    umma_commit(done_bar);
    if (j == pr.n - 1) umma_commit(bars + (L::B_OR + i) * 8);  // O_i final for this unit
    if (i == 1) umma_commit(bars + (L::B_VE + st) * 8);      // both PV have read V_j
    last_commit_bar = done_bar;
    last_commit_par = it & 1;
    return true;
  };

  if (!issue_s(0, 0) || !issue_s(1, 0)) return false;
  for (int j = 0; j < pr.n; ++j) {
#if POD_SHARED_S
    // S0' as soon as the buffer is free, while the softmax of tile 0 still works
    if (j + 1 < pr.n && !issue_s(0, j + 1)) return false;
    if (!issue_pv(0, j)) return false;
    if (j + 1 < pr.n && !issue_s(1, j + 1)) return false;
    if (!issue_pv(1, j)) return false;
#else
    if (!issue_pv(0, j)) return false;
    if (j + 1 < pr.n && !issue_s(0, j + 1)) return false;
    if (!issue_pv(1, j)) return false;
    if (j + 1 < pr.n && !issue_s(1, j + 1)) return false;
#endif
  }
  ps.kv += pr.n;
  return true;
}

// ---- softmax + epilogue, key-split form (POD_SOFTMAX_SPLIT): warps w and
// w + 4 share TMEM lane quarter w & 3 (query rows 32 (w & 3) .. +31) and split
// every 128-key S row: warp w takes keys 0..63, warp w + 4 keys 64..127. All
// eight warps serve tile 0 and then tile 1 of each KV step, so both warps of a
// scheduler partition feed its MUFU with the same tile instead of two tiles
// contending for it. The two halves of a row meet twice per tile:
//   - the half-row maxima, through a 16-byte shared-memory slot per row and a
//     named barrier of the 64 threads of the warp pair; both warps then hold
//     the same row max, reference max and rescale decision;
//   - at the end of the unit, the two partial row sums.
// Each warp writes the P columns of its own keys (P of keys 64 h .. +63 goes to
// P columns 32 h .. +31: P_i's own columns with the shared S buffer, else S_i's,
// where the pair barrier orders that store after the other warp's S load) and
// rescales and stores its half of O's columns.
template <int D>
POD_DEV bool prefill_softmax_split(const Plan& P, const PrefillRange& pr, uint8_t* sm,
                                   uint32_t tmem, PipeState& ps, int tid,
                                   volatile int* abort_flag, int* s_flag) {
  using L = FusedLayout<D>;
  constexpr int OB = D / 64;  // 32-column O blocks per warp (half of O's D columns)
  const uint32_t bars = smem_u32(sm) + L::BAR_OFF;
  const PrefillReq R = P.preq[pr.req];
  const int warp = tid >> 5, lane = tid & 31;
  const int qr = warp & 3, h = warp >> 2;
  const int row = qr * 32 + lane;
  const uint32_t lane_base = (uint32_t)(qr * 32) << 16;
  const int pair_bar = 4 + qr;  // named barrier of warps qr and qr + 4
  volatile float* xs = reinterpret_cast<volatile float*>(sm + L::XCH_OFF + row * L::XCH_STRIDE);
  int lim[2], mask_from[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    lim[i] = R.prior + pr.qtile[i] * kQTile + row;  // last visible key of this row
    mask_from[i] = R.prior + pr.qtile[i] * kQTile;
  }
  const float sc = P.scale_log2;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  bool failed = false;  // warp-uniform; after a failure only the barrier points are kept

  for (int j = 0; j < pr.n; ++j) {
    const uint32_t it = ps.kv + j;
    const int tile0 = (pr.t0 + j) * kKVTile;
    const int key_lo = tile0 + 64 * h;  // this warp's first key
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (!failed && !wait_bar_warp(bars + (L::B_SF + i) * 8, it & 1, P, abort_flag)) failed = true;
      const uint32_t s_col = tmem + lane_base + (POD_SHARED_S ? 256 : 256 + 128 * i);
      const uint32_t p_col = tmem + lane_base + (POD_SHARED_S ? 384 + 64 * i : 256 + 128 * i);
      float s[64];
      float mx = -INFINITY;
      if (!failed) {
        tc_fence_after();
        {
          uint32_t r0[32], r1[32];
          tmem_ld32x2(s_col + 64 * h, r0, r1);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            s[c] = __uint_as_float(r0[c]);
            s[32 + c] = __uint_as_float(r1[c]);
          }
        }
#if POD_SHARED_S
        // this warp's half of S is in registers; the buffer takes the next S
        // once all eight warps have loaded theirs
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + L::B_SE * 8);
#endif
        if (tile0 + kKVTile - 1 > mask_from[i]) {  // uniform over the warp pair
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (key_lo + c > lim[i]) s[c] = -INFINITY;
        }
        // 64 -> 22 -> 8 -> 3 -> 1 with three-input max
        float a[22];
#pragma unroll
        for (int c = 0; c < 21; ++c) a[c] = max3(s[3 * c], s[3 * c + 1], s[3 * c + 2]);
        a[21] = s[63];
        float b[8];
#pragma unroll
        for (int c = 0; c < 7; ++c) b[c] = max3(a[3 * c], a[3 * c + 1], a[3 * c + 2]);
        b[7] = a[21];
        mx = max3(max3(b[0], b[1], b[2]), max3(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
        mx *= sc;
      }
      xs[2 * i + h] = mx;
      asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
      mx = fmaxf(mx, xs[2 * i + (h ^ 1)]);
      if (!failed) {
        // Lazy rescaling, as in the one-warp-per-row form: both warps of the
        // pair compute the same reference from the same row max.
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m_run[i] + 8.f) {
          alpha = ex2(m_run[i] - mx);
          rescale = (m_run[i] != -INFINITY);
          m_run[i] = mx;
        }
        const float m_use = (m_run[i] == -INFINITY) ? 0.f : m_run[i];
        const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(-m_use, -m_use);
        uint64_t acc[4];
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float x0, x1;
          f2_unpack(ffma2(f2_pack(s[2 * c], s[2 * c + 1]), sc2, nm2), x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          pk[c] = POD_PACK(p0, p1);
          const uint64_t p2 = f2_pack(p0, p1);
          acc[c & 3] = (c < 4) ? p2 : fadd2(acc[c & 3], p2);
        }
#if POD_SHARED_S
        // P_i (and O_i, rescaled below) are still read by the previous P_i V
        if (it >= 1) {
          if (wait_bar_warp(bars + (L::B_PE + i) * 8, (it - 1) & 1, P, abort_flag))
            tc_fence_after();
          else
            failed = true;
        }
        if (!failed) tmem_st32(p_col + 32 * h, pk);
#else
        tmem_st32(p_col + 32 * h, pk);
#endif
        float a0, a1;
        f2_unpack(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), a0, a1);
        l_run[i] = l_run[i] * alpha + (a0 + a1);
        // O_i is stable here (S_i of this tile was issued after the previous
        // PV_i completed); each warp rescales its half of O's columns.
        if (!failed && __any_sync(0xffffffffu, rescale)) {
          const float f = rescale ? alpha : 1.f;
          const uint32_t o_col = tmem + lane_base + 128 * i + (D / 2) * h;
#pragma unroll
          for (int cb = 0; cb < OB; ++cb) {
            uint32_t ov[32];
            tmem_ld32(o_col + cb * 32, ov);
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * f);
            tmem_st32(o_col + cb * 32, ov);
          }
        }
      }
      // one arrival per warp, stores complete (tcgen05.wait::st) or none made
      tc_fence_before();
      __syncwarp();
      if (!failed && lane == 0) mbar_arrive(bars + (L::B_PF + i) * 8);
    }
  }
  // O_0 and O_1 complete
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (!failed) {
      if (wait_bar_warp(bars + (L::B_OR + i) * 8, ps.units & 1, P, abort_flag))
        tc_fence_after();
      else
        failed = true;
    }
  }
  ps.kv += pr.n;
  ps.units++;
  // The two halves' row sums. The first barrier keeps this write behind the
  // partner's last read of the max slots.
  asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
  xs[h] = l_run[0];
  xs[2 + h] = l_run[1];
  asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
  const float l_tot[2] = {l_run[0] + xs[h ^ 1], l_run[1] + xs[2 + (h ^ 1)]};

  if (pr.n_split <= 1) {
    if (failed) return false;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const bool tile_ok = (i == 0) || pr.valid1;
      const int q_local = pr.qtile[i] * kQTile + row;
      const bool valid = tile_ok && (q_local < R.chunk);
      const size_t out_row = (size_t)(R.q_row0 + q_local);
      const float inv = 1.f / l_tot[i];
      const uint32_t o_col = tmem + lane_base + 128 * i + (D / 2) * h;
#pragma unroll
      for (int cb = 0; cb < OB; ++cb) {
        uint32_t ov[32];
        tmem_ld32(o_col + cb * 32, ov);
        if (valid) {
          uint16_t* dst = P.o_p + (out_row * P.H + pr.head[i]) * D + (D / 2) * h + cb * 32;
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
      if (valid && h == 0) {
        const float lse2 = (l_tot[i] > 0.f) ? (m_run[i] + log2f(l_tot[i])) : -INFINITY;
        P.lse_p[out_row * P.H + pr.head[i]] = lse2 * kLn2;
      }
    }
    return true;
  }
  // Split partials of both tiles: O normalised by its own sum (fp32), stored
  // [slot][d / 4][row] in float4 units, and the natural-log LSE of the range.
  float4* part = reinterpret_cast<float4*>(P.ppart_o);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool tile_ok = (i == 0) || pr.valid1;
    const bool valid = tile_ok && (pr.qtile[i] * kQTile + row < R.chunk) && !failed;
    const int slot0 = pr.slot_base[i];
    const float inv = (l_tot[i] > 0.f) ? 1.f / l_tot[i] : 0.f;
    float4* po = part + (size_t)(slot0 + pr.split) * (D / 4) * kQTile + row;
    const uint32_t o_col = tmem + lane_base + 128 * i + (D / 2) * h;
#pragma unroll
    for (int cb = 0; cb < OB && !failed; ++cb) {
      uint32_t ov[32];
      tmem_ld32(o_col + cb * 32, ov);
      if (valid) {
        const int c4 = (D / 8) * h + cb * 8;  // first float4 column of this block
#pragma unroll
        for (int q = 0; q < 8; ++q)
          po[(size_t)(c4 + q) * kQTile] =
              make_float4(__uint_as_float(ov[4 * q]) * inv, __uint_as_float(ov[4 * q + 1]) * inv,
                          __uint_as_float(ov[4 * q + 2]) * inv, __uint_as_float(ov[4 * q + 3]) * inv);
      }
    }
    if (valid && h == 0) {
      const float lse2 = (l_tot[i] > 0.f) ? (m_run[i] + log2f(l_tot[i])) : -INFINITY;
      P.ppart_lse[(size_t)(slot0 + pr.split) * kQTile + row] = lse2 * kLn2;
    }
  }
  // Both tiles' partials are written by all eight warps: one barrier of the
  // eight, then one thread per tile counts the split in.
  __threadfence();
  asm volatile("bar.sync 2, %0;" ::"n"(kSoftmaxWarps * 32) : "memory");
  if ((tid & 127) == 0) {
    const int ti = tid >> 7;  // thread 0: tile 0, thread 128: tile 1
    const bool ok_t = (ti == 0) || pr.valid1;
    const int old = (*abort_flag || !ok_t) ? -1 : atomicAdd(P.pgroup_ctr + pr.group[ti], 1);
    s_flag[ti] = (old == pr.n_split - 1);
  }
  asm volatile("bar.sync 2, %0;" ::"n"(kSoftmaxWarps * 32) : "memory");
  // The last split to finish merges: warps 0-3 tile 0, warps 4-7 tile 1, one
  // query row per thread, in split order (the result does not depend on which
  // split finished last).
  const int im = h;
  const bool tile_ok_m = (im == 0) || pr.valid1;
  const int q_local_m = pr.qtile[im] * kQTile + row;
  if (s_flag[im] && !failed && tile_ok_m && q_local_m < R.chunk) {
    __threadfence();
    const size_t out_row = (size_t)(R.q_row0 + q_local_m);
    const int slot0 = pr.slot_base[im];
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
    uint16_t* dst = P.o_p + (out_row * P.H + pr.head[im]) * D;
    const float4* src = part + (size_t)slot0 * (D / 4) * kQTile + row;
#pragma unroll 1
    for (int cb = 0; cb < D / 32; ++cb) {
      float acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0.f;
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
          acc[4 * q] = fmaf(w, x[q].x, acc[4 * q]);
          acc[4 * q + 1] = fmaf(w, x[q].y, acc[4 * q + 1]);
          acc[4 * q + 2] = fmaf(w, x[q].z, acc[4 * q + 2]);
          acc[4 * q + 3] = fmaf(w, x[q].w, acc[4 * q + 3]);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16(acc[8 * q + 0], acc[8 * q + 1]);
        v.y = pack_bf16(acc[8 * q + 2], acc[8 * q + 3]);
        v.z = pack_bf16(acc[8 * q + 4], acc[8 * q + 5]);
        v.w = pack_bf16(acc[8 * q + 6], acc[8 * q + 7]);
        *reinterpret_cast<uint4*>(dst + cb * 32 + 8 * q) = v;
      }
    }
    P.lse_p[out_row * P.H + pr.head[im]] = m + logf(wsum);
  }
  return !failed;
}

// ---- softmax + epilogue: warps 0-3 serve query tile 0, warps 4-7 tile 1; one
// thread per query row (TMEM lane), 128 keys per S tile in two 64-column halves.
template <int D>
POD_DEV bool prefill_softmax(const Plan& P, const PrefillRange& pr, uint8_t* sm, uint32_t tmem,
                             PipeState& ps, int tid, volatile int* abort_flag, int* s_flag) {
  using L = FusedLayout<D>;
  const uint32_t bars = smem_u32(sm) + L::BAR_OFF;
  const PrefillReq R = P.preq[pr.req];
  const int warp = tid >> 5, lane = tid & 31;
  const int i = warp >> 2;  // which query tile of the unit
  const int row = (warp & 3) * 32 + lane;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t s_col = tmem + lane_base + (POD_SHARED_S ? 256 : 256 + 128 * i);
  const uint32_t p_col = tmem + lane_base + (POD_SHARED_S ? 384 + 64 * i : 256 + 128 * i);
  const uint32_t o_col = tmem + lane_base + 128 * i;
  const int head = pr.head[i], qtile = pr.qtile[i];
  const bool tile_ok = (i == 0) || pr.valid1;  // uniform over the warp group
  const int q_local = qtile * kQTile + row;    // token index within the chunk
  const int lim = R.prior + q_local;           // last visible key (inclusive)
  const int mask_from = R.prior + qtile * kQTile;  // KV tiles ending above this need masking
  const float sc = P.scale_log2;
  float m_run = -INFINITY, l_run = 0.f;
  bool failed = false;  // warp-uniform; after a failure only barrier points are kept

  for (int j = 0; j < pr.n; ++j) {
    const uint32_t it = ps.kv + j;
    if (!wait_bar_warp(bars + (L::B_SF + i) * 8, it & 1, P, abort_flag)) {
      failed = true;
      break;
    }
    tc_fence_after();
    const int tile0 = (pr.t0 + j) * kKVTile;
    const bool masked_tile = tile0 + kKVTile - 1 > mask_from;  // uniform over the group
    // The whole 128-key row of S in registers under one TMEM load wait.
    float s[128];
    {
      uint32_t r[128];
      tmem_ld128(s_col, r);
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(r[c]);
    }
#if POD_SHARED_S
    // S is in registers (the load waited): the buffer may take the next S
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + L::B_SE * 8);
#endif
    if (masked_tile) {
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (tile0 + c > lim) s[c] = -INFINITY;
    }
    float mx;
    {  // 128 -> 43 -> 15 -> 5 -> 1 with three-input max
      float a[43];
#pragma unroll
      for (int c = 0; c < 42; ++c) a[c] = max3(s[3 * c], s[3 * c + 1], s[3 * c + 2]);
      a[42] = fmaxf(s[126], s[127]);
      float b[15];
#pragma unroll
      for (int c = 0; c < 14; ++c) b[c] = max3(a[3 * c], a[3 * c + 1], a[3 * c + 2]);
      b[14] = a[42];
      mx = fmaxf(max3(max3(b[0], b[1], b[2]), max3(b[3], b[4], b[5]), max3(b[6], b[7], b[8])),
                 max3(max3(b[9], b[10], b[11]), b[12], fmaxf(b[13], b[14])));
    }
    mx *= sc;
    // Lazy rescaling: the reference m_run is raised only when the row max
    // exceeds it by more than 8 (log2 units), so every weight is <= 2^8.
    float alpha = 1.f;
    bool rescale = false;
    if (mx > m_run + 8.f) {
      alpha = ex2(m_run - mx);         // 0 on the unit's first tile
      rescale = (m_run != -INFINITY);  // O holds earlier tiles' sums
      m_run = mx;
    }
    const float m_use = (m_run == -INFINITY) ? 0.f : m_run;  // fully masked row so far
    // x = s sc - m and the row sums on packed pairs (f32x2)
    const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(-m_use, -m_use);
    uint64_t acc[4];
    // P (bf16 pairs) in 64 columns (over S_i's first 64, already read, or in
    // P_i's own columns with a shared S buffer); the PV MMA reads it as A.
    // Keys 64 hh .. +63 go to columns 32 hh .. +31.
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int k = 64 * hh + 2 * c;
        float x0, x1;
        f2_unpack(ffma2(f2_pack(s[k], s[k + 1]), sc2, nm2), x0, x1);
        const bool soft = !masked_tile && ((c & 7) >= 8 - kSoftPairs);
        uint64_t p2;
        float p0, p1;
        if (soft) {
          p2 = exp2_poly2(x0, x1);
          f2_unpack(p2, p0, p1);
        } else {
          p0 = ex2(x0);
          p1 = ex2(x1);
          p2 = f2_pack(p0, p1);
        }
        pk[c] = POD_PACK(p0, p1);
        // unrounded weights (see the decode path), four running pair sums
        acc[c & 3] = (hh == 0 && c < 4) ? p2 : fadd2(acc[c & 3], p2);
      }
#if POD_SHARED_S
      if (hh == 0 && it >= 1) {
        // P_i (and O_i, rescaled below) are still read by the previous P_i V
        if (!wait_bar_warp(bars + (L::B_PE + i) * 8, (it - 1) & 1, P, abort_flag)) {
          failed = true;
          break;
        }
        tc_fence_after();
      }
#endif
      if (hh == 0)
        tmem_st32_nowait(p_col, pk);
      else
        tmem_st32(p_col + 32, pk);  // waits for both stores
    }
    if (failed) break;
    float lt;
    {
      float a0, a1;
      f2_unpack(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), a0, a1);
      lt = a0 + a1;
    }
    l_run = l_run * alpha + lt;
    // O_i is stable here: the previous PV_i has completed (S_i of this tile was
    // issued only after it, or with a shared S buffer the wait before the P
    // store saw it). tcgen05.ld/st are warp-collective, so the whole warp
    // takes this branch if any row rescales; the others multiply by 1.
    if (__any_sync(0xffffffffu, rescale)) {
      const float f = rescale ? alpha : 1.f;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t ov[32];
        tmem_ld32(o_col + cb * 32, ov);
#pragma unroll
        for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * f);
        tmem_st32(o_col + cb * 32, ov);
      }
    }
    // every lane's stores are complete (tcgen05.wait::st); one arrival per warp
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + (L::B_PF + i) * 8);
  }
  // O_i complete
  if (!failed) {
    if (wait_bar_warp(bars + (L::B_OR + i) * 8, ps.units & 1, P, abort_flag))
      tc_fence_after();
    else
      failed = true;
  }
  ps.kv += pr.n;
  ps.units++;

  const bool valid = tile_ok && (q_local < R.chunk) && !failed;
  const size_t out_row = (size_t)(R.q_row0 + q_local);
  const float lse2 = (l_run > 0.f) ? (m_run + log2f(l_run)) : -INFINITY;
  const int bar_id = 2 + i;  // named barrier of this warp group (128 threads)
  if (pr.n_split <= 1) {
    if (failed) return false;
    const float inv = 1.f / l_run;
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb) {
      uint32_t ov[32];
      tmem_ld32(o_col + cb * 32, ov);
      if (valid) {
        uint16_t* dst = P.o_p + (out_row * P.H + head) * D + cb * 32;
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
    if (valid) P.lse_p[out_row * P.H + head] = lse2 * kLn2;
    return true;
  }
  // Split partial of this tile: O normalised by its own sum (fp32) and the
  // natural-log LSE of its KV range. O is stored [slot][d / 4][row] in float4
  // units, so the 32 rows of a warp touch 512 contiguous bytes per access.
  const int slot0 = pr.slot_base[i];
  const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
  float4* part = reinterpret_cast<float4*>(P.ppart_o);
  {
    float4* po = part + (size_t)(slot0 + pr.split) * (D / 4) * kQTile + row;
#pragma unroll
    for (int cb = 0; cb < D / 32 && !failed; ++cb) {
      uint32_t ov[32];
      tmem_ld32(o_col + cb * 32, ov);
      if (valid) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          po[(size_t)(cb * 8 + q) * kQTile] =
              make_float4(__uint_as_float(ov[4 * q]) * inv, __uint_as_float(ov[4 * q + 1]) * inv,
                          __uint_as_float(ov[4 * q + 2]) * inv, __uint_as_float(ov[4 * q + 3]) * inv);
      }
    }
  }
  if (valid) P.ppart_lse[(size_t)(slot0 + pr.split) * kQTile + row] = lse2 * kLn2;
  __threadfence();
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
  if ((tid & 127) == 0) {
    // a missing tile has no group; after a failure nobody merges
    const int old = (*abort_flag || !tile_ok) ? -1 : atomicAdd(P.pgroup_ctr + pr.group[i], 1);
    s_flag[i] = (old == pr.n_split - 1);
  }
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
  if (s_flag[i] && !failed && valid) {
    // The last split to finish merges all of them, one query row per thread,
    // always in split order so the result does not depend on which split
    // finished last: O = sum_s w_s O_s / sum_s w_s, w_s = exp(LSE_s - max LSE).
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
    uint16_t* dst = P.o_p + (out_row * P.H + head) * D;
    const float4* src = part + (size_t)slot0 * (D / 4) * kQTile + row;
#pragma unroll 1
    for (int cb = 0; cb < D / 32; ++cb) {
      float acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0.f;
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
          acc[4 * q] = fmaf(w, x[q].x, acc[4 * q]);
          acc[4 * q + 1] = fmaf(w, x[q].y, acc[4 * q + 1]);
          acc[4 * q + 2] = fmaf(w, x[q].z, acc[4 * q + 2]);
          acc[4 * q + 3] = fmaf(w, x[q].w, acc[4 * q + 3]);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16(acc[8 * q + 0], acc[8 * q + 1]);
        v.y = pack_bf16(acc[8 * q + 2], acc[8 * q + 3]);
        v.z = pack_bf16(acc[8 * q + 4], acc[8 * q + 5]);
        v.w = pack_bf16(acc[8 * q + 6], acc[8 * q + 7]);
        *reinterpret_cast<uint4*>(dst + cb * 32 + 8 * q) = v;
      }
    }
    P.lse_p[out_row * P.H + head] = m + logf(wsum);
  }
  return !failed;
}

