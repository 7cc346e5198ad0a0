// pod_attn_api.cpp -- C ABI, argument validation and the host planner of
// libpod_attn.so. See include/pod_attn.h for the contract.
//
// Planner (POD-Attention §4.2.2-§4.2.3 and §5.4): splits the hybrid batch into
// prefill units (request, pair of 128-row query tiles sharing K/V, KV split)
// and decode units (request, KV head, KV split), chooses the split counts, and
// sets the role policy the fused kernel's per-SM tickets follow (§4.1, §5.4.2).
// The plan is a pure function of the shapes, the SM count and whether the call
// is one fused launch (which leaves the prefill unsplit when decodes share it);
// on a common plan FUSED, SERIAL and TWO_STREAM compute bitwise-identical
// results.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <new>
#include <vector>

#include "pod_attn.h"
#include "pod_plan.h"

namespace pod {
cudaError_t kernels_init(int D);
int fused_smem_bytes(int D);
int decode_smem_bytes(int D);
cudaError_t launch_fused(const Plan& P, const TmaDescs& T, int grid, int allow_prefill,
                         int allow_decode, cudaStream_t s);
cudaError_t launch_decode(const Plan& P, int max_grid, cudaStream_t s);
cudaError_t decode_occupancy(int D, int* blocks_per_sm);
cudaError_t launch_merge(const Plan& P, cudaStream_t s);
cudaError_t pair_max_clusters(int* clusters);
cudaError_t launch_fused_pair(const Plan& P, const TmaDescs& T, int grid, int allow_prefill,
                              int allow_decode, cudaStream_t s);
}  // namespace pod

using namespace pod;

namespace {

constexpr int kRing = 8;            // pinned host plan slots
constexpr int kMaxPrefillSplit = 16;
constexpr int kDecSplitMax = 1 << 20;
constexpr int kStatsInts = kMaxSmid * 2;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = (prev == dev) || (cudaSetDevice(dev) == cudaSuccess);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// Capacity layout of the plan buffer: its size bounds any call's plan. A call
// packs its plan from the start of the buffer (control words, tickets, stats,
// merge counters, then the tables it uses) and copies only that much; the
// control words, tickets, stats and merge counters (everything before the
// tables) start at zero.
struct PlanLayout {
  size_t ctl, ticket, stats, tables0;                        // fixed part
  size_t pgroup, dgroup, tables, preq, punits, dreq;  // capacities
  size_t end;
};

}  // namespace

struct pod_attn_ctx {
  pod_attn_config cfg{};
  int device = 0, num_sms = 0, slots_per_sm = kFusedSlotsPerSm;
  int decode_grid = 0;  // persistent decode-only grid (SMs x resident CTAs)
  // scheduling levers (defaults; environment overrides exist for ablations)
  int policy = 4;        // 0 proportional, 1 even (50:50), 2 prefill first, 3 decode first,
                         // 4 front (each SM's first tickets take prefill, then 50:50)
                         // 5 balanced (a fixed set of SMs takes prefill first)
  int smid_aware = 1;    // per-SM tickets (1) or one global ticket counter (0)
  int dec_turn = 1;      // decode units each warp claims per decode turn of a fused CTA
  int dec_split = 0;     // 0: cost model; else keys per decode split (multiple of 16)
  int pre_split = 0;     // 0: makespan model; else KV splits per prefill tile
  bool tail_split_fused = false;  // ablation: also split the last wave in fused calls with decodes
  bool split_uncapped = false;  // forced splits ignore the two-wave cap (ablation)
  // prefill tile: a CTA pair on two SMs (M = 256, head_dim 128) or one SM
  bool use_pair = false;
  int pair_clusters = 0;  // clusters of two CTAs resident at once (pair kernel)
  int H = 0, Hk = 0, G = 0, D = 0;
  int cap_punits = 0, cap_pgroups = 0, cap_pslots = 0;
  int cap_dunits = 0, cap_dgroups = 0, cap_dslots = 0, cap_dreqs = 0;
  size_t plan_cap = 0;
  char* d_plan = nullptr;
  float* d_ppart_o = nullptr;
  float* d_ppart_lse = nullptr;
  float* d_dpart_o = nullptr;
  float* d_dpart_lse = nullptr;
  int* d_misc = nullptr;  // [0] status, [1] never-set flag
  char* h_plan[kRing] = {};
  cudaEvent_t h_ev[kRing] = {};
  int ring_i = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  pod_plan_info last{};
  PlanLayout lay{};
  // scratch for the planner (reused, sized at create)
  std::vector<PrefillUnit> units_tmp;
  std::vector<int> units_split;
  std::vector<long long> heap_tmp;
  std::vector<long long> heap2_tmp;
  std::vector<long long> parts_len_tmp;
  std::vector<PrefillUnit> parts_tmp;
  std::vector<PrefillReq> preq_tmp;
  std::vector<DecodeReq> dreq_tmp;
};

namespace {

PlanLayout plan_layout(const pod_attn_ctx* c) {
  PlanLayout L{};
  size_t o = 0;
  L.ctl = o; o += 64;
  L.ticket = o; o += sizeof(int) * kMaxSmid;
  L.stats = o; o += sizeof(int) * kStatsInts;
  L.tables0 = o = align_up(o, 64);
  L.pgroup = o; o = align_up(o + sizeof(int) * (size_t)c->cap_pgroups, 64);
  L.dgroup = o; o = align_up(o + sizeof(int) * (size_t)c->cap_dgroups, 64);
  L.tables = o;
  L.preq = o; o = align_up(o + sizeof(PrefillReq) * kMaxPrefillReqs, 64);
  L.punits = o; o = align_up(o + sizeof(PrefillUnit) * (size_t)c->cap_punits, 64);
  L.dreq = o; o = align_up(o + sizeof(DecodeReq) * (size_t)c->cap_dreqs, 64);
  L.end = o;
  return L;
}

int cuda_fail() { return POD_ECUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int make_map(pod_attn_ctx* c, CUtensorMap* m, const void* base, uint64_t heads, uint64_t rows,
             uint32_t box_rows) {
  const uint64_t D = (uint64_t)c->D;
  cuuint64_t dims[3] = {D, heads, rows};
  cuuint64_t strides[2] = {D * 2, heads * D * 2};
  cuuint32_t box[3] = {64, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = c->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? POD_OK : POD_ECUDA;
}

// ----------------------------------------------------------------- validation
int check_prefill(const pod_attn_ctx* c, const pod_prefill_args* a, long long* total_tokens) {
  *total_tokens = 0;
  if (!a || a->num_reqs == 0) return POD_OK;
  if (a->num_reqs < 0) return POD_EINVAL;
  if (a->num_reqs > c->cfg.max_prefill_reqs || a->num_reqs > kMaxPrefillReqs) return POD_ECAPACITY;
  if (!a->chunk_lens || !a->prior_lens) return POD_EINVAL;
  long long tot = 0;
  for (int i = 0; i < a->num_reqs; ++i) {
    const long long cl = a->chunk_lens[i], pl = a->prior_lens[i];
    if (cl < 0 || pl < 0) return POD_EINVAL;
    if (cl > 0 && cl + pl > c->cfg.max_kv_tokens) return POD_ECAPACITY;
    if (cl + pl > (1LL << 30)) return POD_ECAPACITY;
    tot += cl;
  }
  if (tot > c->cfg.max_prefill_tokens) return POD_ECAPACITY;
  *total_tokens = tot;
  if (tot == 0) return POD_OK;
  if (!a->q || !a->o || !a->lse) return POD_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->o) || (reinterpret_cast<uintptr_t>(a->lse) & 3u))
    return POD_EINVAL;
  if (c->cfg.kv_layout == POD_KV_CONTIGUOUS) {
    if (!a->k_ptrs || !a->v_ptrs) return POD_EINVAL;
    for (int i = 0; i < a->num_reqs; ++i) {
      if (a->chunk_lens[i] == 0) continue;
      if (!a->k_ptrs[i] || !a->v_ptrs[i]) return POD_EINVAL;
      if (!aligned16(a->k_ptrs[i]) || !aligned16(a->v_ptrs[i])) return POD_EINVAL;
    }
  } else {
    if (!a->k_pool || !a->v_pool || !a->block_table || a->pool_blocks <= 0) return POD_EINVAL;
    if (!aligned16(a->k_pool) || !aligned16(a->v_pool)) return POD_EINVAL;
    if (a->pool_blocks * 16 > (1LL << 31)) return POD_ECAPACITY;
    for (int i = 0; i < a->num_reqs; ++i) {
      if (a->chunk_lens[i] == 0) continue;
      const long long need = (a->chunk_lens[i] + (long long)a->prior_lens[i] + 15) / 16;
      if (a->block_table_stride < need) return POD_EINVAL;
    }
  }
  return POD_OK;
}

int check_decode(const pod_attn_ctx* c, const pod_decode_args* a) {
  if (!a || a->num_reqs == 0) return POD_OK;
  if (a->num_reqs < 0) return POD_EINVAL;
  if (a->num_reqs > c->cfg.max_decode_reqs || a->num_reqs > c->cap_dreqs) return POD_ECAPACITY;
  if (!a->ctx_lens || !a->q || !a->o || !a->lse) return POD_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->o) || (reinterpret_cast<uintptr_t>(a->lse) & 3u))
    return POD_EINVAL;
  for (int i = 0; i < a->num_reqs; ++i) {
    if (a->ctx_lens[i] < 1) return POD_EINVAL;
    if (a->ctx_lens[i] > c->cfg.max_kv_tokens) return POD_ECAPACITY;
  }
  if (c->cfg.kv_layout == POD_KV_CONTIGUOUS) {
    if (!a->k_ptrs || !a->v_ptrs) return POD_EINVAL;
    for (int i = 0; i < a->num_reqs; ++i) {
      if (!a->k_ptrs[i] || !a->v_ptrs[i]) return POD_EINVAL;
      if (!aligned16(a->k_ptrs[i]) || !aligned16(a->v_ptrs[i])) return POD_EINVAL;
    }
  } else {
    if (!a->k_pool || !a->v_pool || !a->block_table || a->pool_blocks <= 0) return POD_EINVAL;
    if (!aligned16(a->k_pool) || !aligned16(a->v_pool)) return POD_EINVAL;
    for (int i = 0; i < a->num_reqs; ++i)
      if (a->block_table_stride < (a->ctx_lens[i] + 15) / 16) return POD_EINVAL;
  }
  return POD_OK;
}

// ----------------------------------------------------------------- planner
// Fills the host slot `h` and the kernel parameters. Returns a pod_status.
int build_plan(pod_attn_ctx* c, const pod_prefill_args* pa, const pod_decode_args* da,
               bool fused_call, char* h, Plan* P, TmaDescs* T, size_t* copy_bytes) {
  const PlanLayout& L = c->lay;
  const int H = c->H, Hk = c->Hk;
  const int np = (pa ? pa->num_reqs : 0);
  const int nd = (da ? da->num_reqs : 0);
  const bool paged = c->cfg.kv_layout == POD_KV_PAGED;
  // persistent prefill workers: CTA pairs, or CTAs of one SM each
  const int slots = c->use_pair ? c->pair_clusters : c->num_sms * c->slots_per_sm;

  // ---- prefill
  c->preq_tmp.assign(np, PrefillReq{});
  PrefillReq* preq = c->preq_tmp.data();
  // A unit is two query tiles sharing K/V: a head pair of one KV group at one
  // token tile (G even) or two consecutive token tiles of one head (G odd).
  const bool pair_heads = (c->G % 2) == 0;
  const int qt_step = pair_heads ? 1 : 2;  // token tiles per unit
  const int h_step = pair_heads ? 2 : 1;   // heads per unit
  int q_row = 0;
  c->units_tmp.clear();
  for (int p = 0; p < np; ++p) {
    PrefillReq& R = preq[p];
    const int chunk = pa->chunk_lens[p], prior = pa->prior_lens[p];
    R.prior = prior;
    R.chunk = chunk;
    R.q_row0 = q_row;
    R.n_qtiles = (chunk + kQTile - 1) / kQTile;
    R.kv_len = prior + chunk;
    R.bt_row = p;
    R.pair_heads = pair_heads ? 1 : 0;
    R.n_split = 1;
    q_row += chunk;
    for (int qt = 0; qt < R.n_qtiles; qt += qt_step) {
      const int last_qt = std::min(qt + qt_step, R.n_qtiles) - 1;
      const int kv_hi = prior + std::min(chunk, (last_qt + 1) * kQTile);
      const int work = (kv_hi + kKVTile - 1) / kKVTile;
      for (int hh = 0; hh < H; hh += h_step) {
        c->units_tmp.push_back(PrefillUnit{p, hh, qt, 0, 1, 0, 0, work});
      }
    }
  }
  const int n_draft = (int)c->units_tmp.size();
  // queue order: longest first (LPT), so the tail of the queue is short work;
  // ties in request, token tile, head and split order
  auto queue_order = [](const PrefillUnit& a, const PrefillUnit& b) {
    if (a.work != b.work) return a.work > b.work;
    if (a.req != b.req) return a.req < b.req;
    if (a.qtile != b.qtile) return a.qtile < b.qtile;
    if (a.head != b.head) return a.head < b.head;
    return a.split < b.split;
  };
  std::sort(c->units_tmp.begin(), c->units_tmp.end(), queue_order);
  // KV splits per unit. A split keeps >= 4 KV tiles. Candidates: the same
  // count for every unit (the summary's "at most two full waves": units x
  // splits <= 2 slots), or splitting only the units of the last, partial
  // wave; each is scored by the finish time of a longest-first assignment of
  // the parts to the slots (what the persistent queue does), with two tiles
  // of per-part overhead (query load, pipeline fill, epilogue, merge).
  std::vector<int>& split = c->units_split;
  split.assign(n_draft, 1);
  auto max_split_of = [&](int u) {
    return std::max(1, std::min(kMaxPrefillSplit, c->units_tmp[u].work / 4));
  };
  auto makespan = [&](const std::vector<int>& sp) -> long long {
    // parts in queue order: by part length, longest first
    std::vector<long long>& parts = c->heap_tmp;
    parts.clear();
    for (int u = 0; u < n_draft; ++u) {
      const long long w = c->units_tmp[u].work;
      for (int k = 0; k < sp[u]; ++k)
        parts.push_back((w * (k + 1)) / sp[u] - (w * k) / sp[u] + 2);
    }
    std::sort(parts.begin(), parts.end(), std::greater<long long>());
    // each part goes to the slot that frees first (a min-heap of finish times)
    std::vector<long long>& hp = c->heap2_tmp;
    const size_t n0 = std::min(parts.size(), (size_t)std::max(slots, 1));
    hp.assign(parts.begin(), parts.begin() + n0);
    long long end = n0 ? hp.front() : 0;
    std::make_heap(hp.begin(), hp.end(), std::greater<long long>());
    for (size_t i = n0; i < parts.size(); ++i) {
      std::pop_heap(hp.begin(), hp.end(), std::greater<long long>());
      hp.back() += parts[i];
      end = std::max(end, hp.back());
      std::push_heap(hp.begin(), hp.end(), std::greater<long long>());
    }
    return end;
  };
  auto fits = [&](const std::vector<int>& sp) {
    long long groups = 0, tiles = 0;
    for (int u = 0; u < n_draft; ++u)
      if (sp[u] > 1) {
        groups += 2;
        tiles += 2LL * sp[u];
      }
    return groups <= c->cap_pgroups && tiles <= c->cap_pslots;
  };
  if (n_draft > 0 && c->pre_split > 0) {
    int s_all = c->pre_split;
    while (!c->split_uncapped && s_all > 1 && (long long)n_draft * s_all > 2LL * slots) --s_all;
    for (int u = 0; u < n_draft; ++u) split[u] = std::min(s_all, max_split_of(u));
    if (!fits(split)) split.assign(n_draft, 1);
  } else if (n_draft > 0) {
    const long long base = makespan(split);
    bool consider = true;
    if (fused_call && nd > 0) {
      // One fused launch that also carries decodes: split only when the
      // prefill is the longer phase. Otherwise the decode units fill the
      // slots an unsplit prefill leaves idle, and the prefill holds fewer SMs
      // at once while the others stream decode K/V (measured on B200,
      // Llama-3-8B batch: 242 us unsplit against 257 with 2 splits).
      const double tile_us = c->use_pair ? 0.75 : (c->D == 128 ? 2.0 : 1.2);
      double kv_bytes = 0.0;
      for (int r = 0; r < nd; ++r) kv_bytes += (double)da->ctx_lens[r] * Hk * c->D * 4.0;
      consider = (double)base * tile_us > kv_bytes / 6.0e6;  // decode at ~6 TB/s
    }
    if (consider) {
      long long best = base;
      std::vector<int> cand(n_draft);
      auto try_cand = [&]() {
        if (!fits(cand)) return;
        const long long t = makespan(cand);
        if (t < (best * 97) / 100) {
          best = t;
          split = cand;
        }
      };
      for (int s_all = 2; s_all <= kMaxPrefillSplit && (long long)n_draft * s_all <= 2LL * slots;
           ++s_all) {
        for (int u = 0; u < n_draft; ++u) cand[u] = std::min(s_all, max_split_of(u));
        try_cand();
      }
      // Splitting only the last wave balances a launch that runs prefill
      // alone. In a fused launch that also carries decodes, the SMs an
      // unsplit last wave leaves free run decode turns instead, and the split
      // measured slower (B200, long-context batch: 725 us against 670 us
      // unsplit; prefill alone 587 us against 602 us).
      const int tail =
          (n_draft > slots && (c->tail_split_fused || !(fused_call && nd > 0))) ? n_draft % slots : 0;
      if (tail > 0) {
        // The tail units are the shortest, so their parts queue after every
        // unsplit unit: run the unsplit prefix once, then each tail split.
        std::vector<long long>& hp0 = c->heap_tmp;
        hp0.clear();
        long long end0 = 0;
        const int prefix = n_draft - tail;
        for (int u = 0; u < prefix; ++u) {
          const long long w = c->units_tmp[u].work + 2;
          if ((int)hp0.size() < slots) {
            hp0.push_back(w);
            end0 = std::max(end0, w);
            if ((int)hp0.size() == slots)
              std::make_heap(hp0.begin(), hp0.end(), std::greater<long long>());
            continue;
          }
          std::pop_heap(hp0.begin(), hp0.end(), std::greater<long long>());
          hp0.back() += w;
          end0 = std::max(end0, hp0.back());
          std::push_heap(hp0.begin(), hp0.end(), std::greater<long long>());
        }
        for (int s_tail = 2; s_tail <= 4; ++s_tail) {
          for (int u = 0; u < n_draft; ++u)
            cand[u] = (u >= prefix) ? std::min(s_tail, max_split_of(u)) : 1;
          if (!fits(cand)) continue;
          std::vector<long long>& tp = c->parts_len_tmp;
          tp.clear();
          for (int u = prefix; u < n_draft; ++u) {
            const long long w = c->units_tmp[u].work;
            for (int k = 0; k < cand[u]; ++k)
              tp.push_back((w * (k + 1)) / cand[u] - (w * k) / cand[u] + 2);
          }
          std::sort(tp.begin(), tp.end(), std::greater<long long>());
          std::vector<long long>& hp = c->heap2_tmp;
          hp = hp0;  // prefix >= slots: a full heap of finish times
          long long end = end0;
          for (long long w : tp) {
            std::pop_heap(hp.begin(), hp.end(), std::greater<long long>());
            hp.back() += w;
            end = std::max(end, hp.back());
            std::push_heap(hp.begin(), hp.end(), std::greater<long long>());
          }
          if (end < (best * 97) / 100) {
            best = end;
            split = cand;
          }
        }
      }
    }
  }
  // expand the parts; split units get their merge groups and partial slots
  int n_pg = 0, n_ps = 0, max_split = 1;
  std::vector<PrefillUnit>& parts = c->parts_tmp;
  parts.clear();
  for (int u = 0; u < n_draft; ++u) {
    PrefillUnit U = c->units_tmp[u];
    const int sp = split[u];
    U.n_split = sp;
    if (sp > 1) {
      U.group0 = n_pg;
      U.slot0 = n_ps;
      n_pg += 2;
      n_ps += 2 * sp;
    }
    max_split = std::max(max_split, sp);
    preq[U.req].n_split = std::max(preq[U.req].n_split, sp);
    const int w = U.work;
    for (int k = 0; k < sp; ++k) {
      PrefillUnit part = U;
      part.split = k;
      part.work = (w * (k + 1)) / sp - (w * k) / sp;
      parts.push_back(part);
    }
  }
  const int n_pu = (int)parts.size();
  if (n_pu > c->cap_punits || n_pg > c->cap_pgroups || n_ps > c->cap_pslots) return POD_ECAPACITY;
  std::sort(parts.begin(), parts.end(), queue_order);
  const PrefillUnit* punits = parts.data();

  // ---- decode
  c->dreq_tmp.assign(nd, DecodeReq{});
  DecodeReq* dreq = c->dreq_tmp.data();
  // Keys per decode split (a multiple of the 16-key decode tile): the
  // candidate minimising an estimate of the decode makespan on the persistent
  // decode warps. Units are claimed dynamically, so with U units of at most
  // `mx` keys on W warps the finish time is about min(ceil(U/W) * (mx + o),
  // sum/W + mx + o), o being a per-unit overhead (start-up, partial write,
  // merge) of about 48 keys' worth of streaming.
  auto count_units = [&](int sl) {
    long long n = 0;
    for (int r = 0; r < nd; ++r) n += (long long)((da->ctx_lens[r] + sl - 1) / sl) * Hk;
    return n;
  };
  int split_len = kDecSplitMax;
  if (nd > 0 && c->dec_split > 0) {
    split_len = c->dec_split;
    while (split_len < kDecSplitMax && count_units(split_len) > c->cap_dunits) split_len *= 2;
  } else if (nd > 0) {
    static const int kCands[] = {256, 320, 384, 512, 640, 768, 1024, 1536, 2048, 3072, 4096,
                                 8192, 16384, 32768, 65536, 131072, 262144, 524288, 1048576};
    const double W = (double)std::max(1, c->decode_grid * kDecodeWarps);
    const double o = 48.0;
    int max_len = 1;
    long long keys = 0;
    for (int r = 0; r < nd; ++r) {
      max_len = std::max(max_len, da->ctx_lens[r]);
      keys += (long long)da->ctx_lens[r] * Hk;
    }
    double best = 1e300;
    for (int sl : kCands) {
      const long long U = count_units(sl);
      if (U > c->cap_dunits) continue;
      const double mx = (double)std::min(sl, max_len);
      const double est = std::min(std::ceil((double)U / W) * (mx + o),
                                  ((double)keys + (double)U * o) / W + mx + o);
      if (est < best * 0.999) {
        best = est;
        split_len = sl;
      }
      if (sl >= max_len) break;  // larger splits change nothing
    }
  }
  int n_du = 0, n_dg = 0, n_ds = 0;
  for (int r = 0; r < nd; ++r) {
    DecodeReq& R = dreq[r];
    const int len = da->ctx_lens[r];
    R.k = paged ? nullptr : static_cast<const uint16_t*>(da->k_ptrs[r]);
    R.v = paged ? nullptr : static_cast<const uint16_t*>(da->v_ptrs[r]);
    R.len = len;
    R.n_split = (len + split_len - 1) / split_len;
    R.unit0 = n_du;
    R.bt_row = r;
    if (R.n_split > 1) {
      R.group0 = n_dg;
      R.slot0 = n_ds;
      n_dg += Hk;
      n_ds += R.n_split * Hk;
    }
    const int nu = R.n_split * Hk;
    if (n_du + nu > c->cap_dunits) return POD_ECAPACITY;
    n_du += nu;
  }
  if (n_dg > c->cap_dgroups || n_ds > c->cap_dslots) return POD_ECAPACITY;

  // ---- claim ratio (per-SM Bresenham over tickets): prefill share of claims
  // A fused CTA's decode turn processes up to dec_turn units per warp.
  const long long dclaims =
      (n_du + (long long)kFusedWarps * c->dec_turn - 1) / ((long long)kFusedWarps * c->dec_turn);
  int rho_num = n_pu, rho_den = n_pu + (int)dclaims;  // proportional (summary §5.4.2)
  if (c->policy == 1) { rho_num = 1; rho_den = 2; }
  if (c->policy == 2) { rho_num = 1; rho_den = 1; }
  if (c->policy == 3) { rho_num = 0; rho_den = 1; }
  if (c->policy == 4) { rho_num = 1; rho_den = 2; }  // front: see pod_fused_kernel
  // balanced (POD-Attention §4.1: match the prefill and decode shares of the
  // SMs to their work): CTAs 0..p_cap-1 take prefill first, the others decode
  // first. With the decode side bound by HBM, decode alone takes about
  // bytes / bandwidth on the whole GPU and still about that on the SMs left
  // to it, as long as those are enough to keep HBM busy; prefill needs
  // sum(unit times) SM-microseconds. p_cap is the SM count on which prefill
  // finishes in the decode time (all SMs when prefill dominates).
  int p_cap = slots;
  if (c->policy == 5 && n_pu > 0 && nd > 0) {
    const double tile_us = c->use_pair ? 0.75 : (c->D == 128 ? 2.0 : 1.2), unit_us = 3.0;
    double p_sm_us = 0.0;
    for (int u = 0; u < n_pu; ++u) p_sm_us += punits[u].work * tile_us + unit_us;
    double kv_keys = 0.0;
    for (int r = 0; r < nd; ++r) kv_keys += (double)da->ctx_lens[r];
    const double d_us = kv_keys * Hk * c->D * 4.0 / 6.0e6;  // K and V, bf16, ~6 TB/s
    if (d_us > p_sm_us / slots)
      p_cap = std::max(1, std::min(slots, (int)std::ceil(p_sm_us / d_us)));
  }
  if (rho_den == 0) rho_den = 1;

  // ---- kernel parameters
  Plan& Q = *P;
  std::memset(&Q, 0, sizeof(Q));
  Q.H = H;
  Q.Hk = Hk;
  Q.G = c->G;
  Q.D = c->D;
  Q.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c->D));
  Q.n_prefill_units = n_pu;
  Q.n_decode_units = n_du;
  Q.n_prefill_reqs = np;
  Q.n_decode_reqs = nd;
  Q.dec_split_len = split_len;
  Q.rho_num = rho_num;
  Q.rho_den = rho_den;
  Q.paged = paged ? 1 : 0;
  Q.bt_stride_p = (np && paged) ? pa->block_table_stride : 0;
  Q.bt_stride_d = (nd && paged) ? da->block_table_stride : 0;
  Q.flags = (int)c->cfg.flags | (c->smid_aware ? 0 : kFlagGlobalTicket) | (c->policy == 4 ? kFlagFrontPolicy : 0) |
            (c->policy == 5 ? kFlagBalancedPolicy : 0);
  Q.p_cap = p_cap;
  Q.dec_turn = c->dec_turn;
  Q.wait_budget = kDefaultWaitBudget;
  // ---- pack the plan: zeroed words, merge counters, then the tables in use
  const size_t o_pg = L.tables0;
  const size_t o_dg = align_up(o_pg + sizeof(int) * (size_t)n_pg, 64);
  const size_t o_preq = align_up(o_dg + sizeof(int) * (size_t)n_dg, 64);
  const size_t o_pu = align_up(o_preq + sizeof(PrefillReq) * (size_t)np, 64);
  const size_t o_dreq = align_up(o_pu + sizeof(PrefillUnit) * (size_t)n_pu, 64);
  // (decode units are not listed: a unit finds its request by a search of
  // the requests' first-unit indices, which ascend)
  const size_t o_end = o_dreq + sizeof(DecodeReq) * (size_t)nd;
  if (o_end > c->plan_cap) return POD_ECAPACITY;
  std::memset(h, 0, o_preq);
  if (np) std::memcpy(h + o_preq, preq, sizeof(PrefillReq) * (size_t)np);
  if (n_pu) std::memcpy(h + o_pu, punits, sizeof(PrefillUnit) * (size_t)n_pu);
  if (nd) std::memcpy(h + o_dreq, dreq, sizeof(DecodeReq) * (size_t)nd);
  char* dp = c->d_plan;
  Q.preq = reinterpret_cast<const PrefillReq*>(dp + o_preq);
  Q.punits = reinterpret_cast<const PrefillUnit*>(dp + o_pu);
  Q.dreq = reinterpret_cast<const DecodeReq*>(dp + o_dreq);
  if (np) {
    Q.q_p = static_cast<const uint16_t*>(pa->q);
    Q.o_p = static_cast<uint16_t*>(pa->o);
    Q.lse_p = pa->lse;
    Q.bt_p = paged ? pa->block_table : nullptr;
  }
  if (nd) {
    Q.q_d = static_cast<const uint16_t*>(da->q);
    Q.o_d = static_cast<uint16_t*>(da->o);
    Q.lse_d = da->lse;
    Q.bt_d = paged ? da->block_table : nullptr;
  }
  if (paged) {
    Q.k_pool = static_cast<const uint16_t*>(nd ? da->k_pool : (np ? pa->k_pool : nullptr));
    Q.v_pool = static_cast<const uint16_t*>(nd ? da->v_pool : (np ? pa->v_pool : nullptr));
    Q.pool_blocks = (int)std::min<long long>(nd ? da->pool_blocks : (np ? pa->pool_blocks : 0),
                                             1LL << 30);
  }
  Q.ppart_o = c->d_ppart_o;
  Q.ppart_lse = c->d_ppart_lse;
  Q.dpart_o = c->d_dpart_o;
  Q.dpart_lse = c->d_dpart_lse;
  Q.ctl = reinterpret_cast<int*>(dp + L.ctl);
  Q.sm_ticket = reinterpret_cast<int*>(dp + L.ticket);
  Q.stats = reinterpret_cast<int*>(dp + L.stats);
  Q.pgroup_ctr = reinterpret_cast<int*>(dp + o_pg);
  Q.dgroup_ctr = reinterpret_cast<int*>(dp + o_dg);
  Q.status = c->d_misc;
  Q.never_set = c->d_misc + 1;

  // ---- TMA descriptors (prefill only)
  std::memset(T, 0, sizeof(*T));
  if (n_pu > 0) {
    const long long tp = q_row;
    int rc = make_map(c, &T->q, pa->q, (uint64_t)H, (uint64_t)tp, kQTile);
    if (rc) return rc;
    if (!paged) {
      for (int p = 0; p < np; ++p) {
        if (pa->chunk_lens[p] == 0) continue;
        const uint64_t len = (uint64_t)pa->chunk_lens[p] + (uint64_t)pa->prior_lens[p];
        rc = make_map(c, &T->k[p], pa->k_ptrs[p], (uint64_t)Hk, len,
                      c->use_pair ? kKVTile / 2 : kKVTile);  // the pair loads K in halves
        if (rc) return rc;
        rc = make_map(c, &T->v[p], pa->v_ptrs[p], (uint64_t)Hk, len, kKVTile);
        if (rc) return rc;
      }
    } else {
      const uint64_t rows = (uint64_t)pa->pool_blocks * 16;
      rc = make_map(c, &T->k[0], pa->k_pool, (uint64_t)Hk, rows, 16);
      if (rc) return rc;
      rc = make_map(c, &T->v[0], pa->v_pool, (uint64_t)Hk, rows, 16);
      if (rc) return rc;
    }
  }
  // ---- record
  c->last.num_sms = c->num_sms;
  c->last.slots_per_sm = c->slots_per_sm;
  c->last.prefill_units = n_pu;
  c->last.prefill_split = np ? max_split : 0;
  c->last.decode_units = n_du;
  c->last.decode_split_len = nd ? split_len : 0;
  c->last.ratio_num = rho_num;
  c->last.ratio_den = rho_den;
  c->last.prefill_sm_cap = p_cap;
  c->last.pair_clusters = c->use_pair ? c->pair_clusters : 0;
  *copy_bytes = o_end;
  c->last.plan_bytes = (long long)*copy_bytes;
  return POD_OK;
}

int fused_grid(const pod_attn_ctx* c, const Plan& P, bool allow_decode) {
  long long claims = P.n_prefill_units;
  if (c->use_pair) {  // clusters of two CTAs
    if (allow_decode) claims += (P.n_decode_units + 2 * kFusedWarps - 1) / (2 * kFusedWarps);
    const long long g = std::min<long long>(c->pair_clusters, claims);
    return 2 * (int)std::max<long long>(g, 1);
  }
  if (allow_decode) claims += (P.n_decode_units + kFusedWarps - 1) / kFusedWarps;
  long long g = std::min<long long>((long long)c->num_sms * c->slots_per_sm, claims);
  return (int)std::max<long long>(g, 1);
}

// The persistent fused launch (prefill and / or decode units).
cudaError_t run_fused(const pod_attn_ctx* c, const Plan& P, const TmaDescs& T, bool allow_decode,
                      cudaStream_t s) {
  const int grid = fused_grid(c, P, allow_decode);
  if (c->use_pair) return launch_fused_pair(P, T, grid, 1, allow_decode ? 1 : 0, s);
  return launch_fused(P, T, grid, 1, allow_decode ? 1 : 0, s);
}

// Common front half of every call: pick a ring slot, plan, copy the plan.
int stage_plan(pod_attn_ctx* c, const pod_prefill_args* pa, const pod_decode_args* da,
               bool fused_call, cudaStream_t s, Plan* P, TmaDescs* T) {
  const int slot = c->ring_i;
  c->ring_i = (c->ring_i + 1) % kRing;
  if (cudaEventSynchronize(c->h_ev[slot]) != cudaSuccess) return POD_ECUDA;
  size_t bytes = 0;
  int rc = build_plan(c, pa, da, fused_call, c->h_plan[slot], P, T, &bytes);
  if (rc) return rc;
  if (cudaMemcpyAsync(c->d_plan, c->h_plan[slot], bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return POD_ECUDA;
  if (cudaEventRecord(c->h_ev[slot], s) != cudaSuccess) return POD_ECUDA;
  return POD_OK;
}

// Capacities of the per-call tables and the plan layout, from the config,
// the head counts and the SM count already set in c.
void size_context(pod_attn_ctx* c) {
  const pod_attn_config* cfg = &c->cfg;
  const int slots = c->num_sms * c->slots_per_sm;
  const long long qtiles = (long long)cfg->max_prefill_tokens / kQTile + cfg->max_prefill_reqs;
  c->cap_punits = (int)std::min<long long>(qtiles * c->H * kMaxPrefillSplit, 1 << 24);
  c->cap_pgroups =
      (int)std::min<long long>(std::min<long long>(qtiles * c->H, 2LL * slots), 1 << 24);
  // partial slots (two query tiles per split unit): a uniform split keeps
  // units x splits <= 2 slots (4 x slots); a split of the last, partial wave
  // only has fewer than `slots` units in up to 4 parts (8 x slots)
  c->cap_pslots = 8 * slots;
  if (c->split_uncapped) {     // forced splits past two waves (an ablation lever)
    c->cap_pgroups = (int)std::min<long long>(qtiles * c->H, 1 << 20);
    c->cap_pslots = (int)std::min<long long>(qtiles * c->H * kMaxPrefillSplit, 1 << 20);
  }
  c->cap_pgroups = std::max(c->cap_pgroups, 1);
  c->cap_dreqs = std::max(cfg->max_decode_reqs, 1);
  c->cap_dunits =
      (int)std::max<long long>(16LL * c->num_sms * 8, (long long)c->cap_dreqs * c->Hk * 2);
  c->cap_dgroups = c->cap_dreqs * c->Hk;
  c->cap_dslots = c->cap_dunits;
  c->lay = plan_layout(c);
  c->plan_cap = c->lay.end;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* pod_attn_strerror(int st) {
  switch (st) {
    case POD_OK: return "ok";
    case POD_EINVAL: return "invalid argument";
    case POD_EUNSUPPORTED: return "unsupported shape or layout";
    case POD_ENOMEM: return "out of memory";
    case POD_ECUDA: return "CUDA error";
    case POD_ETIMEOUT: return "device wait timed out";
    case POD_ECAPACITY: return "size exceeds the context's capacity";
    default: return "unknown status";
  }
}

int pod_attn_create(pod_attn_ctx** out, const pod_attn_config* cfg) {
  if (!out || !cfg) return POD_EINVAL;
  *out = nullptr;
  const int H = cfg->num_qo_heads, Hk = cfg->num_kv_heads, D = cfg->head_dim;
  if (H <= 0 || Hk <= 0 || H % Hk != 0) return POD_EINVAL;
  if (cfg->max_prefill_reqs < 0 || cfg->max_prefill_tokens < 0 || cfg->max_decode_reqs < 0 ||
      cfg->max_kv_tokens < 1)
    return POD_EINVAL;
  if (cfg->kv_layout != POD_KV_CONTIGUOUS && cfg->kv_layout != POD_KV_PAGED) return POD_EINVAL;
  if (D != 64 && D != 128) return POD_EUNSUPPORTED;
  if (H / Hk > kMaxGroup) return POD_EUNSUPPORTED;
  if (cfg->kv_layout == POD_KV_PAGED && cfg->page_size != 16) return POD_EUNSUPPORTED;
  if (cfg->max_prefill_reqs > kMaxPrefillReqs) return POD_ECAPACITY;
  if (cfg->max_kv_tokens > (1LL << 30)) return POD_ECAPACITY;

  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return POD_ECUDA;
  if (cfg->device < 0 || cfg->device >= ndev) return POD_EINVAL;
  DeviceGuard guard(cfg->device);
  if (!guard.ok) return POD_ECUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, cfg->device) != cudaSuccess) return POD_ECUDA;
  if (prop.major != 10 || prop.minor != 0) return POD_EUNSUPPORTED;  // built for sm_100a only

  pod_attn_ctx* c = new (std::nothrow) pod_attn_ctx();
  if (!c) return POD_ENOMEM;
  c->cfg = *cfg;
  c->device = cfg->device;
  c->num_sms = prop.multiProcessorCount;
  c->H = H;
  c->Hk = Hk;
  c->G = H / Hk;
  c->D = D;

  auto fail = [&](int code) {
    pod_attn_destroy(c);
    return code;
  };
  if (kernels_init(D) != cudaSuccess) return fail(POD_ECUDA);
  // Scheduling levers for ablations (POD-Attention §5.4): environment overrides.
  if (const char* e = std::getenv("POD_ATTN_POLICY")) {
    if (!std::strcmp(e, "even")) c->policy = 1;
    else if (!std::strcmp(e, "prefill_first")) c->policy = 2;
    else if (!std::strcmp(e, "decode_first")) c->policy = 3;
    else if (!std::strcmp(e, "front")) c->policy = 4;
    else if (!std::strcmp(e, "balanced")) c->policy = 5;
    else if (!std::strcmp(e, "proportional")) c->policy = 0;
  }
  if (const char* e = std::getenv("POD_ATTN_SMID_AWARE")) c->smid_aware = std::atoi(e) != 0;
  if (const char* e = std::getenv("POD_ATTN_DEC_TURN")) c->dec_turn = std::max(1, std::atoi(e));
  if (const char* e = std::getenv("POD_ATTN_PREFILL_SPLIT"))
  {
    // a negative count forces that many splits without the two-wave cap
    const int v = std::atoi(e);
    c->split_uncapped = v < 0;
    c->pre_split = std::max(0, std::min(kMaxPrefillSplit, v < 0 ? -v : v));
  }
  if (const char* e = std::getenv("POD_ATTN_TAIL_SPLIT_FUSED"))
    c->tail_split_fused = std::atoi(e) != 0;
  if (const char* e = std::getenv("POD_ATTN_DEC_SPLIT"))
    c->dec_split = std::max(0, std::atoi(e)) / dec_stage_keys(D) * dec_stage_keys(D);
  // The one-SM prefill tile serves every head_dim by default: it measured
  // faster than the CTA-pair tile on every hybrid workload of the benchmark
  // (the pair's single MMA-issuing thread sets its pace). The pair tile
  // (head_dim 128) is selected with POD_ATTN_PREFILL_TILE=pair; its
  // persistent launch uses every cluster of two that fits at once.
  if (D == 128) {
    const char* e = std::getenv("POD_ATTN_PREFILL_TILE");
    if (e && !std::strcmp(e, "pair")) {
      int clusters = 0;
      if (pair_max_clusters(&clusters) != cudaSuccess) return fail(POD_ECUDA);
      if (clusters >= 1) {
        c->use_pair = true;
        c->pair_clusters = clusters;
        // the pair's prefill tile is fast enough that its units go first:
        // decode streams beside them on every SM's side warps
        if (!std::getenv("POD_ATTN_POLICY")) c->policy = 2;
      }
    }
  }
  int dec_blocks = 0;
  if (decode_occupancy(D, &dec_blocks) != cudaSuccess || dec_blocks < 1) return fail(POD_ECUDA);
  c->decode_grid = c->num_sms * dec_blocks;

  size_context(c);

  if (cudaMalloc(&c->d_plan, c->plan_cap) != cudaSuccess) return fail(POD_ENOMEM);
  if (cudaMalloc(&c->d_ppart_o, sizeof(float) * (size_t)c->cap_pslots * kQTile * D) != cudaSuccess)
    return fail(POD_ENOMEM);
  if (cudaMalloc(&c->d_ppart_lse, sizeof(float) * (size_t)c->cap_pslots * kQTile) != cudaSuccess)
    return fail(POD_ENOMEM);
  if (cudaMalloc(&c->d_dpart_o, sizeof(float) * (size_t)c->cap_dslots * kMaxGroup * D) !=
      cudaSuccess)
    return fail(POD_ENOMEM);
  if (cudaMalloc(&c->d_dpart_lse, sizeof(float) * (size_t)c->cap_dslots * kMaxGroup) != cudaSuccess)
    return fail(POD_ENOMEM);
  if (cudaMalloc(&c->d_misc, 64) != cudaSuccess) return fail(POD_ENOMEM);
  if (cudaMemset(c->d_misc, 0, 64) != cudaSuccess) return fail(POD_ECUDA);
  if (cudaMemset(c->d_plan, 0, c->plan_cap) != cudaSuccess) return fail(POD_ECUDA);
  for (int i = 0; i < kRing; ++i) {
    if (cudaHostAlloc(reinterpret_cast<void**>(&c->h_plan[i]), c->plan_cap,
                      cudaHostAllocDefault) != cudaSuccess)
      return fail(POD_ENOMEM);
    std::memset(c->h_plan[i], 0, c->plan_cap);
    if (cudaEventCreateWithFlags(&c->h_ev[i], cudaEventDisableTiming) != cudaSuccess)
      return fail(POD_ECUDA);
  }
  if (cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking) != cudaSuccess)
    return fail(POD_ECUDA);
  if (cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming) != cudaSuccess)
    return fail(POD_ECUDA);
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                       &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return fail(POD_ECUDA);
  c->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  c->units_tmp.reserve(1024);
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(POD_ECUDA);
  *out = c;
  return POD_OK;
}

int pod_attn_hybrid(pod_attn_ctx* c, const pod_prefill_args* pa, const pod_decode_args* da,
                    int mode, void* stream) {
  if (!c) return POD_EINVAL;
  if (mode != POD_MODE_FUSED && mode != POD_MODE_SERIAL && mode != POD_MODE_TWO_STREAM)
    return POD_EINVAL;
  long long tp = 0;
  int rc = check_prefill(c, pa, &tp);
  if (rc) return rc;
  rc = check_decode(c, da);
  if (rc) return rc;
  DeviceGuard guard(c->device);
  if (!guard.ok) return POD_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Plan P;
  TmaDescs T;
  rc = stage_plan(c, pa, da, mode == POD_MODE_FUSED, s, &P, &T);
  if (rc) return rc;
  const bool has_p = P.n_prefill_units > 0, has_d = P.n_decode_units > 0;
  if (!has_p && !has_d) return POD_OK;
  if (mode == POD_MODE_FUSED) {
    if (run_fused(c, P, T, true, s) != cudaSuccess) return POD_ECUDA;
    return POD_OK;
  }
  if (mode == POD_MODE_SERIAL) {
    if (has_p && run_fused(c, P, T, false, s) != cudaSuccess) return POD_ECUDA;
    if (has_d && (launch_decode(P, c->decode_grid, s) != cudaSuccess || launch_merge(P, s) != cudaSuccess))
      return POD_ECUDA;
    return POD_OK;
  }
  // TWO_STREAM
  if (cudaEventRecord(c->ev_fork, s) != cudaSuccess) return POD_ECUDA;
  if (cudaStreamWaitEvent(c->side, c->ev_fork, 0) != cudaSuccess) return POD_ECUDA;
  if (has_p && run_fused(c, P, T, false, s) != cudaSuccess) return POD_ECUDA;
  if (has_d && (launch_decode(P, c->decode_grid, c->side) != cudaSuccess || launch_merge(P, c->side) != cudaSuccess))
    return POD_ECUDA;
  if (cudaEventRecord(c->ev_join, c->side) != cudaSuccess) return POD_ECUDA;
  if (cudaStreamWaitEvent(s, c->ev_join, 0) != cudaSuccess) return POD_ECUDA;
  return POD_OK;
}

int pod_attn_prefill_only(pod_attn_ctx* c, const pod_prefill_args* pa, void* stream) {
  if (!c) return POD_EINVAL;
  long long tp = 0;
  int rc = check_prefill(c, pa, &tp);
  if (rc) return rc;
  DeviceGuard guard(c->device);
  if (!guard.ok) return POD_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Plan P;
  TmaDescs T;
  rc = stage_plan(c, pa, nullptr, false, s, &P, &T);
  if (rc) return rc;
  if (P.n_prefill_units == 0) return POD_OK;
  return run_fused(c, P, T, false, s) == cudaSuccess ? POD_OK : POD_ECUDA;
}

int pod_attn_decode_only(pod_attn_ctx* c, const pod_decode_args* da, void* stream) {
  if (!c) return POD_EINVAL;
  int rc = check_decode(c, da);
  if (rc) return rc;
  DeviceGuard guard(c->device);
  if (!guard.ok) return POD_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Plan P;
  TmaDescs T;
  rc = stage_plan(c, nullptr, da, false, s, &P, &T);
  if (rc) return rc;
  if (P.n_decode_units == 0) return POD_OK;
  if (launch_decode(P, c->decode_grid, s) != cudaSuccess || launch_merge(P, s) != cudaSuccess) return POD_ECUDA;
  return POD_OK;
}

int pod_attn_status(pod_attn_ctx* c, void* stream) {
  if (!c) return POD_EINVAL;
  DeviceGuard guard(c->device);
  if (!guard.ok) return POD_ECUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return POD_ECUDA;
  int st = 0;
  if (cudaMemcpy(&st, c->d_misc, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return POD_ECUDA;
  if (cudaMemset(c->d_misc, 0, sizeof(int)) != cudaSuccess) return POD_ECUDA;
  return st;
}

int pod_attn_last_plan(const pod_attn_ctx* c, pod_plan_info* out) {
  if (!c || !out) return POD_EINVAL;
  *out = c->last;
  return POD_OK;
}

int pod_attn_get_stats(pod_attn_ctx* c, void* stream, pod_stats* out) {
  if (!c || !out) return POD_EINVAL;
  if (!(c->cfg.flags & POD_FLAG_STATS)) return POD_EINVAL;
  DeviceGuard guard(c->device);
  if (!guard.ok) return POD_ECUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return POD_ECUDA;
  std::vector<int> st(kStatsInts);
  if (cudaMemcpy(st.data(), c->d_plan + c->lay.stats, sizeof(int) * kStatsInts,
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return POD_ECUDA;
  std::memset(out, 0, sizeof(*out));
  out->num_sms = c->num_sms;
  for (int i = 0; i < kMaxSmid; ++i) {
    out->prefill_claims += st[2 * i];
    out->decode_claims += st[2 * i + 1];
    if (st[2 * i] > 0 && st[2 * i + 1] > 0) out->sms_with_both++;
  }
  return POD_OK;
}

int pod_attn_destroy(pod_attn_ctx* c) {
  if (!c) return POD_OK;
  int st = POD_OK;
  {
    DeviceGuard guard(c->device);
    if (cudaDeviceSynchronize() != cudaSuccess) st = POD_ECUDA;
    if (c->d_misc && st == POD_OK) {
      int v = 0;
      if (cudaMemcpy(&v, c->d_misc, sizeof(int), cudaMemcpyDeviceToHost) == cudaSuccess)
        st = v;
      else
        st = POD_ECUDA;
    }
    cudaFree(c->d_plan);
    cudaFree(c->d_ppart_o);
    cudaFree(c->d_ppart_lse);
    cudaFree(c->d_dpart_o);
    cudaFree(c->d_dpart_lse);
    cudaFree(c->d_misc);
    for (int i = 0; i < kRing; ++i) {
      if (c->h_plan[i]) cudaFreeHost(c->h_plan[i]);
      if (c->h_ev[i]) cudaEventDestroy(c->h_ev[i]);
    }
    if (c->side) cudaStreamDestroy(c->side);
    if (c->ev_fork) cudaEventDestroy(c->ev_fork);
    if (c->ev_join) cudaEventDestroy(c->ev_join);
  }
  delete c;
  return st;
}

}  // extern "C"
