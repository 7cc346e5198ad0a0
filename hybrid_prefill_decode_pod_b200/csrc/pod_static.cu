// pod_static.cu -- decode attention that allocates nothing (pod_attn_decode_static).
//
// Some callers cannot allocate device memory at call time: an inference
// engine that reserves nearly all HBM for its KV-cache pool up front (a
// further cudaMalloc fails or fragments that pool), a plugin that may only
// use the buffers its host framework hands it, or a latency-critical loop
// that cannot afford cudaMalloc's implicit device synchronisation. Creating a
// pod_attn context allocates its workspace, so this entry point runs the
// split-KV decode kernel and the LSE merge kernel with all of their scratch
// (plan tables, counters, split partial results) in the file-scope device
// array below instead. The caller still passes every input and output.
//
// The array lives in every GPU that loads the library until the process
// exits. Every call uses the same array and leaves its contents behind; each
// call re-initialises what must start at zero. Two calls that overlap on the
// GPU (different streams, or different host threads) race on it. A call whose
// decode warps gave up on a bounded device wait writes NaN to its outputs.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "pod_attn.h"
#include "pod_plan.h"

namespace pod {
cudaError_t kernels_init(int D);
cudaError_t decode_occupancy(int D, int* blocks_per_sm);
cudaError_t launch_decode(const Plan& P, int max_grid, cudaStream_t s);
cudaError_t launch_merge(const Plan& P, cudaStream_t s);
}  // namespace pod

using namespace pod;

namespace {

constexpr int kMaxReqs = POD_STATIC_MAX_DECODE_REQS;
constexpr int kMaxUnits = POD_STATIC_MAX_UNITS;
constexpr int kMaxKvHeads = POD_STATIC_MAX_KV_HEADS;
constexpr int kMaxDim = 128;

// Byte layout of the scratch array. The head part (control words, merge
// counters, request table) is rewritten by every call; the partial results
// are written before they are read. (A decode unit finds its request by a
// search of the requests' first-unit indices: there is no unit table.)
constexpr size_t kCtlOff = 0;                                        // 16 ints
constexpr size_t kGroupOff = 256;                                    // merge counters
constexpr size_t kReqOff = kGroupOff + sizeof(int) * kMaxReqs * kMaxKvHeads;
constexpr size_t kHeadBytes = kReqOff + sizeof(DecodeReq) * kMaxReqs;
constexpr size_t kLseOff = (kHeadBytes + 255) / 256 * 256;
constexpr size_t kPartOff = kLseOff + sizeof(float) * kMaxUnits * kMaxGroup;
constexpr size_t kScratchBytes = kPartOff + sizeof(float) * kMaxUnits * kMaxGroup * kMaxDim;

}  // namespace

// The scratch array itself: file scope, internal linkage. In host code its
// name is only a stand-in for the symbol; the device address comes from
// cudaGetSymbolAddress (setup_device below).
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

namespace {

// Host staging for the head part (copied with one cudaMemcpyAsync per call).
unsigned char g_host_head[kHeadBytes];

struct DeviceState {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_decode_scratch
  int decode_grid[2] = {0, 0};  // persistent decode grid for d = 64, d = 128
};
constexpr int kMaxDevices = 64;
DeviceState g_state[kMaxDevices];
std::mutex g_mu;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Once per device, with that device current: resolve the array's device
// address (the host-side symbol is only a stand-in) and set the kernels'
// shared-memory limits.
int setup_device(int dev, DeviceState** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_state[dev];
  if (!st.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return POD_ECUDA;
    if (kernels_init(64) != cudaSuccess || kernels_init(128) != cudaSuccess) return POD_ECUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return POD_ECUDA;
    for (int i = 0; i < 2; ++i) {
      int blocks = 0;
      if (decode_occupancy(i ? 128 : 64, &blocks) != cudaSuccess || blocks < 1) return POD_ECUDA;
      st.decode_grid[i] = sms * blocks;
    }
    st.scratch = static_cast<unsigned char*>(p);
    st.ready = true;
  }
  *out = &st;
  return POD_OK;
}

}  // namespace

extern "C" POD_API int pod_attn_decode_static(int num_qo_heads, int num_kv_heads, int head_dim,
                                              int kv_layout, const pod_decode_args* a,
                                              void* stream) {
  const int H = num_qo_heads, Hk = num_kv_heads, D = head_dim;
  if (!a) return POD_EINVAL;
  if (H <= 0 || Hk <= 0 || H % Hk != 0) return POD_EINVAL;
  if (D != 64 && D != 128) return POD_EUNSUPPORTED;
  if (H / Hk > kMaxGroup) return POD_EUNSUPPORTED;
  if (kv_layout != POD_KV_CONTIGUOUS && kv_layout != POD_KV_PAGED) return POD_EINVAL;
  const bool paged = kv_layout == POD_KV_PAGED;
  if (a->num_reqs < 0) return POD_EINVAL;
  if (a->num_reqs == 0) return POD_OK;
  if (a->num_reqs > kMaxReqs || Hk > kMaxKvHeads || (long long)a->num_reqs * Hk > kMaxUnits)
    return POD_ECAPACITY;
  if (!a->ctx_lens || !a->q || !a->o || !a->lse) return POD_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->o) || (reinterpret_cast<uintptr_t>(a->lse) & 3u))
    return POD_EINVAL;
  for (int i = 0; i < a->num_reqs; ++i)
    if (a->ctx_lens[i] < 1 || a->ctx_lens[i] > (1 << 30)) return POD_EINVAL;
  if (!paged) {
    if (!a->k_ptrs || !a->v_ptrs) return POD_EINVAL;
    for (int i = 0; i < a->num_reqs; ++i)
      if (!a->k_ptrs[i] || !a->v_ptrs[i] || !aligned16(a->k_ptrs[i]) || !aligned16(a->v_ptrs[i]))
        return POD_EINVAL;
  } else {
    if (!a->k_pool || !a->v_pool || !a->block_table || a->pool_blocks <= 0) return POD_EINVAL;
    if (!aligned16(a->k_pool) || !aligned16(a->v_pool)) return POD_EINVAL;
    for (int i = 0; i < a->num_reqs; ++i)
      if (a->block_table_stride < (a->ctx_lens[i] + 15) / 16) return POD_EINVAL;
  }

  // keys per split: at least 512, doubled until the units fit the array
  int split_len = 512;
  auto units_for = [&](int sl) {
    long long n = 0;
    for (int r = 0; r < a->num_reqs; ++r) n += (long long)((a->ctx_lens[r] + sl - 1) / sl) * Hk;
    return n;
  };
  while (units_for(split_len) > kMaxUnits) split_len *= 2;  // ends: num_reqs * Hk <= max units

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The per-call plan is copied from one shared host buffer that the next
  // call overwrites, so a captured copy would replay whatever plan the latest
  // call left there: refuse while the stream is being captured.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return POD_ECUDA;
  if (cap != cudaStreamCaptureStatusNone) return POD_EUNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return POD_ECUDA;
  DeviceState* st = nullptr;
  int rc = setup_device(dev, &st);
  if (rc) return rc;

  // head part of the scratch: zeroed control words and merge counters, then
  // the request table
  std::lock_guard<std::mutex> lk(g_mu);
  std::memset(g_host_head, 0, kReqOff);
  DecodeReq* req = reinterpret_cast<DecodeReq*>(g_host_head + kReqOff);
  int n_units = 0, n_groups = 0, n_slots = 0;
  for (int r = 0; r < a->num_reqs; ++r) {
    DecodeReq& R = req[r];
    std::memset(&R, 0, sizeof(R));
    R.k = paged ? nullptr : static_cast<const uint16_t*>(a->k_ptrs[r]);
    R.v = paged ? nullptr : static_cast<const uint16_t*>(a->v_ptrs[r]);
    R.len = a->ctx_lens[r];
    R.n_split = (R.len + split_len - 1) / split_len;
    R.unit0 = n_units;
    R.bt_row = r;
    if (R.n_split > 1) {
      R.group0 = n_groups;
      R.slot0 = n_slots;
      n_groups += Hk;
      n_slots += R.n_split * Hk;
    }
    n_units += R.n_split * Hk;
  }
  const size_t head_bytes = kReqOff + sizeof(DecodeReq) * (size_t)a->num_reqs;
  if (cudaMemcpyAsync(st->scratch, g_host_head, head_bytes, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return POD_ECUDA;

  Plan P;
  std::memset(&P, 0, sizeof(P));
  P.H = H;
  P.Hk = Hk;
  P.G = H / Hk;
  P.D = D;
  P.scale_log2 = 1.4426950408889634f / (D == 128 ? 11.313708498984761f : 8.0f);
  P.n_decode_units = n_units;
  P.n_decode_reqs = a->num_reqs;
  P.dec_split_len = split_len;
  P.paged = paged ? 1 : 0;
  P.bt_stride_d = paged ? a->block_table_stride : 0;
  P.pool_blocks = paged ? (int)(a->pool_blocks < (1LL << 30) ? a->pool_blocks : (1LL << 30)) : 0;
  P.wait_budget = kDefaultWaitBudget;
  // The status word lives in the zeroed head of the array: if a decode warp
  // gives up on a bounded wait in this call, the merge launch writes NaN to
  // every output row instead of merging partials that are incomplete or left
  // over from an earlier call.
  P.flags = kFlagPoisonOnStatus;
  P.dreq = reinterpret_cast<const DecodeReq*>(st->scratch + kReqOff);
  P.q_d = static_cast<const uint16_t*>(a->q);
  P.o_d = static_cast<uint16_t*>(a->o);
  P.lse_d = a->lse;
  P.bt_d = paged ? a->block_table : nullptr;
  P.k_pool = paged ? static_cast<const uint16_t*>(a->k_pool) : nullptr;
  P.v_pool = paged ? static_cast<const uint16_t*>(a->v_pool) : nullptr;
  P.dpart_o = reinterpret_cast<float*>(st->scratch + kPartOff);
  P.dpart_lse = reinterpret_cast<float*>(st->scratch + kLseOff);
  P.ctl = reinterpret_cast<int*>(st->scratch + kCtlOff);
  P.status = reinterpret_cast<int*>(st->scratch + kCtlOff) + 8;
  P.dgroup_ctr = reinterpret_cast<int*>(st->scratch + kGroupOff);
  if (launch_decode(P, st->decode_grid[D == 128 ? 1 : 0], s) != cudaSuccess) return POD_ECUDA;
  if (launch_merge(P, s) != cudaSuccess) return POD_ECUDA;
  return POD_OK;
}
