// planner_harness.cpp -- runs the host planner of libpod_attn without a GPU.
//
// Test infrastructure: includes the library's API translation unit, builds a
// context by hand (no device allocation, a stand-in tensor-map encoder that
// only checks its arguments), plans one call described on the command line
// and prints the plan as JSON for tests/test_planner.py. The kernels are not
// linked; the stubs below fail loudly if anything tries to launch one.
//
// Usage: planner_harness H Hk D sms decode_grid policy fused pre_split dec_split
//                        paged "prior:chunk,..." "len,..." max_prefill_tokens
//                        max_decode_reqs max_kv_tokens pair_clusters
// (pair_clusters 0: prefill units on one SM each; else on that many CTA pairs)
#include "pod_attn_api.cpp"

#include <cstdio>
#include <string>

namespace pod {
cudaError_t kernels_init(int) { return cudaErrorNotSupported; }
int fused_smem_bytes(int) { return 0; }
int decode_smem_bytes(int) { return 0; }
cudaError_t launch_fused(const Plan&, const TmaDescs&, int, int, int, cudaStream_t) {
  std::abort();
}
cudaError_t launch_decode(const Plan&, int, cudaStream_t) { std::abort(); }
cudaError_t decode_occupancy(int, int*) { return cudaErrorNotSupported; }
cudaError_t launch_merge(const Plan&, cudaStream_t) { std::abort(); }
cudaError_t pair_max_clusters(int*) { return cudaErrorNotSupported; }
cudaError_t launch_fused_pair(const Plan&, const TmaDescs&, int, int, int, cudaStream_t) {
  std::abort();
}
}  // namespace pod

static int g_maps = 0;
static std::vector<int> g_boxes;  // rows per box of each map, in encoding order
static CUresult fake_encode(CUtensorMap*, CUtensorMapDataType dt, cuuint32_t rank, void* base,
                            const cuuint64_t* dims, const cuuint64_t* strides,
                            const cuuint32_t* box, const cuuint32_t*, CUtensorMapInterleave,
                            CUtensorMapSwizzle sw, CUtensorMapL2promotion, CUtensorMapFloatOOBfill) {
  ++g_maps;
  // the kernels rely on these: bf16, 3-D, 128-byte swizzle over 64-column boxes,
  // 16-byte-aligned base and strides
  if (dt != CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 || rank != 3 || sw != CU_TENSOR_MAP_SWIZZLE_128B)
    return CUDA_ERROR_INVALID_VALUE;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (strides[0] & 15u) || (strides[1] & 15u))
    return CUDA_ERROR_INVALID_VALUE;
  if (box[0] != 64 || box[1] != 1 || dims[0] % 64) return CUDA_ERROR_INVALID_VALUE;
  if (box[2] != 16 && box[2] != 64 && box[2] != 128) return CUDA_ERROR_INVALID_VALUE;
  g_boxes.push_back((int)box[2]);
  return CUDA_SUCCESS;
}

static std::vector<long long> parse_list(const std::string& s) {
  std::vector<long long> v;
  size_t i = 0;
  while (i < s.size()) {
    size_t j = s.find_first_of(",:", i);
    if (j == std::string::npos) j = s.size();
    if (j > i) v.push_back(std::stoll(s.substr(i, j - i)));
    i = j + 1;
  }
  return v;
}

int main(int argc, char** argv) {
  if (argc != 17) {
    std::fprintf(stderr, "expected 16 arguments\n");
    return 2;
  }
  pod_attn_ctx c;
  c.H = std::atoi(argv[1]);
  c.Hk = std::atoi(argv[2]);
  c.G = c.H / c.Hk;
  c.D = std::atoi(argv[3]);
  c.num_sms = std::atoi(argv[4]);
  c.decode_grid = std::atoi(argv[5]);
  c.policy = std::atoi(argv[6]);
  const bool fused = std::atoi(argv[7]) != 0;
  c.pre_split = std::atoi(argv[8]);
  c.dec_split = std::atoi(argv[9]);
  const bool paged = std::atoi(argv[10]) != 0;
  const std::vector<long long> pre = parse_list(argv[11]);
  const std::vector<long long> dec = parse_list(argv[12]);
  c.cfg.num_qo_heads = c.H;
  c.cfg.num_kv_heads = c.Hk;
  c.cfg.head_dim = c.D;
  c.cfg.kv_layout = paged ? POD_KV_PAGED : POD_KV_CONTIGUOUS;
  c.cfg.page_size = 16;
  c.cfg.max_prefill_tokens = std::atoll(argv[13]);
  c.cfg.max_prefill_reqs = kMaxPrefillReqs;
  c.cfg.max_decode_reqs = std::atoi(argv[14]);
  c.cfg.max_kv_tokens = std::atoll(argv[15]);
  c.pair_clusters = std::atoi(argv[16]);
  c.use_pair = c.pair_clusters > 0;
  c.encode = fake_encode;
  size_context(&c);
  c.units_tmp.reserve(1024);
  std::vector<char> h(c.plan_cap + 64), dplan(c.plan_cap + 64);
  c.d_plan = dplan.data();  // only a base address here: the planner never dereferences it

  // arguments with stand-in device addresses (16-byte aligned, never touched)
  const int np = (int)pre.size() / 2, nd = (int)dec.size();
  std::vector<int> chunk(np), prior(np), ctx(nd);
  std::vector<const void*> kp(np + nd), vp(np + nd);
  long long total_q = 0, max_blocks = 1;
  for (int i = 0; i < np; ++i) {
    prior[i] = (int)pre[2 * i];
    chunk[i] = (int)pre[2 * i + 1];
    total_q += chunk[i];
    max_blocks = std::max(max_blocks, (long long)(prior[i] + chunk[i] + 15) / 16);
  }
  for (int i = 0; i < nd; ++i) {
    ctx[i] = (int)dec[i];
    max_blocks = std::max(max_blocks, (long long)(ctx[i] + 15) / 16);
  }
  for (int i = 0; i < np + nd; ++i) {
    kp[i] = reinterpret_cast<const void*>((uintptr_t)(0x100000 + 0x1000 * i));
    vp[i] = reinterpret_cast<const void*>((uintptr_t)(0x900000 + 0x1000 * i));
  }
  void* const any = reinterpret_cast<void*>((uintptr_t)0x40000);
  pod_prefill_args pa{};
  pa.num_reqs = np;
  pa.chunk_lens = chunk.data();
  pa.prior_lens = prior.data();
  pa.q = any;
  pa.o = any;
  pa.lse = static_cast<float*>(any);
  pod_decode_args da{};
  da.num_reqs = nd;
  da.ctx_lens = ctx.data();
  da.q = any;
  da.o = any;
  da.lse = static_cast<float*>(any);
  if (paged) {
    pa.k_pool = pa.v_pool = da.k_pool = da.v_pool = any;
    pa.block_table = da.block_table = static_cast<const int*>(any);
    pa.block_table_stride = da.block_table_stride = (int)max_blocks;
    pa.pool_blocks = da.pool_blocks = max_blocks * (np + nd);
  } else {
    pa.k_ptrs = kp.data();
    pa.v_ptrs = vp.data();
    da.k_ptrs = kp.data() + np;
    da.v_ptrs = vp.data() + np;
  }
  long long tq = 0;
  int rc = np ? check_prefill(&c, &pa, &tq) : POD_OK;
  if (rc == POD_OK && nd) rc = check_decode(&c, &da);
  Plan P;
  TmaDescs T;
  size_t bytes = 0;
  if (rc == POD_OK)
    rc = build_plan(&c, np ? &pa : nullptr, nd ? &da : nullptr, fused, h.data(), &P, &T, &bytes);

  std::printf("{\"status\": %d", rc);
  if (rc == POD_OK) {
    // the plan's device pointers are offsets from the stand-in buffer base,
    // and the host slot has the same layout
    auto at = [&](const void* dev) { return h.data() + ((const char*)dev - c.d_plan); };
    const PrefillReq* preq = reinterpret_cast<const PrefillReq*>(at(P.preq));
    const PrefillUnit* pu = reinterpret_cast<const PrefillUnit*>(at(P.punits));
    const DecodeReq* dreq = reinterpret_cast<const DecodeReq*>(at(P.dreq));
    // every table lies inside the bytes the call copies, and the zeroed words
    // (queue heads, tickets, merge counters) are zero
    const size_t ends[3] = {(size_t)((const char*)(P.preq + np) - c.d_plan),
                            (size_t)((const char*)(P.punits + P.n_prefill_units) - c.d_plan),
                            (size_t)((const char*)(P.dreq + nd) - c.d_plan)};
    bool inside = true;
    for (size_t e : ends) inside = inside && e <= bytes && e <= c.plan_cap;
    bool zeroed = true;
    for (size_t i = 0; i < (size_t)((const char*)P.preq - c.d_plan); ++i) zeroed = zeroed && !h[i];
    std::printf(", \"tables_inside_copy\": %s, \"counters_zeroed\": %s", inside ? "true" : "false",
                zeroed ? "true" : "false");
    std::printf(", \"slots\": %d, \"flags\": %d, \"p_cap\": %d, \"rho\": [%d, %d]",
                c.use_pair ? c.pair_clusters : c.num_sms * c.slots_per_sm, P.flags, P.p_cap,
                P.rho_num, P.rho_den);
    std::printf(", \"boxes\": [");
    for (size_t i = 0; i < g_boxes.size(); ++i) std::printf("%s%d", i ? ", " : "", g_boxes[i]);
    std::printf("]");
    std::printf(", \"plan_bytes\": %zu, \"maps\": %d, \"dec_split_len\": %d", bytes, g_maps,
                P.dec_split_len);
    std::printf(", \"caps\": {\"punits\": %d, \"pgroups\": %d, \"pslots\": %d, \"dunits\": %d}",
                c.cap_punits, c.cap_pgroups, c.cap_pslots, c.cap_dunits);
    std::printf(", \"preq\": [");
    for (int i = 0; i < np; ++i)
      std::printf("%s{\"prior\": %d, \"chunk\": %d, \"q_row0\": %d, \"n_qtiles\": %d, "
                  "\"kv_len\": %d, \"n_split\": %d, \"pair_heads\": %d}",
                  i ? ", " : "", preq[i].prior, preq[i].chunk, preq[i].q_row0, preq[i].n_qtiles,
                  preq[i].kv_len, preq[i].n_split, preq[i].pair_heads);
    std::printf("], \"punits\": [");
    for (int u = 0; u < P.n_prefill_units; ++u)
      std::printf("%s[%d, %d, %d, %d, %d, %d, %d, %d]", u ? ", " : "", pu[u].req, pu[u].head,
                  pu[u].qtile, pu[u].split, pu[u].n_split, pu[u].group0, pu[u].slot0,
                  pu[u].work);
    std::printf("], \"dreq\": [");
    for (int i = 0; i < nd; ++i)
      std::printf("%s{\"len\": %d, \"n_split\": %d, \"unit0\": %d, \"group0\": %d, \"slot0\": %d}",
                  i ? ", " : "", dreq[i].len, dreq[i].n_split, dreq[i].unit0, dreq[i].group0,
                  dreq[i].slot0);
    // the request of each decode unit, by the rule the kernel applies (the
    // last request whose first unit is <= u)
    std::printf("], \"dunit\": [");
    for (int u = 0, r = 0; u < P.n_decode_units; ++u) {
      while (r + 1 < nd && dreq[r + 1].unit0 <= u) ++r;
      std::printf("%s%d", u ? ", " : "", r);
    }
    std::printf("]");
  }
  std::printf("}\n");
  return 0;
}
