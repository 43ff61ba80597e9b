// api.cu -- the exported C ABI of libddt.so: host-side validation, workspace
// layout and dispatch to the stage kernels.  See include/ddt.h.
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "attn_common.cuh"
#include "ddt.h"
#include "launch.h"

namespace ddt {

// Opt a kernel in to `bytes` of dynamic shared memory when its static plus
// dynamic shared memory exceeds the 48 KB a launch gets by default.
cudaError_t ensure_smem_attr(const void* func, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;      // dynamic bytes opted in
  static std::map<std::pair<const void*, int>, size_t> static_of;  // static bytes of the kernel
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(func, dev);
  auto st = static_of.find(key);
  if (st == static_of.end()) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, func);
    if (e != cudaSuccess) return e;
    st = static_of.emplace(key, fa.sharedSizeBytes).first;
  }
  if (st->second + bytes <= 48 * 1024) return cudaSuccess;
  size_t& have = done[key];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

int device_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  return n > 0 ? n : 148;
}

namespace {
constexpr long long kDefaultWaitCycles = 2000000000LL;  // about one second at 1.9 GHz
std::atomic<long long> g_wait_override{0};
}  // namespace

std::atomic<int> g_attn_kernel{0};

int attn_kernel_choice() { return g_attn_kernel.load(std::memory_order_relaxed); }

long long wait_limit_cycles() {
  const long long v = g_wait_override.load(std::memory_order_relaxed);
  return v > 0 ? v : kDefaultWaitCycles;
}

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int sm_count() { return device_sm_count(); }

bool ws_ok(const void* ws, size_t have, size_t need) {
  if (need == 0) return true;
  return ws != nullptr && have >= need && ((uintptr_t)ws & 255u) == 0;
}

}  // namespace

ddt_status launch_attn_simt(AttnParams& p, cudaStream_t stream);
int attn_simt_rows_per_cta();
bool attn_tc_eligible(const ddt_attn_args* a);
void attn_tc_plan(const ddt_attn_args* a, int sms, int* qtiles, int* nsplit, int* tps);
bool attn_tc_cluster(int nsplit, long clusters);
bool attn_pair_plan(const ddt_attn_args* a, int sms, int* qtiles, int* nsplit, int* tps);
size_t attn_tc_workspace_size(const ddt_attn_args* a, int sms);
ddt_status launch_attn_tc(const ddt_attn_args* a, void* ws, int sms, cudaStream_t stream);

// KV-split plan shared by the workspace query and the launch.
static void attn_plan(const ddt_attn_args* a, int rows_per_cta, int* row_tiles, int* nsplit,
                      int* tps) {
  const int g = a->hq / a->hkv;
  const int R = a->n_max * g;
  *row_tiles = (R + rows_per_cta - 1) / rows_per_cta;
  const long groups = (long)a->batch * a->hkv;
  const long base = (long)*row_tiles * groups;
  const int max_split = a->max_ctx > 0 ? (a->max_ctx + 63) / 64 : 1;
  const long target = 2L * sm_count();
  long ns = (target + base - 1) / (base > 0 ? base : 1);
  if (ns < 1) ns = 1;
  if (ns > max_split) ns = max_split;
  int t = a->max_ctx > 0 ? (int)((a->max_ctx + ns - 1) / ns) : 64;
  t = (t + 63) / 64 * 64;
  *tps = t;
  *nsplit = a->max_ctx > 0 ? (a->max_ctx + t - 1) / t : 1;
}

size_t attn_workspace_size(const ddt_attn_args* a) {
  if (attn_tc_eligible(a)) {
    const size_t n = attn_tc_workspace_size(a, sm_count());
    return n ? (size_t)DDT_WS_COUNTER_BYTES + n : 0;
  }
  int rt, ns, tps;
  attn_plan(a, attn_simt_rows_per_cta(), &rt, &ns, &tps);
  if (ns <= 1) return 0;
  const size_t groups = (size_t)a->batch * a->hkv;
  const size_t R = (size_t)a->n_max * (a->hq / a->hkv);
  return (size_t)DDT_WS_COUNTER_BYTES + align256(sizeof(float2) * groups * ns * R) +
         align256(sizeof(float) * groups * ns * R * a->d);
}

// Counters the CUDA-core attention needs (one ticket per row tile and kv head).
static size_t attn_simt_counters(const ddt_attn_args* a) {
  int rt, ns, tps;
  attn_plan(a, attn_simt_rows_per_cta(), &rt, &ns, &tps);
  return ns > 1 ? (size_t)a->batch * a->hkv * rt : 0;
}

ddt_status launch_attn(const ddt_attn_args* a, void* ws, size_t ws_bytes, cudaStream_t stream) {
  AttnParams p;
  p.q = (const uint16_t*)a->q;
  p.kc = (const uint16_t*)a->k_cache;
  p.vc = (const uint16_t*)a->v_cache;
  p.kt = (const uint16_t*)a->k_tree;
  p.vt = (const uint16_t*)a->v_tree;
  p.page_table = a->page_table;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages;
  p.t_max = a->t_max;
  p.ctx_len = a->ctx_len;
  p.max_ctx = a->max_ctx;
  p.mask = a->mask;
  p.n_nodes = a->n_nodes;
  p.batch = a->batch;
  p.n_max = a->n_max;
  p.hq = a->hq;
  p.hkv = a->hkv;
  p.d = a->d;
  p.g = a->hq / a->hkv;
  p.W = (a->n_max + 31) / 32;
  p.scale_log2 = a->scale * kLog2e;
  p.out = (uint16_t*)a->out;
  p.lse_out = a->lse_out;
  p.status = a->dev_status;
  if (a->batch == 0) return DDT_OK;
  if (attn_tc_eligible(a))
    return launch_attn_tc(a, ws ? (char*)ws + DDT_WS_COUNTER_BYTES : nullptr, sm_count(), stream);
  attn_plan(a, attn_simt_rows_per_cta(), &p.row_tiles, &p.nsplit, &p.tok_per_split);
  const size_t groups = (size_t)a->batch * a->hkv;
  const size_t R = (size_t)a->n_max * p.g;
  char* w = (char*)ws;
  p.tickets = (unsigned*)w;  // counter region
  if (p.nsplit > 1) {
    w += DDT_WS_COUNTER_BYTES;
    p.part_ml = (float2*)w;
    w += align256(sizeof(float2) * groups * p.nsplit * R);
    p.part_o = (float*)w;
  } else {
    p.part_ml = nullptr;
    p.part_o = nullptr;
  }
  return launch_attn_simt(p, stream);
}

}  // namespace ddt

namespace ddt {
// Every check of ddt_topk's arguments but the workspace's (shared with the
// allocation-free entry point, so that both return the same codes).
ddt_status topk_check(const void* logits, ddt_dtype dtype, int batch, int L, int V,
                      int64_t row_stride, int k, float inv_temperature, const int32_t* ids,
                      const float* zk, const float* lse) {
  if (batch < 0 || L < 0 || V < 1 || k < 1 || row_stride < V) return DDT_ERR_INVALID_ARG;
  if (dtype != DDT_BF16 && dtype != DDT_F32) return DDT_ERR_UNSUPPORTED;
  if (k > DDT_TOPK_K_MAX) return DDT_ERR_UNSUPPORTED;
  if (k > V) return DDT_ERR_INVALID_ARG;
  if (!(inv_temperature > 0.f) || !(inv_temperature < INFINITY)) return DDT_ERR_INVALID_ARG;
  const long rows = (long)batch * L;
  if (rows > 65535) return DDT_ERR_UNSUPPORTED;
  if (rows > 0 && (!logits || !ids || !zk || !lse)) return DDT_ERR_INVALID_ARG;
  return DDT_OK;
}
}  // namespace ddt

using namespace ddt;

namespace {
// An NVTX range around each launching entry point, so that a timeline
// (Nsight Systems, ncu's range filters) shows the library's calls by name.
// Without a tool attached the push and pop cost a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace

extern "C" {

const char* ddt_status_string(ddt_status s) {
  switch (s) {
    case DDT_OK: return "DDT_OK";
    case DDT_ERR_INVALID_ARG: return "DDT_ERR_INVALID_ARG: invalid argument";
    case DDT_ERR_UNSUPPORTED: return "DDT_ERR_UNSUPPORTED: outside the implemented range";
    case DDT_ERR_WORKSPACE: return "DDT_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case DDT_ERR_CUDA: return "DDT_ERR_CUDA: a CUDA call failed";
    case DDT_ERR_TIMEOUT: return "DDT_ERR_TIMEOUT: a bounded device wait gave up";
  }
  return "unknown ddt_status";
}

int ddt_mask_words(int n_max) { return n_max > 0 ? (n_max + 31) / 32 : 0; }

long long ddt_debug_set_wait_limit(long long cycles) {
  return g_wait_override.exchange(cycles > 0 ? cycles : 0);
}

int ddt_debug_set_attn_kernel(int which) {
  if (which < 0 || which > 2) return -1;
  return g_attn_kernel.exchange(which);
}

size_t ddt_topk_workspace_size(int batch, int L, int V, int k) {
  if (batch < 0 || L < 0 || V < 1 || k < 1) return 0;
  return topk_workspace_size(batch * L, V, k);
}

ddt_status ddt_topk(const void* logits, ddt_dtype dtype, int batch, int L, int V,
                    int64_t row_stride, int k, float inv_temperature, int32_t* ids, float* zk,
                    float* logp, float* lse, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream) {
  const NvtxRange nvtx("ddt_topk");
  const ddt_status st =
      topk_check(logits, dtype, batch, L, V, row_stride, k, inv_temperature, ids, zk, lse);
  if (st != DDT_OK) return st;
  const long rows = (long)batch * L;
  if (!ws_ok(workspace, workspace_bytes, topk_workspace_size((int)rows, V, k)))
    return DDT_ERR_WORKSPACE;
  return launch_topk(logits, dtype, (int)rows, V, row_stride, k, inv_temperature, ids, zk, logp,
                     lse, workspace, workspace_bytes, stream);
}

ddt_status ddt_build_tree(const int32_t* ids, const float* zk, const float* lse, int batch, int L,
                          int k, float inv_temperature, const int32_t* k_per_seq,
                          const int32_t* budget_per_seq, int B_max, const int32_t* root_token,
                          const int32_t* ctx_len, int32_t* tok, int32_t* parent, int32_t* depth,
                          int32_t* pos, uint32_t* mask, int32_t* n_nodes, double* surrogate,
                          int32_t* dev_status, cudaStream_t stream) {
  const NvtxRange nvtx("ddt_build_tree");
  if (batch < 0 || L < 1 || k < 1 || B_max < 0) return DDT_ERR_INVALID_ARG;
  if (L > DDT_TREE_L_MAX || k > DDT_TOPK_K_MAX || B_max > DDT_TREE_B_MAX) return DDT_ERR_UNSUPPORTED;
  if (!(inv_temperature > 0.f) || !(inv_temperature < INFINITY)) return DDT_ERR_INVALID_ARG;
  if (batch > 65535) return DDT_ERR_UNSUPPORTED;
  if (batch > 0 && (!ids || !zk || !lse || !root_token || !tok || !parent || !depth || !pos ||
                    !mask || !n_nodes))
    return DDT_ERR_INVALID_ARG;
  return launch_build_tree(ids, zk, lse, batch, L, k, inv_temperature, k_per_seq, budget_per_seq,
                           B_max, root_token, ctx_len, tok, parent, depth, pos, mask, n_nodes,
                           surrogate, dev_status, stream);
}

ddt_status ddt_plan_budget(const int32_t* tok, const int32_t* parent, const int32_t* depth,
                           const int32_t* n_nodes, const int32_t* ids, const float* zk,
                           const float* lse, int batch, int L, int k, int n_max,
                           float inv_temperature, int total_budget, double cost_fixed,
                           double cost_per_node, int32_t* budget_per_seq, double* expected_tokens,
                           int32_t* dev_status, cudaStream_t stream) {
  const NvtxRange nvtx("ddt_plan_budget");
  if (batch < 0 || L < 1 || k < 1 || n_max < 1) return DDT_ERR_INVALID_ARG;
  if (L > DDT_TREE_L_MAX || k > DDT_TOPK_K_MAX || n_max > DDT_TREE_B_MAX + 1)
    return DDT_ERR_UNSUPPORTED;
  if ((int64_t)batch * (n_max - 1) > plan_budget_max_nodes()) return DDT_ERR_UNSUPPORTED;
  if (!(inv_temperature > 0.f) || !(inv_temperature < INFINITY)) return DDT_ERR_INVALID_ARG;
  if (!(cost_fixed >= 0.0) || !(cost_fixed < INFINITY) || !(cost_per_node < INFINITY) ||
      cost_per_node != cost_per_node)
    return DDT_ERR_INVALID_ARG;
  if (cost_per_node > 0.0 && !(cost_fixed > 0.0)) return DDT_ERR_INVALID_ARG;
  if (batch > 0 && (!tok || !parent || !depth || !n_nodes || !ids || !zk || !lse ||
                    !budget_per_seq))
    return DDT_ERR_INVALID_ARG;
  return launch_plan_budget(tok, parent, depth, n_nodes, ids, zk, lse, batch, L, k, n_max,
                            inv_temperature, total_budget, cost_fixed, cost_per_node,
                            budget_per_seq, expected_tokens, dev_status, stream);
}

static ddt_status check_attn(const ddt_attn_args* a) {
  if (!a) return DDT_ERR_INVALID_ARG;
  if (a->batch < 0 || a->n_max < 1 || a->hq < 1 || a->hkv < 1 || a->max_ctx < 0)
    return DDT_ERR_INVALID_ARG;
  if (a->hq % a->hkv != 0) return DDT_ERR_INVALID_ARG;
  if (a->d != 64 && a->d != 128) return DDT_ERR_UNSUPPORTED;
  if (a->n_max > DDT_TREE_B_MAX + 1) return DDT_ERR_UNSUPPORTED;
  if (a->batch > 65535) return DDT_ERR_UNSUPPORTED;
  if (!(a->scale > 0.f) || !(a->scale < INFINITY)) return DDT_ERR_INVALID_ARG;
  if (a->batch == 0) return DDT_OK;
  if (!a->q || !a->k_tree || !a->v_tree || !a->mask || !a->n_nodes || !a->ctx_len || !a->out)
    return DDT_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k_tree) || !aligned16(a->v_tree) || !aligned16(a->out))
    return DDT_ERR_INVALID_ARG;
  if (a->max_ctx > 0) {
    if (!a->k_cache || !a->v_cache) return DDT_ERR_INVALID_ARG;
    if (!aligned16(a->k_cache) || !aligned16(a->v_cache)) return DDT_ERR_INVALID_ARG;
    if (a->page_table) {
      if (a->page_size < 16 || a->page_size % 16 != 0) return DDT_ERR_UNSUPPORTED;
      if ((long)a->max_pages * a->page_size < a->max_ctx) return DDT_ERR_INVALID_ARG;
      if (a->num_pages < 0) return DDT_ERR_INVALID_ARG;
    } else if (a->t_max < a->max_ctx) {
      return DDT_ERR_INVALID_ARG;
    }
  }
  return DDT_OK;
}

size_t ddt_tree_attn_workspace_size(const ddt_attn_args* a) {
  if (check_attn(a) != DDT_OK) return 0;
  return attn_workspace_size(a);
}

static const size_t kMaxCounters = DDT_WS_COUNTER_BYTES / sizeof(unsigned);

ddt_status ddt_tree_attn(const ddt_attn_args* a, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
  const NvtxRange nvtx("ddt_tree_attn");
  const ddt_status st = check_attn(a);
  if (st != DDT_OK) return st;
  if (!attn_tc_eligible(a) && attn_simt_counters(a) > kMaxCounters) return DDT_ERR_UNSUPPORTED;
  if (!ws_ok(workspace, workspace_bytes, attn_workspace_size(a))) return DDT_ERR_WORKSPACE;
  return launch_attn(a, workspace, workspace_bytes, stream);
}

ddt_status ddt_tree_attn_plan(const ddt_attn_args* a, int* path, int* kv_splits) {
  const ddt_status st = check_attn(a);
  if (st != DDT_OK) return st;
  int pth, ns;
  if (attn_tc_eligible(a)) {
    int qt, tps;
    if (attn_pair_plan(a, sm_count(), &qt, &ns, &tps)) {
      pth = ns <= 1 ? DDT_ATTN_PATH_TC_PAIRS : DDT_ATTN_PATH_TC_PAIRS_COMBINE;
    } else {
      attn_tc_plan(a, sm_count(), &qt, &ns, &tps);
      if (ns <= 1) pth = DDT_ATTN_PATH_TC;
      else if (attn_tc_cluster(ns, (long)qt * a->batch * a->hkv)) pth = DDT_ATTN_PATH_TC_CLUSTER;
      else pth = DDT_ATTN_PATH_TC_COMBINE;
    }
  } else {
    int rt, tps;
    attn_plan(a, attn_simt_rows_per_cta(), &rt, &ns, &tps);
    pth = DDT_ATTN_PATH_SIMT;
  }
  if (path) *path = pth;
  if (kv_splits) *kv_splits = ns;
  return DDT_OK;
}

size_t ddt_tree_walk_workspace_size(int batch, int n_max, int V) {
  if (batch < 0 || n_max < 1 || V < 1) return 0;
  return walk_workspace_size(batch, n_max, V);
}

namespace {
ddt_status walk_common(const void* logits, ddt_dtype dtype, int batch, int n_max, int V,
                       int64_t row_stride, const int32_t* tok, const int32_t* parent,
                       const int32_t* depth, const int32_t* n_nodes, int L, int mode,
                       int32_t* acc_len, int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status,
                       cudaStream_t stream, const WalkSampling* sampling) {
  if (batch < 0 || n_max < 1 || V < 1 || row_stride < V || L < 0) return DDT_ERR_INVALID_ARG;
  if (mode != DDT_WALK_ALL_ROWS && mode != DDT_WALK_LAZY && mode != DDT_WALK_AUTO)
    return DDT_ERR_INVALID_ARG;
  if (dtype != DDT_BF16 && dtype != DDT_F32) return DDT_ERR_UNSUPPORTED;
  if (n_max > DDT_TREE_B_MAX + 1 || batch > 65535 || L > DDT_TREE_L_MAX) return DDT_ERR_UNSUPPORTED;
  if ((size_t)batch * n_max + batch + 1 > kMaxCounters) return DDT_ERR_UNSUPPORTED;
  if (batch > 0 && (!logits || !tok || !parent || !depth || !n_nodes || !acc_len || !bonus ||
                    (L > 0 && (!acc_nodes || !acc_tok))))
    return DDT_ERR_INVALID_ARG;
  if (!ws_ok(workspace, workspace_bytes, walk_workspace_size(batch, n_max, V)))
    return DDT_ERR_WORKSPACE;
  return launch_tree_walk(logits, dtype, batch, n_max, V, row_stride, tok, parent, depth, n_nodes,
                          L, mode, acc_len, acc_nodes, acc_tok, bonus, workspace, dev_status,
                          stream, sampling);
}
}  // namespace

ddt_status ddt_tree_walk(const void* logits, ddt_dtype dtype, int batch, int n_max, int V,
                         int64_t row_stride, const int32_t* tok, const int32_t* parent,
                         const int32_t* depth, const int32_t* n_nodes, int L, int mode,
                         int32_t* acc_len, int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus,
                         void* workspace, size_t workspace_bytes, int32_t* dev_status,
                         cudaStream_t stream) {
  const NvtxRange nvtx("ddt_tree_walk");
  return walk_common(logits, dtype, batch, n_max, V, row_stride, tok, parent, depth, n_nodes, L,
                     mode, acc_len, acc_nodes, acc_tok, bonus, workspace, workspace_bytes,
                     dev_status, stream, nullptr);
}

int ddt_tree_walk_resolve_mode(int mode, ddt_dtype dtype, int batch, int n_max, int V, int L) {
  if (mode != DDT_WALK_ALL_ROWS && mode != DDT_WALK_LAZY && mode != DDT_WALK_AUTO) return -1;
  if (batch < 0 || n_max < 1 || V < 1 || L < 0) return -1;
  return walk_mode_for(mode, dtype, batch, n_max, V, L);
}

ddt_status ddt_tree_walk_sample(const void* logits, ddt_dtype dtype, int batch, int n_max, int V,
                                int64_t row_stride, const int32_t* tok, const int32_t* parent,
                                const int32_t* depth, const int32_t* n_nodes, int L,
                                float inv_temperature, uint64_t seed, uint64_t step,
                                uint64_t* step_counter, int32_t* acc_len, int32_t* acc_nodes,
                                int32_t* acc_tok, int32_t* bonus, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream) {
  const NvtxRange nvtx("ddt_tree_walk_sample");
  if (!(inv_temperature > 0.f) || !(inv_temperature * kLog2e < INFINITY))
    return DDT_ERR_INVALID_ARG;
  if (step_counter && ((uintptr_t)step_counter & 7u)) return DDT_ERR_INVALID_ARG;
  const WalkSampling smp{inv_temperature, seed, step, step_counter};
  return walk_common(logits, dtype, batch, n_max, V, row_stride, tok, parent, depth, n_nodes, L,
                     DDT_WALK_ALL_ROWS, acc_len, acc_nodes, acc_tok, bonus, workspace,
                     workspace_bytes, dev_status, stream, &smp);
}

int ddt_lm_head_max_rows(void) { return lm_head_max_rows(); }

size_t ddt_lm_head_walk_workspace_size(const ddt_lm_head_walk_args* a) {
  (void)a;
  return DDT_WS_COUNTER_BYTES;
}

ddt_status ddt_lm_head_walk(const ddt_lm_head_walk_args* a, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange nvtx("ddt_lm_head_walk");
  if (!a) return DDT_ERR_INVALID_ARG;
  if (a->batch < 0 || a->n_max < 1 || a->L < 0 || a->K < 1 || a->V < 1) return DDT_ERR_INVALID_ARG;
  if (a->K % 8 != 0 || a->n_max > DDT_TREE_B_MAX + 1 || a->L > DDT_TREE_L_MAX ||
      (int64_t)a->batch * a->n_max > lm_head_max_rows())
    return DDT_ERR_UNSUPPORTED;
  if (a->batch == 0) return DDT_OK;
  if (!a->hidden || !a->weight || !a->tok || !a->parent || !a->depth || !a->n_nodes ||
      !a->acc_len || !a->bonus || (a->L > 0 && (!a->acc_nodes || !a->acc_tok)))
    return DDT_ERR_INVALID_ARG;
  if (!aligned16(a->hidden) || !aligned16(a->weight)) return DDT_ERR_INVALID_ARG;
  if (!ws_ok(workspace, workspace_bytes, DDT_WS_COUNTER_BYTES)) return DDT_ERR_WORKSPACE;
  return launch_lm_head_walk(a, workspace, stream);
}

ddt_status ddt_kv_commit(const ddt_kv_commit_args* a, cudaStream_t stream) {
  const NvtxRange nvtx("ddt_kv_commit");
  if (!a) return DDT_ERR_INVALID_ARG;
  if (a->batch < 0 || a->n_max < 1 || a->hkv < 1 || a->d < 1 || a->L < 0)
    return DDT_ERR_INVALID_ARG;
  if (a->L > DDT_TREE_L_MAX || ((int64_t)a->hkv * a->d) % 8 != 0 ||
      (int64_t)a->hkv * a->d > (1 << 20))
    return DDT_ERR_UNSUPPORTED;
  if (a->batch == 0) return DDT_OK;
  if (!a->k_tree || !a->v_tree || !a->acc_len || !a->ctx_len || !a->k_cache || !a->v_cache ||
      (a->L > 0 && !a->acc_nodes))
    return DDT_ERR_INVALID_ARG;
  if (!aligned16(a->k_tree) || !aligned16(a->v_tree) || !aligned16(a->k_cache) ||
      !aligned16(a->v_cache))
    return DDT_ERR_INVALID_ARG;
  if (a->page_table) {
    if (a->page_size < 1 || a->max_pages < 1 || a->num_pages < 0) return DDT_ERR_INVALID_ARG;
  } else if (a->t_max < 1) {
    return DDT_ERR_INVALID_ARG;
  }
  return launch_kv_commit(a, stream);
}

}  // extern "C"
