// launch.h -- internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "ddt.h"

namespace ddt {

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_smem_attr(const void* func, size_t bytes);

// Multiprocessors of the current device.
int device_sm_count();

// Clock cycles after which a bounded mbarrier wait of the tensor-core kernels
// gives up (about one second by default; see ddt_debug_set_wait_limit), and
// the bound of each wait that drains loads and MMAs in flight after that.
long long wait_limit_cycles();
// The tensor-core attention kernel override (0 auto, 1 one-tile, 2 pairs).
int attn_kernel_choice();
constexpr long long kDrainCycles = 200000000LL;

// Launch with programmatic stream serialization (see pdl_wait/pdl_trigger),
// optionally as clusters of cluster_y CTAs along y.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       int cluster_y, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_y > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = (unsigned)cluster_y;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

size_t topk_workspace_size(int rows, int V, int k);
ddt_status topk_check(const void* logits, ddt_dtype dtype, int batch, int L, int V,
                      int64_t row_stride, int k, float inv_temperature, const int32_t* ids,
                      const float* zk, const float* lse);
ddt_status launch_topk(const void* logits, ddt_dtype dt, int rows, int V, int64_t row_stride,
                       int k, float inv_t, int32_t* ids, float* zk, float* logp, float* lse,
                       void* ws, size_t ws_bytes, cudaStream_t stream);

ddt_status launch_build_tree(const int32_t* ids, const float* zk, const float* lse, int batch,
                             int L, int k, float inv_t, const int32_t* k_per_seq,
                             const int32_t* budget, int B_max, const int32_t* root_token,
                             const int32_t* ctx_len, int32_t* tok, int32_t* parent,
                             int32_t* depth, int32_t* pos, uint32_t* mask, int32_t* n_nodes,
                             double* surrogate, int32_t* dev_status, cudaStream_t stream);

size_t walk_workspace_size(int batch, int n_max, int V);
// The sampling decoding rule of the walk (null: greedy).
struct WalkSampling {
  float inv_temperature;
  uint64_t seed, step;
  uint64_t* step_counter;  // optional device word added to step; advanced by one per call
};
ddt_status launch_tree_walk(const void* logits, ddt_dtype dt, int batch, int n_max, int V,
                            int64_t row_stride, const int32_t* tok, const int32_t* parent,
                            const int32_t* depth, const int32_t* n_nodes, int L, int mode,
                            int32_t* acc_len, int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus,
                            void* ws, int32_t* dev_status, cudaStream_t stream,
                            const WalkSampling* sampling = nullptr);
// The walk DDT_WALK_AUTO resolves to for these sizes on the current device.
int walk_mode_for(int mode, ddt_dtype dt, int batch, int n_max, int V, int L);

ddt_status launch_kv_commit(const ddt_kv_commit_args* a, cudaStream_t stream);
ddt_status launch_lm_head_walk(const ddt_lm_head_walk_args* a, void* ws, cudaStream_t stream);
int lm_head_max_rows();

int plan_budget_max_nodes();
ddt_status launch_plan_budget(const int32_t* tok, const int32_t* parent, const int32_t* depth,
                              const int32_t* n_nodes, const int32_t* ids, const float* zk,
                              const float* lse, int batch, int L, int k, int n_max,
                              float inv_temperature, int total_budget, double c0, double c1,
                              int32_t* budget, double* expected_tokens, int32_t* dev_status,
                              cudaStream_t stream);

struct AttnParams;
size_t attn_workspace_size(const ddt_attn_args* a);
ddt_status launch_attn(const ddt_attn_args* a, void* ws, size_t ws_bytes, cudaStream_t stream);

}  // namespace ddt
