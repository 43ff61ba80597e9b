// launch.h -- internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ddt.h"

namespace ddt {

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_smem_attr(const void* func, size_t bytes);

// Multiprocessors of the current device.
int device_sm_count();

size_t topk_workspace_size(int rows, int V, int k);
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
ddt_status launch_tree_walk(const void* logits, ddt_dtype dt, int batch, int n_max, int V,
                            int64_t row_stride, const int32_t* tok, const int32_t* parent,
                            const int32_t* depth, const int32_t* n_nodes, int L, int32_t* acc_len,
                            int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus, void* ws,
                            int32_t* dev_status, cudaStream_t stream);

struct AttnParams;
size_t attn_workspace_size(const ddt_attn_args* a);
ddt_status launch_attn(const ddt_attn_args* a, void* ws, size_t ws_bytes, cudaStream_t stream);

}  // namespace ddt
