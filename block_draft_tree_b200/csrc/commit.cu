// commit.cu -- after the walk: the root and the accepted rows' K/V join the
// committed context.
//
// DDTree page, section 運作流程 (workflow): each round starts from the bonus
// token that the target produced but has not run yet; the round runs it as
// the tree's root together with the draft rows, and the walk (step 4)
// accepts a path of rows.  So the root and the accepted rows have been
// forwarded and their K/V belong to the context from now on, at the
// positions their rows were scored at (ctx_len + depth); the new bonus
// token has not been forwarded and stays out.  The context grows by
// acc_len + 1.
//
// Design: the copy is a few KB per sequence (rows of hkv * d bf16), so the
// kernel is one CTA per sequence: the CTA resolves the destination of every
// row it commits (dense position or page slot) once, then all its threads
// stream 16-byte vectors of K and V, several in flight each; the CTA reads
// ctx_len[b] before and writes it after the copy, so the in-place update of
// ctx_len races with nothing.
#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 4;  // vectors in flight per thread

struct CommitParams {
  const uint4 *k_tree, *v_tree;
  const int32_t *acc_len, *acc_nodes;
  int32_t* ctx_len;
  uint4 *k_cache, *v_cache;
  const int32_t* page_table;
  int page_size, max_pages, num_pages;
  int64_t t_max;
  int n_max, L, row_vecs;
  int32_t* status;
};

__global__ void __launch_bounds__(kThreads) commit_kernel(CommitParams p) {
  __shared__ int s_row[DDT_TREE_L_MAX + 1];
  __shared__ int64_t s_dst[DDT_TREE_L_MAX + 1];  // destination cache row, -1: not written
  __shared__ int s_a, s_c;
  const int b = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  if (tid == 0) {
    int a = p.acc_len[b];
    if (a < 0 || a > p.L) {
      raise_status(p.status, DDT_ERR_INVALID_ARG);
      a = min(max(a, 0), p.L);
    }
    s_a = a;
    s_c = p.ctx_len[b];
  }
  __syncthreads();
  const int a = s_a, c = s_c;
  if (tid <= a) {
    const int r = tid == 0 ? 0 : p.acc_nodes[(int64_t)b * p.L + tid - 1];
    const int64_t pos = (int64_t)c + tid;
    int64_t dst = -1;
    if (p.page_table == nullptr) {
      if (pos >= 0 && pos < p.t_max) dst = (int64_t)b * p.t_max + pos;
    } else if (pos >= 0) {
      const int64_t pi = pos / p.page_size;
      const int pg = pi < p.max_pages ? p.page_table[(int64_t)b * p.max_pages + pi] : -1;
      if (pg >= 0 && (p.num_pages <= 0 || pg < p.num_pages))
        dst = (int64_t)pg * p.page_size + pos % p.page_size;
    }
    const bool row_ok = r >= 0 && r < p.n_max;
    if (dst < 0 || !row_ok) raise_status(p.status, DDT_ERR_INVALID_ARG);
    s_row[tid] = row_ok ? r : -1;
    s_dst[tid] = row_ok ? dst : -1;
  }
  __syncthreads();
  const int64_t units = (int64_t)(a + 1) * p.row_vecs;
  const int64_t src_base = (int64_t)b * p.n_max;
  for (int64_t u0 = tid; u0 < units; u0 += (int64_t)kThreads * kBatch) {
    uint4 kv[kBatch], vv[kBatch];
    int64_t to[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int64_t u = u0 + (int64_t)q * kThreads;
      to[q] = -1;
      if (u < units) {
        const int i = (int)(u / p.row_vecs), e = (int)(u % p.row_vecs);
        if (s_dst[i] >= 0) {
          const int64_t from = (src_base + s_row[i]) * p.row_vecs + e;
          kv[q] = __ldg(p.k_tree + from);
          vv[q] = __ldg(p.v_tree + from);
          to[q] = s_dst[i] * p.row_vecs + e;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q)
      if (to[q] >= 0) {
        p.k_cache[to[q]] = kv[q];
        p.v_cache[to[q]] = vv[q];
      }
  }
  pdl_trigger();
  if (tid == 0) p.ctx_len[b] = c + a + 1;
}

}  // namespace

ddt_status launch_kv_commit(const ddt_kv_commit_args* a, cudaStream_t stream) {
  if (a->batch == 0) return DDT_OK;
  CommitParams p;
  p.k_tree = (const uint4*)a->k_tree;
  p.v_tree = (const uint4*)a->v_tree;
  p.acc_len = a->acc_len;
  p.acc_nodes = a->acc_nodes;
  p.ctx_len = a->ctx_len;
  p.k_cache = (uint4*)a->k_cache;
  p.v_cache = (uint4*)a->v_cache;
  p.page_table = a->page_table;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages;
  p.num_pages = a->num_pages;
  p.t_max = a->t_max;
  p.n_max = a->n_max;
  p.L = a->L;
  p.row_vecs = a->hkv * a->d * 2 / 16;
  p.status = a->dev_status;
  const cudaError_t e = launch_pdl(commit_kernel, dim3(a->batch), dim3(kThreads), 0, stream, 0, p);
  return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
