// budget.cu -- node budgets across a batch, between two tree builds.
//
// DDTree page, section 實驗結果與權衡 (results and trade-offs): acceptance
// grows with the node budget B and so does the verifier's cost, so the
// round's speed peaks at an intermediate B; section 理論基礎, Proposition 1:
// a tree's expected acceptance length is the sum of its nodes' prefix
// probabilities, and the best tree of a smaller budget is the best-first
// part of the best tree of a larger one.  So, from every sequence's tree
// built with its largest budget, the batch's nodes ranked by prefix
// probability give the split of any total number of nodes that maximises
// the batch's expected acceptance: the first n nodes.  Under a round cost
// c0 + c1 * n the call takes the n that maximises the expected emitted
// tokens per unit of cost, (batch + accepted) / (c0 + c1 * n), and returns
// each sequence's share as its budget for the second build.
//
// One CTA of 1024 threads: each node's score (invT * logit sum - lse sum
// along its path, in depth order, fp64), a bitonic sort of the batch's
// nodes by (score desc, slot asc) in shared memory, an fp64 prefix sum of
// exp(score) in that order, the best n (largest rate, smallest n on ties),
// and per-sequence counts and sums.
#include <cmath>

#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 1024;

struct BudgetParams {
  const int32_t *tok, *parent, *depth, *n_nodes, *ids;
  const float *zk, *lse;
  int batch, L, k, n_max, slots, npow2;
  double inv_t;
  int total_budget;
  double c0, c1;
  int32_t* budget;
  double* expected_tokens;
  int32_t* status;
};

// Order-preserving map of a double onto uint64 (larger -> larger).
__device__ __forceinline__ uint64_t ord64(double d) {
  uint64_t u = (uint64_t)__double_as_longlong(d);
  if (u == 0x8000000000000000ull) u = 0ull;
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double from_ord64(uint64_t k) {
  const uint64_t u = (k & 0x8000000000000000ull) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
  return __longlong_as_double((long long)u);
}

__global__ void __launch_bounds__(kThreads, 1) plan_budget_kernel(BudgetParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* key = (uint64_t*)smem;                    // [npow2] ordered scores (0: no node)
  int* slot = (int*)(key + p.npow2);                  // [npow2]
  double* psum = (double*)(slot + p.npow2 + (p.npow2 & 1));  // [npow2] prefix sums
  int* cnt = (int*)(psum + p.npow2);                  // [batch]
  double* esum = (double*)(((uintptr_t)(cnt + p.batch) + 7) & ~(uintptr_t)7);  // [batch]
  __shared__ double s_wsum[kThreads / 32];
  __shared__ double s_best[kThreads / 32];
  __shared__ int s_bestn[kThreads / 32];
  __shared__ int s_n;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = p.n_max - 1;  // node slots per sequence
  pdl_wait();
  pdl_trigger();
  // each node's score; rows beyond n_nodes (and padding) get key 0
  for (int s = tid; s < p.npow2; s += kThreads) {
    uint64_t kk = 0;
    if (s < p.slots) {
      const int b = s / per, j = 1 + s % per;
      int n = p.n_nodes[b];
      if (n < 1 || n > p.n_max) {
        raise_status(p.status, DDT_ERR_INVALID_ARG);
        n = min(max(n, 1), p.n_max);
      }
      if (j < n) {
        const int64_t base = (int64_t)b * p.n_max;
        const int d = p.depth[base + j];
        int path[DDT_TREE_L_MAX];
        bool ok = d >= 1 && d <= p.L;
        for (int x = j, t = d; ok && t >= 1; --t) {
          path[t - 1] = p.tok[base + x];
          x = p.parent[base + x];
          ok = x >= 0 && x < n;
        }
        double sz = 0.0, S = 0.0;
        for (int t = 0; ok && t < d; ++t) {
          const int64_t row = ((int64_t)b * p.L + t) * p.k;
          int r = 0;
          while (r < p.k && p.ids[row + r] != path[t]) ++r;
          if (r == p.k) {
            ok = false;
            break;
          }
          sz = __dadd_rn(sz, (double)p.zk[row + r]);
          S = __dadd_rn(S, (double)p.lse[(int64_t)b * p.L + t]);
        }
        if (ok) {
          kk = ord64(__dadd_rn(__dmul_rn(p.inv_t, sz), -S));
          if (kk == 0) kk = 1;
        } else {
          raise_status(p.status, DDT_ERR_INVALID_ARG);  // a row that is not a tree node of these candidates
        }
      }
    }
    key[s] = kk;
    slot[s] = s;
  }
  for (int b = tid; b < p.batch; b += kThreads) {
    cnt[b] = 0;
    esum[b] = 0.0;
  }
  __syncthreads();
  // bitonic sort: key descending, slot ascending
  for (int size = 2; size <= p.npow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < p.npow2 / 2; i += kThreads) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t ka = key[lo], kb = key[hi];
        const int sa = slot[lo], sb = slot[hi];
        const bool a_first = ka > kb || (ka == kb && sa < sb);  // a ranks before b
        if (a_first != desc) {
          key[lo] = kb;
          key[hi] = ka;
          slot[lo] = sb;
          slot[hi] = sa;
        }
      }
      __syncthreads();
    }
  }
  // inclusive prefix sums of exp(score) in rank order (blocks of consecutive
  // positions per thread, then a scan of the thread totals)
  const int chunk = (p.npow2 + kThreads - 1) / kThreads;
  const int i0 = tid * chunk;
  double run = 0.0;
  for (int i = i0; i < min(i0 + chunk, p.npow2); ++i) {
    run += key[i] ? exp(from_ord64(key[i])) : 0.0;
    psum[i] = run;
  }
  double incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  double wbase = 0.0;
  for (int w = 0; w < warp; ++w) wbase += s_wsum[w];
  const double tbase = wbase + (incl - run);
  // the best number of nodes n: rate(n) = (batch + P(n)) / (c0 + c1 * n);
  // position i holds P(i + 1)
  int navail = 0;
  for (int i = tid; i < p.npow2; i += kThreads) navail += key[i] != 0;
  navail = __reduce_add_sync(0xFFFFFFFFu, navail);
  if (lane == 0) s_bestn[warp] = navail;
  __syncthreads();
  int avail = 0;
  for (int w = 0; w < kThreads / 32; ++w) avail += s_bestn[w];
  const int cap = p.total_budget >= 0 ? min(avail, p.total_budget) : avail;
  __syncthreads();
  int best_n;
  if (p.c1 > 0.0) {
    double best = -1.0;
    int bn = INT_MAX;
    if (tid == 0) {
      best = (double)p.batch / p.c0;
      bn = 0;
    }
    for (int i = i0; i < min(i0 + chunk, cap); ++i) {
      psum[i] += tbase;
      const double f = ((double)p.batch + psum[i]) / (p.c0 + p.c1 * (double)(i + 1));
      if (f > best) {
        best = f;
        bn = i + 1;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double f2 = __shfl_xor_sync(0xFFFFFFFFu, best, o);
      const int n2 = __shfl_xor_sync(0xFFFFFFFFu, bn, o);
      if (f2 > best || (f2 == best && n2 < bn)) {
        best = f2;
        bn = n2;
      }
    }
    if (lane == 0) {
      s_best[warp] = best;
      s_bestn[warp] = bn;
    }
    __syncthreads();
    if (tid == 0) {
      double b2 = s_best[0];
      int n2 = s_bestn[0];
      for (int w = 1; w < kThreads / 32; ++w)
        if (s_best[w] > b2 || (s_best[w] == b2 && s_bestn[w] < n2)) {
          b2 = s_best[w];
          n2 = s_bestn[w];
        }
      s_n = n2;
    }
    __syncthreads();
    best_n = s_n;
  } else {
    best_n = cap;
  }
  // each sequence's share of the first best_n nodes
  for (int i = tid; i < best_n; i += kThreads) {
    const int b = slot[i] / per;
    atomicAdd(&cnt[b], 1);
    atomicAdd(&esum[b], exp(from_ord64(key[i])));
  }
  __syncthreads();
  for (int b = tid; b < p.batch; b += kThreads) {
    p.budget[b] = cnt[b];
    if (p.expected_tokens) p.expected_tokens[b] = 1.0 + esum[b];
  }
}

}  // namespace

int plan_budget_max_nodes() { return 8192; }

size_t plan_budget_smem(int batch, int npow2) {
  return (size_t)npow2 * (8 + 4 + 8) + 8 + (size_t)batch * (4 + 8) + 16;
}

ddt_status launch_plan_budget(const int32_t* tok, const int32_t* parent, const int32_t* depth,
                              const int32_t* n_nodes, const int32_t* ids, const float* zk,
                              const float* lse, int batch, int L, int k, int n_max,
                              float inv_temperature, int total_budget, double c0, double c1,
                              int32_t* budget, double* expected_tokens, int32_t* dev_status,
                              cudaStream_t stream) {
  BudgetParams p;
  p.tok = tok;
  p.parent = parent;
  p.depth = depth;
  p.n_nodes = n_nodes;
  p.ids = ids;
  p.zk = zk;
  p.lse = lse;
  p.batch = batch;
  p.L = L;
  p.k = k;
  p.n_max = n_max;
  p.slots = batch * (n_max - 1);
  int np2 = 2;
  while (np2 < p.slots) np2 <<= 1;
  p.npow2 = np2;
  p.inv_t = (double)inv_temperature;
  p.total_budget = total_budget;
  p.c0 = c0;
  p.c1 = c1;
  p.budget = budget;
  p.expected_tokens = expected_tokens;
  p.status = dev_status;
  if (batch == 0) return DDT_OK;
  const size_t smem = plan_budget_smem(batch, np2);
  if (ensure_smem_attr((const void*)plan_budget_kernel, smem) != cudaSuccess) return DDT_ERR_CUDA;
  return launch_pdl(plan_budget_kernel, dim3(1), dim3(kThreads), smem, stream, 0, p) == cudaSuccess
             ? DDT_OK
             : DDT_ERR_CUDA;
}

}  // namespace ddt
