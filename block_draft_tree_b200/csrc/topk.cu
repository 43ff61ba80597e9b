// topk.cu -- stage 1 of the verification round: per-position softmax
// normaliser (log-sum-exp) and top-k candidates of the draft marginals.
//
// DDTree page, section 運作流程 step 1: the drafter returns one marginal q_i
// per position; the tree's candidates at depth i are the k most likely
// tokens of q_i (logit descending, smaller token id first on ties).
//
// Design (HBM-bound single pass over the logits):
//   * grid = (chunks of 8192 logits, rows); 256 threads; each thread keeps
//     32 logits in registers, loaded with 16-byte streaming loads.
//   * from registers: thread max, thread sum of exp2((z-max)*c), and the
//     thread maximum's order key;
//   * the k-th largest thread maximum over the CTA (16 or 32 rounds of
//     __syncthreads_count bisection) is a threshold that at least k logits
//     of the chunk reach and that few others do (about k+1 on random rows);
//     those candidates go to shared memory and are ranked exactly by the
//     64-bit key (value, then smaller id);
//   * per chunk partials (k keys, max, sum) go to the workspace; the last
//     CTA of a row (atomic ticket, no waiting) merges them, writes the row's
//     outputs and returns its ticket to zero.
// Degenerate rows (many equal values beyond the candidate capacity) fall
// back to k rounds of block-wide argmax: slower, same result.
#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8192;
constexpr int kCandCap = 1024;

struct TopkParams {
  const void* logits;
  int V;
  int64_t row_stride;  // elements
  int k;
  float inv_t;
  float c;             // inv_t * log2(e)
  int S;               // chunks per row
  int vec_ok;          // 16-byte aligned rows
  uint64_t* part_keys; // [rows][S][k]
  float2* part_ms;     // [rows][S]
  unsigned* tickets;   // [rows]
  int32_t* ids;
  float* zk;
  float* logp;
  float* lse;
};

__device__ __forceinline__ void block_ms_reduce(float& m, float& s, float c, float* sm_m,
                                                float* sm_s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    float s2 = __shfl_xor_sync(0xFFFFFFFFu, s, o);
    ms_merge(m, s, m2, s2, c);
  }
  if (lane == 0) {
    sm_m[warp] = m;
    sm_s[warp] = s;
  }
  __syncthreads();
  m = -INFINITY;
  s = 0.f;
  for (int w = 0; w < kThreads / 32; ++w) ms_merge(m, s, sm_m[w], sm_s[w], c);
}

__device__ __forceinline__ uint64_t block_max_u64(uint64_t v, uint64_t* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    uint64_t u = shfl_xor_u64(v, o);
    v = u > v ? u : v;
  }
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  uint64_t r = 0;
  for (int w = 0; w < kThreads / 32; ++w) r = sm[w] > r ? sm[w] : r;
  return r;
}

// Exact rank selection of the k largest of n distinct keys in s_cand.
__device__ void rank_select(const uint64_t* s_cand, int n, int k, uint64_t* s_top) {
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint64_t key = s_cand[i];
    int r = 0;
    for (int j = 0; j < n; ++j) r += (s_cand[j] > key);
    if (r < k) s_top[r] = key;
  }
  for (int i = n + threadIdx.x; i < k; i += kThreads) s_top[i] = 0;
}

// Row log-sum-exp, rounded up to f32: inv_t*max + log(sum) in fp64, so that
// no candidate gets a positive log-probability when the tree builder widens
// the f32 lse back to fp64 (its prefix scores must never grow with depth).
__device__ __forceinline__ float row_lse_up(float inv_t, float m, float s) {
  if (m == -INFINITY) return -INFINITY;
  return __double2float_ru(__dadd_ru(__dmul_ru((double)inv_t, (double)m), (double)logf(s)));
}

__device__ void write_row(const TopkParams& p, int row, const uint64_t* s_top, float row_lse) {
  for (int r = threadIdx.x; r < p.k; r += kThreads) {
    const uint64_t key = s_top[r];
    const int64_t o = (int64_t)row * p.k + r;
    const float z = key ? key_val(key) : -INFINITY;
    p.ids[o] = key ? (int32_t)key_id(key) : -1;
    p.zk[o] = z;
    if (p.logp) p.logp[o] = p.inv_t * z - row_lse;
  }
  if (threadIdx.x == 0) p.lse[row] = row_lse;
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkParams p) {
  constexpr int EPV = BF16 ? 8 : 4;           // elements per 16-byte vector
  constexpr int EPT = kChunk / kThreads;      // 32 elements per thread
  constexpr int VPT = EPT / EPV;
  constexpr int ES = BF16 ? 2 : 4;

  __shared__ uint64_t s_cand[kCandCap];
  __shared__ uint64_t s_top[DDT_TOPK_K_MAX];
  __shared__ uint64_t s_red[kThreads / 32];
  __shared__ float s_wm[kThreads / 32], s_wsum[kThreads / 32];
  __shared__ int s_count, s_last;

  const int tid = threadIdx.x;
  const int chunk = blockIdx.x, row = blockIdx.y;
  const int64_t c0 = (int64_t)chunk * kChunk;
  const char* rowp = (const char*)p.logits + (int64_t)row * p.row_stride * ES;

  // element e of vector j of this thread has index c0 + (j*kThreads + tid)*EPV + e
  float x[EPT];
  const bool full = p.vec_ok && (c0 + kChunk <= p.V);
  if (full) {
    uint4 v[VPT];
#pragma unroll
    for (int j = 0; j < VPT; ++j)
      v[j] = ld_stream_v4(rowp + (c0 + (int64_t)(j * kThreads + tid) * EPV) * ES);
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (BF16) {
          x[j * EPV + 2 * q] = bf16_lo(w[q]);
          x[j * EPV + 2 * q + 1] = bf16_hi(w[q]);
        } else {
          x[j * EPV + q] = __uint_as_float(w[q]);
        }
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        const int64_t idx = c0 + (int64_t)(j * kThreads + tid) * EPV + e;
        float val = -INFINITY;
        if (idx < p.V) {
          if (BF16)
            val = bf16_to_f32(((const uint16_t*)rowp)[idx]);
          else
            val = ((const float*)rowp)[idx];
        }
        x[j * EPV + e] = val;
      }
    }
  }
  auto index_of = [&](int i) -> int64_t {
    return c0 + (int64_t)((i / EPV) * kThreads + tid) * EPV + (i % EPV);
  };
  int nvalid = 0;
  if (full) {
    nvalid = EPT;
  } else {
#pragma unroll
    for (int i = 0; i < EPT; ++i) nvalid += (index_of(i) < p.V);
  }

  // thread max and thread sum of exp2((z - max) * c)
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < EPT; ++i) m = fmaxf(m, x[i]);
  float s = 0.f;
  if (m != -INFINITY) {
    const float mc = m * p.c;
#pragma unroll
    for (int i = 0; i < EPT; ++i) s += ex2(fmaf(x[i], p.c, -mc));
  }
  // order key of the thread maximum (0: thread holds no element)
  uint32_t tk = 0;
  if (nvalid > 0) {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPT; ++i)
      if (full || index_of(i) < p.V) mx = fmaxf(mx, x[i]);
    tk = BF16 ? ord16(__float_as_uint(mx) >> 16) : ord32(mx);
    if (tk == 0) tk = 1;  // keep "holds an element" distinct from "holds none"
  }
  if (tid == 0) s_count = 0;

  // the k-th largest thread maximum over the CTA
  constexpr int KB = BF16 ? 16 : 32;
  uint32_t tau = 0;
#pragma unroll 1
  for (int bit = KB - 1; bit >= 0; --bit) {
    const uint32_t cand = tau | (1u << bit);
    if (__syncthreads_count(tk >= cand) >= p.k) tau = cand;
  }
  if (tau == 0) tau = 1;  // fewer than k threads hold elements: take them all

  // candidates: elements whose order key reaches tau
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    const int64_t idx = index_of(i);
    if (!full && idx >= p.V) continue;
    uint32_t ok = BF16 ? ord16(__float_as_uint(x[i]) >> 16) : ord32(x[i]);
    if (ok == 0) ok = 1;
    if (ok >= tau) {
      const int pos = atomicAdd(&s_count, 1);
      if (pos < kCandCap) s_cand[pos] = cand_key(x[i], (uint32_t)idx);
    }
  }
  block_ms_reduce(m, s, p.c, s_wm, s_wsum);  // contains __syncthreads
  const int n = s_count;
  if (n <= kCandCap) {
    rank_select(s_cand, n, p.k, s_top);
  } else {
    // degenerate chunk: k rounds of block-wide argmax below the previous pick
    uint64_t prev = ~0ull;
    for (int r = 0; r < p.k; ++r) {
      uint64_t best = 0;
#pragma unroll
      for (int i = 0; i < EPT; ++i) {
        const int64_t idx = index_of(i);
        if (!full && idx >= p.V) continue;
        const uint64_t key = cand_key(x[i], (uint32_t)idx);
        if (key < prev && key > best) best = key;
      }
      best = block_max_u64(best, s_red);
      if (tid == 0) s_top[r] = best;
      prev = best;
    }
  }
  __syncthreads();

  if (p.S == 1) {
    write_row(p, row, s_top, row_lse_up(p.inv_t, m, s));
    return;
  }

  // publish this chunk's partial, then take a ticket
  const int64_t pbase = (int64_t)row * p.S + chunk;
  for (int r = tid; r < p.k; r += kThreads) p.part_keys[pbase * p.k + r] = s_top[r];
  if (tid == 0) p.part_ms[pbase] = make_float2(m, s);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.tickets[row], 1u) == (unsigned)(p.S - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // last CTA of the row: merge the S partials
  if (tid == 0) s_count = 0;
  float M = -INFINITY, Ssum = 0.f;
  for (int cc = tid; cc < p.S; cc += kThreads) {
    const float2 ms = ld_cg_f2(&p.part_ms[(int64_t)row * p.S + cc]);
    ms_merge(M, Ssum, ms.x, ms.y, p.c);
  }
  // threshold: the best k-th key of any single chunk (each chunk has k keys >= it)
  uint64_t t = 0;
  for (int cc = tid; cc < p.S; cc += kThreads) {
    const uint64_t kk = ld_cg_u64(&p.part_keys[((int64_t)row * p.S + cc) * p.k + p.k - 1]);
    t = kk > t ? kk : t;
  }
  t = block_max_u64(t, s_red);
  if (t == 0) t = 1;
  const int tot = p.S * p.k;
  for (int i = tid; i < tot; i += kThreads) {
    const uint64_t key = ld_cg_u64(&p.part_keys[(int64_t)row * tot + i]);
    if (key >= t) {
      const int pos = atomicAdd(&s_count, 1);
      if (pos < kCandCap) s_cand[pos] = key;
    }
  }
  block_ms_reduce(M, Ssum, p.c, s_wm, s_wsum);
  const int n2 = s_count;
  if (n2 <= kCandCap) {
    rank_select(s_cand, n2, p.k, s_top);
  } else {
    uint64_t prev = ~0ull;
    for (int r = 0; r < p.k; ++r) {
      uint64_t best = 0;
      for (int i = tid; i < tot; i += kThreads) {
        const uint64_t key = ld_cg_u64(&p.part_keys[(int64_t)row * tot + i]);
        if (key < prev && key > best) best = key;
      }
      best = block_max_u64(best, s_red);
      if (tid == 0) s_top[r] = best;
      prev = best;
    }
  }
  __syncthreads();
  write_row(p, row, s_top, row_lse_up(p.inv_t, M, Ssum));
  // leave the workspace as it was found: all zero
  for (int i = tid; i < tot; i += kThreads) p.part_keys[(int64_t)row * tot + i] = 0ull;
  for (int cc = tid; cc < p.S; cc += kThreads)
    p.part_ms[(int64_t)row * p.S + cc] = make_float2(0.f, 0.f);
  if (tid == 0) p.tickets[row] = 0u;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

size_t topk_workspace_size(int rows, int V, int k) {
  const int S = (V + kChunk - 1) / kChunk;
  if (S <= 1) return 0;
  return align256(sizeof(unsigned) * rows) + align256(sizeof(float2) * (size_t)rows * S) +
         align256(sizeof(uint64_t) * (size_t)rows * S * k);
}

ddt_status launch_topk(const void* logits, ddt_dtype dt, int rows, int V, int64_t row_stride,
                       int k, float inv_t, int32_t* ids, float* zk, float* logp, float* lse,
                       void* ws, size_t ws_bytes, cudaStream_t stream) {
  TopkParams p;
  p.logits = logits;
  p.V = V;
  p.row_stride = row_stride;
  p.k = k;
  p.inv_t = inv_t;
  p.c = inv_t * kLog2e;
  p.S = (V + kChunk - 1) / kChunk;
  const int es = dt == DDT_BF16 ? 2 : 4;
  p.vec_ok = ((uintptr_t)logits % 16 == 0) && ((row_stride * es) % 16 == 0);
  char* w = (char*)ws;
  p.tickets = (unsigned*)w;
  w += align256(sizeof(unsigned) * rows);
  p.part_ms = (float2*)w;
  w += align256(sizeof(float2) * (size_t)rows * p.S);
  p.part_keys = (uint64_t*)w;
  p.ids = ids;
  p.zk = zk;
  p.logp = logp;
  p.lse = lse;
  if (rows == 0) return DDT_OK;
  dim3 grid(p.S, rows);
  if (dt == DDT_BF16)
    topk_kernel<true><<<grid, kThreads, 0, stream>>>(p);
  else
    topk_kernel<false><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
