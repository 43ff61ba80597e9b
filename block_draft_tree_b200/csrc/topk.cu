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

// Block merge of per-thread (max, sum of exp2((z-max)*c)): the block maximum
// from a REDUX on the ordered keys, one rescale per thread, then a sum.  Two
// barriers; every thread gets the result.
__device__ __forceinline__ void block_ms_reduce(float& m, float& s, float c, float* sm_m,
                                                float* sm_s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t wk = __reduce_max_sync(0xFFFFFFFFu, ord32(m));
  if (lane == 0) sm_m[warp] = from_ord32(wk);
  __syncthreads();
  float M = sm_m[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) M = fmaxf(M, sm_m[w]);
  float t = (m == -INFINITY || M == -INFINITY) ? 0.f : s * ex2((m - M) * c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
  if (lane == 0) sm_s[warp] = t;
  __syncthreads();
  float S = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) S += sm_s[w];
  m = M;
  s = S;
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

// MIN_CTAS: CTAs per SM the registers are budgeted for.  Three keep every
// value in registers; four (64 registers, a few spilled) hide more of the
// per-chunk compute behind other CTAs' loads when the grid spans many waves.
template <bool BF16, int MIN_CTAS>
__global__ void __launch_bounds__(kThreads, MIN_CTAS) topk_kernel(TopkParams p) {
  constexpr int EPV = BF16 ? 8 : 4;           // elements per 16-byte vector
  constexpr int EPT = kChunk / kThreads;      // 32 elements per thread
  constexpr int VPT = EPT / EPV;
  constexpr int ES = BF16 ? 2 : 4;
  constexpr int NW = EPT * ES / 4;            // 32-bit words held per thread

  __shared__ uint64_t s_cand[kCandCap];
  __shared__ uint64_t s_top[DDT_TOPK_K_MAX];
  __shared__ uint64_t s_red[kThreads / 32];
  __shared__ float s_wm[kThreads / 32], s_wsum[kThreads / 32];
  __shared__ int s_count, s_last;

  const int tid = threadIdx.x;
  const int chunk = blockIdx.x, row = blockIdx.y;
  const int64_t c0 = (int64_t)chunk * kChunk;
  pdl_wait();
  const char* rowp = (const char*)p.logits + (int64_t)row * p.row_stride * ES;

  // word j of vector q of this thread holds elements starting at index
  // c0 + (q*kThreads + tid)*EPV + j*(EPV/4); out-of-range elements read as -inf
  uint32_t w[NW];
  const bool full = p.vec_ok && (c0 + kChunk <= p.V);
  if (full) {
#pragma unroll
    for (int q = 0; q < VPT; ++q) {
      const uint4 v = ld_stream_v4(rowp + (c0 + (int64_t)(q * kThreads + tid) * EPV) * ES);
      w[4 * q] = v.x;
      w[4 * q + 1] = v.y;
      w[4 * q + 2] = v.z;
      w[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < VPT; ++q)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t e0 = c0 + (int64_t)(q * kThreads + tid) * EPV + j * (EPV / 4);
        if (BF16) {
          const uint32_t lo = e0 < p.V ? ((const uint16_t*)rowp)[e0] : 0xFF80u;
          const uint32_t hi = e0 + 1 < p.V ? ((const uint16_t*)rowp)[e0 + 1] : 0xFF80u;
          w[4 * q + j] = lo | (hi << 16);
        } else {
          w[4 * q + j] = e0 < p.V ? __float_as_uint(((const float*)rowp)[e0]) : 0xFF800000u;
        }
      }
  }
  const int ibase = (int)c0 + tid * EPV;
  auto index_of = [&](int e) -> int {  // element e (0..EPT) of this thread
    return ibase + (e / EPV) * kThreads * EPV + (e % EPV);
  };
  auto value_of = [&](int e) -> float {
    if (BF16) return (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]);
    return __uint_as_float(w[e]);
  };
  int nvalid = EPT;
  if (!full) {
    nvalid = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) nvalid += (index_of(e) < p.V);
  }

  // thread max (packed bf16 pairs where possible) and sum of exp2((z-max)*c)
  float m;
  if (BF16) {
    __nv_bfloat162 m2 = *(const __nv_bfloat162*)&w[0];
#pragma unroll
    for (int j = 1; j < NW; ++j) m2 = __hmax2(m2, *(const __nv_bfloat162*)&w[j]);
    m = fmaxf(__low2float(m2), __high2float(m2));
  } else {
    m = -INFINITY;
#pragma unroll
    for (int e = 0; e < EPT; ++e) m = fmaxf(m, value_of(e));
  }
  float s = 0.f;
  if (m != -INFINITY) {
    const float mc = m * p.c;
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < EPT; ++e) s4[e & 3] += ex2(fmaf(value_of(e), p.c, -mc));
    s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  }
  // order key of the thread maximum (0: thread holds no element)
  uint32_t tk = 0;
  if (nvalid > 0) {
    tk = BF16 ? ord16(__float_as_uint(m) >> 16) : ord32(m);
    if (tk == 0) tk = 1;
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

  // candidates: elements whose order key reaches tau; with a float threshold
  // this is one compare per element (ties included, -0 == +0 as in the keys)
  {
    const uint32_t tb = BF16 ? (tau & 0xFFFFu) : tau;
    const uint32_t tbits = BF16 ? (((tb & 0x8000u) ? (tb & 0x7FFFu) : (~tb & 0xFFFFu)) << 16)
                                : ((tb & 0x80000000u) ? (tb & 0x7FFFFFFFu) : ~tb);
    // keys below the key of -inf only come from the take-everything sentinel
    const float tf = tb < (BF16 ? 0x7Fu : 0x007FFFFFu) ? -INFINITY : __uint_as_float(tbits);
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const float v = value_of(e);
      if (v >= tf) {
        const int idx = index_of(e);
        if (!full && idx >= p.V) continue;
        const int pos = atomicAdd(&s_count, 1);
        if (pos < kCandCap) s_cand[pos] = cand_key(v, (uint32_t)idx);
      }
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
      for (int e = 0; e < EPT; ++e) {
        const int idx = index_of(e);
        if (!full && idx >= p.V) continue;
        const uint64_t key = cand_key(value_of(e), (uint32_t)idx);
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

  pdl_trigger();
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

  // last CTA of the row: every chunk's keys and (max, sum) in one round of
  // loads, then the k best keys of the row ranked directly
  const int tot = p.S * p.k;
  float M = -INFINITY, Ssum = 0.f;
  for (int cc = tid; cc < p.S; cc += kThreads) {
    const float2 ms = ld_cg_f2(&p.part_ms[(int64_t)row * p.S + cc]);
    ms_merge(M, Ssum, ms.x, ms.y, p.c);
  }
  if (tot <= kCandCap) {
    for (int i = tid; i < tot; i += kThreads) s_cand[i] = ld_cg_u64(&p.part_keys[(int64_t)row * tot + i]);
    block_ms_reduce(M, Ssum, p.c, s_wm, s_wsum);  // its barriers publish s_cand
    rank_select(s_cand, tot, p.k, s_top);
  } else {
    // many chunks: a threshold first (the best k-th key of any chunk: each
    // chunk has k keys at or above it), then the keys that reach it
    if (tid == 0) s_count = 0;
    uint64_t t = 0;
    for (int cc = tid; cc < p.S; cc += kThreads) {
      const uint64_t kk = ld_cg_u64(&p.part_keys[((int64_t)row * p.S + cc) * p.k + p.k - 1]);
      t = kk > t ? kk : t;
    }
    t = block_max_u64(t, s_red);
    if (t == 0) t = 1;
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
  }
  __syncthreads();
  write_row(p, row, s_top, row_lse_up(p.inv_t, M, Ssum));
  if (tid == 0) p.tickets[row] = 0u;  // the counter region is left zero
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

size_t topk_workspace_size(int rows, int V, int k) {
  const int S = (V + kChunk - 1) / kChunk;
  if (S <= 1) return 0;
  return (size_t)DDT_WS_COUNTER_BYTES + align256(sizeof(float2) * (size_t)rows * S) +
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
  p.tickets = (unsigned*)w;  // counter region: one ticket per row
  w += DDT_WS_COUNTER_BYTES;
  p.part_ms = (float2*)w;
  w += align256(sizeof(float2) * (size_t)rows * p.S);
  p.part_keys = (uint64_t*)w;
  p.ids = ids;
  p.zk = zk;
  p.logp = logp;
  p.lse = lse;
  if (rows == 0) return DDT_OK;
  dim3 grid(p.S, rows);
  // many waves of chunks: the higher-occupancy build; a few: the spill-free one
  const bool many = (long)p.S * rows > 4L * 3 * device_sm_count();
  cudaError_t e;
  if (dt == DDT_BF16)
    e = many ? launch_pdl(topk_kernel<true, 4>, grid, dim3(kThreads), 0, stream, 0, p)
             : launch_pdl(topk_kernel<true, 3>, grid, dim3(kThreads), 0, stream, 0, p);
  else
    e = many ? launch_pdl(topk_kernel<false, 4>, grid, dim3(kThreads), 0, stream, 0, p)
             : launch_pdl(topk_kernel<false, 3>, grid, dim3(kThreads), 0, stream, 0, p);
  return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
