// topk.cu -- stage 1 of the verification round: per-position softmax
// normaliser (log-sum-exp) and top-k candidates of the draft marginals.
//
// DDTree page, section 運作流程 step 1: the drafter returns one marginal q_i
// per position; the tree's candidates at depth i are the k most likely
// tokens of q_i (logit descending, smaller token id first on ties).
//
// Design (an HBM-bound stream over the logits):
//   * the rows are cut into 16 KB chunks and the chunks, in row order, into
//     one contiguous range per CTA, as many CTAs as fit on the device at
//     once; every CTA streams its range through a 3-deep ring of shared
//     memory filled by 16-byte asynchronous copies (each thread copies and
//     later reads the same 64 bytes of a chunk, so no barrier guards the
//     ring), so that two chunks per CTA are always in flight;
//   * per chunk, each thread folds its 32 (bf16) or 16 (f32) logits into a
//     running (max, sum of 2^((z - max) * c)) and compares its chunk maximum
//     with the CTA's current bound on the k-th best key: only a thread whose
//     maximum beats it looks at its logits again and appends the ones that
//     do to a shared candidate buffer.  The buffer is ranked (exactly, by
//     the 64-bit keys) only when it fills past half its size -- which also
//     raises the bound -- and at the end of the CTA's part of the row;
//   * the first chunk of each row a CTA sees starts from a bound k logits
//     are sure to reach: the largest over warps of the k-th largest lane
//     maximum (a sort of 32 keys inside each warp);
//   * a CTA's part of a row ends in a partial (k best keys, max, sum) in the
//     workspace; the last CTA of the row (atomic ticket, no waiting) merges
//     the partials, writes the row's outputs and returns its ticket to zero.
// The order key is 64 bits: the float's order-preserving bits, then the
// complement of the token id, so ties go to the smaller id and every key is
// distinct.  No CTA ever waits for another, so nothing can hang.
#include <climits>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 256;
constexpr int kChunkBytes = 16384;             // one chunk: 64 bytes per thread
constexpr int kVecPerThread = kChunkBytes / 16 / kThreads;  // 4 vectors of 16 bytes
constexpr int kStages = 3;                     // chunks of the ring
constexpr int kCandCap = 1024;

struct TopkParams {
  const void* logits;
  int rows, V;
  int64_t row_stride;  // elements
  int k;
  float inv_t;
  float c;             // inv_t * log2(e)
  int S;               // chunks per row
  int G;               // CTAs
  int64_t T;           // chunks in all (rows * S)
  int pmax;            // partial slots per row
  int vec_ok;          // 16-byte aligned rows
  uint64_t* part_keys; // [rows][pmax][k]
  float2* part_ms;     // [rows][pmax]
  unsigned* tickets;   // [rows]
  int32_t* ids;
  float* zk;
  float* logp;
  float* lse;
};

// First chunk of CTA g's range, and the CTA whose range holds chunk ch.
__host__ __device__ __forceinline__ int64_t range_lo(int64_t g, int64_t T, int64_t G) {
  return g * T / G;
}
__host__ __device__ __forceinline__ int64_t owner_of(int64_t ch, int64_t T, int64_t G) {
  return ((ch + 1) * G - 1) / T;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Block merge of per-thread (max, sum of exp2((z-max)*c)); every thread gets
// the result.  Two barriers.
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
    const uint64_t u = shfl_xor_u64(v, o);
    v = u > v ? u : v;
  }
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  uint64_t r = 0;
  for (int w = 0; w < kThreads / 32; ++w) r = sm[w] > r ? sm[w] : r;
  return r;
}

// The k largest of the distinct nonzero keys a[0..na) and b[0..nb) (either
// may hold zeros: "no element"), in descending order, into out[0..k).
__device__ void rank_select2(const uint64_t* a, int na, const uint64_t* b, int nb, int k,
                             uint64_t* out) {
  const int n = na + nb;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint64_t key = i < na ? a[i] : b[i - na];
    if (key == 0) continue;
    int r = 0;
    for (int j = 0; j < na; ++j) r += (a[j] > key);
    for (int j = 0; j < nb; ++j) r += (b[j] > key);
    if (r < k) out[r] = key;
  }
}

// The k-th largest key of the warp's lanes (0 when fewer than k lanes hold
// one): a bitonic sort of the 32 keys, descending.
__device__ __forceinline__ uint64_t warp_kth_key(uint64_t v, int k) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t o = shfl_xor_u64(v, stride);
      const bool up = (lane & stride) == 0;            // the lower lane of the pair
      const bool desc = (lane & size) == 0;            // this block sorts descending
      const bool keep_max = (up == desc);
      v = keep_max ? (o > v ? o : v) : (o < v ? o : v);
    }
  }
  const uint32_t lo = __shfl_sync(0xFFFFFFFFu, (uint32_t)v, k - 1);
  const uint32_t hi = __shfl_sync(0xFFFFFFFFu, (uint32_t)(v >> 32), k - 1);
  return ((uint64_t)hi << 32) | lo;
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

struct Smem {
  uint64_t cand[kCandCap];
  uint64_t top[DDT_TOPK_K_MAX];
  uint64_t top2[DDT_TOPK_K_MAX];
  uint64_t red[kThreads / 32];
  float wm[kThreads / 32], wsum[kThreads / 32];
  int count, last, overflow;
};

// Issue this thread's copies of chunk ch into ring slot `slot` (vectors
// entirely inside the row only; the one that straddles V is read from
// global memory when the chunk is used).  Always commits one group.
template <bool BF16>
__device__ __forceinline__ void prefetch_chunk(const TopkParams& p, unsigned char* ring, int slot,
                                               int64_t ch) {
  constexpr int ES = BF16 ? 2 : 4, EPV = 16 / ES, EPC = kChunkBytes / ES;
  if (p.vec_ok && ch < p.T) {
    const int row = (int)(ch / p.S), cidx = (int)(ch % p.S);
    const char* rowp = (const char*)p.logits + (int64_t)row * p.row_stride * ES;
    const int e0 = cidx * EPC;
#pragma unroll
    for (int q = 0; q < kVecPerThread; ++q) {
      const int v = q * kThreads + (int)threadIdx.x;
      const int e = e0 + v * EPV;
      if (e + EPV <= p.V) cp_async16(ring + slot * kChunkBytes + v * 16, rowp + (int64_t)e * ES);
    }
  }
  cp_async_commit();
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 3) topk_kernel(TopkParams p) {
  constexpr int ES = BF16 ? 2 : 4, EPV = 16 / ES, EPC = kChunkBytes / ES;
  constexpr int NW = kVecPerThread * 4;  // 32-bit words of logits per thread per chunk
  constexpr int PER = EPV / 4;           // elements per word
  constexpr int NE = NW * PER;           // elements per thread per chunk
  extern __shared__ __align__(16) unsigned char ring[];
  __shared__ Smem sm;

  const int tid = threadIdx.x;
  const int64_t c_lo = range_lo(blockIdx.x, p.T, p.G), c_hi = range_lo(blockIdx.x + 1, p.T, p.G);
  pdl_wait();
  for (int i = 0; i < kStages; ++i) prefetch_chunk<BF16>(p, ring, i, c_lo + i < c_hi ? c_lo + i : p.T);
  pdl_trigger();

  float m = -INFINITY, s = 0.f;  // this thread's running (max, sum) for the current row
  uint64_t tau = 0;              // a lower bound of the segment's k-th best key (0: none yet)
  bool first = true;             // next chunk is the first of a row for this CTA
  int row = (int)(c_lo / p.S), cidx = (int)(c_lo % p.S), slot = 0;
  for (int64_t ch = c_lo; ch < c_hi; ++ch, slot = slot == kStages - 1 ? 0 : slot + 1) {
    if (ch > c_lo && ++cidx == p.S) {  // the next chunk (no division per chunk)
      cidx = 0;
      ++row;
    }
    const int e0 = cidx * EPC;
    const char* rowp = (const char*)p.logits + (int64_t)row * p.row_stride * ES;
    cp_async_wait<kStages - 1>();
    // this thread's logits: word j of vector q holds elements
    // e0 + (q*kThreads + tid)*EPV + j*PER ...; absent ones read as -inf
    uint32_t w[NW];
#pragma unroll
    for (int q = 0; q < kVecPerThread; ++q) {
      const int v = q * kThreads + tid;
      const int e = e0 + v * EPV;
      if (p.vec_ok && e + EPV <= p.V) {
        const uint4 u = *(const uint4*)(ring + slot * kChunkBytes + v * 16);
        w[4 * q] = u.x;
        w[4 * q + 1] = u.y;
        w[4 * q + 2] = u.z;
        w[4 * q + 3] = u.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ej = e + j * PER;
          if (BF16) {
            const uint32_t lo = ej < p.V ? ((const uint16_t*)rowp)[ej] : 0xFF80u;
            const uint32_t hi = ej + 1 < p.V ? ((const uint16_t*)rowp)[ej + 1] : 0xFF80u;
            w[4 * q + j] = lo | (hi << 16);
          } else {
            w[4 * q + j] = ej < p.V ? __float_as_uint(((const float*)rowp)[ej]) : 0xFF800000u;
          }
        }
      }
    }
    // element i (0..NE) of this thread: vector i / (4 PER), in increasing index order
    auto index_of = [&](int i) -> int {
      const int q = i / (4 * PER), r = i % (4 * PER);
      return e0 + (q * kThreads + tid) * EPV + r;
    };
    auto value_of = [&](int i) -> float {
      if (BF16) return (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
      return __uint_as_float(w[i]);
    };

    // chunk maximum of this thread (-inf pads never exceed a real logit)
    float mc;
    if (BF16) {
      __nv_bfloat162 m2 = *(const __nv_bfloat162*)&w[0];
#pragma unroll
      for (int j = 1; j < NW; ++j) m2 = __hmax2(m2, *(const __nv_bfloat162*)&w[j]);
      mc = fmaxf(__low2float(m2), __high2float(m2));
    } else {
      mc = __uint_as_float(w[0]);
#pragma unroll
      for (int j = 1; j < NW; ++j) mc = fmaxf(mc, __uint_as_float(w[j]));
    }
    // running (max, sum of 2^((z - max) * c)), two logits per packed instruction
    if (mc > m) {
      if (m != -INFINITY) s *= ex2((m - mc) * p.c);
      m = mc;
    }
    if (m != -INFINITY) {
      const uint64_t c2 = pack2(p.c, p.c), nm2 = pack2(-m * p.c, -m * p.c);
      uint64_t acc[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
      for (int i = 0; i < NE; i += 2) {
        const uint64_t x2 = ffma2(pack2(value_of(i), value_of(i + 1)), c2, nm2);
        float xa, xb;
        unpack2(x2, xa, xb);
        acc[(i >> 1) & 1] = fadd2(acc[(i >> 1) & 1], pack2(ex2(xa), ex2(xb)));
      }
      float a0, a1, b0, b1;
      unpack2(acc[0], a0, a1);
      unpack2(acc[1], b0, b1);
      s += (a0 + a1) + (b0 + b1);
    }

    // Candidates: every logit of the row segment that can still be among
    // the k best goes to a shared buffer, which is only ranked when it
    // fills past half its size and at the end of the segment.  The first
    // chunk of a row starts from a threshold k logits of the CTA reach: the
    // largest over warps of the k-th largest lane maximum (a lane maximum's
    // key: its value at the smallest index holding it); later chunks take
    // the logits above the current k-th best key's value (a logit equal to
    // it comes later, so it ranks below it).
    float tv;
    int ti;
    bool take_all;
    if (first) {
      uint64_t kmax = 0;
#pragma unroll
      for (int i = NE - 1; i >= 0; --i)
        if (value_of(i) == mc && index_of(i) < p.V) kmax = cand_key(mc, (uint32_t)index_of(i));
      const uint64_t tw = warp_kth_key(kmax, p.k);
      tau = block_max_u64(tw, sm.red);  // barriers; a lower bound of the k-th best
      if (tid == 0) {
        sm.count = 0;
        sm.overflow = 0;
      }
      __syncthreads();
      tv = tau ? key_val(tau) : -INFINITY;
      ti = tau ? (int)key_id(tau) : INT_MAX;
      take_all = tau == 0;  // fewer than k lanes hold logits
    } else {
      tv = tau ? key_val(tau) : -INFINITY;
      ti = -1;
      take_all = tau == 0;
    }
    // this thread's candidates as a bit mask over its elements; only a
    // thread whose chunk maximum reaches the bound looks at them again
    uint32_t mask = 0;
    if (take_all || mc > tv || (mc == tv && ti >= 0)) {
#pragma unroll
      for (int i = 0; i < NE; ++i) {
        const float v = value_of(i);
        const bool c = take_all ? index_of(i) < p.V
                                : (v > tv || (v == tv && ti >= 0 && index_of(i) <= ti));
        mask |= (uint32_t)c << i;
      }
    }
    // append them: one reservation per warp (a warp scan of the threads'
    // counts and one atomic); each set bit re-reads its logit from this
    // thread's own bytes of the ring (or from global memory for a vector
    // the ring does not hold), so no register array is indexed at run time
    if (__ballot_sync(0xFFFFFFFFu, mask != 0u)) {
      const int lane = tid & 31;
      const int cnt = __popc(mask);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += u;
      }
      int base = 0;
      if (lane == 31) base = atomicAdd(&sm.count, incl);
      base = __shfl_sync(0xFFFFFFFFu, base, 31);
      int pos = base + incl - cnt;
      while (mask) {
        const int i = __ffs(mask) - 1;
        mask &= mask - 1u;
        const int vq = (i / EPV) * kThreads + tid, r = i % EPV;  // vector of the chunk, element in it
        const int e = e0 + vq * EPV + r;
        float v;
        if (p.vec_ok && e - r + EPV <= p.V) {
          const unsigned char* src = ring + slot * kChunkBytes + vq * 16 + r * ES;
          v = BF16 ? __uint_as_float((uint32_t)(*(const uint16_t*)src) << 16) : *(const float*)src;
        } else {
          v = BF16 ? __uint_as_float((uint32_t)((const uint16_t*)rowp)[e] << 16) : ((const float*)rowp)[e];
        }
        if (pos < kCandCap) sm.cand[pos] = cand_key(v, (uint32_t)e);
        else sm.overflow = 1;
        ++pos;
      }
    }
    // this thread is done with its bytes of the slot: refill it with the
    // chunk kStages ahead
    prefetch_chunk<BF16>(p, ring, slot, ch + kStages < c_hi ? ch + kStages : p.T);
    __syncthreads();
    const int n = sm.count;
    // the first chunk ranks at once, so that later chunks compare with the
    // exact k-th best so far; later ones only when the buffer is half full
    if (first || sm.overflow || n > kCandCap / 2) {
      // compact the buffer to the k best (when it overflowed, this chunk's
      // logits join by k rounds of block-wide argmax)
      if (tid < DDT_TOPK_K_MAX) sm.top2[tid] = 0;
      __syncthreads();
      if (!sm.overflow) {
        rank_select2(sm.cand, n, nullptr, 0, p.k, sm.top2);
      } else {
        uint64_t prev = ~0ull;
        for (int r = 0; r < p.k; ++r) {
          uint64_t best = 0;
          for (int i = tid; i < kCandCap; i += kThreads) {
            const uint64_t key = sm.cand[i];
            if (key < prev && key > best) best = key;
          }
#pragma unroll
          for (int i = 0; i < NE; ++i) {
            const int idx = index_of(i);
            if (idx >= p.V) continue;
            const uint64_t key = cand_key(value_of(i), (uint32_t)idx);
            if (key < prev && key > best) best = key;
          }
          best = block_max_u64(best, sm.red);
          if (tid == 0) sm.top2[r] = best;
          prev = best;
        }
      }
      __syncthreads();
      if (tid < p.k) sm.cand[tid] = sm.top2[tid];
      if (tid == 0) {
        sm.count = p.k;
        sm.overflow = 0;
      }
      __syncthreads();
      tau = sm.top2[p.k - 1];
      if (tau == 0) {  // fewer than k logits so far: keep them all
        if (tid == 0) {
          int c = 0;
          while (c < p.k && sm.top2[c] != 0) ++c;
          sm.count = c;
        }
        __syncthreads();
      }
    }
    first = false;

    // end of this CTA's part of the row: rank the buffer, publish (or
    // finish the row)
    if (cidx == p.S - 1 || ch == c_hi - 1) {
      float M = m, Ssum = s;
      block_ms_reduce(M, Ssum, p.c, sm.wm, sm.wsum);  // barriers
      if (tid < DDT_TOPK_K_MAX) sm.top[tid] = 0;
      __syncthreads();
      rank_select2(sm.cand, min(sm.count, kCandCap), nullptr, 0, p.k, sm.top);
      __syncthreads();
      const int64_t g_first = owner_of((int64_t)row * p.S, p.T, p.G);
      const int64_t g_last = owner_of((int64_t)row * p.S + p.S - 1, p.T, p.G);
      if (g_first == g_last) {
        write_row(p, row, sm.top, row_lse_up(p.inv_t, M, Ssum));
      } else {
        const int slot_p = (int)(blockIdx.x - g_first);
        const int64_t pb = (int64_t)row * p.pmax + slot_p;
        for (int r = tid; r < p.k; r += kThreads) p.part_keys[pb * p.k + r] = sm.top[r];
        if (tid == 0) p.part_ms[pb] = make_float2(M, Ssum);
        __syncthreads();
        // one acquire-release ticket for the CTA: it releases the partial the
        // barrier ordered before it and, for the last CTA, acquires the others
        const int np = (int)(g_last - g_first + 1);
        if (tid == 0) sm.last = (atom_add_acq_rel_gpu(&p.tickets[row], 1u) == (unsigned)(np - 1));
        __syncthreads();
        if (sm.last) {
          // every partial's keys and (max, sum) in one round of loads, then
          // the row's k best ranked directly
          const int tot = np * p.k;
          float Mr = -INFINITY, Sr = 0.f;
          for (int cc = tid; cc < np; cc += kThreads) {
            const float2 ms = ld_cg_f2(&p.part_ms[(int64_t)row * p.pmax + cc]);
            ms_merge(Mr, Sr, ms.x, ms.y, p.c);
          }
          if (tid == 0) sm.count = 0;
          if (tot <= kCandCap) {
            for (int i = tid; i < tot; i += kThreads)
              sm.cand[i] = ld_cg_u64(&p.part_keys[(int64_t)row * p.pmax * p.k + i]);
          } else {
            // many partials: each has k keys at or above its k-th, so the
            // largest k-th key bounds the row's k-th from below
            uint64_t t = 0;
            for (int cc = tid; cc < np; cc += kThreads) {
              const uint64_t kk = ld_cg_u64(&p.part_keys[((int64_t)row * p.pmax + cc) * p.k + p.k - 1]);
              t = kk > t ? kk : t;
            }
            t = block_max_u64(t, sm.red);
            for (int i = tid; i < tot; i += kThreads) {
              const uint64_t key = ld_cg_u64(&p.part_keys[(int64_t)row * p.pmax * p.k + i]);
              if (key != 0 && key >= t) {
                const int pos = atomicAdd(&sm.count, 1);
                if (pos < kCandCap) sm.cand[pos] = key;
              }
            }
          }
          if (tid < DDT_TOPK_K_MAX) sm.top2[tid] = 0;
          block_ms_reduce(Mr, Sr, p.c, sm.wm, sm.wsum);  // its barriers publish cand / count
          const int n = tot <= kCandCap ? tot : sm.count;
          rank_select2(sm.cand, min(n, kCandCap), nullptr, 0, p.k, sm.top2);
          __syncthreads();
          write_row(p, row, sm.top2, row_lse_up(p.inv_t, Mr, Sr));
          if (tid == 0) p.tickets[row] = 0u;  // the counter region is left zero
        }
      }
      __syncthreads();
      m = -INFINITY;
      s = 0.f;
      tau = 0;
      first = true;
    }
  }
  cp_async_wait<0>();
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// CTAs the device runs at once (per SM, from the occupancy calculator).
int ctas_per_sm(bool bf16) {
  static std::mutex mu;
  static int known[2] = {0, 0};
  std::lock_guard<std::mutex> lock(mu);
  int& n = known[bf16 ? 1 : 0];
  if (n == 0) {
    const void* fn = bf16 ? (const void*)topk_kernel<true> : (const void*)topk_kernel<false>;
    const size_t smem = (size_t)kStages * kChunkBytes;
    int v = 0;
    if (ensure_smem_attr(fn, smem) == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fn, kThreads, smem) == cudaSuccess && v > 0)
      n = v;
    else
      n = 1;
    cudaGetLastError();  // a failed query must not leave a sticky error behind
  }
  return n;
}

struct Plan {
  int S, G, pmax;
  int64_t T;
};

Plan plan_for(int rows, int V, int es, bool bf16) {
  Plan pl;
  const int epc = kChunkBytes / es;
  pl.S = (V + epc - 1) / epc;
  pl.T = (int64_t)rows * pl.S;
  const int64_t slots = (int64_t)device_sm_count() * ctas_per_sm(bf16);
  pl.G = (int)(pl.T < slots ? pl.T : slots);
  if (pl.G < 1) pl.G = 1;
  // the CTAs a row's chunks can span: CTAs hold floor or ceil of T/G chunks
  // each, so those wholly inside a row number fewer than (S + 1) G / T
  pl.pmax = (int)(((int64_t)pl.S + 1) * pl.G / (pl.T > 0 ? pl.T : 1)) + 3;
  return pl;
}

}  // namespace

size_t topk_workspace_size(int rows, int V, int k) {
  // bf16 rows have half as many chunks; size for the larger (f32) plan
  const Plan pl = plan_for(rows, V, 4, false);
  const Plan pb = plan_for(rows, V, 2, true);
  const int pmax = pl.pmax > pb.pmax ? pl.pmax : pb.pmax;
  if (pl.S <= 1 && pb.S <= 1) return 0;
  return (size_t)DDT_WS_COUNTER_BYTES + align256(sizeof(float2) * (size_t)rows * pmax) +
         align256(sizeof(uint64_t) * (size_t)rows * pmax * k);
}

ddt_status launch_topk(const void* logits, ddt_dtype dt, int rows, int V, int64_t row_stride,
                       int k, float inv_t, int32_t* ids, float* zk, float* logp, float* lse,
                       void* ws, size_t ws_bytes, cudaStream_t stream) {
  (void)ws_bytes;
  if (rows == 0) return DDT_OK;
  const bool bf16 = dt == DDT_BF16;
  const int es = bf16 ? 2 : 4;
  const Plan pl = plan_for(rows, V, es, bf16);
  // the workspace is sized for the larger of the two dtypes' plans
  const Plan pf = plan_for(rows, V, 4, false), pb = plan_for(rows, V, 2, true);
  TopkParams p;
  p.logits = logits;
  p.rows = rows;
  p.V = V;
  p.row_stride = row_stride;
  p.k = k;
  p.inv_t = inv_t;
  p.c = inv_t * kLog2e;
  p.S = pl.S;
  p.G = pl.G;
  p.T = pl.T;
  p.pmax = pf.pmax > pb.pmax ? pf.pmax : pb.pmax;
  p.vec_ok = ((uintptr_t)logits % 16 == 0) && ((row_stride * es) % 16 == 0);
  char* w = (char*)ws;
  p.tickets = (unsigned*)w;  // counter region: one ticket per row
  if (w) w += DDT_WS_COUNTER_BYTES;
  p.part_ms = (float2*)w;
  if (w) w += align256(sizeof(float2) * (size_t)rows * p.pmax);
  p.part_keys = (uint64_t*)w;
  p.ids = ids;
  p.zk = zk;
  p.logp = logp;
  p.lse = lse;
  const size_t smem = (size_t)kStages * kChunkBytes;
  const void* fn = bf16 ? (const void*)topk_kernel<true> : (const void*)topk_kernel<false>;
  if (ensure_smem_attr(fn, smem) != cudaSuccess) return DDT_ERR_CUDA;
  const cudaError_t e =
      bf16 ? launch_pdl(topk_kernel<true>, dim3(pl.G), dim3(kThreads), smem, stream, 0, p)
           : launch_pdl(topk_kernel<false>, dim3(pl.G), dim3(kThreads), smem, stream, 0, p);
  return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
