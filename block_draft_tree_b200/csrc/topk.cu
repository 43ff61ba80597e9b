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
//     later reads the same 64 bytes of a chunk, so no block barrier guards
//     the ring), so that two chunks per CTA are always in flight;
//   * per chunk, each thread folds its 32 (bf16) or 16 (f32) logits into a
//     running (max, sum of 2^((z - max) * c)) and compares its chunk maximum
//     with the CTA's current bound on the k-th best key.  The lanes whose
//     maximum reaches it are rare, but a warp that holds one is not, so the
//     warp takes its hot lanes together: one hot lane at a time, every lane
//     checks one of its logits (re-read from the ring) and the candidates
//     go to a shared buffer with one ballot and one atomic.  The buffer is
//     ranked (exactly, by the 64-bit keys) whenever it holds more than 4k
//     keys -- which raises the bound to the exact k-th best so far -- and at
//     the end of the CTA's part of the row;
//   * the first chunk of each row a CTA sees starts from a bound k logits
//     are sure to reach: the k-th largest lane maximum of the CTA (a sort of
//     32 keys inside each warp, then a rank over the warps' sorted lists);
//   * a CTA's part of a row ends in a partial (k best keys, sorted, max,
//     sum) in the workspace; the last CTA of the row (one acquire-release
//     ticket, no waiting) merges the partials by rank (a binary search in
//     each sorted list), writes the row's outputs and returns its ticket to
//     zero.
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
constexpr int kOneChunk = 8192;                // logits per CTA of the one-chunk kernel
constexpr int kWarps = kThreads / 32;

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

// First chunk of CTA g's range, and the CTA whose range holds chunk ch
// (32-bit arithmetic: the host keeps T * G below 2^32).
__host__ __device__ __forceinline__ uint32_t range_lo(uint32_t g, uint32_t T, uint32_t G) {
  return g * T / G;
}
__host__ __device__ __forceinline__ uint32_t owner_of(uint32_t ch, uint32_t T, uint32_t G) {
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

// The k largest of the distinct nonzero keys a[0..n) (zeros: "no
// element"), in descending order, into out[0..k): each key's rank is the
// number of keys above it (16-byte loads, eight keys per step, so that the
// shared-memory loads overlap; a is 16-byte aligned).
__device__ void rank_select(const uint64_t* a, int n, int k, uint64_t* out) {
  const int n2 = n & ~7;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint64_t key = a[i];
    if (key == 0) continue;
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
    for (int j = 0; j < n2; j += 8) {
      const ulonglong2 x0 = *(const ulonglong2*)(a + j), x1 = *(const ulonglong2*)(a + j + 2);
      const ulonglong2 x2 = *(const ulonglong2*)(a + j + 4), x3 = *(const ulonglong2*)(a + j + 6);
      r0 += (x0.x > key) + (x0.y > key);
      r1 += (x1.x > key) + (x1.y > key);
      r2 += (x2.x > key) + (x2.y > key);
      r3 += (x3.x > key) + (x3.y > key);
    }
    for (int j = n2; j < n; ++j) r0 += a[j] > key;
    const int r = (r0 + r1) + (r2 + r3);
    if (r < k) out[r] = key;
  }
}

// The warp's 32 keys sorted descending across the lanes (lane i gets the
// i-th largest): a bitonic network on 64-bit keys.
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t v) {
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
  return v;
}

// The k-th largest nonzero key over the CTA's lanes (0 when fewer than k
// lanes hold one; keys may repeat), from each warp's k largest, sorted: a
// key is the k-th when fewer than k keys lie above it and at least k at or
// above it, both counted by binary searches in every warp's list.  Barriers:
// two.  wtop: kWarps * k keys of shared scratch.
__device__ uint64_t block_kth_key(uint64_t v, int k, uint64_t* wtop, uint64_t* result) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t sorted = warp_sort_desc(v);
  if (lane < k) wtop[warp * k + lane] = sorted;
  if (threadIdx.x == 0) *result = 0;
  __syncthreads();
  if ((int)threadIdx.x < kWarps * k) {
    const uint64_t key = wtop[threadIdx.x];
    if (key != 0) {
      int gt = 0, ge = 0;
      for (int w = 0; w < kWarps; ++w) {
        const uint64_t* l = wtop + w * k;
        int lo = 0, hi = k;  // first position not above key
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (l[mid] > key) lo = mid + 1;
          else hi = mid;
        }
        gt += lo;
        hi = k;  // first position below key
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (l[mid] >= key) lo = mid + 1;
          else hi = mid;
        }
        ge += lo;
      }
      if (gt < k && ge >= k) *result = key;  // equal keys write the same value
    }
  }
  __syncthreads();
  return *result;
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
  __align__(16) uint64_t cand[kCandCap];  // 16-byte loads in rank_select
  uint64_t top[DDT_TOPK_K_MAX];
  uint64_t top2[DDT_TOPK_K_MAX];
  uint64_t red[kThreads / 32];
  uint64_t wtop[kThreads / 32 * DDT_TOPK_K_MAX];  // each warp's largest lane maxima
  uint64_t kth;
  float wm[kThreads / 32], wsum[kThreads / 32];
  int count, last, overflow;
};

// The last CTA of a row merges the row's np partials (k keys, sorted, and
// (max, sum) each): every partial in one round of loads (above the buffer's
// capacity, only the keys that reach the largest k-th key of any partial:
// each partial has k keys at or above it), the k best ranked exactly, the
// row written, and the row's ticket returned to zero.
__device__ void merge_row(const TopkParams& p, int row, int np, Smem& sm) {
  const int tid = threadIdx.x;
  const int tot = np * p.k;
  const uint64_t* keys = p.part_keys + (int64_t)row * p.pmax * p.k;
  float Mr = -INFINITY, Sr = 0.f;
  for (int cc = tid; cc < np; cc += kThreads) {
    const float2 ms = ld_cg_f2(&p.part_ms[(int64_t)row * p.pmax + cc]);
    ms_merge(Mr, Sr, ms.x, ms.y, p.c);
  }
  if (tid == 0) sm.count = 0;
  if (tot <= kCandCap) {
    for (int i = tid; i < tot; i += kThreads) sm.cand[i] = ld_cg_u64(&keys[i]);
  } else {
    uint64_t t = 0;
    for (int cc = tid; cc < np; cc += kThreads) {
      const uint64_t kk = ld_cg_u64(&keys[cc * p.k + p.k - 1]);
      t = kk > t ? kk : t;
    }
    t = block_max_u64(t, sm.red);
    for (int i = tid; i < tot; i += kThreads) {
      const uint64_t key = ld_cg_u64(&keys[i]);
      if (key != 0 && key >= t) {
        const int pos = atomicAdd(&sm.count, 1);
        if (pos < kCandCap) sm.cand[pos] = key;
      }
    }
  }
  if (tid < DDT_TOPK_K_MAX) sm.top2[tid] = 0;
  block_ms_reduce(Mr, Sr, p.c, sm.wm, sm.wsum);  // its barriers publish cand / count
  rank_select(sm.cand, tot <= kCandCap ? tot : min(sm.count, kCandCap), p.k, sm.top2);
  __syncthreads();
  write_row(p, row, sm.top2, row_lse_up(p.inv_t, Mr, Sr));
  if (tid == 0) p.tickets[row] = 0u;  // the counter region is left zero
}

// Issue this thread's copies of chunk cidx of row `row` into ring slot
// `slot` when `live` (vectors entirely inside the row only; the one that
// straddles V is read from global memory when the chunk is used).  Always
// commits one group.
template <bool BF16>
__device__ __forceinline__ void prefetch_chunk(const TopkParams& p, unsigned char* ring, int slot,
                                               bool live, int row, int cidx) {
  constexpr int ES = BF16 ? 2 : 4, EPV = 16 / ES, EPC = kChunkBytes / ES;
  if (p.vec_ok && live) {
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

// Append the candidates of the warp's hot lanes (those whose chunk maximum
// reaches the bound) to the shared buffer, one hot lane at a time: lane l
// takes the hot lane's element l (elements in increasing index order within
// each of its 16-byte vectors), re-read from the hot lane's bytes of the
// ring slot, or from global memory for a vector the ring does not hold; a
// ballot counts the candidates, the leader reserves them with one atomic,
// and each lane writes its own key.  A candidate is a logit above tv, or
// equal to it at an index <= ti (ti >= 0 on a row's first chunk only), or,
// with take_all, every logit of the row.  Called by whole warps after the
// hot lanes waited for their copies; ends with __syncwarp, after which the
// hot lanes may refill their bytes of the slot.
template <bool BF16>
__device__ __forceinline__ void append_hot_lanes(uint32_t hot, int vec_ok, int V,
                                                 const unsigned char* ring_slot, const char* rowp,
                                                 int e0, float tv, int ti, bool take_all, Smem& sm) {
  constexpr int ES = BF16 ? 2 : 4, EPV = 16 / ES, NE = kChunkBytes / ES / kThreads;
  const int lane = threadIdx.x & 31, wbase = threadIdx.x & ~31;
  __syncwarp();  // the hot lanes' copies are visible to the warp
  const int q = lane / EPV, r = lane % EPV;  // this lane's element: vector q, element r
  while (hot) {
    const int h = __ffs(hot) - 1;
    hot &= hot - 1u;
    const int vq = q * kThreads + wbase + h;  // vector of the chunk
    const int e = e0 + vq * EPV + r;
    bool c = false;
    float v = -INFINITY;
    if (lane < NE && e < V) {
      if (vec_ok && e - r + EPV <= V) {
        const unsigned char* src = ring_slot + vq * 16 + r * ES;
        v = BF16 ? __uint_as_float((uint32_t)(*(const uint16_t*)src) << 16) : *(const float*)src;
      } else {
        v = BF16 ? __uint_as_float((uint32_t)((const uint16_t*)rowp)[e] << 16) : ((const float*)rowp)[e];
      }
      c = take_all || v > tv || (v == tv && ti >= 0 && e <= ti);
    }
    const uint32_t cm = __ballot_sync(0xFFFFFFFFu, c);
    int base = 0;
    if (lane == 0) base = atomicAdd(&sm.count, __popc(cm));
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
    if (c) {
      const int pos = base + __popc(cm & ((1u << lane) - 1u));
      if (pos < kCandCap) sm.cand[pos] = cand_key(v, (uint32_t)e);
      else sm.overflow = 1;
    }
  }
  __syncwarp();
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
  const uint32_t T32 = (uint32_t)p.T, G32 = (uint32_t)p.G;
  const int c_lo = (int)range_lo(blockIdx.x, T32, G32), c_hi = (int)range_lo(blockIdx.x + 1, T32, G32);
  int row = (int)((uint32_t)c_lo / (uint32_t)p.S), cidx = c_lo - row * p.S, slot = 0;
  // the prefetch cursor runs kStages chunks ahead (no division per chunk)
  int pf_ch = c_lo;
  int pf_row = row, pf_cidx = cidx;
  auto pf_next = [&]() {
    const bool live = pf_ch < c_hi;
    const int r = pf_row, c = pf_cidx;
    ++pf_ch;
    if (++pf_cidx == p.S) {
      pf_cidx = 0;
      ++pf_row;
    }
    return make_int3(live, r, c);
  };
  pdl_wait();
  for (int i = 0; i < kStages; ++i) {
    const int3 f = pf_next();
    prefetch_chunk<BF16>(p, ring, i, f.x != 0, f.y, f.z);
  }
  pdl_trigger();

  float m = -INFINITY, s = 0.f;  // this thread's running (max, sum) for the current row
  uint64_t tau = 0;              // a lower bound of the segment's k-th best key (0: none yet)
  bool first = true;             // next chunk is the first of a row for this CTA
  for (int ch = c_lo; ch < c_hi; ++ch, slot = slot == kStages - 1 ? 0 : slot + 1) {
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
    if (p.vec_ok && e0 + EPC <= p.V) {  // the whole chunk is in the ring
#pragma unroll
      for (int q = 0; q < kVecPerThread; ++q) {
        const uint4 u = *(const uint4*)(ring + slot * kChunkBytes + (q * kThreads + tid) * 16);
        w[4 * q] = u.x;
        w[4 * q + 1] = u.y;
        w[4 * q + 2] = u.z;
        w[4 * q + 3] = u.w;
      }
    } else {  // the row's last chunk, or rows the ring cannot copy
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
    // the k best goes to a shared buffer, which is ranked whenever it holds
    // more than 4k keys and at the end of the segment.  The first chunk of
    // a row starts from a threshold k logits of the CTA reach: the k-th
    // largest lane maximum over the CTA (a lane maximum's key: its value at
    // the smallest index holding it); later chunks take the logits above
    // the current k-th best key's value (a logit equal to it comes later,
    // so it ranks below it).
    float tv;
    int ti;
    bool take_all;
    if (first) {
      // the lane's bound: the smallest key a logit of value mc can have (its
      // maximum's key is at least that); 0 for a lane past the row's end
      uint64_t kmax = 0;
      if (index_of(0) < p.V) {
        kmax = cand_key(mc, 0xFFFFFFFFu);
        if (kmax == 0) kmax = 1;
      }
      if (tid == 0) {
        sm.count = 0;
        sm.overflow = 0;
      }
      // k lanes hold a logit at or above the k-th largest lane maximum: a
      // lower bound of the k-th best (barriers)
      tau = block_kth_key(kmax, p.k, sm.wtop, &sm.kth);
      tv = tau ? key_val(tau) : -INFINITY;
      ti = INT_MAX;         // a logit equal to the bound may rank above it
      take_all = tau == 0;  // fewer than k lanes hold logits
    } else {
      tv = tau ? key_val(tau) : -INFINITY;
      ti = -1;
      take_all = tau == 0;
    }
    // candidates: only the lanes whose chunk maximum reaches the bound hold
    // any; their warp takes them one lane at a time
    const bool need = take_all || mc > tv || (mc == tv && ti >= 0);
    const uint32_t hot = __ballot_sync(0xFFFFFFFFu, need);
    if (hot)
      append_hot_lanes<BF16>(hot, p.vec_ok, p.V, ring + slot * kChunkBytes, rowp, e0, tv, ti, take_all,
                             sm);
    // this thread is done with its bytes of the slot: refill it with the
    // chunk kStages ahead
    {
      const int3 f = pf_next();
      prefetch_chunk<BF16>(p, ring, slot, f.x != 0, f.y, f.z);
    }
    __syncthreads();
    const int n = sm.count;
    // the first chunk ranks at once, so that later chunks compare with the
    // exact k-th best so far; later ones once the buffer holds more than 4k
    // keys, so that the bound keeps up with the row and the lists stay short
    if (first || sm.overflow || n > 4 * p.k) {
      // compact the buffer to the k best (when it overflowed, this chunk's
      // logits join by k rounds of block-wide argmax)
      if (tid < DDT_TOPK_K_MAX) sm.top2[tid] = 0;
      __syncthreads();
      if (!sm.overflow) {
        rank_select(sm.cand, n, p.k, sm.top2);
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
      rank_select(sm.cand, min(sm.count, kCandCap), p.k, sm.top);
      __syncthreads();
      const int g_first = (int)owner_of((uint32_t)(row * p.S), T32, G32);
      const int g_last = (int)owner_of((uint32_t)(row * p.S + p.S - 1), T32, G32);
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
        if (sm.last) merge_row(p, row, np, sm);
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

// One CTA per (row, 8192-logit chunk), for grids that the device holds at
// once (small batches): every thread loads its 32 logits straight into
// registers, the CTA's bound on its k-th best is the k-th largest thread
// maximum (a bisection on the order bits with a counting barrier), the
// logits that reach it are ranked exactly, and the last CTA of the row
// merges the chunks' partials as the streaming kernel does.  One pass over
// the logits, no ring and no per-chunk state: the latency of a single chunk
// is all there is.
template <bool BF16>
__global__ void __launch_bounds__(kThreads, 3) topk_chunk_kernel(TopkParams p) {
  constexpr int EPV = BF16 ? 8 : 4;             // elements per 16-byte vector
  constexpr int EPT = kOneChunk / kThreads;     // 32 elements per thread
  constexpr int VPT = EPT / EPV;
  constexpr int ES = BF16 ? 2 : 4;
  constexpr int NW = EPT * ES / 4;              // 32-bit words held per thread
  __shared__ Smem sm;

  const int tid = threadIdx.x;
  const int chunk = blockIdx.x, row = blockIdx.y;
  const int c0 = chunk * kOneChunk;
  pdl_wait();
  const char* rowp = (const char*)p.logits + (int64_t)row * p.row_stride * ES;

  // word j of vector q of this thread holds elements from index
  // c0 + (q*kThreads + tid)*EPV + j*(EPV/4); elements past V read as -inf
  uint32_t w[NW];
  const bool full = p.vec_ok && c0 + kOneChunk <= p.V;
  if (full) {
#pragma unroll
    for (int q = 0; q < VPT; ++q) {
      const uint4 v = ld_stream_v4(rowp + ((int64_t)c0 + (q * kThreads + tid) * EPV) * ES);
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
        const int e0 = c0 + (q * kThreads + tid) * EPV + j * (EPV / 4);
        if (BF16) {
          const uint32_t lo = e0 < p.V ? ((const uint16_t*)rowp)[e0] : 0xFF80u;
          const uint32_t hi = e0 + 1 < p.V ? ((const uint16_t*)rowp)[e0 + 1] : 0xFF80u;
          w[4 * q + j] = lo | (hi << 16);
        } else {
          w[4 * q + j] = e0 < p.V ? __float_as_uint(((const float*)rowp)[e0]) : 0xFF800000u;
        }
      }
  }
  pdl_trigger();
  const int ibase = c0 + tid * EPV;
  auto index_of = [&](int e) -> int { return ibase + (e / EPV) * kThreads * EPV + (e % EPV); };
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
  // thread max and sum of 2^((z - max) * c), two logits per packed FFMA
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
    const uint64_t c2 = pack2(p.c, p.c), nm2 = pack2(-m * p.c, -m * p.c);
    uint64_t acc[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < EPT; i += 2) {
      const uint64_t x2 = ffma2(pack2(value_of(i), value_of(i + 1)), c2, nm2);
      float xa, xb;
      unpack2(x2, xa, xb);
      acc[(i >> 1) & 1] = fadd2(acc[(i >> 1) & 1], pack2(ex2(xa), ex2(xb)));
    }
    float a0, a1, b0, b1;
    unpack2(acc[0], a0, a1);
    unpack2(acc[1], b0, b1);
    s = (a0 + a1) + (b0 + b1);
  }
  // the order bits of the thread maximum (0: the thread holds no element)
  uint32_t tk = 0;
  if (nvalid > 0) {
    tk = BF16 ? ord16(__float_as_uint(m) >> 16) : ord32(m);
    if (tk == 0) tk = 1;
  }
  if (tid == 0) {
    sm.count = 0;
    sm.overflow = 0;
  }
  // the k-th largest thread maximum over the CTA: k threads hold a logit
  // at or above it, so it bounds the chunk's k-th best from below
  constexpr int KB = BF16 ? 16 : 32;
  uint32_t tau = 0;
#pragma unroll 1
  for (int bit = KB - 1; bit >= 0; --bit) {
    const uint32_t cand = tau | (1u << bit);
    if (__syncthreads_count(tk >= cand) >= p.k) tau = cand;
  }
  if (tau == 0) tau = 1;  // fewer than k threads hold logits: take them all
  {
    const uint32_t tb = BF16 ? (tau & 0xFFFFu) : tau;
    const uint32_t tbits = BF16 ? (((tb & 0x8000u) ? (tb & 0x7FFFu) : (~tb & 0xFFFFu)) << 16)
                                : ((tb & 0x80000000u) ? (tb & 0x7FFFFFFFu) : ~tb);
    // order bits below those of -inf only come from the take-everything case
    const float tf = tb < (BF16 ? 0x7Fu : 0x007FFFFFu) ? -INFINITY : __uint_as_float(tbits);
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const float v = value_of(e);
      if (v >= tf) {
        const int idx = index_of(e);
        if (!full && idx >= p.V) continue;
        const int pos = atomicAdd(&sm.count, 1);
        if (pos < kCandCap) sm.cand[pos] = cand_key(v, (uint32_t)idx);
      }
    }
  }
  if (tid < DDT_TOPK_K_MAX) sm.top[tid] = 0;
  block_ms_reduce(m, s, p.c, sm.wm, sm.wsum);  // its barriers publish the candidates
  const int n = sm.count;
  if (n <= kCandCap) {
    rank_select(sm.cand, n, p.k, sm.top);
  } else {
    // a degenerate chunk (many equal logits): k rounds of block argmax
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
      best = block_max_u64(best, sm.red);
      if (tid == 0) sm.top[r] = best;
      prev = best;
    }
  }
  __syncthreads();
  if (p.S == 1) {
    write_row(p, row, sm.top, row_lse_up(p.inv_t, m, s));
    return;
  }
  // publish this chunk's partial (sorted), then one acquire-release ticket
  const int64_t pb = (int64_t)row * p.pmax + chunk;
  for (int r = tid; r < p.k; r += kThreads) p.part_keys[pb * p.k + r] = sm.top[r];
  if (tid == 0) p.part_ms[pb] = make_float2(m, s);
  __syncthreads();
  if (tid == 0) sm.last = (atom_add_acq_rel_gpu(&p.tickets[row], 1u) == (unsigned)(p.S - 1));
  __syncthreads();
  if (sm.last) merge_row(p, row, p.S, sm);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// CTAs the device runs at once (per SM, from the occupancy calculator) of
// the streaming kernel (chunk = false) or the one-chunk kernel.
int ctas_per_sm(bool bf16, bool chunk = false) {
  static std::mutex mu;
  static int known[2][2] = {{0, 0}, {0, 0}};
  std::lock_guard<std::mutex> lock(mu);
  int& n = known[chunk ? 1 : 0][bf16 ? 1 : 0];
  if (n == 0) {
    const void* fn = chunk ? (bf16 ? (const void*)topk_chunk_kernel<true> : (const void*)topk_chunk_kernel<false>)
                           : (bf16 ? (const void*)topk_kernel<true> : (const void*)topk_kernel<false>);
    const size_t smem = chunk ? 0 : (size_t)kStages * kChunkBytes;
    int v = 0;
    if ((chunk || ensure_smem_attr(fn, smem) == cudaSuccess) &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fn, kThreads, smem) == cudaSuccess && v > 0)
      n = v;
    else
      n = 1;
    cudaGetLastError();  // a failed query must not leave a sticky error behind
  }
  return n;
}

// Chunks of the one-chunk kernel per row, and whether its grid fits on the
// device at once (then it serves the call: one pass, no ring).
int one_chunks(int V) { return (V + kOneChunk - 1) / kOneChunk; }
bool one_chunk_fits(int rows, int V, bool bf16) {
  return (int64_t)rows * one_chunks(V) <= (int64_t)device_sm_count() * ctas_per_sm(bf16, true);
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
  // the device partitions chunks in 32-bit arithmetic: T * G < 2^32
  if (pl.T > 0 && (int64_t)pl.G > 0xFFFFFFFFll / pl.T) pl.G = (int)(0xFFFFFFFFll / pl.T);
  if (pl.G < 1) pl.G = 1;
  // the CTAs a row's chunks can span: CTAs hold floor or ceil of T/G chunks
  // each, so those wholly inside a row number fewer than (S + 1) G / T
  pl.pmax = (int)(((int64_t)pl.S + 1) * pl.G / (pl.T > 0 ? pl.T : 1)) + 3;
  return pl;
}

}  // namespace

namespace {
// Partial slots per row the workspace holds: enough for either kernel and
// either dtype (0: no call needs a workspace).
int partial_slots(int rows, int V) {
  const Plan pl = plan_for(rows, V, 4, false);
  const Plan pb = plan_for(rows, V, 2, true);
  int pmax = pl.pmax > pb.pmax ? pl.pmax : pb.pmax;
  if (one_chunks(V) > pmax) pmax = one_chunks(V);
  if (pl.S <= 1 && pb.S <= 1 && one_chunks(V) <= 1) return 0;
  return pmax;
}
}  // namespace

size_t topk_workspace_size(int rows, int V, int k) {
  const int pmax = partial_slots(rows, V);
  if (pmax == 0) return 0;
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
  // more than 2^31 chunks of 16 KB (32 TB of logits) cannot be resident
  if (pl.T >= (int64_t)1 << 31) return DDT_ERR_UNSUPPORTED;
  const bool one = one_chunk_fits(rows, V, bf16);
  const int slots = partial_slots(rows, V);  // the workspace's partial slots per row
  TopkParams p;
  p.logits = logits;
  p.rows = rows;
  p.V = V;
  p.row_stride = row_stride;
  p.k = k;
  p.inv_t = inv_t;
  p.c = inv_t * kLog2e;
  p.S = one ? one_chunks(V) : pl.S;
  p.G = pl.G;
  p.T = pl.T;
  p.pmax = one ? one_chunks(V) : slots;  // partial slots per row (the row stride)
  p.vec_ok = ((uintptr_t)logits % 16 == 0) && ((row_stride * es) % 16 == 0);
  char* w = (char*)ws;
  p.tickets = (unsigned*)w;  // counter region: one ticket per row
  if (w) w += DDT_WS_COUNTER_BYTES;
  p.part_ms = (float2*)w;
  if (w) w += align256(sizeof(float2) * (size_t)rows * slots);
  p.part_keys = (uint64_t*)w;
  p.ids = ids;
  p.zk = zk;
  p.logp = logp;
  p.lse = lse;
  if (one) {
    const dim3 grid((unsigned)one_chunks(V), (unsigned)rows);
    const cudaError_t e = bf16 ? launch_pdl(topk_chunk_kernel<true>, grid, dim3(kThreads), 0, stream, 0, p)
                               : launch_pdl(topk_chunk_kernel<false>, grid, dim3(kThreads), 0, stream, 0, p);
    return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
  }
  const size_t smem = (size_t)kStages * kChunkBytes;
  const void* fn = bf16 ? (const void*)topk_kernel<true> : (const void*)topk_kernel<false>;
  if (ensure_smem_attr(fn, smem) != cudaSuccess) return DDT_ERR_CUDA;
  const cudaError_t e =
      bf16 ? launch_pdl(topk_kernel<true>, dim3(pl.G), dim3(kThreads), smem, stream, 0, p)
           : launch_pdl(topk_kernel<false>, dim3(pl.G), dim3(kThreads), smem, stream, 0, p);
  return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
