// walk.cu -- stage 4 of the verification round: the greedy tree walk.
//
// DDTree page, section 運作流程 step 4: from the root, take the target's
// next token under its decoding rule; if the current node has a child with
// that token, accept it and continue; the first token that matches no child
// is carried into the next round as the bonus token.  The greedy rule is
// argmax with the smaller token id on ties.
//
// Design: the walk needs the argmax of the rows it visits, and each argmax
// is a full scan of V logits, so the kernel is an HBM-bound scan of every
// tree row followed by a walk that costs nothing:
//   * grid = (chunks of 8192 logits, rows, sequences); each CTA scans one
//     chunk with 16-byte streaming loads and reduces a 64-bit key
//     (value, then smaller id);
//   * the last CTA of a row (atomic ticket) merges the chunk keys into the
//     row's argmax; the last row of a sequence to finish (a second ticket)
//     stages the sequence's argmaxes and tree in shared memory with one
//     coalesced pass and walks it with one warp.
// No CTA ever waits on another, so there is no spin and nothing to time out.
//
// Sampling rule (target temperature T > 0): the walk stays lossless when each
// visited row draws its token from softmax(z / T) with a fresh uniform, so
// the token of row j of sequence b is the inverse-CDF draw over token ids in
// increasing order with u from Philox4x64-10 (Salmon, Moraes, Dror and Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) at counter
// (j, b, 0, 0) under key (seed, step [+ *step_counter]): u = (top 52 bits of word 0 + 1/2)
// * 2^-52.  The scan then keeps, per chunk, the pair (R, s): an integer
// reference R (the largest exponent) and the fp64 sum s of the chunk's
// weights against R, instead of an argmax key; the row's last CTA merges
// the pairs, finds the chunk whose cumulative weight first exceeds u times
// the total, and rescans that one chunk (from L2) with a block prefix sum
// to find the token.  Each weight is an fp32 evaluation of 2^(t - R),
// t = z*log2(e)/T (with the rounding of t added back), that is exact in
// fp64 by construction (see draw_weight),
// so weights against different references differ by exact powers of two
// and only the fp64 sums round: the draws land on tokens of probability
// ~1/V, where an fp32 cumulative sum (~1e-7 relative error) would move a
// fair share of them to a neighbour.
#include <climits>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8192;

struct WalkParams {
  const void* logits;
  int batch, n_max, V, S, vec_ok, L;
  int64_t row_stride;
  const int32_t *tok, *parent, *depth, *n_nodes;
  int32_t *acc_len, *acc_nodes, *acc_tok, *bonus;
  uint64_t* part;        // [batch*n_max][S]
  int32_t* amax;         // [batch*n_max]
  unsigned* row_ticket;  // [batch*n_max]
  unsigned* seq_count;   // [batch]
  unsigned* draw_count;  // sampling with a step counter: rows drawn so far
  int32_t* status;
  float a, a_lo;         // sampling: fl32(log2(e) / T) and fl32 of the rest
  uint64_t seed, step;   // sampling: Philox key
  uint64_t* step_counter;  // sampling: optional device word added to step, advanced per call
};

__device__ __forceinline__ uint64_t block_max_key(uint64_t v, uint64_t* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t u = shfl_xor_u64(v, o);
    v = u > v ? u : v;
  }
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  uint64_t r = 0;
  for (int w = 0; w < kThreads / 32; ++w) r = sm[w] > r ? sm[w] : r;
  return r;
}

// One warp walks sequence b with its argmaxes and tree staged in shared memory.
__device__ void walk_sequence(const WalkParams& p, int b, int n, const int* s_amax, const int* s_tok,
                              const int* s_par, const int* s_dep) {
  const int lane = threadIdx.x & 31;
  int x = 0, a = 0, bonus = 0;
#pragma unroll 1
  for (;;) {
    const int t = s_amax[x];
    int next = -1;
    if (a < p.L && s_dep[x] < p.L) {
      // children of x come after x (rows are breadth-first)
      for (int c0 = x + 1; c0 < n; c0 += 32) {
        const int c = c0 + lane;
        const bool hit = c < n && s_par[c] == x && s_tok[c] == t;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, hit);
        if (bal) {
          next = c0 + __ffs(bal) - 1;
          break;
        }
      }
    }
    if (next < 0) {
      bonus = t;
      break;
    }
    if (lane == 0) {
      p.acc_nodes[(int64_t)b * p.L + a] = next;
      p.acc_tok[(int64_t)b * p.L + a] = t;
    }
    ++a;
    x = next;
  }
  for (int i = a + lane; i < p.L; i += 32) {
    p.acc_nodes[(int64_t)b * p.L + i] = -1;
    p.acc_tok[(int64_t)b * p.L + i] = -1;
  }
  if (lane == 0) {
    p.acc_len[b] = a;
    p.bonus[b] = bonus;
  }
}

template <bool BF16>
struct Chunk {
  static constexpr int EPV = BF16 ? 8 : 4;
  static constexpr int VPT = kChunk / kThreads / EPV;
  uint4 v[VPT];
};

// Issue the loads of one (row, chunk) item (full chunks only).
template <bool BF16>
__device__ __forceinline__ void load_chunk(Chunk<BF16>& c, const char* rowp, int64_t c0) {
  constexpr int EPV = Chunk<BF16>::EPV, ES = BF16 ? 2 : 4;
#pragma unroll
  for (int q = 0; q < Chunk<BF16>::VPT; ++q)
    c.v[q] = ld_stream_v4(rowp + (c0 + (int64_t)(q * kThreads + threadIdx.x) * EPV) * ES);
}

// Loads of a chunk that may run past V: whole 16-byte vectors inside the
// row, element loads for the one that straddles V, and -inf beyond it.
template <bool BF16>
__device__ __forceinline__ void load_chunk_tail(Chunk<BF16>& c, const char* rowp, int c0, int V) {
  constexpr int EPV = Chunk<BF16>::EPV, ES = BF16 ? 2 : 4;
#pragma unroll
  for (int q = 0; q < Chunk<BF16>::VPT; ++q) {
    const int idx = c0 + (q * kThreads + threadIdx.x) * EPV;
    if (idx + EPV <= V) {
      c.v[q] = ld_stream_v4(rowp + (int64_t)idx * ES);
    } else {
      uint32_t w[4];
      for (int e = 0; e < 4; ++e) {
        if (BF16) {
          const uint32_t lo = idx + 2 * e < V ? ((const uint16_t*)rowp)[idx + 2 * e] : 0xFF80u;
          const uint32_t hi = idx + 2 * e + 1 < V ? ((const uint16_t*)rowp)[idx + 2 * e + 1] : 0xFF80u;
          w[e] = lo | (hi << 16);
        } else {
          w[e] = idx + e < V ? ((const uint32_t*)rowp)[idx + e] : 0xFF800000u;
        }
      }
      c.v[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Thread-local argmax of a loaded chunk; each thread sees its indices in
// increasing order, so strict > keeps the smallest index among equal values.
template <bool BF16>
__device__ __forceinline__ void argmax_chunk(const Chunk<BF16>& c, int c0, float& bv, int& bi) {
  constexpr int EPV = Chunk<BF16>::EPV;
#pragma unroll
  for (int q = 0; q < Chunk<BF16>::VPT; ++q) {
    const int base = c0 + (q * kThreads + (int)threadIdx.x) * EPV;
    const uint32_t w[4] = {c.v[q].x, c.v[q].y, c.v[q].z, c.v[q].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (BF16) {
        const float lo = bf16_lo(w[e]), hi = bf16_hi(w[e]);
        if (lo > bv || bi < 0) { bv = lo; bi = base + 2 * e; }
        if (hi > bv) { bv = hi; bi = base + 2 * e + 1; }
      } else {
        const float f = __uint_as_float(w[e]);
        if (f > bv || bi < 0) { bv = f; bi = base + e; }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Sampling rule
// ---------------------------------------------------------------------------

// Word 0 of the Philox4x64-10 block at counter (c0, c1, c2, c3) under key
// (k0, k1).  A round multiplies counter words 0 and 2 by the round
// multipliers; the new word 0 is hi(M1*x2) ^ x1 ^ k0, the new word 2 is
// hi(M0*x0) ^ x3 ^ k1, the low halves become words 1 and 3, and the key
// advances by the Weyl increments between rounds.
__device__ __forceinline__ uint64_t philox4x64_10_w0(uint64_t x0, uint64_t x1, uint64_t x2,
                                                     uint64_t x3, uint64_t k0, uint64_t k1) {
  constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t hi0 = __umul64hi(M0, x0), lo0 = M0 * x0;
    const uint64_t hi1 = __umul64hi(M1, x2), lo1 = M1 * x2;
    x0 = hi1 ^ x1 ^ k0;
    x1 = lo1;
    x2 = hi0 ^ x3 ^ k1;
    x3 = lo0;
    k0 += W0;
    k1 += W1;
  }
  return x0;
}

// The uniform in (0, 1) that tree row j of sequence b draws.
__device__ __forceinline__ double row_uniform(const WalkParams& p, int b, int j) {
  const uint64_t step = p.step + (p.step_counter ? __ldcg((const unsigned long long*)p.step_counter) : 0ull);
  const uint64_t w = philox4x64_10_w0((uint32_t)j, (uint32_t)b, 0, 0, p.seed, step);
  return ((double)(w >> 12) + 0.5) * 0x1.0p-52;
}

// The draw's weights.  The token is an integer decided by floating point,
// so its arithmetic is fixed exactly.  With A = log2(e)/T, a = fl32(A) and
// a_lo = fl32(A - a): t = fl32(a*z), k = nearest integer to t (ties to
// even), r = t - k (exact), P = fp32 Horner evaluation with fused
// multiply-adds of the degree-7 Taylor polynomial of 2^r (coefficients
// (ln 2)^i / i! rounded to fp32), then P += P * ln2 * e with
// e = fma(a_lo, z, fma(a, z, -t)), the part of A*z that t lost (an exact
// residual plus the rounding of A), and w = P * 2^(k - R), an exact normal
// fp32 number, for an integer reference R >= k (0 when k - R < -120 or
// z = -inf).  So a weight's error is the polynomial's (a few fp32 ulps) and
// does not grow with |A*z|.  Weights taken against different references
// differ by exact powers of two, so every chunk and thread sums against its
// own maximum and the sums merge without rounding the weights again.  A
// thread sums its 32 weights as two double-float sums of 16 (an exact
// TwoSum per term; the low part, below 2^-20 of the high part, rounds at
// 2^-24 of itself per term: relative error below 2^-40), and everything
// after that is fp64.
__device__ __forceinline__ float draw_poly(float r) {
  float p = 0x1.ffcbfcp-17f;
  p = fmaf(p, r, 0x1.430912p-13f);
  p = fmaf(p, r, 0x1.5d87fep-10f);
  p = fmaf(p, r, 0x1.3b2ab6p-7f);
  p = fmaf(p, r, 0x1.c6b08ep-5f);
  p = fmaf(p, r, 0x1.ebfbep-3f);
  p = fmaf(p, r, 0x1.62e43p-1f);
  return fmaf(p, r, 1.0f);
}

constexpr float kRoundShift = 12582912.0f;  // 1.5 * 2^23: t + shift rounds t to an integer
constexpr int kRoundShiftBits = 0x4B400000;
constexpr int kNoRef = -(1 << 30);          // reference of a thread with no finite logit
constexpr float kLn2f = 0.693147182f;       // ln 2 rounded to fp32

// R = nearest integer to t (|t| < 2^22).
__device__ __forceinline__ int draw_ref(float t) {
  return t >= -4.0e6f ? __float_as_int(__fadd_rn(t, kRoundShift)) - kRoundShiftBits : kNoRef;
}

// The weight of logit z against the reference R >= -4e6.  Branch free: for
// t below -2^22 (and -inf) the rounding trick yields an exponent far below
// R - 120, so the final select discards it (with whatever the correction
// made of it).
__device__ __forceinline__ float draw_weight(float z, float a, float a_lo, int R) {
  const float t = __fmul_rn(a, z);
  const float e_lo = __fmaf_rn(a_lo, z, __fmaf_rn(a, z, -t));
  const float sh = __fadd_rn(t, kRoundShift);
  const int e = __float_as_int(sh) - (kRoundShiftBits + R);
  const float r = __fsub_rn(t, __fsub_rn(sh, kRoundShift));
  float P = draw_poly(r);
  P = __fmaf_rn(P, __fmul_rn(e_lo, kLn2f), P);
  const float w = __int_as_float(__float_as_int(P) + (e << 23));
  return e >= -120 ? w : 0.f;
}

// The weights of a pair of logits z (packed), as draw_weight.
__device__ __forceinline__ uint64_t draw_weight2(uint64_t z2, uint64_t a2, uint64_t alo2, int R) {
  const uint64_t t2 = fmul2(a2, z2);
  const uint64_t e2 = ffma2(alo2, z2, ffma2(a2, z2, t2 ^ 0x8000000080000000ull));
  const uint64_t sh2 = fadd2(t2, pack2(kRoundShift, kRoundShift));
  const uint64_t r2 = fsub2(t2, fadd2(sh2, pack2(-kRoundShift, -kRoundShift)));
  uint64_t p2 = ffma2(pack2(0x1.ffcbfcp-17f, 0x1.ffcbfcp-17f), r2, pack2(0x1.430912p-13f, 0x1.430912p-13f));
  p2 = ffma2(p2, r2, pack2(0x1.5d87fep-10f, 0x1.5d87fep-10f));
  p2 = ffma2(p2, r2, pack2(0x1.3b2ab6p-7f, 0x1.3b2ab6p-7f));
  p2 = ffma2(p2, r2, pack2(0x1.c6b08ep-5f, 0x1.c6b08ep-5f));
  p2 = ffma2(p2, r2, pack2(0x1.ebfbep-3f, 0x1.ebfbep-3f));
  p2 = ffma2(p2, r2, pack2(0x1.62e43p-1f, 0x1.62e43p-1f));
  p2 = ffma2(p2, r2, pack2(1.f, 1.f));
  p2 = ffma2(p2, fmul2(e2, pack2(kLn2f, kLn2f)), p2);
  float sa, sb, pa, pb;
  unpack2(sh2, sa, sb);
  unpack2(p2, pa, pb);
  const int ea = __float_as_int(sa) - (kRoundShiftBits + R);
  const int eb = __float_as_int(sb) - (kRoundShiftBits + R);
  const float wa = ea >= -120 ? __int_as_float(__float_as_int(pa) + (ea << 23)) : 0.f;
  const float wb = eb >= -120 ? __int_as_float(__float_as_int(pb) + (eb << 23)) : 0.f;
  return pack2(wa, wb);
}

// hi + lo += w lane by lane, with hi + w split exactly (Knuth's TwoSum).
__device__ __forceinline__ void two_sum_add2(uint64_t& hi, uint64_t& lo, uint64_t w) {
  const uint64_t s = fadd2(hi, w);
  const uint64_t bp = fsub2(s, hi);
  const uint64_t err = fadd2(fsub2(hi, fsub2(s, bp)), fsub2(w, bp));
  hi = s;
  lo = fadd2(lo, err);
}



// s * 2^d for d <= 0, exact (0 below 2^-1000).
__device__ __forceinline__ double scale2(double s, int d) {
  return d < -1000 ? 0.0 : s * __hiloint2double((1023 + d) << 20, 0);
}

// Merge the pair (R2, s2) into (R, s); s is a sum of weights against R.
__device__ __forceinline__ void rs_add(int& R, double& s, int R2, double s2) {
  if (R2 == kNoRef) return;
  if (R == kNoRef) {
    R = R2;
    s = s2;
  } else if (R2 > R) {
    s = scale2(s, R - R2) + s2;
    R = R2;
  } else {
    s += scale2(s2, R2 - R);
  }
}

// Thread pair (R, sum of weights against R) over a loaded chunk, two
// tokens per packed instruction.  The thread's 32 weights are summed as two
// interleaved double-float sums of 16.
template <bool BF16>
__device__ __forceinline__ void rs_chunk(const Chunk<BF16>& c, float a, float a_lo, int& R, double& s) {
  float zm = -INFINITY;
#pragma unroll
  for (int q = 0; q < Chunk<BF16>::VPT; ++q) {
    const uint32_t w[4] = {c.v[q].x, c.v[q].y, c.v[q].z, c.v[q].w};
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      if (BF16) {
        zm = fmax3(zm, bf16_lo(w[i]), bf16_hi(w[i]));
        zm = fmax3(zm, bf16_lo(w[i + 1]), bf16_hi(w[i + 1]));
      } else {
        zm = fmax3(zm, __uint_as_float(w[i]), __uint_as_float(w[i + 1]));
      }
    }
  }
  R = draw_ref(__fmul_rn(a, zm));  // fl32(a*z) is monotone in z
  s = 0.0;
  if (R == kNoRef) return;
  const uint64_t a2 = pack2(a, a), alo2 = pack2(a_lo, a_lo);
  uint64_t hi = pack2(0.f, 0.f), lo = pack2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < Chunk<BF16>::VPT; ++q) {
    const uint32_t w[4] = {c.v[q].x, c.v[q].y, c.v[q].z, c.v[q].w};
    if (BF16) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        two_sum_add2(hi, lo, draw_weight2(pack2(bf16_lo(w[i]), bf16_hi(w[i])), a2, alo2, R));
    } else {
#pragma unroll
      for (int i = 0; i < 4; i += 2)
        two_sum_add2(hi, lo, draw_weight2(pack2(__uint_as_float(w[i]), __uint_as_float(w[i + 1])), a2, alo2, R));
    }
  }
  float ha, hb, la, lb;
  unpack2(hi, ha, hb);
  unpack2(lo, la, lb);
  s = ((double)ha + (double)la) + ((double)hb + (double)lb);
}

// Block merge of the threads' pairs; the result is valid in thread 0.
__device__ __forceinline__ void block_rs(int& R, double& s, double2* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const int R2 = __shfl_xor_sync(0xFFFFFFFFu, R, o);
    const double s2 = __shfl_xor_sync(0xFFFFFFFFu, s, o);
    rs_add(R, s, R2, s2);
  }
  if (lane == 0) sm[warp] = make_double2((double)R, s);
  __syncthreads();
  R = (int)sm[0].x;
  s = sm[0].y;
  for (int w = 1; w < kThreads / 32; ++w) rs_add(R, s, (int)sm[w].x, sm[w].y);
}

// Inclusive prefix sum over the lanes of a warp.
__device__ __forceinline__ double warp_incl_scan(double v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double u = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// One more row of the call has drawn (or has nothing to draw); the last of
// all batch * n_max rows advances the step counter, once every draw of the
// call has read it, and leaves the draw count zero.
__device__ __forceinline__ void count_draw(const WalkParams& p) {
  __threadfence();
  if (atomicAdd(p.draw_count, 1u) == (unsigned)(p.batch * p.n_max - 1)) {
    __threadfence();
    *p.step_counter += 1ull;
    *p.draw_count = 0u;
  }
}

struct SampleSmem {
  double P, theta;
  int R, cstar;
  double wsum[kThreads / 32];
  int hit, last;
};

__device__ __forceinline__ float load_logit(const char* rowp, int idx, bool bf16) {
  return bf16 ? bf16_to_f32(((const uint16_t*)rowp)[idx]) : ((const float*)rowp)[idx];
}

// The token drawn for row (b, j) once every chunk pair of the row is in
// `part`; called by the whole block, returns the token in every thread.
template <bool BF16>
__device__ int sample_row_token(const WalkParams& p, int b, int j, int64_t row, const char* rowp,
                                SampleSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double2* part = (const double2*)p.part + row * p.S;
  if (warp == 0) {
    int R = kNoRef;
    for (int c = lane; c < p.S; c += 32) R = max(R, (int)__ldcg(&part[c]).x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) R = max(R, __shfl_xor_sync(0xFFFFFFFFu, R, o));
    // two identical passes of the chunk prefix sum: the total, then the
    // first chunk whose inclusive prefix exceeds theta
    double theta = 0.0, P = 0.0, Plast = 0.0;
    int cstar = -1, clast = -1;
    for (int pass = 0; pass < 2 && R != kNoRef; ++pass) {
      double carry = 0.0;
      for (int g = 0; g < p.S; g += 32) {
        const int c = g + lane;
        double W = 0.0;
        if (c < p.S) {
          const double2 rs = __ldcg(&part[c]);
          if ((int)rs.x != kNoRef) W = scale2(rs.y, (int)rs.x - R);
        }
        const double incl = carry + warp_incl_scan(W);
        double excl = __shfl_up_sync(0xFFFFFFFFu, incl, 1);
        if (lane == 0) excl = carry;
        if (pass == 1) {
          const unsigned hit = __ballot_sync(0xFFFFFFFFu, c < p.S && incl > theta);
          const unsigned pos = __ballot_sync(0xFFFFFFFFu, W > 0.0);
          if (pos) {
            const int l = 31 - __clz(pos);
            clast = g + l;
            Plast = __shfl_sync(0xFFFFFFFFu, excl, l);
          }
          if (hit) {
            const int l = __ffs(hit) - 1;
            cstar = g + l;
            P = __shfl_sync(0xFFFFFFFFu, excl, l);
            break;
          }
        }
        carry = __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      if (pass == 0) theta = row_uniform(p, b, j) * carry;
    }
    if (cstar < 0) {  // theta rounded onto the total: the last chunk of positive weight
      cstar = clast;
      P = Plast;
    }
    if (lane == 0) {
      sm.R = R;
      sm.P = P;
      sm.theta = theta;
      sm.cstar = cstar;
      sm.hit = INT_MAX;
      sm.last = -1;
    }
  }
  __syncthreads();
  const int cstar = sm.cstar;
  if (cstar < 0) return 0;  // no finite logit in the row
  const int R = sm.R;
  const double theta = sm.theta;
  const float a = p.a, a_lo = p.a_lo;
  // each thread owns kPer consecutive tokens of chunk cstar
  constexpr int kPer = kChunk / kThreads;
  const int e0 = cstar * kChunk + tid * kPer;
  const int e1 = min(e0 + kPer, p.V);
  double local = 0.0;
  int last = -1;
  for (int i = e0; i < e1; ++i) {
    const double w = (double)draw_weight(load_logit(rowp, i, BF16), a, a_lo, R);
    local += w;
    if (w > 0.0) last = i;
  }
  // block exclusive prefix of the threads' sums
  const double incl = warp_incl_scan(local);
  if (lane == 31) sm.wsum[warp] = incl;
  __syncthreads();
  double wbase = 0.0;
  for (int v = 0; v < warp; ++v) wbase += sm.wsum[v];
  double excl = __shfl_up_sync(0xFFFFFFFFu, incl, 1);
  if (lane == 0) excl = 0.0;
  const double base = sm.P + (wbase + excl);
  if (base + local > theta) {
    // the crossing may be in this thread's tokens: walk them in order
    double cum = base;
    int hit = last;
    for (int i = e0; i < e1; ++i) {
      cum += (double)draw_weight(load_logit(rowp, i, BF16), a, a_lo, R);
      if (cum > theta) {
        hit = i;
        break;
      }
    }
    if (hit >= 0) atomicMin(&sm.hit, hit);
  }
  if (last >= 0) atomicMax(&sm.last, last);
  __syncthreads();
  return sm.hit != INT_MAX ? sm.hit : sm.last;
}

template <bool BF16, bool SAMPLE>
__global__ void __launch_bounds__(kThreads) walk_kernel(WalkParams p) {
  constexpr int EPV = Chunk<BF16>::EPV;
  constexpr int ES = BF16 ? 2 : 4;
  __shared__ uint64_t s_red[kThreads / 32];
  __shared__ __align__(16) uint64_t s_red2[2 * (kThreads / 32)];
  __shared__ int s_flag;
  __shared__ int s_amax[DDT_TREE_B_MAX + 1], s_tok[DDT_TREE_B_MAX + 1];
  __shared__ int s_par[DDT_TREE_B_MAX + 1], s_dep[DDT_TREE_B_MAX + 1];

  const int chunk = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  pdl_wait();
  int n = p.n_nodes[b];
  if (n < 1 || n > p.n_max) {
    if (chunk == 0 && j == 0 && tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    n = min(max(n, 1), p.n_max);
  }
  if (j >= n) {
    if (SAMPLE && p.step_counter && chunk == 0 && tid == 0) count_draw(p);  // a row without a draw
    return;
  }
  const int64_t row = (int64_t)b * p.n_max + j;
  const char* rowp = (const char*)p.logits + row * p.row_stride * ES;
  const int c0 = chunk * kChunk;

  if constexpr (SAMPLE) {
    __shared__ SampleSmem sm;
    // chunk pair (reference R, sum of weights against R)
    int R = kNoRef;
    double sum = 0.0;
    if (p.vec_ok) {
      Chunk<BF16> cur;
      if (c0 + kChunk <= p.V) load_chunk<BF16>(cur, rowp, c0);
      else load_chunk_tail<BF16>(cur, rowp, c0, p.V);
      rs_chunk<BF16>(cur, p.a, p.a_lo, R, sum);
    } else {
      for (int q = 0; q < Chunk<BF16>::VPT; ++q)
        for (int i = 0; i < EPV; ++i) {
          const int idx = c0 + (q * kThreads + tid) * EPV + i;
          if (idx >= p.V) continue;
          const float z = load_logit(rowp, idx, BF16);
          const int Rv = draw_ref(__fmul_rn(p.a, z));
          rs_add(R, sum, Rv, Rv == kNoRef ? 0.0 : (double)draw_weight(z, p.a, p.a_lo, Rv));
        }
    }
    pdl_trigger();
    block_rs(R, sum, (double2*)s_red2);
    const double2 rs = make_double2((double)R, sum);
    if (p.S > 1) {
      if (tid == 0) {
        ((double2*)p.part)[row * p.S + chunk] = rs;
        s_flag = (atom_add_acq_rel_gpu(&p.row_ticket[row], 1u) == (unsigned)(p.S - 1));
      }
      __syncthreads();
      if (!s_flag) return;
    } else {
      if (tid == 0) ((double2*)p.part)[row] = rs;
      __syncthreads();
    }
    const int t = sample_row_token<BF16>(p, b, j, row, rowp, sm);
    if (tid == 0) {
      p.amax[row] = t;
      if (p.S > 1) p.row_ticket[row] = 0u;  // the counter region is left zero
      if (p.step_counter) count_draw(p);
    }
  } else {
    float bv = -INFINITY;
    int bi = -1;
    if (p.vec_ok && c0 + kChunk <= p.V) {
      Chunk<BF16> cur;
      load_chunk<BF16>(cur, rowp, c0);
      argmax_chunk<BF16>(cur, c0, bv, bi);
    } else {
      for (int q = 0; q < Chunk<BF16>::VPT; ++q)
        for (int e = 0; e < EPV; ++e) {
          const int idx = c0 + (q * kThreads + tid) * EPV + e;
          if (idx >= p.V) continue;
          const float f = BF16 ? bf16_to_f32(((const uint16_t*)rowp)[idx]) : ((const float*)rowp)[idx];
          if (f > bv || bi < 0) { bv = f; bi = idx; }
        }
    }
    pdl_trigger();
    uint64_t key = bi < 0 ? 0ull : cand_key(bv, (uint32_t)bi);
    key = block_max_key(key, s_red);

    if (p.S == 1) {
      if (tid == 0) p.amax[row] = (int32_t)key_id(key);
    } else {
      if (tid == 0) {
        p.part[row * p.S + chunk] = key;
        // acquire-release ticket: releases this thread's partial, and for the
        // last CTA acquires the others' (its barrier then orders the block)
        s_flag = (atom_add_acq_rel_gpu(&p.row_ticket[row], 1u) == (unsigned)(p.S - 1));
      }
      __syncthreads();
      if (!s_flag) return;
      uint64_t m = 0;
      for (int c = tid; c < p.S; c += kThreads) {
        const uint64_t u = ld_cg_u64(&p.part[row * p.S + c]);
        m = u > m ? u : m;
      }
      __syncthreads();
      m = block_max_key(m, s_red);
      if (tid == 0) {
        p.amax[row] = (int32_t)key_id(m);
        p.row_ticket[row] = 0u;  // the counter region is left zero
      }
    }
  }
  // the row is done; the last row of the sequence walks it
  if (tid == 0)  // thread 0 wrote the row's token: the ticket releases it
    s_flag = (atom_add_acq_rel_gpu(&p.seq_count[b], 1u) == (unsigned)(n - 1));
  __syncthreads();
  if (!s_flag) return;
  for (int r = tid; r < n; r += kThreads) {
    s_amax[r] = __ldcg(&p.amax[(int64_t)b * p.n_max + r]);
    s_tok[r] = p.tok[(int64_t)b * p.n_max + r];
    s_par[r] = p.parent[(int64_t)b * p.n_max + r];
    s_dep[r] = p.depth[(int64_t)b * p.n_max + r];
  }
  __syncthreads();
  if (tid < 32) walk_sequence(p, b, n, s_amax, s_tok, s_par, s_dep);
  if (tid == 0) p.seq_count[b] = 0u;  // the counter region is left zero
}

// ---------------------------------------------------------------------------
// Path-only walk
// ---------------------------------------------------------------------------
// The walk only ever needs the argmax of the rows it visits: the root and
// the accepted rows, acc_len + 1 <= L + 1 of them, against every row of the
// tree for the all-rows scan.  The path-only walk reads just those rows, at
// the price of one dependent row after another.  One thread-block cluster
// walks one sequence: every step, each CTA of the cluster takes the argmax
// of its slice of the current row (16-byte streaming loads, all issued
// before any is used), the CTAs exchange their 64-bit (value, smaller id)
// keys through distributed shared memory with one cluster barrier, and
// every CTA then finds the same child to descend to in its own copy of the
// tree.  The CTAs take the same decisions on the same data, so every one of
// them meets the same number of barriers.
constexpr int kLazyThreads = 512;
constexpr int kLazyBatch = 8;  // 16-byte vectors in flight per thread per pass
constexpr int kLazyMaxCluster = 16;

__device__ __forceinline__ uint32_t lz_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void lz_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Store a 64-bit key into the shared memory of CTA `rank` of the cluster.
__device__ __forceinline__ void st_cluster_u64(uint64_t* local, uint32_t rank, uint64_t v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote)
               : "r"((uint32_t)__cvta_generic_to_shared(local)), "r"(rank));
  asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(remote), "l"(v) : "memory");
}

// Argmax key of elements [e0, e1) of a row (e0 a multiple of the vector
// width); each thread visits its indices in increasing order, so a strict >
// keeps the smallest index among equal values.
template <bool BF16>
__device__ __forceinline__ uint64_t lazy_slice_key(const char* rowp, int e0, int e1, int V,
                                                   bool vec_ok) {
  constexpr int EPV = BF16 ? 8 : 4, ES = BF16 ? 2 : 4;
  float bv = -INFINITY;
  int bi = -1;
  if (vec_ok) {
    const int nvec = (e1 - e0 + EPV - 1) / EPV;
    for (int v0 = 0; v0 < nvec; v0 += kLazyBatch * kLazyThreads) {
      uint4 buf[kLazyBatch];
#pragma unroll
      for (int q = 0; q < kLazyBatch; ++q) {
        const int v = v0 + q * kLazyThreads + (int)threadIdx.x;
        const int idx = e0 + v * EPV;
        if (v < nvec && idx + EPV <= V) buf[q] = ld_stream_v4(rowp + (int64_t)idx * ES);
      }
#pragma unroll
      for (int q = 0; q < kLazyBatch; ++q) {
        const int v = v0 + q * kLazyThreads + (int)threadIdx.x;
        const int idx = e0 + v * EPV;
        if (v >= nvec) continue;
        if (idx + EPV <= V) {
          const uint32_t w[4] = {buf[q].x, buf[q].y, buf[q].z, buf[q].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (BF16) {
              const float lo = bf16_lo(w[e]), hi = bf16_hi(w[e]);
              if (lo > bv || bi < 0) { bv = lo; bi = idx + 2 * e; }
              if (hi > bv) { bv = hi; bi = idx + 2 * e + 1; }
            } else {
              const float f = __uint_as_float(w[e]);
              if (f > bv || bi < 0) { bv = f; bi = idx + e; }
            }
          }
        } else {  // the vector that straddles V: element loads inside the row only
          for (int i = idx; i < min(idx + EPV, e1); ++i) {
            const float f = BF16 ? bf16_to_f32(((const uint16_t*)rowp)[i]) : ((const float*)rowp)[i];
            if (f > bv || bi < 0) { bv = f; bi = i; }
          }
        }
      }
    }
  } else {
    for (int i = e0 + (int)threadIdx.x; i < e1; i += kLazyThreads) {
      const float f = BF16 ? bf16_to_f32(((const uint16_t*)rowp)[i]) : ((const float*)rowp)[i];
      if (f > bv || bi < 0) { bv = f; bi = i; }
    }
  }
  return bi < 0 ? 0ull : cand_key(bv, (uint32_t)bi);
}

template <bool BF16>
__global__ void __launch_bounds__(kLazyThreads) walk_lazy_kernel(WalkParams p, int slice) {
  constexpr int ES = BF16 ? 2 : 4;
  __shared__ uint64_t s_keys[2][kLazyMaxCluster];
  __shared__ uint64_t s_red[kLazyThreads / 32];
  __shared__ int s_tok[DDT_TREE_B_MAX + 1], s_first[DDT_TREE_B_MAX + 1], s_cnt[DDT_TREE_B_MAX + 1];
  __shared__ int s_dep[DDT_TREE_B_MAX + 1];
  __shared__ int s_next, s_t;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y;
  const uint32_t rank = lz_cluster_rank();
  const int csize = (int)gridDim.x;
  pdl_wait();
  pdl_trigger();
  int n = p.n_nodes[b];
  if (n < 1 || n > p.n_max) {
    if (rank == 0 && tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    n = min(max(n, 1), p.n_max);
  }
  // the tree, with each row's first child and child count (rows are
  // breadth-first, so a row's children are consecutive)
  for (int r = tid; r < n; r += kLazyThreads) {
    s_tok[r] = p.tok[(int64_t)b * p.n_max + r];
    s_dep[r] = p.depth[(int64_t)b * p.n_max + r];
    s_first[r] = INT_MAX;
    s_cnt[r] = 0;
  }
  __syncthreads();
  for (int r = 1 + tid; r < n; r += kLazyThreads) {
    const int par = p.parent[(int64_t)b * p.n_max + r];
    if (par >= 0 && par < r) {
      atomicMin(&s_first[par], r);
      atomicAdd(&s_cnt[par], 1);
    }
  }
  __syncthreads();
  const int e0 = (int)rank * slice, e1 = min(p.V, e0 + slice);
  int x = 0, a = 0, t = 0;
#pragma unroll 1
  for (int step = 0;; ++step) {
    const char* rowp = (const char*)p.logits + ((int64_t)b * p.n_max + x) * p.row_stride * ES;
    uint64_t key = e0 < e1 ? lazy_slice_key<BF16>(rowp, e0, e1, p.V, p.vec_ok) : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t u = shfl_xor_u64(key, o);
      key = u > key ? u : key;
    }
    if (lane == 0) s_red[warp] = key;
    __syncthreads();
    if (warp == 0) {
      uint64_t k2 = lane < kLazyThreads / 32 ? s_red[lane] : 0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint64_t u = shfl_xor_u64(k2, o);
        k2 = u > k2 ? u : k2;
      }
      if (lane < csize) st_cluster_u64(&s_keys[step & 1][rank], (uint32_t)lane, k2);
    }
    lz_cluster_sync();
    if (warp == 0) {
      uint64_t k2 = lane < csize ? s_keys[step & 1][lane] : 0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint64_t u = shfl_xor_u64(k2, o);
        k2 = u > k2 ? u : k2;
      }
      const int tt = (int)key_id(k2);
      int next = -1;
      if (a < p.L && s_dep[x] < p.L && s_cnt[x] > 0) {
        for (int c0 = s_first[x]; c0 < s_first[x] + s_cnt[x]; c0 += 32) {
          const int c = c0 + lane;
          const bool hit = c < s_first[x] + s_cnt[x] && s_tok[c] == tt;
          const unsigned bal = __ballot_sync(0xFFFFFFFFu, hit);
          if (bal) {
            next = c0 + __ffs(bal) - 1;
            break;
          }
        }
      }
      if (lane == 0) {
        s_next = next;
        s_t = tt;
        if (rank == 0 && next >= 0) {
          p.acc_nodes[(int64_t)b * p.L + a] = next;
          p.acc_tok[(int64_t)b * p.L + a] = tt;
        }
      }
    }
    __syncthreads();
    const int next = s_next;
    t = s_t;
    if (next < 0) break;
    x = next;
    ++a;
  }
  if (rank == 0) {
    for (int i = a + tid; i < p.L; i += kLazyThreads) {
      p.acc_nodes[(int64_t)b * p.L + i] = -1;
      p.acc_tok[(int64_t)b * p.L + i] = -1;
    }
    if (tid == 0) {
      p.acc_len[b] = a;
      p.bonus[b] = t;
    }
  }
}

// Largest cluster (16, else 8) of path-only walk CTAs the device can run,
// and how many such clusters it runs at once.
struct LazyShape {
  int csize, active;
};
LazyShape lazy_shape() {
  static std::mutex mu;
  static LazyShape cached = {0, 0};
  std::lock_guard<std::mutex> lock(mu);
  if (cached.csize) return cached;
  auto* fn = (const void*)walk_lazy_kernel<false>;
  auto* fn2 = (const void*)walk_lazy_kernel<true>;
  const bool big = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
                   cudaFuncSetAttribute(fn2, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  LazyShape r = {8, 1};
  for (int cs : {16, 8}) {
    if (cs == 16 && !big) continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs, 1, 1);
    cfg.blockDim = dim3(kLazyThreads, 1, 1);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = cs;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, fn, &cfg) == cudaSuccess && nc > 0) {
      r = {cs, nc};
      break;
    }
  }
  cudaGetLastError();  // a refused query must not leave a sticky error behind
  cached = r;
  return r;
}
int lazy_cluster_size() { return lazy_shape().csize; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

size_t walk_workspace_size(int batch, int n_max, int V) {
  const int S = (V + kChunk - 1) / kChunk;
  const size_t rows = (size_t)batch * n_max;
  return (size_t)DDT_WS_COUNTER_BYTES + align256(sizeof(int32_t) * rows) +
         align256(2 * sizeof(uint64_t) * rows * S);
}

// Path-only or all-rows for DDT_WALK_AUTO, from times measured on B200: the
// all-rows scan costs its bytes at about 5.8 TB/s plus a few microseconds of
// merging; the path-only walk costs about 3.5 us per dependent step (one
// row per sequence), per wave of clusters the device runs at once, and up
// to L + 1 steps.  AUTO takes the path-only walk when even its worst case
// (every row down to depth L accepted) is the cheaper.  (Both pay the same
// launch latency, which cancels.)
constexpr double kAllRowsGBs = 5800.0, kAllRowsMergeUs = 4.0;
constexpr double kLazyStepUs = 3.5;

int walk_mode_for(int mode, ddt_dtype dt, int batch, int n_max, int V, int L) {
  if (mode != DDT_WALK_AUTO) return mode;
  const double bytes = (double)batch * n_max * V * (dt == DDT_BF16 ? 2 : 4);
  const double all_us = bytes / (kAllRowsGBs * 1e3) + kAllRowsMergeUs;
  const LazyShape ls = lazy_shape();
  const double waves = std::ceil((double)batch / (double)(ls.active > 0 ? ls.active : 1));
  const double lazy_us = (L + 1) * kLazyStepUs * waves;
  return lazy_us < all_us ? DDT_WALK_LAZY : DDT_WALK_ALL_ROWS;
}

ddt_status launch_tree_walk(const void* logits, ddt_dtype dt, int batch, int n_max, int V,
                            int64_t row_stride, const int32_t* tok, const int32_t* parent,
                            const int32_t* depth, const int32_t* n_nodes, int L, int mode,
                            int32_t* acc_len, int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus,
                            void* ws, int32_t* dev_status, cudaStream_t stream,
                            const WalkSampling* sampling) {
  WalkParams p;
  const double A = sampling ? (double)sampling->inv_temperature * 1.4426950408889634074 : 0.0;
  p.a = (float)A;
  p.a_lo = (float)(A - (double)p.a);
  p.seed = sampling ? sampling->seed : 0;
  p.step = sampling ? sampling->step : 0;
  p.step_counter = sampling ? sampling->step_counter : nullptr;
  p.logits = logits;
  p.batch = batch;
  p.n_max = n_max;
  p.V = V;
  p.S = (V + kChunk - 1) / kChunk;
  p.L = L;
  p.row_stride = row_stride;
  const int es = dt == DDT_BF16 ? 2 : 4;
  p.vec_ok = ((uintptr_t)logits % 16 == 0) && ((row_stride * es) % 16 == 0);
  p.tok = tok;
  p.parent = parent;
  p.depth = depth;
  p.n_nodes = n_nodes;
  p.acc_len = acc_len;
  p.acc_nodes = acc_nodes;
  p.acc_tok = acc_tok;
  p.bonus = bonus;
  p.status = dev_status;
  const size_t rows = (size_t)batch * n_max;
  char* w = (char*)ws;
  p.row_ticket = (unsigned*)w;  // counter region: rows tickets, then batch counters
  p.seq_count = (unsigned*)w + rows;
  p.draw_count = p.seq_count + batch;
  w += DDT_WS_COUNTER_BYTES;
  p.amax = (int32_t*)w;
  w += align256(sizeof(int32_t) * rows);
  p.part = (uint64_t*)w;
  if (batch == 0) return DDT_OK;
  cudaError_t e;
  if (!sampling && walk_mode_for(mode, dt, batch, n_max, V, L) == DDT_WALK_LAZY) {
    const int csize = lazy_cluster_size();
    // each CTA's slice: a multiple of 8 elements (whole 16-byte vectors)
    const int slice = ((V + csize - 1) / csize + 7) / 8 * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize, batch, 1);
    cfg.blockDim = dim3(kLazyThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)csize;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = dt == DDT_BF16 ? cudaLaunchKernelEx(&cfg, walk_lazy_kernel<true>, p, slice)
                       : cudaLaunchKernelEx(&cfg, walk_lazy_kernel<false>, p, slice);
    return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
  }
  dim3 grid(p.S, n_max, batch);
  if (sampling)
    e = dt == DDT_BF16 ? launch_pdl(walk_kernel<true, true>, grid, dim3(kThreads), 0, stream, 0, p)
                       : launch_pdl(walk_kernel<false, true>, grid, dim3(kThreads), 0, stream, 0, p);
  else
    e = dt == DDT_BF16 ? launch_pdl(walk_kernel<true, false>, grid, dim3(kThreads), 0, stream, 0, p)
                       : launch_pdl(walk_kernel<false, false>, grid, dim3(kThreads), 0, stream, 0, p);
  return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
