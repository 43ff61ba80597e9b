// tree.cu -- stage 2 of the verification round: the B most probable prefixes
// of the factorised draft, compiled into target-model inputs.
//
// DDTree page: section 核心創新 (best-first selection under a node budget B),
// 運作流程 step 2 (maximise the expected acceptance length under the
// factorised draft; the optimum is the set of highest-probability prefixes,
// which is prefix-closed), 理論基礎 Propositions 1-2, and step 3 (compile
// the tree into target inputs with an ancestor-only mask).
//
// Order K (best first): equal depth -> larger fp64 sum of raw logits, then
// reverse-lexicographic token ids; different depths -> larger fp64 score
// inv_t*sum(z) - sum(lse), then the shallower prefix.  At equal depth the
// score is a monotone function of the sum, so K is the lexicographic order
// on (score desc, depth asc, sum desc, reversed tokens); comparisons use the
// score as a 64-bit integer key and fall back to the rest only on equal keys.
//
// One CTA of 256 threads per sequence; thread t owns nodes t, t+256, ...
// Selection runs in frontier rounds and selects exactly the set a one-node-
// at-a-time best-first search would:
//   * every selected node x keeps nnext[x], its selected-children count; they
//     are ranks 0..nnext[x]-1, since siblings come in candidate order, which
//     is K (the candidates of a position are sorted by logit, then id);
//   * the frontier is, per node, the run of ranks nnext[x]..k-1; the best
//     prefix not in any run is the first child of some run head, so
//     theta = the K-best run-head first child bounds everything ungenerated;
//   * every run item that precedes theta is among the best remaining
//     prefixes: each node counts its run's items before theta, one scan
//     numbers them, and they are created together (three barriers a round);
//   * when they overshoot the budget, the R best are kept by a radix select
//     on their score keys (8 bits a pass), exact ties ranked under K.
// Each round selects at least the best run head, so the loop ends.
// Breadth-first rows are then the order of (depth, rank path): each node
// carries its path of candidate ranks as a packed key and its row is its
// rank by key within its depth, so no level-by-level pass is needed; the
// ancestor masks follow the parent rows.
#include <climits>

#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;           // radix-select digit
constexpr int kTieList = 256;        // exact ties ranked by counting
constexpr int kItemCapMax = 16384;
constexpr int kWide = 64;            // wider levels are numbered from their parents' rows
constexpr size_t kSmemMax = 227 * 1024;
constexpr unsigned kFull = 0xFFFFFFFFu;

struct TreeParams {
  const int32_t* ids;
  const float* zk;
  const float* lse;
  int L, k;
  double inv_t;
  const int32_t* k_per_seq;
  const int32_t* budget;
  int B_max, n_max, W, icap, kw, rb;
  const int32_t* root_token;
  const int32_t* ctx_len;
  int32_t *tok, *parent, *depth, *pos;
  uint32_t* mask;
  int32_t* n_nodes;
  double* surrogate;
  int32_t* status;
};

struct Smem {
  double* zt;      // [L*k] raw logits of the candidates
  double* S;       // [L+1] prefix sums of lse
  double* nsz;     // [n_max] node logit sums
  double* nsc;     // [n_max] node scores
  int* tt;         // [L*k] candidate token ids
  int* npar;       // [n_max] parent node (creation index)
  int* ndep;       // [n_max]
  int* nrank;      // [n_max] candidate rank at the node's own position
  int* nnext;      // [n_max] selected-children count
  int* nrow;       // [n_max] breadth-first row of a node
  int* ninv;       // [n_max] row -> node; also the depth buckets
  int* prow;       // [n_max] row -> parent row
  uint64_t* pkey;  // [n_max*kw] rank path, most significant word first
  uint64_t* nrk;   // [n_max] reversed id-rank path (own position first), top 64 bits
  int* idr;        // [L*k] rank of each candidate's token id within its position
  uint64_t* ckey;  // [icap] cut candidates: score key
  uint32_t* cid;   // [icap] cut candidates: node << 8 | rank, bit 31 = kept
  int k, kw, rb;
};

// A prefix under the order K in integer form (see pk_before).
struct PK {
  uint64_t sk, rk;
  double sz;
  int dep;
  uint32_t h;
};

// Shared scratch of the reductions, scans and the cut.
struct Red {
  uint64_t wkey[kWarps];
  uint32_t wid[kWarps];
  int wtie[kWarps];
  int wsum[kWarps];
  uint64_t wmn[kWarps], wmx[kWarps];
  double wd[kWarps];
  PK wpk[kWarps];
  double csz[kTieList];
  uint64_t crk[kTieList];
  int cdep[kTieList];
  uint32_t chd[kTieList];
  int hist[2][kBins];
  int digit, above, hcount, nlist;
  int list[kTieList];
  int list2[kTieList];
  __align__(16) uint64_t lkey[kTieList];
  int lvl[DDT_TREE_L_MAX + 2];
};

// fp64 score as an integer key: larger score <-> larger key; -0 == +0.
__device__ __forceinline__ uint64_t score_key(double sc) {
  uint64_t u = (uint64_t)__double_as_longlong(sc);
  if ((u << 1) == 0) u = 0;
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ double score_of(const Smem& s, double inv_t, double sz, int t) {
  return __dsub_rn(__dmul_rn(inv_t, sz), s.S[t]);
}

// A prefix given as a selected node plus one or two appended ranks.
struct VP {
  double sz, sc;
  int depth, base, r1, r2;
};

__device__ __forceinline__ int vp_token(const Smem& s, const VP& v, int t) {
  const int db = s.ndep[v.base];
  if (t == db + 2) return s.tt[(t - 1) * s.k + v.r2];
  if (t == db + 1) return s.tt[(t - 1) * s.k + v.r1];
  int x = v.base;
  while (s.ndep[x] > t) x = s.npar[x];
  return s.tt[(t - 1) * s.k + s.nrank[x]];
}

// true iff a strictly precedes b under K (full comparison).
__device__ __forceinline__ bool vp_before(const Smem& s, const VP& a, const VP& b) {
  if (a.depth == b.depth) {
    if (a.sz != b.sz) return a.sz > b.sz;
    for (int t = a.depth; t >= 1; --t) {
      const int ta = vp_token(s, a, t), tb = vp_token(s, b, t);
      if (ta != tb) return ta < tb;
    }
    return false;
  }
  if (a.sc != b.sc) return a.sc > b.sc;
  return a.depth < b.depth;
}

// Packed prefix handle: node << 16 | r1 << 8 | (r2 + 1); r2 = -1 is an item
// (one appended rank), r2 = 0 a run head's first child.
__device__ __forceinline__ uint32_t pack_vp(int x, int r1, int r2) {
  return ((uint32_t)x << 16) | ((uint32_t)r1 << 8) | (uint32_t)(r2 + 1);
}

__device__ __forceinline__ VP unpack_vp(const Smem& s, double inv_t, uint32_t h) {
  VP v;
  v.base = (int)(h >> 16);
  v.r1 = (int)((h >> 8) & 0xFFu);
  v.r2 = (int)(h & 0xFFu) - 1;
  const int d = s.ndep[v.base];
  v.sz = __dadd_rn(s.nsz[v.base], s.zt[d * s.k + v.r1]);
  v.depth = d + 1;
  if (v.r2 >= 0) {
    v.sz = __dadd_rn(v.sz, s.zt[(d + 1) * s.k + v.r2]);
    v.depth = d + 2;
  }
  v.sc = score_of(s, inv_t, v.sz, v.depth);
  return v;
}

// The CTA's shared-memory layout, published once for the out-of-line full
// comparison, so that its call sites pass two handles and nothing else.
__shared__ Smem g_layout;
__shared__ double g_inv_t;

// Full comparison of two prefix handles (only equal score keys get here).
__device__ __noinline__ bool slow_before(uint32_t ha, uint32_t hb) {
  const Smem s = g_layout;
  const double inv_t = g_inv_t;
  return vp_before(s, unpack_vp(s, inv_t, ha), unpack_vp(s, inv_t, hb));
}

__device__ __forceinline__ bool handle_before(const Smem&, double, uint32_t ha, uint32_t hb) {
  return slow_before(ha, hb);
}

// (ka, ha) strictly before (kb, hb); key 0 means "none" (last).
__device__ __forceinline__ bool key_before(const Smem& s, double inv_t, uint64_t ka, uint32_t ha,
                                           uint64_t kb, uint32_t hb) {
  if (ka != kb) return ka > kb;
  if (ka == 0 || ha == hb) return false;
  return handle_before(s, inv_t, ha, hb);
}

// The order K as integers: (score key desc, depth asc, logit sum desc,
// reversed id-rank path asc).  Within a position, token order is id-rank
// order, so the reversed path compares like the reversed token ids; it keeps
// the deepest 64 bits, and only prefixes that agree on all of them go to the
// out-of-line comparison.
__device__ __forceinline__ uint64_t rev_key(const Smem& s, uint64_t parent_rk, int t, int r) {
  return ((uint64_t)s.idr[t * s.k + r] << (64 - s.rb)) | (parent_rk >> s.rb);
}

__device__ __forceinline__ PK make_pk(const Smem& s, double inv_t, uint32_t h) {
  PK v;
  const int x = (int)(h >> 16), r1 = (int)((h >> 8) & 0xFFu), r2 = (int)(h & 0xFFu) - 1;
  const int d = s.ndep[x];
  v.sz = __dadd_rn(s.nsz[x], s.zt[d * s.k + r1]);
  v.rk = rev_key(s, s.nrk[x], d, r1);
  v.dep = d + 1;
  if (r2 >= 0) {
    v.sz = __dadd_rn(v.sz, s.zt[(d + 1) * s.k + r2]);
    v.rk = rev_key(s, v.rk, d + 1, r2);
    v.dep = d + 2;
  }
  v.sk = score_key(score_of(s, inv_t, v.sz, v.dep));
  v.h = h;
  return v;
}

__device__ __forceinline__ PK no_pk() {
  PK v;
  v.sk = v.rk = 0ull;
  v.sz = 0.0;
  v.dep = 0;
  v.h = 0u;
  return v;
}

// a strictly before b under K; sk == 0 is "none" (last).
__device__ __forceinline__ bool pk_before(const Smem& s, const PK& a, const PK& b) {
  if (a.sk != b.sk) return a.sk > b.sk;
  if (a.sk == 0) return false;
  if (a.dep != b.dep) return a.dep < b.dep;
  if (a.sz != b.sz) return a.sz > b.sz;
  if (a.rk != b.rk) return a.rk < b.rk;
  if (a.dep * s.rb <= 64 || a.h == b.h) return false;  // whole path compared: same prefix
  return slow_before(a.h, b.h);
}

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int o) {
  const uint32_t lo = __shfl_xor_sync(kFull, (uint32_t)v, o);
  const uint32_t hi = __shfl_xor_sync(kFull, (uint32_t)(v >> 32), o);
  return ((uint64_t)hi << 32) | lo;
}

// Block-wide maximum of the score keys with the handle of one holder,
// returned to every thread; `tie` is set when the maximum is held by more
// than one candidate (or by a thread that flagged a tie of its own), so that
// the caller resolves it under the full order; `flag` is ORed over the block.
// One barrier; the caller must barrier before the next call.
__device__ __forceinline__ void block_max_key(uint64_t& key, uint32_t& h, int& tie, int& flag,
                                              Red* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t hi = (uint32_t)(key >> 32);
  uint32_t mhi = __reduce_max_sync(kFull, hi);
  uint32_t mlo = __reduce_max_sync(kFull, hi == mhi ? (uint32_t)key : 0u);
  uint64_t wk = ((uint64_t)mhi << 32) | mlo;
  unsigned bal = __ballot_sync(kFull, key == wk);
  const uint32_t wh = __shfl_sync(kFull, h, __ffs(bal) - 1);
  const int wt = (__popc(bal) > 1) | __any_sync(kFull, tie && key == wk);
  if (lane == 0) {
    red->wkey[warp] = wk;
    red->wid[warp] = wh;
    red->wtie[warp] = wt;
  }
  flag = __syncthreads_or(flag);
  // every warp reduces the per-warp results the same way
  const uint64_t k8 = lane < kWarps ? red->wkey[lane] : 0ull;
  const uint32_t h8 = lane < kWarps ? red->wid[lane] : 0u;
  const int t8 = lane < kWarps ? red->wtie[lane] : 0;
  hi = (uint32_t)(k8 >> 32);
  mhi = __reduce_max_sync(kFull, hi);
  mlo = __reduce_max_sync(kFull, hi == mhi ? (uint32_t)k8 : 0u);
  wk = ((uint64_t)mhi << 32) | mlo;
  bal = __ballot_sync(kFull, lane < kWarps && k8 == wk);
  h = __shfl_sync(kFull, h8, __ffs(bal) - 1);
  tie = wk != 0 && ((__popc(bal) > 1) | __any_sync(kFull, t8 && k8 == wk));
  key = wk;
}

struct KeyHandle {
  uint64_t key;
  uint32_t h;
};

// K-best (key, handle) over the block under the full order, returned to
// every thread (the rare paths: exact ties and degenerate inputs).  One
// barrier; the caller must barrier before the next reduction.
__device__ __noinline__ KeyHandle block_best_slow(uint64_t key, uint32_t h, Red* red) {
  const Smem s = g_layout;
  const double inv_t = g_inv_t;
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t ok = shfl_u64(key, o);
    const uint32_t oh = __shfl_xor_sync(kFull, h, o);
    if (key_before(s, inv_t, ok, oh, key, h)) {
      key = ok;
      h = oh;
    }
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red->wkey[warp] = key;
    red->wid[warp] = h;
  }
  __syncthreads();
  key = red->wkey[0];
  h = red->wid[0];
  for (int w = 1; w < kWarps; ++w) {
    const uint64_t ok = red->wkey[w];
    const uint32_t oh = red->wid[w];
    if (key_before(s, inv_t, ok, oh, key, h)) {
      key = ok;
      h = oh;
    }
  }
  return KeyHandle{key, h};
}

// K-best prefix over the block by pk_before, returned to every thread.  One
// barrier; the caller must barrier before the next reduction.
__device__ __forceinline__ PK block_best_pk(const Smem& s, PK v, Red* red) {
  for (int o = 16; o > 0; o >>= 1) {
    PK u;
    u.sk = shfl_u64(v.sk, o);
    u.rk = shfl_u64(v.rk, o);
    u.sz = __shfl_xor_sync(kFull, v.sz, o);
    u.dep = __shfl_xor_sync(kFull, v.dep, o);
    u.h = __shfl_xor_sync(kFull, v.h, o);
    if (pk_before(s, u, v)) v = u;
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red->wpk[warp] = v;
  __syncthreads();
  PK b = red->wpk[0];
  for (int w = 1; w < kWarps; ++w)
    if (pk_before(s, red->wpk[w], b)) b = red->wpk[w];
  return b;
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// Exclusive scan of one value per thread in thread order; returns the
// thread's offset, sets `total` and ORs `flag` over the block.  One barrier;
// the caller must barrier before the next call.
__device__ __forceinline__ int block_exscan1(int v, int& total, int& flag, Red* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int inc = warp_incl_scan(v, lane);
  if (lane == 31) red->wsum[warp] = inc;
  flag = __syncthreads_or(flag);
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int c = red->wsum[w];
    before += (w < warp) ? c : 0;
    tot += c;
  }
  total = tot;
  return before + inc - v;
}

// Rank the nl candidates list[0..nl) (indices into ckey/cid, all with the
// same score key) among themselves under K and keep the `need` best (bit 30
// of cid).  Each candidate's (depth, sum, reversed path) is published once,
// so the ranking compares shared-memory words.  nl <= kTieList.
__device__ void rank_ties(const Smem& s, double inv_t, const int* list, int nl, int need, Red* red) {
  const int tid = threadIdx.x;
  for (int q = tid; q < nl; q += kThreads) {
    const PK v = make_pk(s, inv_t, (s.cid[list[q]] & 0x3FFFFFFFu) << 8);
    red->csz[q] = v.sz;
    red->crk[q] = v.rk;
    red->cdep[q] = v.dep;
    red->chd[q] = v.h;
  }
  __syncthreads();
  for (int q = tid; q < nl; q += kThreads) {
    const int dq = red->cdep[q];
    const double zq = red->csz[q];
    const uint64_t rq = red->crk[q];
    const bool exact = dq * s.rb <= 64;
    int rank = 0;
    for (int u = 0; u < nl; ++u) {
      const int du = red->cdep[u];
      const double zu = red->csz[u];
      const uint64_t ru = red->crk[u];
      bool b;
      if (du != dq) b = du < dq;
      else if (zu != zq) b = zu > zq;
      else if (ru != rq) b = ru < rq;
      else b = !exact && u != q && slow_before(red->chd[u], red->chd[q]);
      rank += b;
    }
    if (rank < need) s.cid[list[q]] |= 0x40000000u;
  }
  __syncthreads();
}

// Among nl <= kThreads candidates (score keys keys[q], candidate index
// idx[q], or q when idx is null) keep the `need` K-best (bit 30 of cid).
// Candidate q has `above` candidates with larger keys and `eq` with equal
// ones (itself included): kept if above + eq <= need, dropped if
// above >= need; only the one group of equal keys that straddles `need` is
// ranked under the full order.
__device__ void keep_best_of(const Smem& s, const uint64_t* keys, const int* idx, int nl, int need,
                             Red* red) {
  const int tid = threadIdx.x;
  int above = 0, eq = 0;
  if (tid == 0) red->nlist = 0;
  if (tid < nl) {
    const uint64_t ki = keys[tid];
    int u = 0;
    for (; u + 8 <= nl; u += 8) {  // eight keys a step, loads first
      ulonglong2 v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = *reinterpret_cast<const ulonglong2*>(keys + u + 2 * e);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        above += (v[e].x > ki) + (v[e].y > ki);
        eq += (v[e].x == ki) + (v[e].y == ki);
      }
    }
    for (; u < nl; ++u) {
      above += keys[u] > ki;
      eq += keys[u] == ki;
    }
  }
  const int me = tid < nl ? (idx ? idx[tid] : tid) : 0;
  const bool bnd = tid < nl && above < need && above + eq > need;
  if (__syncthreads_or(bnd)) {
    if (bnd) {
      red->list2[atomicAdd(&red->nlist, 1)] = me;
      red->digit = need - above;  // the same in every member of the group
    }
    __syncthreads();
    rank_ties(s, g_inv_t, red->list2, red->nlist, red->digit, red);
  }
  if (tid < nl && above + eq <= need) s.cid[me] |= 0x40000000u;
  __syncthreads();
}

// Final round with at most one candidate per thread.
__device__ void cut_small(const Smem& s, int T, int R, Red* red) {
  keep_best_of(s, s.ckey, nullptr, T, R, red);
  if (threadIdx.x < T) {
    const uint32_t c = s.cid[threadIdx.x];
    if (c & 0x40000000u) s.cid[threadIdx.x] = (c & 0x3FFFFFFFu) | 0x80000000u;
  }
  __syncthreads();
}

// Final round: keep the R K-best of the T > R candidates in ckey/cid (bit 31
// of cid set on the kept ones).  Radix select on the score keys, 8 bits a
// pass below the bits all keys share, until the bucket holding the R-th key
// has at most kTieList candidates; those are gathered and ranked like a
// small cut.
__device__ void cut_best(const Smem& s, double inv_t, int T, int R, Red* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t mn = ~0ull, mx = 0;
  for (int i0 = tid; i0 < T; i0 += 4 * kThreads) {
    uint64_t kk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) kk[e] = i0 + e * kThreads < T ? s.ckey[i0 + e * kThreads] : s.ckey[i0];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      mn = kk[e] < mn ? kk[e] : mn;
      mx = kk[e] > mx ? kk[e] : mx;
    }
  }
  {
    uint32_t hi = (uint32_t)(mx >> 32);
    const uint32_t mhi = __reduce_max_sync(kFull, hi);
    const uint32_t mlo = __reduce_max_sync(kFull, hi == mhi ? (uint32_t)mx : 0u);
    hi = (uint32_t)(mn >> 32);
    const uint32_t nhi = __reduce_min_sync(kFull, hi);
    const uint32_t nlo = __reduce_min_sync(kFull, hi == nhi ? (uint32_t)mn : ~0u);
    if (lane == 0) {
      red->wmx[warp] = ((uint64_t)mhi << 32) | mlo;
      red->wmn[warp] = ((uint64_t)nhi << 32) | nlo;
    }
  }
  red->hist[0][tid] = 0;
  __syncthreads();
  mn = red->wmn[0];
  mx = red->wmx[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) {
    mn = red->wmn[w] < mn ? red->wmn[w] : mn;
    mx = red->wmx[w] > mx ? red->wmx[w] : mx;
  }
  int need = R, bucket = T;
  uint64_t prefix = mx, pmask = ~0ull;
  if (mn != mx) {
    int hb = 63 - __clzll((long long)(mn ^ mx));
    pmask = hb == 63 ? 0ull : (~0ull << (hb + 1));
    prefix = mx & pmask;
    int buf = 0;
    for (;;) {
      const int shift = hb >= 7 ? hb - 7 : 0;
      const uint64_t dmask = (1ull << (hb - shift + 1)) - 1;
      red->hist[buf ^ 1][tid] = 0;  // the next pass's histogram
      // warp-aggregated: one atomic per distinct digit in a warp; four keys
      // loaded per step
      for (int i0 = warp * 32; i0 < T; i0 += 4 * kThreads) {
        uint64_t kk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i0 + e * kThreads + lane;
          kk[e] = i < T ? s.ckey[i] : 0ull;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i0 + e * kThreads + lane;
          const int dg = (i < T && (kk[e] & pmask) == prefix) ? (int)((kk[e] >> shift) & dmask) : -1;
          const unsigned grp = __match_any_sync(kFull, dg);
          if (dg >= 0 && lane == __ffs(grp) - 1) atomicAdd(&red->hist[buf][dg], __popc(grp));
        }
      }
      __syncthreads();
      // thread t holds bin 255 - t: scan from the top bin down
      const int hcnt = red->hist[buf][kBins - 1 - tid];
      int tot, nof = 0;
      const int excl = block_exscan1(hcnt, tot, nof, red);
      if (excl < need && excl + hcnt >= need) {
        red->digit = kBins - 1 - tid;
        red->above = excl;
        red->hcount = hcnt;
      }
      __syncthreads();
      need -= red->above;
      bucket = red->hcount;
      prefix |= (uint64_t)red->digit << shift;
      pmask |= dmask << shift;
      buf ^= 1;
      if (bucket <= kTieList || shift == 0) break;
      hb = shift - 1;
    }
  }
  // above the bucket: kept; the bucket: gathered and ranked
  if (tid == 0) red->nlist = 0;
  __syncthreads();
  for (int i = tid; i < T; i += kThreads) {
    const uint64_t km = s.ckey[i] & pmask;
    if (km > prefix) s.cid[i] |= 0x80000000u;
    if (km == prefix) {
      const int q = atomicAdd(&red->nlist, 1);
      if (q < kTieList) {
        red->list[q] = i;
        red->lkey[q] = s.ckey[i];
      }
    }
  }
  __syncthreads();
  const int nl = red->nlist;
  __syncthreads();  // every thread has read nlist before it is reused
  if (nl <= kTieList) {
    keep_best_of(s, red->lkey, red->list, nl, need, red);
  } else {
    // a very large exact tie: take the K-best undecided tied candidate, need times
    for (int t = 0; t < need; ++t) {
      uint64_t key = 0;
      uint32_t h = 0;
      for (int i = tid; i < T; i += kThreads) {
        if (s.ckey[i] != prefix || (s.cid[i] & 0x40000000u)) continue;
        const uint32_t hi = (s.cid[i] & 0x3FFFFFFFu) << 8;
        if (key_before(s, inv_t, prefix, hi, key, h)) {
          key = prefix;
          h = hi;
        }
      }
      h = block_best_slow(key, h, red).h;
      for (int i = tid; i < T; i += kThreads)
        if (s.ckey[i] == prefix && ((s.cid[i] & 0x3FFFFFFFu) << 8) == h) s.cid[i] |= 0x40000000u;
      __syncthreads();
    }
  }
  for (int i = tid; i < T; i += kThreads)
    if (s.cid[i] & 0x40000000u) s.cid[i] = (s.cid[i] & 0x3FFFFFFFu) | 0x80000000u;
  __syncthreads();
}

// Rank path key of a new node at depth d+1 with rank r: its parent's key with
// r placed in field d (rb bits per field, fields from the most significant
// bit of word 0 on; a field may straddle two words).
__device__ __forceinline__ void make_path_key(const Smem& s, int parent, int id, int d, int r) {
  const uint64_t* pk = s.pkey + (size_t)parent * s.kw;
  uint64_t* ck = s.pkey + (size_t)id * s.kw;
  for (int w = 0; w < s.kw; ++w) ck[w] = pk[w];
  const int o = d * s.rb, w = o >> 6, sh = 64 - (o & 63) - s.rb;
  if (sh >= 0) {
    ck[w] |= (uint64_t)r << sh;
  } else {
    ck[w] |= (uint64_t)r >> (-sh);
    ck[w + 1] |= (uint64_t)r << (64 + sh);
  }
}

__device__ __forceinline__ bool path_less(const Smem& s, int a, int b) {
  const uint64_t* ka = s.pkey + (size_t)a * s.kw;
  const uint64_t* kb = s.pkey + (size_t)b * s.kw;
  for (int w = 0; w < s.kw; ++w)
    if (ka[w] != kb[w]) return ka[w] < kb[w];
  return false;
}

// Item (x, r): key of the child of node x (depth d) with candidate rank r.
__device__ __forceinline__ uint64_t item_key(const Smem& s, double inv_t, double base_sz, int d, int r) {
  return score_key(score_of(s, inv_t, __dadd_rn(base_sz, s.zt[d * s.k + r]), d + 1));
}

// Items of node x's run from rank r0 (below rend) whose keys exceed tk, up
// to the first one that does not; `tie` is set when that one's key equals
// tk, which only the full order can decide.  Four keys at a time, so that
// their shared-memory loads overlap.
__device__ __forceinline__ int count_fast(const Smem& s, double inv_t, int x, int d, int r0, int rend,
                                          uint64_t tk, int& tie) {
  const double base = s.nsz[x];
  int c = 0;
  for (int r = r0; r < rend; r += 4) {
    uint64_t kk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) kk[e] = r + e < rend ? item_key(s, inv_t, base, d, r + e) : 0ull;
    bool go = true;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (go) {
        if (r + e < rend && kk[e] > tk) {
          ++c;
        } else {
          tie |= (r + e < rend && kk[e] == tk);
          go = false;
        }
      }
    }
    if (!go) break;
  }
  return c;
}

// The same count under the full order (the rare paths).
__device__ __noinline__ int count_slow(int x, int r0, int rend, uint64_t tk, uint32_t th) {
  const Smem s = g_layout;
  const double inv_t = g_inv_t;
  const int d = s.ndep[x];
  const double base = s.nsz[x];
  int c = 0;
  for (int r = r0; r < rend; ++r) {
    if (!key_before(s, inv_t, item_key(s, inv_t, base, d, r), pack_vp(x, r, -1), tk, th)) break;
    ++c;
  }
  return c;
}

__global__ void __launch_bounds__(kThreads, 1) build_tree_kernel(TreeParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ Red red;

  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = p.L, k = p.k, NM = p.n_max, icap = p.icap;
  pdl_wait();
  const double inv_t = p.inv_t;

  Smem s;
  s.k = k;
  s.kw = p.kw;
  s.rb = p.rb;
  {
    unsigned char* q = smem_raw;
    auto take = [&](size_t bytes) {
      unsigned char* r = q;
      q += (bytes + 15) & ~(size_t)15;
      return r;
    };
    s.S = (double*)take(sizeof(double) * (L + 1));
    s.zt = (double*)take(sizeof(double) * L * k);
    s.nsz = (double*)take(sizeof(double) * NM);
    s.nsc = (double*)take(sizeof(double) * NM);
    s.pkey = (uint64_t*)take(sizeof(uint64_t) * NM * p.kw);
    s.nrk = (uint64_t*)take(sizeof(uint64_t) * NM);
    s.ckey = (uint64_t*)take(sizeof(uint64_t) * icap);  // ckey and cid adjacent: the
    s.cid = (uint32_t*)take(sizeof(uint32_t) * icap);   // mask staging area
    s.tt = (int*)take(sizeof(int) * L * k);
    s.npar = (int*)take(sizeof(int) * NM);
    s.ndep = (int*)take(sizeof(int) * NM);
    s.nrank = (int*)take(sizeof(int) * NM);
    s.nnext = (int*)take(sizeof(int) * NM);
    s.nrow = (int*)take(sizeof(int) * NM);
    s.ninv = (int*)take(sizeof(int) * NM);
    s.prow = (int*)take(sizeof(int) * NM);
    s.idr = (int*)take(sizeof(int) * L * k);
  }
  if (tid == 0) {
    g_layout = s;
    g_inv_t = inv_t;
  }

  // global loads first; the budget and candidate count are only needed later
  for (int i = tid; i < L * k; i += kThreads) {
    s.zt[i] = (double)p.zk[(int64_t)b * L * k + i];
    s.tt[i] = p.ids[(int64_t)b * L * k + i];
  }
  for (int t = tid; t < L; t += kThreads) s.S[t + 1] = (double)p.lse[(int64_t)b * L + t];
  int kb = p.k_per_seq ? p.k_per_seq[b] : k;
  int Bb = p.budget ? p.budget[b] : p.B_max;
  for (int w = tid; w < p.kw; w += kThreads) s.pkey[w] = 0ull;
  if (tid == 0) {
    s.nsz[0] = 0.0;
    s.nsc[0] = 0.0;
    s.npar[0] = -1;
    s.ndep[0] = 0;
    s.nrank[0] = 0;
    s.nnext[0] = 0;
    s.nrk[0] = 0ull;
    s.ninv[0] = 0;
  }
  if (tid < L + 2) red.lvl[tid] = tid == 0 ? 1 : 0;
  __shared__ int s_emax, s_emin;
  if (tid == 0) {
    s_emax = INT_MIN;
    s_emin = INT_MAX;
  }
  __syncthreads();
  // Siblings are taken in candidate order, which is K only while every fp64
  // sum of logits along a path is exact: then two children of one node
  // compare as their own logits do.  With f32 logits that holds when the
  // binary exponents of the nonzero finite candidates span at most
  // 29 - ceil(log2 L) (24-bit significands inside a 53-bit sum of L terms).
  {
    int emax = INT_MIN, emin = INT_MAX;
    for (int i = tid; i < L * k; i += kThreads) {
      const uint32_t u = __float_as_uint(p.zk[(int64_t)b * L * k + i]);
      const int ef = (int)((u >> 23) & 0xFFu);
      if (ef == 0xFF || (u & 0x7FFFFFFFu) == 0) continue;  // inf, nan, +-0: exact in any sum
      const int e = ef == 0 ? -126 : ef - 127;             // subnormals: lowest bit 2^-149
      emax = max(emax, e);
      emin = min(emin, e);
    }
    emax = __reduce_max_sync(kFull, emax);
    emin = __reduce_min_sync(kFull, emin);
    if ((tid & 31) == 0 && emax != INT_MIN) {
      atomicMax(&s_emax, emax);
      atomicMin(&s_emin, emin);
    }
  }
  // id ranks: within a position, token order is id-rank order
  for (int i = tid; i < L * k; i += kThreads) {
    const int t = i / k, tok = s.tt[i];
    int below = 0;
#pragma unroll 8
    for (int r = 0; r < k; ++r) below += s.tt[t * k + r] < tok;
    s.idr[i] = below;
  }
  if (tid == 0) {  // S[t] = lse_1 + ... + lse_t, summed in position order
    double acc = 0.0;
    s.S[0] = 0.0;
    for (int t0 = 1; t0 <= L; t0 += 8) {
      double v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = t0 + e <= L ? s.S[t0 + e] : 0.0;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (t0 + e <= L) {
          acc = __dadd_rn(acc, v[e]);
          s.S[t0 + e] = acc;
        }
    }
  }
  // per-sequence candidate count and budget (clamped, flagged)
  if (kb < 1 || kb > k || Bb < 0 || Bb > p.B_max) {
    if (tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    kb = min(max(kb, 1), k);
    Bb = min(max(Bb, 0), p.B_max);
  }
  __syncthreads();
  if (tid == 0 && s_emax != INT_MIN && s_emax - s_emin > 29 - (32 - __clz(L - 1 > 0 ? L - 1 : 0)))
    raise_status(p.status, DDT_ERR_UNSUPPORTED);  // path sums may round: the order may differ

  // ---------------- selection ----------------
  // ncnt[x] (in nrow, free until numbering): the items of x's run taken
  // this round
  int* ncnt = s.nrow;
  int nn = 1, nsel = 0;
  if (kb == 1) {
    // one candidate per position: the tree is the chain of the first B positions
    const int len = min(Bb, L);
    for (int t = 1 + tid; t <= len; t += kThreads) {
      double sz = 0.0;
      for (int u = 0; u < t; ++u) sz = __dadd_rn(sz, s.zt[u * k]);
      s.nsz[t] = sz;
      s.nsc[t] = score_of(s, inv_t, sz, t);
      s.npar[t] = t - 1;
      s.ndep[t] = t;
      s.nrank[t] = 0;
      s.nnext[t] = t < len ? 1 : 0;
      for (int w = 0; w < p.kw; ++w) s.pkey[(size_t)t * p.kw + w] = 0ull;
      s.nrk[t] = 0ull;  // one node per depth: never compared
      s.ninv[t] = 0;
      red.lvl[t] = 1;
    }
    if (tid == 0) s.nnext[0] = len > 0 ? 1 : 0;
    nn = 1 + len;
    nsel = Bb;  // no other prefix exists
    __syncthreads();
  }
#pragma unroll 1
  while (nsel < Bb) {
    // theta: the K-best first child of a run head
    uint64_t tk = 0;
    uint32_t th = 0;
    int ttie = 0, front = 0;
    for (int x = tid; x < nn; x += kThreads) {
      const int d = s.ndep[x], nx = s.nnext[x];
      if (d < L && nx < kb) {
        front = 1;
        if (d + 1 < L) {
          const double sz = __dadd_rn(__dadd_rn(s.nsz[x], s.zt[d * k + nx]), s.zt[(d + 1) * k]);
          const uint64_t kk = score_key(score_of(s, inv_t, sz, d + 2));
          if (kk > tk) {
            tk = kk;
            th = pack_vp(x, nx, 0);
            ttie = 0;
          } else if (kk == tk) {
            ttie = 1;
          }
        }
      }
    }
    block_max_key(tk, th, ttie, front, &red);
    if (!front) break;
    if (ttie) {
      // several first children share the best score: the full order decides
      __syncthreads();
      PK best = no_pk();
      for (int x = tid; x < nn; x += kThreads) {
        const int d = s.ndep[x], nx = s.nnext[x];
        if (d < L - 1 && nx < kb) {
          const PK c = make_pk(s, inv_t, pack_vp(x, nx, 0));
          if (c.sk == tk && pk_before(s, c, best)) best = c;
        }
      }
      th = block_best_pk(s, best, &red).h;
    }
    // run items before theta (tk == 0: no first child exists, all are)
    int sum = 0, ctie = 0;
    if (nn <= kWarps) {
      // few nodes: a warp per node, a lane per rank of its run
      if (warp < nn) {
        const int x = warp, d = s.ndep[x], nx = s.nnext[x];
        const int len = d < L ? kb - nx : 0;
        const bool in = lane < len;
        const uint64_t kk = in ? item_key(s, inv_t, s.nsz[x], d, nx + lane) : 0ull;
        const unsigned gt = __ballot_sync(kFull, in && kk > tk);
        const unsigned eqb = __ballot_sync(kFull, in && kk == tk);
        const int c = gt == kFull ? 32 : __ffs(~gt) - 1;
        if (c < len && ((eqb >> c) & 1u)) ctie = 1;
        if (lane == 0) ncnt[x] = c;
      }
      ctie = __syncthreads_or(ctie);
      sum = tid < nn ? ncnt[tid] : 0;
    } else {
      for (int x = tid; x < nn; x += kThreads) {
        const int d = s.ndep[x];
        const int c = d < L ? count_fast(s, inv_t, x, d, s.nnext[x], kb, tk, ctie) : 0;
        ncnt[x] = c;
        sum += c;
      }
    }
    int T;
    int off = block_exscan1(sum, T, ctie, &red);
    if (ctie) {
      // an item scores exactly like theta: count again under the full order
      __syncthreads();
      const PK tp = make_pk(s, inv_t, th);
      sum = 0;
      for (int x = tid; x < nn; x += kThreads) {
        int c = 0;
        if (s.ndep[x] < L)
          for (int r = s.nnext[x]; r < kb && pk_before(s, make_pk(s, inv_t, pack_vp(x, r, -1)), tp); ++r) ++c;
        ncnt[x] = c;
        sum += c;
      }
      int nof = 0;
      off = block_exscan1(sum, T, nof, &red);
    }
    if (T == 0) {
      // Only reachable when a candidate scores above its parent (an lse below
      // some inv_t*z): take the K-best run head so that the loop progresses.
      uint64_t bk = 0;
      uint32_t bh = 0;
      for (int x = tid; x < nn; x += kThreads) {
        const int d = s.ndep[x], nx = s.nnext[x];
        if (d < L && nx < kb) {
          const uint64_t kk = item_key(s, inv_t, s.nsz[x], d, nx);
          const uint32_t hh = pack_vp(x, nx, -1);
          if (key_before(s, inv_t, kk, hh, bk, bh)) {
            bk = kk;
            bh = hh;
          }
        }
      }
      bh = block_best_slow(bk, bh, &red).h;
      sum = 0;
      for (int x = tid; x < nn; x += kThreads) {
        ncnt[x] = x == (int)(bh >> 16) ? 1 : 0;
        sum += ncnt[x];
      }
      int nof = 0;
      off = block_exscan1(sum, T, nof, &red);
      if (tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    }
    const int R = Bb - nsel;
    if (T > R && T > icap) {
      // Too many to stage: keep at most m items per run.  The first item cut
      // from a run bounds this round too, so theta becomes the K-best of
      // theta and those items, and the count is redone within the first m.
      const int m = max(1, icap / nn);
      uint64_t k2 = tk;
      uint32_t h2 = th;
      for (int x = tid; x < nn; x += kThreads)
        if (ncnt[x] > m) {
          const int r = s.nnext[x] + m;
          const uint64_t kk = item_key(s, inv_t, s.nsz[x], s.ndep[x], r);
          const uint32_t hh = pack_vp(x, r, -1);
          if (key_before(s, inv_t, kk, hh, k2, h2)) {
            k2 = kk;
            h2 = hh;
          }
        }
      const KeyHandle b2 = block_best_slow(k2, h2, &red);
      sum = 0;
      for (int x = tid; x < nn; x += kThreads) {
        int c = ncnt[x];
        if (c > 0) {
          const int nx = s.nnext[x];
          c = count_slow(x, nx, nx + min(c, m), b2.key, b2.h);
        }
        ncnt[x] = c;
        sum += c;
      }
      int nof = 0;
      off = block_exscan1(sum, T, nof, &red);
    }
    if (T > R) {
      // final round: stage the T candidates and keep the R best
      int o = off;
      for (int x = tid; x < nn; x += kThreads) {
        const int c = ncnt[x], nx = s.nnext[x];
        for (int i = 0; i < c; ++i) s.cid[o + i] = ((uint32_t)x << 8) | (uint32_t)(nx + i);
        o += c;
      }
      __syncthreads();
#pragma unroll 4
      for (int j = tid; j < T; j += kThreads) {
        const uint32_t e = s.cid[j];
        const int x = (int)(e >> 8);
        s.ckey[j] = item_key(s, inv_t, s.nsz[x], s.ndep[x], (int)(e & 0xFFu));
      }
      __syncthreads();
      if (T <= kThreads)
        cut_small(s, T, R, &red);
      else
        cut_best(s, inv_t, T, R, &red);
      o = off;
      sum = 0;
      for (int x = tid; x < nn; x += kThreads) {
        const int c = ncnt[x];
        int kept = 0;
        for (int i = 0; i < c; ++i) kept += (int)(s.cid[o + i] >> 31);
        o += c;
        ncnt[x] = kept;
        sum += kept;
      }
      int nof = 0;
      off = block_exscan1(sum, T, nof, &red);
    }
    // create the selected items as nodes: the owners write parent and rank,
    // then one thread per new node fills in the rest
    int id = nn + off;
    for (int x = tid; x < nn; x += kThreads) {
      const int c = ncnt[x];
      if (c > 0) {
        const int nx = s.nnext[x];
        for (int i = 0; i < c; ++i) {
          s.npar[id + i] = x;
          s.nrank[id + i] = nx + i;
        }
        id += c;
        s.nnext[x] = nx + c;
      }
    }
    __syncthreads();
    for (int j = tid; j < T; j += kThreads) {
      const int idn = nn + j, x = s.npar[idn], r = s.nrank[idn], d = s.ndep[x];
      const double sz = __dadd_rn(s.nsz[x], s.zt[d * k + r]);
      s.nsz[idn] = sz;
      s.nsc[idn] = score_of(s, inv_t, sz, d + 1);
      s.ndep[idn] = d + 1;
      s.nnext[idn] = 0;
      s.ninv[idn] = atomicAdd(&red.lvl[d + 1], 1);  // slot within its depth
      s.nrk[idn] = rev_key(s, s.nrk[x], d, r);
      if (s.kw == 1)
        s.pkey[idn] = s.pkey[x] | ((uint64_t)r << (64 - (d + 1) * s.rb));
      else
        make_path_key(s, x, idn, d, r);
    }
    __syncthreads();
    nn += T;
    nsel += T;
  }

  // surrogate: sum of exp(score) over the draft nodes (nsc is free after this)
  {
    double acc = 0.0;
    for (int x = 1 + tid; x < nn; x += kThreads) acc += exp(s.nsc[x]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    if (lane == 0) red.wd[warp] = acc;
  }

  // ---------------- breadth-first numbering ----------------
  // Rows are ordered by (depth, rank path).  lvl[t] holds the node count of
  // depth t and ninv[x] node x's slot among them, both kept since the node
  // was created.  A level of at most kWide nodes is ranked by counting the
  // same-depth nodes with smaller path keys (all such levels at once); a
  // wider level takes its rows from its parents' rows: the children of the
  // parent in row j follow those of rows < j, in rank order.
  if (warp == 0) {  // lvl[t] <- first row of depth t, for t = 0..L+1
    int v[3], sm = 0;
#pragma unroll
    for (int e = 0; e < 3; ++e) {
      const int t = 3 * lane + e;
      v[e] = t < L + 2 ? red.lvl[t] : 0;
      sm += v[e];
    }
    int run = warp_incl_scan(sm, lane) - sm;
#pragma unroll
    for (int e = 0; e < 3; ++e) {
      const int t = 3 * lane + e;
      if (t < L + 2) red.lvl[t] = run;
      run += v[e];
    }
  }
  __syncthreads();
  // depth buckets: node ids (in prow, free until the parent rows are
  // written) and, when they fit, a copy of the path keys in bucket order (in
  // the free cut buffer) so that the ranking reads them with broadcasts
  int* bucket = s.prow;
  const int kw = s.kw;
  const bool copy_keys = (int64_t)nn * kw * 8 <= 12 * (int64_t)icap;
  uint64_t* bkey = s.ckey;
  for (int x = tid; x < nn; x += kThreads) {
    const int d = s.ndep[x];
    const int q = red.lvl[d] + s.ninv[x];
    bucket[q] = x;
    if (copy_keys && red.lvl[d + 1] - red.lvl[d] <= kWide)
      for (int w = 0; w < kw; ++w) bkey[(size_t)q * kw + w] = s.pkey[(size_t)x * kw + w];
  }
  __syncthreads();
  // narrow levels: rank bucket position q among its depth; threads of a warp
  // take consecutive positions, so they mostly scan the same bucket together
  for (int q = tid; q < nn; q += kThreads) {
    const int x = bucket[q];
    const int d = s.ndep[x], lo = red.lvl[d], hi = red.lvl[d + 1];
    if (hi - lo > kWide) continue;
    int below = 0;
    if (copy_keys && kw == 1) {
      const uint64_t kx = bkey[q];
      int u = lo;
      if ((u & 1) && u < hi) below += bkey[u++] < kx;  // then 16-byte aligned
      for (; u + 8 <= hi; u += 8) {                      // eight keys a step
        ulonglong2 v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = *reinterpret_cast<const ulonglong2*>(bkey + u + 2 * e);
#pragma unroll
        for (int e = 0; e < 4; ++e) below += (v[e].x < kx) + (v[e].y < kx);
      }
      for (; u < hi; ++u) below += bkey[u] < kx;
    } else if (copy_keys && kw == 2) {
      const uint64_t k0 = bkey[2 * q], k1 = bkey[2 * q + 1];
      for (int u = lo; u < hi; ++u) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(bkey + 2 * u);
        below += (int)(v.x < k0) | ((int)(v.x == k0) & (int)(v.y < k1));
      }
    } else {
      for (int u = lo; u < hi; ++u) below += path_less(s, bucket[u], x);
    }
    s.nrow[x] = lo + below;
    s.ninv[lo + below] = x;
  }
  __syncthreads();
  // wide levels, in depth order: first-child rows of the level above by a
  // scan of its child counts in row order, then each node's row
  int* nfc = reinterpret_cast<int*>(s.nsc);
  for (int d = 1; d <= L; ++d) {
    const int lo = red.lvl[d], hi = red.lvl[d + 1];
    if (hi - lo <= kWide) continue;
    const int plo = red.lvl[d - 1], pw = lo - plo;
    const int c = (pw + kThreads - 1) / kThreads;
    const int r0 = plo + min(tid * c, pw), r1 = plo + min((tid + 1) * c, pw);
    int sum = 0;
    for (int j = r0; j < r1; ++j) sum += s.nnext[s.ninv[j]];
    int tot, nof = 0;
    int run = lo + block_exscan1(sum, tot, nof, &red);
    for (int j = r0; j < r1; ++j) {
      const int x = s.ninv[j];
      nfc[x] = run;
      run += s.nnext[x];
    }
    __syncthreads();
    for (int q = lo + tid; q < hi; q += kThreads) {
      const int x = bucket[q];
      const int row = nfc[s.npar[x]] + s.nrank[x];
      s.nrow[x] = row;
      s.ninv[row] = x;
    }
    __syncthreads();
  }

  // ---------------- outputs ----------------
  const int32_t ctx = p.ctx_len ? p.ctx_len[b] : 0;
  int32_t* o_tok = p.tok + (int64_t)b * NM;
  int32_t* o_par = p.parent + (int64_t)b * NM;
  int32_t* o_dep = p.depth + (int64_t)b * NM;
  int32_t* o_pos = p.pos + (int64_t)b * NM;
  for (int j = tid; j < NM; j += kThreads) {
    if (j < nn) {
      const int x = s.ninv[j];
      const int d = s.ndep[x];
      const int pr = x == 0 ? -1 : s.nrow[s.npar[x]];
      o_tok[j] = x == 0 ? p.root_token[b] : s.tt[(d - 1) * k + s.nrank[x]];
      o_par[j] = pr;
      o_dep[j] = d;
      o_pos[j] = ctx + d;
      s.prow[j] = pr;
    } else {
      o_tok[j] = -1;
      o_par[j] = -1;
      o_dep[j] = -1;
      o_pos[j] = -1;
    }
  }
  __syncthreads();
  // ancestor-or-self masks: row j walks its parent rows, which decrease, so
  // each mask word is complete when the walk moves below it and is written
  // once; staged in the (now free) cut buffer when it holds them
  const int W = p.W;
  uint32_t* o_mask = p.mask + (int64_t)b * NM * W;
  const bool staged = (int64_t)nn * W <= 3 * (int64_t)icap;
  uint32_t* m = staged ? (uint32_t*)s.ckey : o_mask;
  for (int j = tid; j < nn; j += kThreads) {
    uint32_t* row = m + (int64_t)j * W;
    int wcur = j >> 5;
    for (int w = wcur + 1; w < W; ++w) row[w] = 0u;
    uint32_t acc = 0u;
    for (int a = j;;) {
      const int wa = a >> 5;
      while (wa < wcur) {
        row[wcur--] = acc;
        acc = 0u;
      }
      acc |= 1u << (a & 31);
      if (a == 0) break;
      a = s.prow[a];
    }
    row[wcur] = acc;  // wcur == 0 here: the root is row 0
  }
  if (staged) {
    __syncthreads();
    for (int i = tid; i < NM * W; i += kThreads) o_mask[i] = i < nn * W ? m[i] : 0u;
  } else {
    for (int i = nn * W + tid; i < NM * W; i += kThreads) o_mask[i] = 0u;
  }
  pdl_trigger();  // the outputs are being written: the next kernel may be scheduled
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += red.wd[w];
    p.n_nodes[b] = nn;
    if (p.surrogate) p.surrogate[b] = t;
  }
}

size_t tree_smem_bytes(int L, int k, int n_max, int kw, int icap) {
  auto a = [](size_t x) { return (x + 15) & ~(size_t)15; };
  return a(sizeof(double) * (L + 1)) + a(sizeof(double) * L * k) + 2 * a(sizeof(double) * n_max) +
         a(sizeof(uint64_t) * n_max * kw) + a(sizeof(uint64_t) * n_max) + a(sizeof(uint64_t) * icap) +
         a(sizeof(uint32_t) * icap) + a(sizeof(int) * L * k) +
         a(sizeof(int) * L * k) + 7 * a(sizeof(int) * n_max);
}

// Cut buffer: the biggest frontier (n_max*k items), within the shared memory
// left by everything else; never fewer than n_max items (a truncated round
// keeps at least one item per run).
int item_cap(int L, int k, int n_max, int kw) {
  int cap = n_max * k;
  if (cap > kItemCapMax) cap = kItemCapMax;
  if (cap < n_max) cap = n_max;
  const size_t fixed = tree_smem_bytes(L, k, n_max, kw, 0) + 2 * 16 + sizeof(Red);
  const size_t per_item = sizeof(uint64_t) + sizeof(uint32_t);
  const int fit = (int)((kSmemMax - 1024 - fixed) / per_item);
  if (cap > fit) cap = fit;
  return cap;
}

int rank_bits(int k) {
  int rb = 1;
  while ((1 << rb) < k) ++rb;
  return rb;
}

}  // namespace

ddt_status launch_build_tree(const int32_t* ids, const float* zk, const float* lse, int batch,
                             int L, int k, float inv_t, const int32_t* k_per_seq,
                             const int32_t* budget, int B_max, const int32_t* root_token,
                             const int32_t* ctx_len, int32_t* tok, int32_t* parent,
                             int32_t* depth, int32_t* pos, uint32_t* mask, int32_t* n_nodes,
                             double* surrogate, int32_t* dev_status, cudaStream_t stream) {
  TreeParams p;
  p.ids = ids;
  p.zk = zk;
  p.lse = lse;
  p.L = L;
  p.k = k;
  p.inv_t = (double)inv_t;
  p.k_per_seq = k_per_seq;
  p.budget = budget;
  p.B_max = B_max;
  p.n_max = B_max + 1;
  p.W = (p.n_max + 31) / 32;
  p.rb = rank_bits(k);
  p.kw = (L * p.rb + 63) / 64;
  if (p.kw < 1) p.kw = 1;
  p.icap = item_cap(L, k, p.n_max, p.kw);
  p.root_token = root_token;
  p.ctx_len = ctx_len;
  p.tok = tok;
  p.parent = parent;
  p.depth = depth;
  p.pos = pos;
  p.mask = mask;
  p.n_nodes = n_nodes;
  p.surrogate = surrogate;
  p.status = dev_status;
  if (batch == 0) return DDT_OK;
  const size_t smem = tree_smem_bytes(L, k, p.n_max, p.kw, p.icap);
  if (ensure_smem_attr((const void*)build_tree_kernel, smem) != cudaSuccess) return DDT_ERR_CUDA;
  return launch_pdl(build_tree_kernel, dim3(batch), dim3(kThreads), smem, stream, 0, p) == cudaSuccess
             ? DDT_OK
             : DDT_ERR_CUDA;
}

}  // namespace ddt
