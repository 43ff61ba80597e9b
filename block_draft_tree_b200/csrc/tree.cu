// tree.cu -- stage 2 of the verification round: the B most probable prefixes
// of the factorised draft, compiled into target-model inputs.
//
// DDTree page: section 核心創新 (best-first selection under a node budget B),
// 運作流程 step 2 (maximise the expected acceptance length under the
// factorised draft; the optimum is the set of highest-probability prefixes,
// which is prefix-closed), 理論基礎 Propositions 1-2, and step 3 (compile
// the tree into target inputs with an ancestor-only mask).
//
// One CTA of 256 threads per sequence.  Selection proceeds in frontier
// rounds instead of popping a heap one node at a time, and selects exactly
// the same set:
//   * every selected node x keeps n_next[x], the number of its children
//     already selected; they are always ranks 0..n_next[x]-1 because
//     siblings come in the candidate order, which is the total order K;
//   * the unselected children of selected nodes (the frontier) are, per x,
//     the run of ranks n_next[x]..k-1, sorted by K;
//   * each round lays the frontier items out in shared memory, one thread
//     per item: theta = the K-best child any of them could have; every item
//     that precedes theta precedes everything not yet generated, so all of
//     them are among the best remaining prefixes and are selected together;
//   * when they would overshoot the budget, the last round keeps the R best
//     of them: histograms of their fp64 scores narrow the cut to one bin,
//     whose few items are ranked exactly under K.
// Each round selects at least the K-best frontier item, so the loop ends.
// A frontier too large for the item buffer is truncated per run, and the
// first item cut from each run joins theta, so truncation never lets a
// worse prefix in ahead of a better one.  The selected set is then numbered
// breadth-first, level by level, and the ancestor masks are built level by
// level (in shared memory when they fit).
//
// Order K (best first): equal depth -> larger fp64 sum of raw logits, then
// reverse-lexicographic token ids; different depths -> larger fp64 score
// inv_t*sum(z) - sum(lse), then the shallower prefix.
#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;        // histogram bins of the final-round cut
constexpr int kExactMax = 16;     // boundary items ranked exactly
constexpr int kMaxPasses = 4;     // histogram passes before ranking what is left
constexpr int kItemCapMax = 10240;
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
  int B_max, n_max, W, icap;
  const int32_t* root_token;
  const int32_t* ctx_len;
  int32_t *tok, *parent, *depth, *pos;
  uint32_t* mask;
  int32_t* n_nodes;
  double* surrogate;
  int32_t* status;
};

struct Smem {
  double* zt;       // [L*k] raw logits of the candidates
  int* tt;          // [L*k] candidate token ids
  double* S;        // [L+1] prefix sums of lse
  double* nsz;      // [n_max] node logit sums
  double* nsc;      // [n_max] node scores
  int* npar;        // [n_max] parent node (creation index)
  int* ndep;        // [n_max]
  int* nrank;       // [n_max] candidate rank at the node's own position
  int* nnext;       // [n_max] selected-children count
  int* nlen;        // [n_max] items of the run this round / BFS row
  int* noff;        // [n_max] offset of the run's items / first-child row
  int* ninv;        // [n_max] BFS row -> node
  uint32_t* iown;   // [icap] item: node << 8 | rank
  double* isc;      // [icap] item score
  int* iflag;       // [icap] item selected this round
  int* ipos;        // [icap] scan of iflag
  int* hist;        // [kBins]
  int k;
};

// A prefix given as a selected node plus up to two appended ranks.
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

// true iff a strictly precedes b under K.  depth < 0 marks "no prefix" (last).
__device__ __forceinline__ bool vp_before(const Smem& s, const VP& a, const VP& b) {
  if (b.depth < 0) return a.depth >= 0;
  if (a.depth < 0) return false;
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

__device__ __forceinline__ double score_of(const Smem& s, double inv_t, double sz, int t) {
  return __dsub_rn(__dmul_rn(inv_t, sz), s.S[t]);
}

// Frontier item (x, r): the child of node x with candidate rank r.
__device__ __forceinline__ VP make_item(const Smem& s, double inv_t, int x, int r) {
  VP v;
  v.base = x;
  v.r1 = r;
  v.r2 = -1;
  const int d = s.ndep[x];
  v.depth = d + 1;
  v.sz = __dadd_rn(s.nsz[x], s.zt[d * s.k + r]);
  v.sc = score_of(s, inv_t, v.sz, v.depth);
  return v;
}

// Item i of the item buffer (its score already computed).
__device__ __forceinline__ VP item_vp(const Smem& s, int i) {
  VP v;
  const uint32_t e = s.iown[i];
  v.base = (int)(e >> 8);
  v.r1 = (int)(e & 0xFFu);
  v.r2 = -1;
  const int d = s.ndep[v.base];
  v.depth = d + 1;
  v.sz = __dadd_rn(s.nsz[v.base], s.zt[d * s.k + v.r1]);
  v.sc = s.isc[i];
  return v;
}

__device__ __forceinline__ VP no_vp() {
  VP v;
  v.sz = v.sc = 0.0;
  v.depth = -1;
  v.base = 0;
  v.r1 = v.r2 = -1;
  return v;
}

__device__ __forceinline__ VP shfl_vp(const VP& v, int o) {
  VP r;
  r.sz = __shfl_xor_sync(kFull, v.sz, o);
  r.sc = __shfl_xor_sync(kFull, v.sc, o);
  r.depth = __shfl_xor_sync(kFull, v.depth, o);
  r.base = __shfl_xor_sync(kFull, v.base, o);
  r.r1 = __shfl_xor_sync(kFull, v.r1, o);
  r.r2 = __shfl_xor_sync(kFull, v.r2, o);
  return r;
}

// K-best over the block; every thread gets the result.
__device__ VP block_best(const Smem& s, VP v, VP* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const VP u = shfl_vp(v, o);
    if (vp_before(s, u, v)) v = u;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  VP b = red[0];
  for (int w = 1; w < kWarps; ++w)
    if (vp_before(s, red[w], b)) b = red[w];
  __syncthreads();
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

// out[i] = in[0] + ... + in[i-1] for i < n (out may alias in); returns the
// total.  Thread t scans the contiguous block [t*c, (t+1)*c).
__device__ int block_exscan(const int* in, int* out, int n, int* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = (n + kThreads - 1) / kThreads;
  const int lo = min(tid * c, n), hi = min(lo + c, n);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += in[i];
  const int inc = warp_incl_scan(sum, lane);
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  int before = 0, total = 0;
  for (int w = 0; w < kWarps; ++w) {
    before += (w < warp) ? red[w] : 0;
    total += red[w];
  }
  int run = before + inc - sum;
  for (int i = lo; i < hi; ++i) {
    const int v = in[i];
    out[i] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

__device__ int block_sum(int v, int* red) {
  v = __reduce_add_sync(kFull, v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  int t = 0;
  for (int w = 0; w < kWarps; ++w) t += red[w];
  __syncthreads();
  return t;
}

// One histogram pass of the final-round cut.
struct Pass {
  double lo, scale;
  int bstar;
};

// Position of a score relative to the cut: 1 above it (kept), -1 below it
// (dropped), 0 in the boundary bin of every pass so far.  Each pass bins
// with the same arithmetic, so an item's state never depends on rounding
// of a recomputed bin edge.
__device__ __forceinline__ int cut_state(double sc, const Pass* ps, int np) {
  for (int q = 0; q < np; ++q) {
    int bin = (int)((sc - ps[q].lo) * ps[q].scale);
    bin = min(max(bin, 0), kBins - 1);
    if (bin > ps[q].bstar) return 1;
    if (bin < ps[q].bstar) return -1;
  }
  return 0;
}

struct CutShared {
  Pass ps[kMaxPasses];
  int np, above, in_cut, nb;
  double lo, hi;
  int list[kBins];
};

// Final round: among the F items with iflag set (more than R of them), keep
// the R K-best (iflag cleared on the others).  The kept items of a run are a
// prefix of it, since a run is K-ordered.
__device__ void keep_best(const Smem& s, int F, int R, CutShared* cs, double* dred, int* red,
                          VP* vred) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double lo = INFINITY, hi = -INFINITY;
  int in_cut = 0;
  for (int i = tid; i < F; i += kThreads)
    if (s.iflag[i]) {
      lo = fmin(lo, s.isc[i]);
      hi = fmax(hi, s.isc[i]);
      ++in_cut;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(kFull, lo, o));
    hi = fmax(hi, __shfl_xor_sync(kFull, hi, o));
  }
  if (lane == 0) {
    dred[warp] = lo;
    dred[kWarps + warp] = hi;
  }
  in_cut = block_sum(in_cut, red);  // its barriers also publish dred
  if (tid == 0) {
    double l = INFINITY, h = -INFINITY;
    for (int w = 0; w < kWarps; ++w) {
      l = fmin(l, dred[w]);
      h = fmax(h, dred[kWarps + w]);
    }
    cs->lo = l;
    cs->hi = h;
    cs->np = 0;
    cs->above = 0;
    cs->in_cut = in_cut;
  }
  __syncthreads();
  // narrow the cut with score histograms
  for (;;) {
    const int np = cs->np;
    if (np >= kMaxPasses || cs->in_cut <= kExactMax || !(cs->hi > cs->lo)) break;
    for (int bn = tid; bn < kBins; bn += kThreads) s.hist[bn] = 0;
    __syncthreads();
    Pass pass;
    pass.lo = cs->lo;
    pass.scale = (double)kBins / (cs->hi - cs->lo);
    for (int i = tid; i < F; i += kThreads) {
      if (!s.iflag[i]) continue;
      const double sc = s.isc[i];
      if (cut_state(sc, cs->ps, np) != 0) continue;
      atomicAdd(&s.hist[min(max((int)((sc - pass.lo) * pass.scale), 0), kBins - 1)], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins [8l, 8l+8); find the bin holding the R-th best from the top
      int h[8], lt = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        h[e] = s.hist[8 * lane + e];
        lt += h[e];
      }
      int suf = lt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_down_sync(kFull, suf, o);
        if (lane + o < 32) suf += u;
      }
      const int above_lane = cs->above + suf - lt;
      const bool mine = above_lane < R && above_lane + lt >= R;
      const unsigned who = __ballot_sync(kFull, mine);
      const int src = who ? __ffs(who) - 1 : 0;
      if (lane == src) {
        int acc = above_lane, bs = 0, cnt = 0;
        for (int e = 7; e >= 0; --e) {
          if (acc + h[e] >= R) {
            bs = 8 * lane + e;
            cnt = h[e];
            break;
          }
          acc += h[e];
        }
        pass.bstar = bs;
        cs->ps[np] = pass;
        cs->np = np + 1;
        cs->above = acc;
        cs->in_cut = cnt;
        cs->lo = pass.lo + bs / pass.scale;
        cs->hi = pass.lo + (bs + 1) / pass.scale;
      }
    }
    __syncthreads();
  }
  const int np = cs->np;
  const int need = R - cs->above;
  // gather the boundary items
  if (tid == 0) cs->nb = 0;
  __syncthreads();
  for (int i = tid; i < F; i += kThreads)
    if (s.iflag[i] && cut_state(s.isc[i], cs->ps, np) == 0) {
      const int q = atomicAdd(&cs->nb, 1);
      if (q < kBins) cs->list[q] = i;
    }
  __syncthreads();
  const int nb = cs->nb;
  if (nb <= kBins) {
    // rank each boundary item among them; keep the `need` best
    for (int t = tid; t < nb; t += kThreads) {
      const int i = cs->list[t];
      const VP vi = item_vp(s, i);
      int rank = 0;
      for (int u = 0; u < nb; ++u)
        if (u != t) rank += vp_before(s, item_vp(s, cs->list[u]), vi);
      s.ipos[i] = rank < need;  // verdict for boundary items
    }
    __syncthreads();
    for (int i = tid; i < F; i += kThreads)
      if (s.iflag[i]) {
        const int st = cut_state(s.isc[i], cs->ps, np);
        s.iflag[i] = st == 1 || (st == 0 && s.ipos[i]);
      }
    __syncthreads();
  } else {
    // many exact score ties: take the K-best undecided boundary item, need times
    for (int i = tid; i < F; i += kThreads)
      if (s.iflag[i]) {
        const int st = cut_state(s.isc[i], cs->ps, np);
        s.iflag[i] = st == 1 ? 1 : (st == 0 ? 2 : 0);  // 2: boundary, undecided
      }
    __syncthreads();
    for (int t = 0; t < need; ++t) {
      VP best = no_vp();
      int bi = -1;
      for (int i = tid; i < F; i += kThreads)
        if (s.iflag[i] == 2) {
          const VP v = item_vp(s, i);
          if (vp_before(s, v, best)) {
            best = v;
            bi = i;
          }
        }
      const VP bb = block_best(s, best, vred);
      if (bi >= 0 && bb.base == best.base && bb.r1 == best.r1 && bb.depth == best.depth)
        s.iflag[bi] = 3;  // taken
      __syncthreads();
    }
    for (int i = tid; i < F; i += kThreads) s.iflag[i] = (s.iflag[i] == 1 || s.iflag[i] == 3);
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads) build_tree_kernel(TreeParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int s_lvl[DDT_TREE_L_MAX + 2];
  __shared__ int s_red[kWarps + 1];
  __shared__ double s_dred[2 * kWarps];
  __shared__ VP s_vred[kWarps];
  __shared__ CutShared s_cut;
  __shared__ int s_maxd;

  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = p.L, k = p.k, NM = p.n_max, icap = p.icap;
  const double inv_t = p.inv_t;

  Smem s;
  s.k = k;
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
    s.isc = (double*)take(sizeof(double) * icap);
    s.tt = (int*)take(sizeof(int) * L * k);
    s.npar = (int*)take(sizeof(int) * NM);
    s.ndep = (int*)take(sizeof(int) * NM);
    s.nrank = (int*)take(sizeof(int) * NM);
    s.nnext = (int*)take(sizeof(int) * NM);
    s.nlen = (int*)take(sizeof(int) * NM);
    s.noff = (int*)take(sizeof(int) * NM);
    s.ninv = (int*)take(sizeof(int) * NM);
    s.iown = (uint32_t*)take(sizeof(uint32_t) * icap);
    s.iflag = (int*)take(sizeof(int) * icap);
    s.ipos = (int*)take(sizeof(int) * icap);
    s.hist = (int*)take(sizeof(int) * kBins);
  }

  // per-sequence candidate count and budget (clamped, flagged)
  int kb = p.k_per_seq ? p.k_per_seq[b] : k;
  int Bb = p.budget ? p.budget[b] : p.B_max;
  if (kb < 1 || kb > k || Bb < 0 || Bb > p.B_max) {
    if (tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    kb = min(max(kb, 1), k);
    Bb = min(max(Bb, 0), p.B_max);
  }
  for (int i = tid; i < L * k; i += kThreads) {
    s.zt[i] = (double)p.zk[(int64_t)b * L * k + i];
    s.tt[i] = p.ids[(int64_t)b * L * k + i];
  }
  if (tid == 32) {
    double acc = 0.0;
    s.S[0] = 0.0;
    for (int t = 1; t <= L; ++t) {
      acc = __dadd_rn(acc, (double)p.lse[(int64_t)b * L + t - 1]);
      s.S[t] = acc;
    }
  }
  if (tid == 0) {
    s.nsz[0] = 0.0;
    s.nsc[0] = 0.0;
    s.npar[0] = -1;
    s.ndep[0] = 0;
    s.nrank[0] = 0;
    s.nnext[0] = 0;
  }
  __syncthreads();

  // ---------------- selection ----------------
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
    }
    if (tid == 0) s.nnext[0] = len > 0 ? 1 : 0;
    nn = 1 + len;
    nsel = Bb;  // no other prefix exists
    __syncthreads();
  }
#pragma unroll 1
  while (nsel < Bb) {
    // runs of this round, truncated to fit the item buffer
    int tot = 0;
    for (int x = tid; x < nn; x += kThreads) {
      const int len = (s.ndep[x] < L) ? max(0, kb - s.nnext[x]) : 0;
      s.nlen[x] = len;
      tot += len;
    }
    tot = block_sum(tot, s_red);
    if (tot == 0) break;
    const int cap = tot <= icap ? DDT_TOPK_K_MAX : max(1, icap / nn);
    VP th = no_vp();
    if (tot > icap) {
      for (int x = tid; x < nn; x += kThreads) {
        const int len = s.nlen[x];
        if (len > cap) {  // the first item cut from the run bounds the round too
          const VP v = make_item(s, inv_t, x, s.nnext[x] + cap);
          if (vp_before(s, v, th)) th = v;
          s.nlen[x] = cap;
        }
      }
      __syncthreads();
    }
    const int F = block_exscan(s.nlen, s.noff, nn, s_red);
    for (int x = tid; x < nn; x += kThreads) {
      const int o = s.noff[x], r0 = s.nnext[x], len = s.nlen[x];
      for (int i = 0; i < len; ++i) s.iown[o + i] = ((uint32_t)x << 8) | (uint32_t)(r0 + i);
    }
    __syncthreads();
    // item scores; theta = the K-best first child of any item
    for (int i = tid; i < F; i += kThreads) {
      const uint32_t e = s.iown[i];
      const int x = (int)(e >> 8), r = (int)(e & 0xFFu);
      const int d = s.ndep[x];
      const double sz = __dadd_rn(s.nsz[x], s.zt[d * k + r]);
      s.isc[i] = score_of(s, inv_t, sz, d + 1);
      if (d + 1 < L) {
        VP c;
        c.base = x;
        c.r1 = r;
        c.r2 = 0;
        c.depth = d + 2;
        c.sz = __dadd_rn(sz, s.zt[(d + 1) * k]);
        c.sc = score_of(s, inv_t, c.sz, c.depth);
        if (vp_before(s, c, th)) th = c;
      }
    }
    th = block_best(s, th, s_vred);
    // safe items: those that precede theta
    for (int i = tid; i < F; i += kThreads) s.iflag[i] = vp_before(s, item_vp(s, i), th);
    __syncthreads();
    int T = block_exscan(s.iflag, s.ipos, F, s_red);
    if (T == 0) {
      // Only reachable when a candidate scores above its parent (an lse below
      // some inv_t*z): take the K-best item so that the loop progresses.
      VP best = no_vp();
      for (int i = tid; i < F; i += kThreads) {
        const VP v = item_vp(s, i);
        if (vp_before(s, v, best)) best = v;
      }
      best = block_best(s, best, s_vred);
      for (int i = tid; i < F; i += kThreads) {
        const uint32_t e = s.iown[i];
        s.iflag[i] = (int)(e >> 8) == best.base && (int)(e & 0xFFu) == best.r1;
      }
      __syncthreads();
      T = block_exscan(s.iflag, s.ipos, F, s_red);
      if (tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    }
    const int R = Bb - nsel;
    const bool last = T >= R;
    if (T > R) {
      keep_best(s, F, R, &s_cut, s_dred, s_red, s_vred);
      T = block_exscan(s.iflag, s.ipos, F, s_red);
    }
    // create the selected items as nodes
    for (int i = tid; i < F; i += kThreads)
      if (s.iflag[i]) {
        const uint32_t e = s.iown[i];
        const int x = (int)(e >> 8), r = (int)(e & 0xFFu);
        const int id = nn + s.ipos[i];
        const int d = s.ndep[x];
        s.nsz[id] = __dadd_rn(s.nsz[x], s.zt[d * k + r]);
        s.nsc[id] = s.isc[i];
        s.npar[id] = x;
        s.ndep[id] = d + 1;
        s.nrank[id] = r;
        s.nnext[id] = 0;
        atomicAdd(&s.nnext[x], 1);
      }
    __syncthreads();
    nn += T;
    nsel += T;
    if (last) break;
  }

  // ---------------- breadth-first numbering ----------------
  // nlen[x] <- row of x, ninv[row] <- x, noff[x] <- row of x's first child
  if (tid < DDT_TREE_L_MAX + 2) s_lvl[tid] = 0;
  __syncthreads();
  int maxd = 0;
  for (int x = tid; x < nn; x += kThreads) {
    atomicAdd(&s_lvl[s.ndep[x]], 1);
    maxd = max(maxd, s.ndep[x]);
  }
  maxd = __reduce_max_sync(kFull, maxd);
  if (lane == 0) s_red[warp] = maxd;
  __syncthreads();
  if (tid == 0) {  // s_lvl[t] <- number of nodes of depth < t (= first row of depth t)
    int acc = 0;
    for (int t = 0; t <= L + 1; ++t) {
      const int c = s_lvl[t];
      s_lvl[t] = acc;
      acc += c;
    }
    int md = 0;
    for (int w = 0; w < kWarps; ++w) md = max(md, s_red[w]);
    s_maxd = md;
    s.nlen[0] = 0;
    s.noff[0] = 1;
    s.ninv[0] = 0;
  }
  __syncthreads();
  const int md = s_maxd;
  for (int t = 1; t <= md; ++t) {
    const int lstart = s_lvl[t], lend = s_lvl[t + 1];
    for (int x = tid; x < nn; x += kThreads)
      if (s.ndep[x] == t) {
        const int j = s.noff[s.npar[x]] + s.nrank[x];
        s.nlen[x] = j;
        s.ninv[j] = x;
      }
    __syncthreads();
    // first-child rows of level t: lend + exclusive scan of child counts
    for (int j = lstart + tid; j < lend; j += kThreads) s.iflag[j - lstart] = s.nnext[s.ninv[j]];
    __syncthreads();
    block_exscan(s.iflag, s.ipos, lend - lstart, s_red);
    for (int j = lstart + tid; j < lend; j += kThreads) s.noff[s.ninv[j]] = lend + s.ipos[j - lstart];
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
      o_tok[j] = x == 0 ? p.root_token[b] : s.tt[(d - 1) * k + s.nrank[x]];
      o_par[j] = x == 0 ? -1 : s.nlen[s.npar[x]];
      o_dep[j] = d;
      o_pos[j] = ctx + d;
    } else {
      o_tok[j] = -1;
      o_par[j] = -1;
      o_dep[j] = -1;
      o_pos[j] = -1;
    }
  }
  // ancestor-or-self masks, level by level: row j = row(parent j) | bit j,
  // staged in the (now free) item buffer when it holds them
  const int W = p.W;
  uint32_t* o_mask = p.mask + (int64_t)b * NM * W;
  const bool staged = (int64_t)nn * W <= 2 * (int64_t)icap;
  uint32_t* m = staged ? (uint32_t*)s.isc : o_mask;
  for (int i = tid; i < (staged ? nn * W : NM * W); i += kThreads) m[i] = (i == 0) ? 1u : 0u;
  __syncthreads();
  for (int t = 1; t <= md; ++t) {
    const int lstart = s_lvl[t], lend = s_lvl[t + 1];
    for (int i = tid; i < (lend - lstart) * W; i += kThreads) {
      const int j = lstart + i / W, w = i % W;
      uint32_t word = m[(int64_t)s.nlen[s.npar[s.ninv[j]]] * W + w];
      if ((j >> 5) == w) word |= 1u << (j & 31);
      m[(int64_t)j * W + w] = word;
    }
    __syncthreads();
  }
  if (staged)
    for (int i = tid; i < NM * W; i += kThreads) o_mask[i] = i < nn * W ? m[i] : 0u;
  // surrogate: sum of exp(score) over the draft nodes
  double acc = 0.0;
  for (int x = 1 + tid; x < nn; x += kThreads) acc += exp(s.nsc[x]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
  if (lane == 0) s_dred[warp] = acc;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += s_dred[w];
    p.n_nodes[b] = nn;
    if (p.surrogate) p.surrogate[b] = t;
  }
}

size_t tree_smem_bytes(int L, int k, int n_max, int icap) {
  auto a = [](size_t x) { return (x + 15) & ~(size_t)15; };
  return a(sizeof(double) * (L + 1)) + a(sizeof(double) * L * k) + 2 * a(sizeof(double) * n_max) +
         a(sizeof(double) * icap) + a(sizeof(int) * L * k) + 7 * a(sizeof(int) * n_max) +
         3 * a(sizeof(int) * icap) + a(sizeof(int) * kBins);
}

// Item buffer: the biggest frontier (n_max*k items), within the shared
// memory left by everything else; never fewer than n_max items (a truncated
// round keeps at least one item per run).
int item_cap(int L, int k, int n_max) {
  int cap = n_max * k;
  if (cap > kItemCapMax) cap = kItemCapMax;
  if (cap < n_max) cap = n_max;
  const size_t fixed = tree_smem_bytes(L, k, n_max, 0) + 4 * 16;
  const size_t per_item = sizeof(double) + 3 * sizeof(int);
  const int fit = (int)((kSmemMax - 4096 - fixed) / per_item);
  if (cap > fit) cap = fit;
  return cap;
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
  p.icap = item_cap(L, k, p.n_max);
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
  const size_t smem = tree_smem_bytes(L, k, p.n_max, p.icap);
  if (ensure_smem_attr((const void*)build_tree_kernel, smem) != cudaSuccess) return DDT_ERR_CUDA;
  build_tree_kernel<<<batch, kThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
