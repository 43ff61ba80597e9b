// tree.cu -- stage 2 of the verification round: the B most probable prefixes
// of the factorised draft, compiled into target-model inputs.
//
// DDTree page: section 核心創新 (best-first selection under a node budget B),
// 運作流程 step 2 (maximise the expected acceptance length under the
// factorised draft; the optimum is the set of highest-probability prefixes,
// which is prefix-closed), 理論基礎 Propositions 1-2, and step 3 (compile
// the tree into target inputs with an ancestor-only mask).
//
// One CTA per sequence.  Instead of popping a heap one node at a time, the
// selection proceeds in frontier rounds that are exact:
//   * every selected node p keeps n_next[p], the number of its children
//     already selected; they are always ranks 0..n_next[p]-1 because
//     siblings come in the candidate order, which is the total order K;
//   * the unselected children of selected nodes (the frontier) are, per p,
//     the run of ranks n_next[p]..k-1, sorted by K;
//   * theta = the K-best child any frontier node could have (the first child
//     of each run head).  Every frontier item that precedes theta under K
//     precedes everything not yet generated, so all of them are among the
//     best remaining prefixes and are selected together;
//   * when they would overshoot the budget, the final round sorts them
//     (bitonic, shared memory) and keeps the best.
// Each round selects at least the K-best frontier item, so the loop ends.
// The selected set is then numbered breadth-first, level by level.
//
// Order K (best first): equal depth -> larger exact fp64 sum of raw logits,
// then reverse-lexicographic token ids; different depths -> larger fp64
// score inv_t*sum(z) - sum(lse), then the shallower prefix.
#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 512;
constexpr int kSafeCap = 4096;

struct TreeParams {
  const int32_t* ids;
  const float* zk;
  const float* lse;
  int L, k;
  double inv_t;
  const int32_t* k_per_seq;
  const int32_t* budget;
  int B_max, n_max, W;
  const int32_t* root_token;
  const int32_t* ctx_len;
  int32_t *tok, *parent, *depth, *pos;
  uint32_t* mask;
  int32_t* n_nodes;
  double* surrogate;
  int32_t* status;
};

struct Smem {
  float* zt;      // [L*k] raw logits of the candidates
  int* tt;        // [L*k] candidate token ids
  double* S;      // [L+1] prefix sums of lse
  double* nsz;    // [n_max] node logit sums
  double* nsc;    // [n_max] node scores
  int* npar;      // [n_max] parent node (creation index)
  int* ndep;      // [n_max]
  int* nrank;     // [n_max] candidate rank at the node's own position
  int* nnext;     // [n_max] selected-children count
  int* ncnt;      // [n_max] round scratch: safe-item count / BFS index
  int* noff;      // [n_max] round scratch: scan / first-child index
  int* ninv;      // [n_max] BFS row -> node
  uint32_t* safe; // [kSafeCap] final-round list (node << 8 | rank)
  int L, k;
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
__device__ bool vp_before(const Smem& s, const VP& a, const VP& b) {
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

__device__ __forceinline__ VP make_item(const Smem& s, double inv_t, int p, int r) {
  VP v;
  v.base = p;
  v.r1 = r;
  v.r2 = -1;
  const int d = s.ndep[p];
  v.depth = d + 1;
  v.sz = __dadd_rn(s.nsz[p], (double)s.zt[d * s.k + r]);
  v.sc = score_of(s, inv_t, v.sz, v.depth);
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

__device__ VP shfl_vp(const VP& v, int o) {
  VP r;
  r.sz = __shfl_xor_sync(0xFFFFFFFFu, v.sz, o);
  r.sc = __shfl_xor_sync(0xFFFFFFFFu, v.sc, o);
  r.depth = __shfl_xor_sync(0xFFFFFFFFu, v.depth, o);
  r.base = __shfl_xor_sync(0xFFFFFFFFu, v.base, o);
  r.r1 = __shfl_xor_sync(0xFFFFFFFFu, v.r1, o);
  r.r2 = __shfl_xor_sync(0xFFFFFFFFu, v.r2, o);
  return r;
}

// K-best over the block.  Every thread gets the result.
__device__ VP block_best(const Smem& s, VP v, VP* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
  for (int o = 16; o > 0; o >>= 1) {
    VP u = shfl_vp(v, o);
    if (vp_before(s, u, v)) v = u;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  VP b = red[0];
  for (int w = 1; w < kThreads / 32; ++w)
    if (vp_before(s, red[w], b)) b = red[w];
  return b;
}

// Exclusive scan of a[0..n) in place (n <= 2*kThreads); returns the total.
__device__ int block_exscan(int* a, int n, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i0 = 2 * threadIdx.x;
  const int v0 = i0 < n ? a[i0] : 0;
  const int v1 = i0 + 1 < n ? a[i0 + 1] : 0;
  const int t = v0 + v1;
  int inc = t;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += u;
  }
  __syncthreads();
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  int wofs = 0, total = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) wofs += red[w];
    total += red[w];
  }
  const int ex = wofs + inc - t;
  if (i0 < n) a[i0] = ex;
  if (i0 + 1 < n) a[i0 + 1] = ex + v0;
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kThreads) build_tree_kernel(TreeParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ VP s_red_vp[kThreads / 32];
  __shared__ int s_red_i[kThreads / 32];
  __shared__ double s_red_d[kThreads / 32];
  __shared__ int s_lvl[DDT_TREE_L_MAX + 2];

  const int b = blockIdx.x, tid = threadIdx.x;
  const int L = p.L, k = p.k, NM = p.n_max;

  Smem s;
  s.L = L;
  s.k = k;
  {
    unsigned char* q = smem_raw;
    auto take = [&](size_t bytes) {
      unsigned char* r = q;
      q += (bytes + 15) & ~(size_t)15;
      return r;
    };
    s.S = (double*)take(sizeof(double) * (L + 1));
    s.nsz = (double*)take(sizeof(double) * NM);
    s.nsc = (double*)take(sizeof(double) * NM);
    s.zt = (float*)take(sizeof(float) * L * k);
    s.tt = (int*)take(sizeof(int) * L * k);
    s.npar = (int*)take(sizeof(int) * NM);
    s.ndep = (int*)take(sizeof(int) * NM);
    s.nrank = (int*)take(sizeof(int) * NM);
    s.nnext = (int*)take(sizeof(int) * NM);
    s.ncnt = (int*)take(sizeof(int) * NM);
    s.noff = (int*)take(sizeof(int) * NM);
    s.ninv = (int*)take(sizeof(int) * NM);
    s.safe = (uint32_t*)take(sizeof(uint32_t) * kSafeCap);
  }
  const double inv_t = p.inv_t;

  // per-sequence candidate count and budget (clamped, flagged)
  int kb = p.k_per_seq ? p.k_per_seq[b] : k;
  int Bb = p.budget ? p.budget[b] : p.B_max;
  if (kb < 1 || kb > k || Bb < 0 || Bb > p.B_max) {
    if (tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    kb = min(max(kb, 1), k);
    Bb = min(max(Bb, 0), p.B_max);
  }

  for (int i = tid; i < L * k; i += kThreads) {
    s.zt[i] = p.zk[(int64_t)b * L * k + i];
    s.tt[i] = p.ids[(int64_t)b * L * k + i];
  }
  if (tid == 0) {
    double acc = 0.0;
    s.S[0] = 0.0;
    for (int t = 1; t <= L; ++t) {
      acc = __dadd_rn(acc, (double)p.lse[(int64_t)b * L + t - 1]);
      s.S[t] = acc;
    }
    s.nsz[0] = 0.0;
    s.nsc[0] = 0.0;
    s.npar[0] = -1;
    s.ndep[0] = 0;
    s.nrank[0] = 0;
    s.nnext[0] = 0;
  }
  __syncthreads();

  int nn = 1;       // nodes including the root
  int nsel = 0;     // draft nodes
  // ---------------- frontier rounds ----------------
#pragma unroll 1
  while (nsel < Bb) {
    // theta: the K-best first child of any run head
    VP th = no_vp();
    int has_head = 0;
    for (int x = tid; x < nn; x += kThreads) {
      const int d = s.ndep[x], r = s.nnext[x];
      if (d < L && r < kb) {
        has_head = 1;
        if (d + 1 < L) {
          VP c;
          c.base = x;
          c.r1 = r;
          c.r2 = 0;
          c.depth = d + 2;
          c.sz = __dadd_rn(__dadd_rn(s.nsz[x], (double)s.zt[d * k + r]),
                           (double)s.zt[(d + 1) * k + 0]);
          c.sc = score_of(s, inv_t, c.sz, c.depth);
          if (vp_before(s, c, th)) th = c;
        }
      }
    }
    if (!__syncthreads_or(has_head)) break;
    th = block_best(s, th, s_red_vp);

    // safe items per run: ranks n_next[x].. that precede theta
    for (int x = tid; x < nn; x += kThreads) {
      const int d = s.ndep[x];
      int c = 0;
      if (d < L) {
        for (int r = s.nnext[x]; r < kb; ++r) {
          if (!vp_before(s, make_item(s, inv_t, x, r), th)) break;
          ++c;
        }
      }
      s.ncnt[x] = c;
      s.noff[x] = c;
    }
    __syncthreads();
    int total = block_exscan(s.noff, nn, s_red_i);
    const int R = Bb - nsel;
    if (total == 0) {
      // Only reachable when a candidate scores above its parent (inputs whose
      // lse is below some inv_t*z): take the K-best run head so that every
      // round selects something and the loop ends.
      VP best = no_vp();
      int bx = -1;
      for (int x = tid; x < nn; x += kThreads)
        if (s.ndep[x] < L && s.nnext[x] < kb) {
          const VP v = make_item(s, inv_t, x, s.nnext[x]);
          if (vp_before(s, v, best)) best = v;
        }
      best = block_best(s, best, s_red_vp);
      bx = best.base;
      for (int x = tid; x < nn; x += kThreads) {
        s.ncnt[x] = (x == bx) ? 1 : 0;
        s.noff[x] = (x == bx) ? 1 : 0;
      }
      __syncthreads();
      total = block_exscan(s.noff, nn, s_red_i);
      if (tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    }
    if (total <= R) {
      for (int x = tid; x < nn; x += kThreads) {
        const int c = s.ncnt[x];
        const int r0 = s.nnext[x];
        for (int i = 0; i < c; ++i) {
          const int id = nn + s.noff[x] + i;
          const VP v = make_item(s, inv_t, x, r0 + i);
          s.nsz[id] = v.sz;
          s.nsc[id] = v.sc;
          s.npar[id] = x;
          s.ndep[id] = v.depth;
          s.nrank[id] = r0 + i;
          s.nnext[id] = 0;
        }
      }
      __syncthreads();
      for (int x = tid; x < nn; x += kThreads) s.nnext[x] += s.ncnt[x];
      __syncthreads();
      nn += total;
      nsel += total;
      continue;
    }

    // final round: keep the R K-best safe items
    for (int x = tid; x < nn; x += kThreads) {
      const int c = min(s.ncnt[x], R);
      s.noff[x] = c;
    }
    __syncthreads();
    const int m = block_exscan(s.noff, nn, s_red_i);
    if (m <= kSafeCap) {
      int npow = 1;
      while (npow < m) npow <<= 1;
      for (int x = tid; x < nn; x += kThreads) {
        const int c = min(s.ncnt[x], R);
        for (int i = 0; i < c; ++i) s.safe[s.noff[x] + i] = ((uint32_t)x << 8) | (uint32_t)(s.nnext[x] + i);
      }
      for (int i = m + tid; i < npow; i += kThreads) s.safe[i] = 0xFFFFFFFFu;
      __syncthreads();
      auto item = [&](uint32_t e) -> VP {
        if (e == 0xFFFFFFFFu) return no_vp();
        return make_item(s, inv_t, (int)(e >> 8), (int)(e & 0xFF));
      };
      for (int size = 2; size <= npow; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int i = tid; i < npow / 2; i += kThreads) {
            const int lo = 2 * i - (i & (stride - 1));
            const int hi = lo + stride;
            const bool up = (lo & size) == 0;
            const uint32_t ea = s.safe[lo], eb = s.safe[hi];
            const VP va = item(ea), vb = item(eb);
            const bool sw = up ? vp_before(s, vb, va) : vp_before(s, va, vb);
            if (sw) {
              s.safe[lo] = eb;
              s.safe[hi] = ea;
            }
          }
          __syncthreads();
        }
      }
      for (int i = tid; i < R; i += kThreads) {
        const uint32_t e = s.safe[i];
        const int x = (int)(e >> 8), r = (int)(e & 0xFF);
        const VP v = make_item(s, inv_t, x, r);
        const int id = nn + i;
        s.nsz[id] = v.sz;
        s.nsc[id] = v.sc;
        s.npar[id] = x;
        s.ndep[id] = v.depth;
        s.nrank[id] = r;
        s.nnext[id] = 0;
      }
      __syncthreads();
      for (int i = tid; i < R; i += kThreads) {
        const uint32_t e = s.safe[i];
        atomicMax(&s.nnext[e >> 8], (int)(e & 0xFF) + 1);
      }
      __syncthreads();
    } else {
      // very large final round: take the K-best safe head, R times
      for (int x = tid; x < nn; x += kThreads) s.noff[x] = 0;  // taken per run
      __syncthreads();
      for (int i = 0; i < R; ++i) {
        VP best = no_vp();
        for (int x = tid; x < nn; x += kThreads)
          if (s.noff[x] < s.ncnt[x]) {
            const VP v = make_item(s, inv_t, x, s.nnext[x]);
            if (vp_before(s, v, best)) best = v;
          }
        best = block_best(s, best, s_red_vp);
        if (tid == 0) {
          const int id = nn + i;
          s.nsz[id] = best.sz;
          s.nsc[id] = best.sc;
          s.npar[id] = best.base;
          s.ndep[id] = best.depth;
          s.nrank[id] = best.r1;
          s.nnext[id] = 0;
          s.nnext[best.base] += 1;
          s.noff[best.base] += 1;
        }
        __syncthreads();
      }
    }
    nn += R;
    nsel += R;
    break;
  }

  // ---------------- breadth-first numbering ----------------
  if (tid < DDT_TREE_L_MAX + 2) s_lvl[tid] = 0;
  __syncthreads();
  int maxd = 0;
  for (int x = tid; x < nn; x += kThreads) {
    atomicAdd(&s_lvl[s.ndep[x]], 1);
    maxd = max(maxd, s.ndep[x]);
  }
  __syncthreads();
  if (tid == 0) {  // s_lvl[t] <- number of nodes of depth < t
    int acc = 0;
    for (int t = 0; t <= L + 1; ++t) {
      const int c = s_lvl[t];
      s_lvl[t] = acc;
      acc += c;
    }
  }
  maxd = __reduce_max_sync(0xFFFFFFFFu, maxd);
  if ((tid & 31) == 0) s_red_i[tid >> 5] = maxd;
  __syncthreads();
  maxd = 0;
  for (int w = 0; w < kThreads / 32; ++w) maxd = max(maxd, s_red_i[w]);
  __syncthreads();
  if (tid == 0) {
    s.ncnt[0] = 0;   // BFS index of the root
    s.noff[0] = 1;   // first child of the root
    s.ninv[0] = 0;
  }
  __syncthreads();
  for (int t = 1; t <= maxd; ++t) {
    const int lstart = s_lvl[t], lend = s_lvl[t + 1];
    // BFS index of level-t nodes; stage their child counts in BFS order
    for (int x = tid; x < nn; x += kThreads)
      if (s.ndep[x] == t) {
        const int j = s.noff[s.npar[x]] + s.nrank[x];
        s.ncnt[x] = j;
        s.ninv[j] = x;
      }
    __syncthreads();
    // first-child index of each level-t node: exclusive scan of child counts
    int* tmp = (int*)s.safe;
    for (int j = lstart + tid; j < lend; j += kThreads) tmp[j - lstart] = s.nnext[s.ninv[j]];
    __syncthreads();
    // levels can exceed 2*kThreads rows only when n_max > 1024 (not allowed)
    block_exscan(tmp, lend - lstart, s_red_i);
    for (int j = lstart + tid; j < lend; j += kThreads) s.noff[s.ninv[j]] = lend + tmp[j - lstart];
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
      o_par[j] = x == 0 ? -1 : s.ncnt[s.npar[x]];
      o_dep[j] = d;
      o_pos[j] = ctx + d;
    } else {
      o_tok[j] = -1;
      o_par[j] = -1;
      o_dep[j] = -1;
      o_pos[j] = -1;
    }
  }
  const int W = p.W;
  uint32_t* o_mask = p.mask + (int64_t)b * NM * W;
  for (int i = tid; i < NM * W; i += kThreads) {
    const int j = i / W, w = i - j * W;
    uint32_t word = 0;
    if (j < nn && w <= (j >> 5)) {
      for (int x = s.ninv[j]; x >= 0; x = s.npar[x]) {
        const int a = s.ncnt[x];
        if (a < 32 * w) break;
        if ((a >> 5) == w) word |= 1u << (a & 31);
      }
    }
    o_mask[i] = word;
  }
  // surrogate: sum of exp(score) over the draft nodes
  double acc = 0.0;
  for (int x = 1 + tid; x < nn; x += kThreads) acc += exp(s.nsc[x]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((tid & 31) == 0) s_red_d[tid >> 5] = acc;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) t += s_red_d[w];
    p.n_nodes[b] = nn;
    if (p.surrogate) p.surrogate[b] = t;
  }
}

size_t tree_smem_bytes(int L, int k, int n_max) {
  auto a = [](size_t x) { return (x + 15) & ~(size_t)15; };
  return a(sizeof(double) * (L + 1)) + 2 * a(sizeof(double) * n_max) + a(sizeof(float) * L * k) +
         a(sizeof(int) * L * k) + 7 * a(sizeof(int) * n_max) + a(sizeof(uint32_t) * kSafeCap);
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
  const size_t smem = tree_smem_bytes(L, k, p.n_max);
  if (ensure_smem_attr((const void*)build_tree_kernel, smem) != cudaSuccess) return DDT_ERR_CUDA;
  build_tree_kernel<<<batch, kThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
