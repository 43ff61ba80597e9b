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
  int32_t* status;
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

template <bool BF16>
__global__ void __launch_bounds__(kThreads) walk_kernel(WalkParams p) {
  constexpr int EPV = Chunk<BF16>::EPV;
  constexpr int ES = BF16 ? 2 : 4;
  __shared__ uint64_t s_red[kThreads / 32];
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
  if (j >= n) return;
  const int64_t row = (int64_t)b * p.n_max + j;
  const char* rowp = (const char*)p.logits + row * p.row_stride * ES;
  const int c0 = chunk * kChunk;

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
      __threadfence();
      s_flag = (atomicAdd(&p.row_ticket[row], 1u) == (unsigned)(p.S - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
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
  // the row is done; the last row of the sequence walks it
  if (tid == 0) {
    __threadfence();
    s_flag = (atomicAdd(&p.seq_count[b], 1u) == (unsigned)(n - 1));
  }
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
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

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

size_t walk_workspace_size(int batch, int n_max, int V) {
  const int S = (V + kChunk - 1) / kChunk;
  const size_t rows = (size_t)batch * n_max;
  return (size_t)DDT_WS_COUNTER_BYTES + align256(sizeof(int32_t) * rows) +
         align256(sizeof(uint64_t) * rows * S);
}

ddt_status launch_tree_walk(const void* logits, ddt_dtype dt, int batch, int n_max, int V,
                            int64_t row_stride, const int32_t* tok, const int32_t* parent,
                            const int32_t* depth, const int32_t* n_nodes, int L, int32_t* acc_len,
                            int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus, void* ws,
                            int32_t* dev_status, cudaStream_t stream) {
  WalkParams p;
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
  w += DDT_WS_COUNTER_BYTES;
  p.amax = (int32_t*)w;
  w += align256(sizeof(int32_t) * rows);
  p.part = (uint64_t*)w;
  if (batch == 0) return DDT_OK;
  dim3 grid(p.S, n_max, batch);
  const cudaError_t e = dt == DDT_BF16 ? launch_pdl(walk_kernel<true>, grid, dim3(kThreads), 0, stream, 0, p)
                                      : launch_pdl(walk_kernel<false>, grid, dim3(kThreads), 0, stream, 0, p);
  return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
