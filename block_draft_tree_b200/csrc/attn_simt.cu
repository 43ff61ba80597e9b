// attn_simt.cu -- stage 3 of the verification round, CUDA-core path.
//
// DDTree page, section 核心創新 third bullet and 運作流程 step 3: the target
// scores every tree row in one pass; a row attends to the committed context
// and to its own ancestors (and itself) only.
//
// This path serves trees with few query rows per kv head (rows * (hq/hkv)
// below a tensor-core tile) and is the reference layout for the tensor-core
// path: split-KV flash decoding.
//   * query rows of one kv head are (tree row j, head-in-group hh), row index
//     j*g + hh, in tiles of 32; grid = (row tiles, KV splits, batch*hkv);
//   * each CTA streams its context range (dense or paged) and, in the last
//     split, the tree's own K/V under the ancestor bitset, through shared
//     memory in tiles of 64 tokens, with an online softmax in base 2;
//   * per-split partials (unnormalised O, running max, running sum) go to
//     the workspace; the last split of a row tile (atomic ticket, no wait)
//     combines them with the usual log-sum-exp weights and writes bf16.
#include "attn_common.cuh"
#include "common.cuh"
#include "launch.h"

namespace ddt {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 32;   // query rows per CTA (8 warps x 4 rows)
constexpr int kTok = 64;    // KV tokens per shared-memory tile

template <int D>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnParams p) {
  constexpr int DV = D / 32;  // output dims per lane
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Qs = (float*)smem_raw;           // [kRows][D], pre-scaled by scale*log2(e)
  float* Ks = Qs + kRows * D;             // [kTok][D+1]
  float* Vs = Ks + kTok * (D + 1);        // [kTok][D]
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rt = blockIdx.x, split = blockIdx.y;
  const int b = blockIdx.z / p.hkv, kvh = blockIdx.z % p.hkv;
  pdl_wait();
  const int g = p.g;
  const int R = p.n_max * g;
  int n = p.n_nodes[b];
  n = min(max(n, 1), p.n_max);
  int T = p.ctx_len[b];
  if (T < 0 || T > p.max_ctx) {
    if (rt == 0 && split == 0 && kvh == 0 && tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    T = min(max(T, 0), p.max_ctx);
  }
  const int t_begin = min(split * p.tok_per_split, T);
  const int t_end = min(t_begin + p.tok_per_split, T);
  const bool last_split = (split == p.nsplit - 1);
  const int n_tree = last_split ? n : 0;

  // query tile
  for (int i = tid; i < kRows * D; i += kThreads) {
    const int r = i / D, e = i % D;
    const int qr = rt * kRows + r;
    float v = 0.f;
    if (qr < R) {
      const int j = qr / g, h = kvh * g + qr % g;
      if (j < n) v = bf16_to_f32(p.q[(((int64_t)b * p.n_max + j) * p.hq + h) * D + e]) * p.scale_log2;
    }
    Qs[i] = v;
  }

  float o[4][DV];
  float m[4], l[4];
  int jrow[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
    const int qr = rt * kRows + warp * 4 + r;
    jrow[r] = (qr < R && qr / g < n) ? qr / g : -1;
#pragma unroll
    for (int i = 0; i < DV; ++i) o[r][i] = 0.f;
  }

  const int n_ctx_tiles = (t_end - t_begin + kTok - 1) / kTok;
  const int n_tree_tiles = (n_tree + kTok - 1) / kTok;
  for (int tile = 0; tile < n_ctx_tiles + n_tree_tiles; ++tile) {
    const bool is_tree = tile >= n_ctx_tiles;
    const int base = is_tree ? (tile - n_ctx_tiles) * kTok : t_begin + tile * kTok;
    const int cnt = is_tree ? min(kTok, n_tree - base) : min(kTok, t_end - base);
    __syncthreads();
    for (int i = tid; i < kTok * (D / 8); i += kThreads) {
      const int t = i / (D / 8), e8 = (i % (D / 8)) * 8;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (t < cnt) {
        const uint16_t *kp, *vp;
        if (is_tree) {
          const int64_t off = (((int64_t)b * p.n_max + base + t) * p.hkv + kvh) * D + e8;
          kp = p.kt + off;
          vp = p.vt + off;
        } else {
          const int64_t off = (kv_row(p, b, base + t) * p.hkv + kvh) * D + e8;
          kp = p.kc + off;
          vp = p.vc + off;
        }
        kv = *(const uint4*)kp;
        vv = *(const uint4*)vp;
      }
      const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        Ks[t * (D + 1) + e8 + 2 * q] = bf16_lo(kw[q]);
        Ks[t * (D + 1) + e8 + 2 * q + 1] = bf16_hi(kw[q]);
        Vs[t * D + e8 + 2 * q] = bf16_lo(vw[q]);
        Vs[t * D + e8 + 2 * q + 1] = bf16_hi(vw[q]);
      }
    }
    __syncthreads();

    // scores: this lane's tokens lane and lane+32 for the warp's 4 rows
    float sc[4][2];
#pragma unroll
    for (int r = 0; r < 4; ++r) sc[r][0] = sc[r][1] = 0.f;
    const float* q0 = Qs + (warp * 4) * D;
#pragma unroll 4
    for (int e = 0; e < D; ++e) {
      const float k0 = Ks[lane * (D + 1) + e], k1 = Ks[(lane + 32) * (D + 1) + e];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float qv = q0[r * D + e];
        sc[r][0] = fmaf(qv, k0, sc[r][0]);
        sc[r][1] = fmaf(qv, k1, sc[r][1]);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = lane + 32 * u;
        bool vis = t < cnt && jrow[r] >= 0;
        if (vis && is_tree) {
          const int i = base + t;
          vis = (p.mask[((int64_t)b * p.n_max + jrow[r]) * p.W + (i >> 5)] >> (i & 31)) & 1u;
        }
        if (!vis) sc[r][u] = -INFINITY;
      }
      float tmax = fmaxf(sc[r][0], sc[r][1]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, off));
      const float mnew = fmaxf(m[r], tmax);
      float pr0 = 0.f, pr1 = 0.f, alpha = 1.f;
      if (mnew != -INFINITY) {
        alpha = ex2(m[r] - mnew);  // m = -inf -> 0
        pr0 = ex2(sc[r][0] - mnew);
        pr1 = ex2(sc[r][1] - mnew);
      }
      float ps = pr0 + pr1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, off);
      l[r] = l[r] * alpha + ps;
      m[r] = mnew;
#pragma unroll
      for (int i = 0; i < DV; ++i) o[r][i] *= alpha;
      sc[r][0] = pr0;
      sc[r][1] = pr1;
    }
    // O += P V
#pragma unroll 4
    for (int t = 0; t < kTok; ++t) {
      float vv[DV];
#pragma unroll
      for (int i = 0; i < DV; ++i) vv[i] = Vs[t * D + lane + 32 * i];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float pt = __shfl_sync(0xFFFFFFFFu, sc[r][t >> 5], t & 31);
#pragma unroll
        for (int i = 0; i < DV; ++i) o[r][i] = fmaf(pt, vv[i], o[r][i]);
      }
    }
  }

  // publish or finish
  const int64_t grp = (int64_t)b * p.hkv + kvh;
  if (p.nsplit == 1) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int qr = rt * kRows + warp * 4 + r;
      if (qr < R) write_row_final<DV>(p, b, kvh, qr, o[r], m[r], l[r], lane);
    }
    return;
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int qr = rt * kRows + warp * 4 + r;
    if (qr >= R) continue;
    float* po = p.part_o + ((grp * p.nsplit + split) * R + qr) * D;
#pragma unroll
    for (int i = 0; i < DV; ++i) po[lane + 32 * i] = o[r][i];
    if (lane == 0) p.part_ml[(grp * p.nsplit + split) * R + qr] = make_float2(m[r], l[r]);
  }
  pdl_trigger();
  __threadfence();
  __syncthreads();
  if (tid == 0)
    s_last = (atomicAdd(&p.tickets[grp * p.row_tiles + rt], 1u) == (unsigned)(p.nsplit - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int qr = rt * kRows + warp * 4 + r;
    if (qr < R) combine_row<DV>(p, grp, b, kvh, qr, lane);
  }
  if (tid == 0) p.tickets[grp * p.row_tiles + rt] = 0u;  // the counter region is left zero
}

}  // namespace

size_t attn_simt_smem(int d) { return sizeof(float) * (kRows * d + kTok * (d + 1) + kTok * d); }
int attn_simt_rows_per_cta() { return kRows; }

ddt_status launch_attn_simt(AttnParams& p, cudaStream_t stream) {
  const size_t smem = attn_simt_smem(p.d);
  dim3 grid(p.row_tiles, p.nsplit, p.batch * p.hkv);
  if (p.d == 128) {
    if (ensure_smem_attr((const void*)attn_simt_kernel<128>, smem) != cudaSuccess) return DDT_ERR_CUDA;
    return launch_pdl(attn_simt_kernel<128>, grid, dim3(kThreads), smem, stream, 0, p) == cudaSuccess
               ? DDT_OK
               : DDT_ERR_CUDA;
  }
  if (ensure_smem_attr((const void*)attn_simt_kernel<64>, smem) != cudaSuccess) return DDT_ERR_CUDA;
  return launch_pdl(attn_simt_kernel<64>, grid, dim3(kThreads), smem, stream, 0, p) == cudaSuccess
             ? DDT_OK
             : DDT_ERR_CUDA;
}

}  // namespace ddt
