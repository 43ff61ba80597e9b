// attn_tc.cu -- stage 3 of the verification round on the 5th-generation tensor
// cores: tcgen05 MMAs with TMEM accumulators, K/V tiles staged by TMA.
//
// DDTree page, section 核心創新 third bullet and 運作流程 step 3: the target
// scores every tree row in one pass; each row attends to the committed
// context and to its own ancestors (and itself) only.
//
// Once the tree has N*g >= 64 query rows per kv head (g = hq/hkv) the
// attention is a dense contraction Q[rows x d] K^T[d x tokens] followed by
// P[rows x tokens] V[tokens x d], so it runs as tiles of 128 query rows x 128
// tokens (d = 128):
//   * grid = (query tiles, KV splits, batch*hkv); one CTA per SM (TMEM: 512
//     columns = S double buffer 2x128, O 128, P 64; smem 224 KB: Q + a 3-deep K/V ring);
//   * warp 0 issues TMA loads (Q once; K and V per token tile, 128B-swizzled,
//     dense rows, 64-token pages, or the tree's own rows), warp 1 issues the
//     MMAs from one thread, warps 2-9 are the softmax: two warps per TMEM lane
//     quarter (one query row per lane), 64 score columns each;
//   * S = Q K^T lands in TMEM; the softmax warps read it, apply the
//     context-length / ancestor-bitset mask, keep a base-2 running max that
//     only moves (and rescales O) when it grows by more than 2^8, write
//     P = 2^(S - m) as bf16 back into TMEM, and the MMA warp computes
//     O += P V with P as the TMEM-resident A operand and V as an MN-major
//     shared-memory B operand;
//   * with one split the CTA normalises and writes bf16 rows; with several
//     the splits of a query tile merge on chip as one cluster, or write
//     (O, m, l) partials that a second kernel merges.
// Every mbarrier wait is bounded (about one second); a wait that gives up
// raises DDT_ERR_TIMEOUT in the status word and the CTA stops issuing work,
// lets its loads and MMAs in flight complete (bounded too), frees TMEM and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "attn_common.cuh"
#include "common.cuh"
#include "launch.h"
#include "tcgen05.cuh"

namespace ddt {
namespace tc {

constexpr int BM = 128;                   // query rows per tile (MMA M)
constexpr int BN = 128;                   // tokens per tile (MMA N of QK^T, K of PV)
constexpr int D = 128;                    // head dim
constexpr int kStages = 3;                // K/V ring depth
constexpr int kThreads = 320;             // warp 0 TMA, warp 1 MMA, warps 2-9 softmax
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP = 384;
constexpr uint32_t kColX = 448;  // exchange columns of the softmax warp pairs
constexpr int kHalf = BN * 128;           // one 64-wide d half: 128 rows x 128 B
constexpr int kTile = 2 * kHalf;          // 32 KB
constexpr float kRescaleLog2 = 8.f;       // move the running max only when it grows by > 2^8

struct Params {
  int batch, n_max, hq, hkv, g, W, max_ctx;
  int paged, page_size, max_pages, rows_per_box, boxes_per_tile;
  int64_t t_max;
  float scale_log2;
  const int32_t* ctx_len;
  const int32_t* n_nodes;
  const uint32_t* mask;
  const int32_t* page_table;
  uint16_t* out;
  float* lse_out;
  int32_t* status;
  int nsplit, tiles_per_split, qtiles;
  int cluster;      // the splits of a query tile form a cluster and merge on chip
  float* part_o;    // [grp][qtile][split][BM][D] (split partials without a cluster)
  float2* part_ml;  // [grp][qtile][split][BM]
  long long wait_cycles;  // bound of every mbarrier wait
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t drain;  // after a wait gave up: completion of every MMA issued
  long long wait_cycles;
  uint32_t tmem_base;
  int abort;
};

// ---------------------------------------------------------------- PTX helpers
// (the shared tcgen05 / TMA / mbarrier wrappers are in tcgen05.cuh)
// Bounded wait: false (and the CTA-wide abort flag set) if the phase does not
// complete within the launch's wait bound or another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, Bars* bars) {
  return mbar_wait_bounded(b, parity, &bars->abort, bars->wait_cycles);
}
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// AND of `pred` over a softmax warp pair (through a spare TMEM column).
__device__ __forceinline__ bool __syncthreads_and_pair(bool pred, int bar_id, uint32_t taddr, int half) {
  const bool w = __all_sync(0xFFFFFFFFu, pred);
  tmem_st1(taddr + half, w ? 1u : 0u);
  tmem_st_wait();
  fence_before();
  named_bar_sync(bar_id, 64);
  fence_after();
  return w && tmem_ld1(taddr + (half ^ 1)) != 0u;
}

// Distributed shared memory of the cluster (the KV splits of one query tile).
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ float2 ld_cluster_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}


// 2^x for a packed pair on the FMA pipe, to relieve the MUFU pipe in the
// softmax.  Cody-Waite reduction: n = rint(x) from the 1.5*2^23 rounding
// constant, f = x - n in [-1/2, 1/2]; 2^f from a cubic fitted here by least
// squares to 2^f at 256 Chebyshev nodes of [-1/2, 1/2] with relative
// weighting (largest relative error 7.8e-5 in fp32, far below the bf16
// rounding of P); 2^n added to the exponent field.  x <= 8 here (the running
// maximum lags the true one by at most 2^8); x below -126 is raised to -126:
// masked scores give 2^-126, far below the output's precision.
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& a, float& b) {
  float xa, xb;
  unpack2(x2, xa, xb);
  const uint64_t xx = pack2(fmaxf(xa, -126.f), fmaxf(xb, -126.f));
  const uint64_t t2 = fadd2(xx, pack2(12582912.f, 12582912.f));
  const uint64_t f2 = ffma2(fadd2(t2, pack2(-12582912.f, -12582912.f)), pack2(-1.f, -1.f), xx);
  uint64_t q2 = ffma2(pack2(5.508868396e-02f, 5.508868396e-02f), f2, pack2(2.426040471e-01f, 2.426040471e-01f));
  q2 = ffma2(q2, f2, pack2(6.932762265e-01f, 6.932762265e-01f));
  q2 = ffma2(q2, f2, pack2(9.999289513e-01f, 9.999289513e-01f));
  float ta, tb, qa, qb;
  unpack2(t2, ta, tb);
  unpack2(q2, qa, qb);
  a = __int_as_float(__float_as_int(qa) + ((__float_as_int(ta) - 0x4B400000) << 23));
  b = __int_as_float(__float_as_int(qb) + ((__float_as_int(tb) - 0x4B400000) << 23));
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, M = 128, N = 128,
// A K-major; B K-major (QK^T) or MN-major (PV).
__host__ __device__ constexpr uint32_t idesc_bf16(bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

struct TileInfo {
  int tree;   // 0: context tile, 1: tree tile
  int base;   // first token (context position or tree row)
  int cnt;    // valid tokens in the tile
};

__device__ __forceinline__ TileInfo tile_info(int t, int nct, int T, int n) {
  TileInfo ti;
  if (t < nct) {
    ti.tree = 0;
    ti.base = t * BN;
    ti.cnt = min(BN, T - ti.base);
  } else {
    ti.tree = 1;
    ti.base = (t - nct) * BN;
    ti.cnt = min(BN, n - ti.base);
  }
  return ti;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
                   const __grid_constant__ CUtensorMap tm_vt, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* sQ = smem;                              // [2][128][128 B]
  unsigned char* sK = smem + kTile;                      // [kStages][2][128][128 B]
  unsigned char* sV = sK + kStages * kTile;              // [kStages][2][128][128 B]
  Bars* bars = (Bars*)(sV + kStages * kTile);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qtile = blockIdx.x, split = blockIdx.y, grp = blockIdx.z;
  const int b = grp / p.hkv, kvh = grp % p.hkv;

  // set-up that reads no input runs before the wait for the previous kernel
  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->p_full, 256);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->drain, 1);
    bars->wait_cycles = p.wait_cycles;
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_kt);
      prefetch_tmap(&tm_vt);
    }
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();
  const int g = p.g;
  const int R = p.n_max * g;
  const int q0 = qtile * BM;
  int n = p.n_nodes[b];
  n = min(max(n, 1), p.n_max);
  int T = p.ctx_len[b];
  if (T < 0 || T > p.max_ctx) {
    if (qtile == 0 && split == 0 && kvh == 0 && tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    T = min(max(T, 0), p.max_ctx);
  }
  const int nct = (T + BN - 1) / BN;
  const int ntt = (n + BN - 1) / BN;
  const int t_lo = min(split * p.tiles_per_split, nct + ntt);
  const int t_hi = min(t_lo + p.tiles_per_split, nct + ntt);
  const int ntiles = t_hi - t_lo;
  const int64_t part_row0 = (((int64_t)grp * p.qtiles + qtile) * p.nsplit + split) * BM;

  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bars->tmem_base;

  // nothing to compute: an empty split, or a tile whose rows are all past
  // n_nodes (zero rows, written once: by split 0 of a cluster)
  const bool dead = q0 / g >= n;
  if ((ntiles == 0 && !p.cluster) || dead) {
    if (tid >= 64 && tid < 64 + BM && !(p.cluster && split != 0)) {
      const int row = tid - 64;
      const int qr = q0 + row;
      if (p.nsplit > 1 && !p.cluster) {
        // an empty partial (m = -inf: the combine never reads its O) for the
        // tree's rows; the combine writes rows past the tree by itself
        if (qr < R && qr / g < n) p.part_ml[part_row0 + row] = make_float2(-INFINITY, 0.f);
      } else if (qr < R) {
        const int j = qr / g, h = kvh * g + qr % g;
        uint4* dst = (uint4*)(p.out + (((int64_t)b * p.n_max + j) * p.hq + h) * D);
        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        if (p.lse_out) p.lse_out[((int64_t)b * p.n_max + j) * p.hq + h] = -INFINITY;
      }
    }
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                   : "memory");
    return;
  }

  const bool work = ntiles > 0;

  if (!work) {
    // an empty split of a cluster: nothing to compute, an empty partial below
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int j0 = q0 / g;
      mbar_expect_tx(&bars->q_full, (uint32_t)kTile);
      tma_load_3d(sQ, &tm_q, 0, kvh * g, b * p.n_max + j0, &bars->q_full);
      tma_load_3d(sQ + kHalf, &tm_q, 64, kvh * g, b * p.n_max + j0, &bars->q_full);
      int issued = 0;  // K/V tiles whose loads were issued
      for (int i = 0; i < ntiles; ++i, issued = i) {
        const int s = i % kStages;
        const uint32_t ph = (uint32_t)(i / kStages) & 1u;
        if (!mbar_wait(&bars->kv_empty[s], ph ^ 1u, bars)) break;
        const TileInfo ti = tile_info(t_lo + i, nct, T, n);
        unsigned char* k_dst = sK + s * kTile;
        unsigned char* v_dst = sV + s * kTile;
        if (ti.tree) {
          const int row = b * p.n_max + ti.base;
          mbar_expect_tx(&bars->kv_full[s], (uint32_t)(2 * kTile));
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(k_dst + h * kHalf, &tm_kt, 64 * h, kvh, row, &bars->kv_full[s]);
            tma_load_3d(v_dst + h * kHalf, &tm_vt, 64 * h, kvh, row, &bars->kv_full[s]);
          }
        } else if (!p.paged) {
          const int row = (int)((int64_t)b * p.t_max + ti.base);
          mbar_expect_tx(&bars->kv_full[s], (uint32_t)(2 * kTile));
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(k_dst + h * kHalf, &tm_k, 64 * h, kvh, row, &bars->kv_full[s]);
            tma_load_3d(v_dst + h * kHalf, &tm_v, 64 * h, kvh, row, &bars->kv_full[s]);
          }
        } else {
          // boxes of rows_per_box tokens; boxes past the context are not loaded
          const int rpb = p.rows_per_box;
          int nbox = 0;
          for (int bx = 0; bx < p.boxes_per_tile; ++bx)
            if (ti.base + bx * rpb < T) ++nbox;
          mbar_expect_tx(&bars->kv_full[s], (uint32_t)(nbox * rpb * 128 * 2 * 2));
          for (int bx = 0; bx < nbox; ++bx) {
            const int tok = ti.base + bx * rpb;
            const int page = p.page_table[(int64_t)b * p.max_pages + tok / p.page_size];
            const int slot = tok % p.page_size;
            for (int h = 0; h < 2; ++h) {
              tma_load_4d(k_dst + h * kHalf + bx * rpb * 128, &tm_k, 64 * h, kvh, slot, page,
                          &bars->kv_full[s]);
              tma_load_4d(v_dst + h * kHalf + bx * rpb * 128, &tm_v, 64 * h, kvh, slot, page,
                          &bars->kv_full[s]);
            }
          }
        }
      }
      if (*(volatile int*)&bars->abort) {
        // a wait gave up: let the loads still in flight land before the CTA
        // (and its shared memory) goes away.  The Q tile and the last
        // kStages K/V tiles issued are the only ones that can be outstanding;
        // each of their stages has exactly one phase pending.
        int keep_going = 0;
        mbar_wait_bounded(&bars->q_full, 0u, &keep_going, kDrainCycles);
        for (int q = issued > kStages ? issued - kStages : 0; q < issued; ++q)
          mbar_wait_bounded(&bars->kv_full[q % kStages], (uint32_t)(q / kStages) & 1u, &keep_going,
                            kDrainCycles);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = idesc_bf16(false);
      constexpr uint32_t kIdPV = idesc_bf16(true);
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(&bars->q_full, 0, bars);
      for (int i = 0; ok && i <= ntiles; ++i) {
        if (i < ntiles) {
          const int s = i % kStages;
          if (!mbar_wait(&bars->kv_full[s], (uint32_t)(i / kStages) & 1u, bars)) break;
          fence_after();
          const uint32_t k_addr = smem_u32(sK + s * kTile);
          const uint32_t d_tm = tmem + ((i & 1) ? kColS1 : kColS0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)((kk >> 2) * kHalf + (kk & 3) * 32);
            mma_ss(d_tm, sdesc(q_addr + off, 16, 1024), sdesc(k_addr + off, 16, 1024), kIdQK,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full[i & 1]);
        }
        if (i > 0) {
          const int ip = i - 1;
          if (!mbar_wait(&bars->p_full, (uint32_t)ip & 1u, bars)) break;
          fence_after();
          const int sp = ip % kStages;
          const uint32_t v_addr = smem_u32(sV + sp * kTile);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ts(tmem + kColO, tmem + kColP + kk * 8, sdesc(v_addr + kk * 2048, kHalf, 1024), kIdPV,
                   (ip > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars->pv_done);
          mma_commit(&bars->kv_empty[sp]);
        }
      }
      if (*(volatile int*)&bars->abort) {
        // a wait gave up: every MMA issued completes before TMEM is freed
        int keep_going = 0;
        mma_commit(&bars->drain);
        mbar_wait_bounded(&bars->drain, 0u, &keep_going, kDrainCycles);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // Two warps per TMEM lane quarter: warp w serves rows 32*(w%4)..+31 and
    // the 64 score columns of half h = (w-2)/4.  The pair exchanges its row
    // maxima (and, at the end, row sums) through spare TMEM columns and a
    // 64-thread named barrier, every iteration, so the pair always meets the
    // same barriers, also after a bounded wait gave up.
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int qr = q0 + row;
    const int j = qr / g;
    const bool row_valid = qr < R && j < n;
    const uint32_t* mrow = p.mask + ((int64_t)b * p.n_max + (j < p.n_max ? j : 0)) * p.W;
    const int bar_id = 1 + quarter;
    const int c0 = half * (BN / 2);  // first score column of this half
    float m_used = -INFINITY, l = 0.f;
    uint32_t r[BN / 2];
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const TileInfo ti = tile_info(t_lo + i, nct, T, n);
      if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full[i & 1], (uint32_t)(i >> 1) & 1u, bars));
      float mx_raw = -INFINITY;
      const float c_log2 = p.scale_log2;
      if (ok) {
        fence_after();
        const uint32_t s_col = ((i & 1) ? kColS1 : kColS0) + c0;
        tmem_ld32(lane_base + s_col, r);
        tmem_ld32(lane_base + s_col + 32, r + 32);
        tmem_ld_wait();
        // Full context tiles need no masking; partial and tree tiles mask
        // with -inf, which the exp below turns into 0.
        const bool full_tile = !ti.tree && ti.cnt == BN && row_valid;
        if (!full_tile) {
          uint32_t mw[2] = {0u, 0u};
          if (ti.tree && row_valid) {
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const int word = ((ti.base + c0) >> 5) + w;
              mw[w] = word < p.W ? mrow[word] : 0u;
            }
          } else if (!ti.tree && row_valid) {
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const int lo = c0 + 32 * w;
              mw[w] = ti.cnt >= lo + 32 ? 0xFFFFFFFFu : (ti.cnt > lo ? ((1u << (ti.cnt - lo)) - 1u) : 0u);
            }
          }
#pragma unroll
          for (int c = 0; c < BN / 2; ++c)
            if (!((mw[c >> 5] >> (c & 31)) & 1u)) r[c] = 0xFF800000u;  // -inf
        }
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(r[e]);
#pragma unroll
        for (int c = 8; c < BN / 2; c += 2)
          mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
        mx_raw = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      }
      // exchange the half-row maxima (raw score domain; scale > 0 commutes with max)
      const uint32_t xcol = kColX + 2 * (i & 1);
      tmem_st1(lane_base + xcol + half, __float_as_uint(mx_raw));
      tmem_st_wait();
      fence_before();
      named_bar_sync(bar_id, 64);
      fence_after();
      const float other = __uint_as_float(tmem_ld1(lane_base + xcol + (half ^ 1)));
      if (!ok) continue;
      const float mx = fmaxf(mx_raw, other) * c_log2;
      const float m_new = fmaxf(m_used, mx);
      const bool move = m_new > m_used + kRescaleLog2 || (m_used == -INFINITY && m_new != -INFINITY);
      const float m_tgt = move ? m_new : m_used;
      uint64_t rs2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) rs2[e] = 0ull;  // (+0, +0)
      if (m_tgt == -INFINITY) {
#pragma unroll
        for (int c = 0; c < BN / 4; ++c) r[c] = 0u;
      } else {
        // p = 2^(s*c - m), two scores at a time: a packed FFMA for the
        // exponents, then MUFU ex2 -- or, for 3 pairs in 8, exp2_poly2 on the
        // FMA pipe, so that neither pipe waits on the other; packed sums;
        // bf16 pairs packed in place
        const uint64_t c2 = pack2(c_log2, c_log2), nm2 = pack2(-m_tgt, -m_tgt);
#pragma unroll
        for (int c = 0; c < BN / 2; c += 2) {
          const uint64_t x2 = ffma2(pack2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), c2, nm2);
          float a, bb;
          if (((c >> 1) & 7) < 3) {
            exp2_poly2(x2, a, bb);
          } else {
            float xa, xb;
            unpack2(x2, xa, xb);
            a = ex2(xa);
            bb = ex2(xb);
          }
          rs2[(c >> 1) & 3] = fadd2(rs2[(c >> 1) & 3], pack2(a, bb));
          __nv_bfloat162 pk = __floats2bfloat162_rn(a, bb);
          r[c >> 1] = *(uint32_t*)&pk;
        }
      }
      float rs8[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) unpack2(rs2[e], rs8[2 * e], rs8[2 * e + 1]);
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      // PV of the previous tile must be done before P and O are touched
      if (i > 0) {
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->pv_done, (uint32_t)(i - 1) & 1u, bars));
        if (!ok) continue;
      }
      fence_after();
      // rows whose maximum moved rescale O; the whole warp takes part in the
      // TMEM accesses (they are warp-collective), the other rows by 1
      const bool resc = move && i > 0 && m_used != -INFINITY;
      if (__any_sync(0xFFFFFFFFu, resc)) {
        const float alpha = resc ? ex2(m_used - m_new) : 1.f;
        uint32_t o[32];
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const uint32_t oc = kColO + half * (D / 2) + 32 * c;
          tmem_ld32(lane_base + oc, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_base + oc, o);
        }
        l *= alpha;
      }
      if (move) m_used = m_new;
      l += rs;
      tmem_st32(lane_base + kColP + half * (BN / 4), r);
      // token row `row` of a partial tile: zero its V row (this half's 64
      // dims) so that 0 * garbage cannot turn into NaN in the PV product
      if (row >= ti.cnt) {
        uint4* vrow = (uint4*)(sV + (i % kStages) * kTile + half * kHalf + row * 128);
#pragma unroll
        for (int e = 0; e < 8; ++e) vrow[e] = make_uint4(0, 0, 0, 0);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tmem_st_wait();
      fence_before();
      mbar_arrive(&bars->p_full);
    }
    if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->pv_done, (uint32_t)(ntiles - 1) & 1u, bars));
    // the row sum over both halves
    tmem_st1(lane_base + kColX + 4 + half, __float_as_uint(l));
    tmem_st_wait();
    fence_before();
    named_bar_sync(bar_id, 64);
    fence_after();
    const float l_row = l + __uint_as_float(tmem_ld1(lane_base + kColX + 4 + (half ^ 1)));
    const bool ok_row = __syncthreads_and_pair(ok, bar_id, lane_base + kColX + 6, half);
    // epilogue: this half's 64 dims of the O row -> final output, a cluster
    // partial in shared memory, or a partial in the workspace
    float* po = p.cluster ? (float*)(sK) + row * D : p.part_o + (part_row0 + row) * D;
    const bool final_out = p.nsplit == 1;
    const float inv = (l_row > 0.f) ? 1.f / l_row : 0.f;
    uint16_t* dst = nullptr;
    if (final_out && qr < R)
      dst = p.out + (((int64_t)b * p.n_max + j) * p.hq + (kvh * g + qr % g)) * D;
#pragma unroll
    for (int cc = 0; cc < D / 64; ++cc) {
      const int c = half * (D / 64) + cc;  // 32-column block of O
      uint32_t o[32];
      tmem_ld32(lane_base + kColO + 32 * c, o);
      tmem_ld_wait();
      if (!ok_row || !row_valid) {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (p.cluster) {
        // 16-byte chunk k of the row goes to slot k ^ (row & 31), so that the
        // 32 rows of a warp hit different banks
        float4* q4 = (float4*)po;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          q4[(8 * c + e) ^ (row & 31)] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                                     __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
      } else if (!final_out) {
        float4* q4 = (float4*)(po + 32 * c);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          q4[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                              __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
      } else if (dst) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                   __uint_as_float(o[2 * e + 1]) * inv);
          pk[e] = *(uint32_t*)&h2;
        }
        uint4* d4 = (uint4*)(dst + 32 * c);
#pragma unroll
        for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
    }
    const bool has = ok_row && row_valid && l_row > 0.f;
    if (half == 0) {
      if (p.cluster) {
        ((float2*)(sK + BM * D * 4))[row] = has ? make_float2(m_used, l_row) : make_float2(-INFINITY, 0.f);
      } else if (!final_out) {
        p.part_ml[part_row0 + row] = has ? make_float2(m_used, l_row) : make_float2(-INFINITY, 0.f);
      } else if (dst && p.lse_out) {
        p.lse_out[((int64_t)b * p.n_max + j) * p.hq + (kvh * g + qr % g)] =
            has ? (m_used + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  pdl_trigger();
  if (!work && tid >= 64 && tid < 64 + BM)  // empty split of a cluster
    ((float2*)(sK + BM * D * 4))[tid - 64] = make_float2(-INFINITY, 0.f);

  fence_before();
  __syncthreads();
  if (work && bars->abort && tid == 0) raise_status(p.status, DDT_ERR_TIMEOUT);
  if (warp == 0) {
    __syncwarp();
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
  if (!p.cluster) return;

  // ---------------- on-chip merge of the cluster's split partials ----------------
  // CTA r of the cluster owns query rows [r*rpc, (r+1)*rpc) of the tile; each
  // warp takes two rows at a time, a lane 4 of their 128 dims, and loads every
  // split's (m, l) and O slice of both from the peers' shared memory in one go
  // (O rows are stored with their 16-byte chunks XOR-swizzled by row).
  cluster_sync();
  {
    const int S = p.nsplit;  // 2..8
    const int rank = (int)cluster_rank();
    const int rpc = (BM + S - 1) / S;
    const uint32_t o_base = smem_u32(sK), ml_base = smem_u32(sK + BM * D * 4);
    const int r_end = min(min(BM, (rank + 1) * rpc), R - q0);
    for (int r0 = rank * rpc + 2 * warp; r0 < r_end; r0 += 2 * (kThreads / 32)) {
      // two rows: every split's (m, l) and O slice of both, loaded together
      float2 ml[2][8];
      float4 v[2][8];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int r = min(r0 + q, r_end - 1);
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < S) {
            ml[q][s2] = ld_cluster_f2(map_to_rank(ml_base + r * 8, s2));
            v[q][s2] = ld_cluster_f4(map_to_rank(o_base + (r * D + 4 * (lane ^ (r & 31))) * 4, s2));
          }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int r = r0 + q;
        if (r >= r_end) break;
        const int qr2 = q0 + r;
        const int j2 = qr2 / g, h2 = kvh * g + qr2 % g;
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < S) M = fmaxf(M, ml[q][s2].x);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float Lsum = 0.f;
        if (M != -INFINITY && j2 < n) {
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
            if (s2 < S && ml[q][s2].x != -INFINITY) {
              const float wgt = ex2(ml[q][s2].x - M);
              Lsum += ml[q][s2].y * wgt;
              acc.x = fmaf(wgt, v[q][s2].x, acc.x);
              acc.y = fmaf(wgt, v[q][s2].y, acc.y);
              acc.z = fmaf(wgt, v[q][s2].z, acc.z);
              acc.w = fmaf(wgt, v[q][s2].w, acc.w);
            }
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        uint2* dst2 = (uint2*)(p.out + (((int64_t)b * p.n_max + j2) * p.hq + h2) * D);
        dst2[lane] = make_uint2(*(uint32_t*)&h0, *(uint32_t*)&h1);
        if (lane == 0 && p.lse_out)
          p.lse_out[((int64_t)b * p.n_max + j2) * p.hq + h2] =
              Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
  cluster_sync();  // peers' shared memory stays alive until every CTA has read it
}

// ---------------------------------------------------------------------------
// Two query tiles per CTA
// ---------------------------------------------------------------------------
// Where a kv head has at least two query tiles, one CTA takes a pair of them
// (A and B: 256 query rows) over its KV range: every K/V tile is loaded once
// for both, so each byte staged feeds twice the MMA work, and the two tiles'
// softmax work overlaps the other tile's MMAs.  Warp 0 loads (Q_A and Q_B
// once; K_i and V_i into a ring of four 32 KB slots, two tiles ahead), warp 1
// issues the MMAs, warps 2-5 are tile A's softmax and warps 6-9 tile B's, one
// query row per thread (the thread's TMEM lane), all 128 scores of a tile
// in registers.  TMEM: S_A, S_B (128 columns each), O_A, O_B (128 each); a
// tile's P (bf16 pairs, 64 columns) overwrites the first half of its S.
// MMA order per KV tile i:  [P_A(i) ready] PV_A(i), QK_A(i+1);
// [P_B(i) ready] PV_B(i), QK_B(i+1): while one tile's softmax runs, the
// tensor cores work for the other.  A commit after QK_t(i+1) completes after
// PV_t(i) too (commits cover every earlier MMA of the thread), so the softmax
// of tile i+1 may rescale O_t without another wait.
constexpr int kPairThreads = 320;
constexpr uint32_t kColSA = 0, kColSB = 128, kColOA = 256, kColOB = 384;

struct __align__(8) PairBars {
  uint64_t q_full;
  uint64_t kv_full[4];
  uint64_t kv_empty[4];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full;
  uint64_t drain;
  long long wait_cycles;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool pair_wait(uint64_t* b, uint32_t parity, PairBars* bars) {
  return mbar_wait_bounded(b, parity, &bars->abort, bars->wait_cycles);
}

// Load the K (kind 0) or V (kind 1) rows of KV tile `ti` into `dst`.
__device__ __forceinline__ void pair_load_kv(const Params& p, const TileInfo& ti, int b, int kvh, int T,
                                             int kind, unsigned char* dst, uint64_t* bar,
                                             const CUtensorMap* tm_c, const CUtensorMap* tm_t) {
  if (ti.tree) {
    const int row = b * p.n_max + ti.base;
    mbar_expect_tx(bar, (uint32_t)kTile);
    for (int h = 0; h < 2; ++h) tma_load_3d(dst + h * kHalf, tm_t, 64 * h, kvh, row, bar);
  } else if (!p.paged) {
    const int row = (int)((int64_t)b * p.t_max + ti.base);
    mbar_expect_tx(bar, (uint32_t)kTile);
    for (int h = 0; h < 2; ++h) tma_load_3d(dst + h * kHalf, tm_c, 64 * h, kvh, row, bar);
  } else {
    const int rpb = p.rows_per_box;
    int nbox = 0;
    for (int bx = 0; bx < p.boxes_per_tile; ++bx)
      if (ti.base + bx * rpb < T) ++nbox;
    mbar_expect_tx(bar, (uint32_t)(nbox * rpb * 128 * 2));
    for (int bx = 0; bx < nbox; ++bx) {
      const int tok = ti.base + bx * rpb;
      const int page = p.page_table[(int64_t)b * p.max_pages + tok / p.page_size];
      const int slot = tok % p.page_size;
      for (int h = 0; h < 2; ++h)
        tma_load_4d(dst + h * kHalf + bx * rpb * 128, tm_c, 64 * h, kvh, slot, page, bar);
    }
  }
  (void)kind;
}

__global__ void __launch_bounds__(kPairThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
                     const __grid_constant__ CUtensorMap tm_vt, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* sQ = smem;                 // [2 tiles][2 halves][128][128 B]
  unsigned char* sKV = smem + 2 * kTile;    // [4 slots][2 halves][128][128 B]
  PairBars* bars = (PairBars*)(sKV + 4 * kTile);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.x, split = blockIdx.y, grp = blockIdx.z;
  const int b = grp / p.hkv, kvh = grp % p.hkv;
  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    bars->wait_cycles = p.wait_cycles;
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_kt);
      prefetch_tmap(&tm_vt);
    }
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();
  const int g = p.g;
  const int R = p.n_max * g;
  const int q0 = pair * 2 * BM;
  int n = p.n_nodes[b];
  n = min(max(n, 1), p.n_max);
  // tile B exists when it holds query rows; a tile works when one of its
  // rows belongs to a tree row (rows past n_nodes only get zeros)
  const bool a_work = q0 / g < n;
  const bool b_exists = q0 + BM < R;
  const bool has_b = b_exists && (q0 + BM) / g < n;
  int T = p.ctx_len[b];
  if (T < 0 || T > p.max_ctx) {
    if (pair == 0 && split == 0 && kvh == 0 && tid == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    T = min(max(T, 0), p.max_ctx);
  }
  const int nct = (T + BN - 1) / BN;
  const int ntt = (n + BN - 1) / BN;
  const int t_lo = min(split * p.tiles_per_split, nct + ntt);
  const int t_hi = min(t_lo + p.tiles_per_split, nct + ntt);
  const int ntiles = a_work ? t_hi - t_lo : 0;  // KV tiles this CTA processes

  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntiles > 0) {
      const int j0 = q0 / g;
      mbar_expect_tx(&bars->q_full, (uint32_t)((has_b ? 2 : 1) * kTile));
      for (int t = 0; t < (has_b ? 2 : 1); ++t)
        for (int h = 0; h < 2; ++h)
          tma_load_3d(sQ + t * kTile + h * kHalf, &tm_q, 64 * h, kvh * g, b * p.n_max + j0 + t * (BM / g),
                      &bars->q_full);
      int issued = 0;  // K/V loads issued (two per tile)
      for (int i = 0; i < ntiles; ++i) {
        const TileInfo ti = tile_info(t_lo + i, nct, T, n);
        bool ok = true;
        for (int kind = 0; kind < 2 && ok; ++kind) {
          const int s = (2 * i + kind) & 3;
          if (!pair_wait(&bars->kv_empty[s], ((uint32_t)(i >> 1) & 1u) ^ 1u, bars)) {
            ok = false;
            break;
          }
          pair_load_kv(p, ti, b, kvh, T, kind, sKV + s * kTile, &bars->kv_full[s],
                       kind ? &tm_v : &tm_k, kind ? &tm_vt : &tm_kt);
          ++issued;
        }
        if (!ok) break;
      }
      if (*(volatile int*)&bars->abort) {
        // a wait gave up: let the loads in flight land before the CTA (and
        // its shared memory) goes away; only the Q tiles and the last four
        // K/V loads can be outstanding, each on a slot with one phase pending
        int keep_going = 0;
        mbar_wait_bounded(&bars->q_full, 0u, &keep_going, kDrainCycles);
        for (int c = issued > 4 ? issued - 4 : 0; c < issued; ++c)
          mbar_wait_bounded(&bars->kv_full[c & 3], (uint32_t)(c >> 2) & 1u, &keep_going, kDrainCycles);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t kIdQK = idesc_bf16(false);
      constexpr uint32_t kIdPV = idesc_bf16(true);
      const int nt = has_b ? 2 : 1;
      auto qk = [&](int t, int i) {  // S_t = Q_t K_i^T
        const uint32_t q_addr = smem_u32(sQ + t * kTile);
        const uint32_t k_addr = smem_u32(sKV + ((2 * i) & 3) * kTile);
        const uint32_t d_tm = tmem + (t ? kColSB : kColSA);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kHalf + (kk & 3) * 32);
          mma_ss(d_tm, sdesc(q_addr + off, 16, 1024), sdesc(k_addr + off, 16, 1024), kIdQK,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[t]);
      };
      auto pv = [&](int t, int i) {  // O_t += P_t V_i, P_t in the first half of S_t
        const uint32_t v_addr = smem_u32(sKV + ((2 * i + 1) & 3) * kTile);
        const uint32_t s_col = t ? kColSB : kColSA, o_col = t ? kColOB : kColOA;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + o_col, tmem + s_col + kk * 8, sdesc(v_addr + kk * 2048, kHalf, 1024), kIdPV,
                 (i > 0 || kk > 0) ? 1u : 0u);
      };
      // Each K/V slot is released (a commit on its kv_empty) as soon as the
      // last MMA that reads it is issued: K_i after the QKs of step i - 1,
      // V_i after the PVs of step i, so the producer refills K slots a step
      // earlier than it could if both waited for the end of step i.
      bool ok = pair_wait(&bars->q_full, 0, bars) && pair_wait(&bars->kv_full[0], 0, bars);
      if (ok) {
        fence_after();
        for (int t = 0; t < nt; ++t) qk(t, 0);
        mma_commit(&bars->kv_empty[0]);  // K_0
      }
      for (int i = 0; ok && i < ntiles; ++i) {
        const int vs = (2 * i + 1) & 3;
        const uint32_t ph = (uint32_t)(i >> 1) & 1u;
        const bool next = i + 1 < ntiles;
        const int ks1 = (2 * i + 2) & 3;
        const uint32_t ph1 = (uint32_t)((i + 1) >> 1) & 1u;
        if (!pair_wait(&bars->kv_full[vs], ph, bars)) break;
        for (int t = 0; t < nt; ++t) {
          if (!pair_wait(&bars->p_full[t], (uint32_t)i & 1u, bars) ||
              (next && t == 0 && !pair_wait(&bars->kv_full[ks1], ph1, bars))) {
            ok = false;
            break;
          }
          fence_after();
          pv(t, i);
          if (next) qk(t, i + 1);
        }
        if (!ok) break;
        mma_commit(&bars->kv_empty[vs]);  // V_i: every PV of step i issued
        if (next) mma_commit(&bars->kv_empty[ks1]);  // K_{i+1}: every QK of step i + 1 issued
      }
      if (ok) mma_commit(&bars->o_full);
      if (*(volatile int*)&bars->abort) {
        int keep_going = 0;
        mma_commit(&bars->drain);
        mbar_wait_bounded(&bars->drain, 0u, &keep_going, kDrainCycles);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int t = (warp - 2) >> 2;         // tile 0 (A) or 1 (B)
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_col = t ? kColSB : kColSA, o_col = t ? kColOB : kColOA;
    const int qr = q0 + t * BM + row;
    const int j = qr / g;
    const bool tile_live = t == 0 || has_b;     // the tile has tree rows to compute
    const bool tile_rows = t == 0 || b_exists;  // the tile has query rows to write
    const bool row_valid = tile_live && qr < R && j < n;
    const uint32_t* mrow = p.mask + ((int64_t)b * p.n_max + (j < p.n_max ? j : 0)) * p.W;
    const float c_log2 = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; tile_live && i < ntiles; ++i) {
      const TileInfo ti = tile_info(t_lo + i, nct, T, n);
      if (ok) ok = __all_sync(0xFFFFFFFFu, pair_wait(&bars->s_full[t], (uint32_t)i & 1u, bars));
      if (!ok) break;
      fence_after();
      // the tile's mask words for this row (all ones for full context tiles)
      uint32_t mw[BN / 32];
      const bool masked = ti.tree || ti.cnt < BN || !row_valid;
#pragma unroll
      for (int w = 0; w < BN / 32; ++w) {
        mw[w] = 0xFFFFFFFFu;
        if (masked) {
          mw[w] = 0u;
          if (row_valid) {
            if (ti.tree) {
              const int word = (ti.base >> 5) + w;
              mw[w] = word < p.W ? mrow[word] : 0u;
            } else {
              const int lo = 32 * w;
              mw[w] = ti.cnt >= lo + 32 ? 0xFFFFFFFFu : (ti.cnt > lo ? ((1u << (ti.cnt - lo)) - 1u) : 0u);
            }
          }
        }
      }
      // the row's 128 scores in registers: four TMEM loads, one wait
      uint32_t r[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(lane_base + s_col + 32 * c, r + 32 * c);
      tmem_ld_wait();
      if (masked) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (!((mw[e >> 5] >> (e & 31)) & 1u)) r[e] = 0xFF800000u;  // -inf
      }
      // the row maximum (three-input max, four independent chains)
      float m4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) m4[e] = __uint_as_float(r[e]);
#pragma unroll
      for (int e = 4; e < BN; e += 2)
        m4[(e >> 1) & 3] = fmax3(m4[(e >> 1) & 3], __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c_log2;
      const float m_new = fmaxf(m_used, mx);
      const bool move = m_new > m_used + kRescaleLog2 || (m_used == -INFINITY && m_new != -INFINITY);
      const float m_tgt = move ? m_new : m_used;
      // p = 2^(s*c - m), two scores at a time: a packed FFMA for the
      // exponents, then MUFU ex2 -- or, for 2 pairs in 8, exp2_poly2 on the
      // FMA pipe; packed sums; bf16 pairs stored over the scores, 32 scores
      // (16 columns) per store
      uint64_t rs2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) rs2[e] = 0ull;
      const uint64_t c2 = pack2(c_log2, c_log2), nm2 = pack2(-m_tgt, -m_tgt);
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t pk[16];
        if (m_tgt == -INFINITY) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        } else {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t x2 = ffma2(pack2(__uint_as_float(r[32 * c + e]), __uint_as_float(r[32 * c + e + 1])),
                                      c2, nm2);
            float a, bb;
            if (((e >> 1) & 7) < 2) {
              exp2_poly2(x2, a, bb);
            } else {
              float xa, xb;
              unpack2(x2, xa, xb);
              a = ex2(xa);
              bb = ex2(xb);
            }
            rs2[(e >> 1) & 3] = fadd2(rs2[(e >> 1) & 3], pack2(a, bb));
            __nv_bfloat162 h2 = __floats2bfloat162_rn(a, bb);
            pk[e >> 1] = *(uint32_t*)&h2;
          }
        }
        tmem_st16(lane_base + s_col + 16 * c, pk);
      }
      float rs8[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) unpack2(rs2[e], rs8[2 * e], rs8[2 * e + 1]);
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      // O_t already holds PV_t(i-1) (complete: the commit behind s_full covers
      // it); rows whose maximum moved rescale it -- the whole warp takes part
      // in the TMEM accesses (they are warp-collective), the others by 1
      const bool resc = move && i > 0 && m_used != -INFINITY;
      if (__any_sync(0xFFFFFFFFu, resc)) {
        const float alpha = resc ? ex2(m_used - m_new) : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + o_col + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_base + o_col + 32 * c, o);
        }
        l *= alpha;
      }
      if (move) m_used = m_new;
      l += rs;
      // token row `row` of a partial KV tile: zero its V row (both halves)
      // so that 0 * garbage cannot turn into NaN in the PV product; tile A's
      // threads do it, once V_i has landed, before PV_A(i), which comes first
      if (t == 0 && ti.cnt < BN &&
          !__all_sync(0xFFFFFFFFu, pair_wait(&bars->kv_full[(2 * i + 1) & 3], (uint32_t)(i >> 1) & 1u, bars))) {
        ok = false;
        break;
      }
      if (t == 0 && row >= ti.cnt) {
        unsigned char* vt = sKV + ((2 * i + 1) & 3) * kTile;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4* vrow = (uint4*)(vt + h * kHalf + row * 128);
#pragma unroll
          for (int e = 0; e < 8; ++e) vrow[e] = make_uint4(0, 0, 0, 0);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tmem_st_wait();
      fence_before();
      mbar_arrive(&bars->p_full[t]);
    }
    if (tile_live && ok && ntiles > 0)
      ok = __all_sync(0xFFFFFFFFu, pair_wait(&bars->o_full, 0, bars));
    // epilogue: the O row -> final output or a split partial
    const bool final_out = p.nsplit == 1;
    const int qt = 2 * pair + t;  // query tile index of this tile
    const int64_t prow = (((int64_t)grp * p.qtiles + qt) * p.nsplit + split) * BM + row;
    const bool has = ok && row_valid && l > 0.f && ntiles > 0;
    const float inv = has ? 1.f / l : 0.f;
    // (TMEM loads by every lane of the warp: they are warp-collective)
    // final rows: every query row (zeros past the tree); partials: the tree's
    // rows only (the combine writes the others without reading partials)
    const bool writes = final_out ? qr < R : (qt < p.qtiles && qr < R && j < n);
    if (tile_rows) {
      fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (tile_live && ntiles > 0) {
          tmem_ld32(lane_base + o_col + 32 * c, o);
          tmem_ld_wait();
        }
        if (!has) {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (!writes) {
        } else if (final_out) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                     __uint_as_float(o[2 * e + 1]) * inv);
            pk[e] = *(uint32_t*)&h2;
          }
          uint4* d4 = (uint4*)(p.out + (((int64_t)b * p.n_max + j) * p.hq + (kvh * g + qr % g)) * D + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        } else {
          float4* q4 = (float4*)(p.part_o + prow * D + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            q4[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
        }
      }
      if (writes && final_out) {
        if (p.lse_out)
          p.lse_out[((int64_t)b * p.n_max + j) * p.hq + (kvh * g + qr % g)] =
              has ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      } else if (writes) {
        p.part_ml[prow] = has ? make_float2(m_used, l) : make_float2(-INFINITY, 0.f);
      }
    }
  }

  pdl_trigger();
  fence_before();
  __syncthreads();
  if (bars->abort && tid == 0) raise_status(p.status, DDT_ERR_TIMEOUT);
  if (warp == 0) {
    __syncwarp();
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

size_t pair_smem_bytes() { return 1024 + (size_t)6 * kTile + sizeof(PairBars) + 64; }

// Merge the per-split partials: one warp per query row, 4 dims per lane.
__global__ void __launch_bounds__(256) attn_tc_combine(const Params p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x * 8 + warp;          // row within the query tile
  const int qtile = row / BM, r = row % BM;
  const int grp = blockIdx.y;
  const int b = grp / p.hkv, kvh = grp % p.hkv;
  const int g = p.g;
  const int R = p.n_max * g;
  const int qr = qtile * BM + r;
  if (qtile >= p.qtiles || qr >= R) return;
  int n = p.n_nodes[b];
  n = min(max(n, 1), p.n_max);
  const int j = qr / g, h = kvh * g + qr % g;
  if (j >= n) {  // a row past the tree: zeros, and no partial to read (none was written)
    uint2* dst = (uint2*)(p.out + (((int64_t)b * p.n_max + j) * p.hq + h) * D);
    dst[lane] = make_uint2(0u, 0u);
    if (lane == 0 && p.lse_out) p.lse_out[((int64_t)b * p.n_max + j) * p.hq + h] = -INFINITY;
    return;
  }
  const int64_t base = (((int64_t)grp * p.qtiles + qtile) * p.nsplit) * BM + r;
  float M = -INFINITY;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
  // splits in groups of 8, each group's (m, l) and O slices loaded together
  for (int s0 = 0; s0 < p.nsplit; s0 += 8) {
    float2 ml[8];
    float4 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (s0 + e < p.nsplit) {
        ml[e] = p.part_ml[base + (int64_t)(s0 + e) * BM];
        v[e] = ((const float4*)(p.part_o + (base + (int64_t)(s0 + e) * BM) * D))[lane];
      } else {
        ml[e] = make_float2(-INFINITY, 0.f);
      }
    float Mg = M;
#pragma unroll
    for (int e = 0; e < 8; ++e) Mg = fmaxf(Mg, ml[e].x);
    if (Mg == -INFINITY) continue;
    const float rescale = M == -INFINITY ? 0.f : ex2(M - Mg);
    L *= rescale;
    acc.x *= rescale;
    acc.y *= rescale;
    acc.z *= rescale;
    acc.w *= rescale;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (ml[e].x != -INFINITY) {
        const float w = ex2(ml[e].x - Mg);
        L += ml[e].y * w;
        acc.x = fmaf(w, v[e].x, acc.x);
        acc.y = fmaf(w, v[e].y, acc.y);
        acc.z = fmaf(w, v[e].z, acc.z);
        acc.w = fmaf(w, v[e].w, acc.w);
      }
    M = Mg;
  }
  if (j >= n) {
    L = 0.f;
    acc = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat162 h0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  __nv_bfloat162 h1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2* dst = (uint2*)(p.out + (((int64_t)b * p.n_max + j) * p.hq + h) * D);
  dst[lane] = make_uint2(*(uint32_t*)&h0, *(uint32_t*)&h1);
  if (lane == 0 && p.lse_out)
    p.lse_out[((int64_t)b * p.n_max + j) * p.hq + h] =
        L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)f;
  });
  return fn;
}

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
            strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t smem_bytes() { return 1024 + (size_t)(1 + 2 * kStages) * kTile + sizeof(Bars) + 64; }

}  // namespace tc

// Can the tensor-core path serve this call?
bool attn_tc_eligible(const ddt_attn_args* a) {
  if (a->d != 128) return false;
  const int g = a->hq / a->hkv;
  if (g > 128 || 128 % g != 0) return false;
  if ((long)a->n_max * g < 64) return false;
  if (a->page_table) {
    const int ps = a->page_size;
    if (a->num_pages <= 0) return false;
    if (ps <= 128 ? (128 % ps != 0) : (ps % 128 != 0)) return false;
  }
  return tc::encode_fn() != nullptr;
}

bool attn_tc_cluster(int nsplit, long clusters);

// KV-split plan of the tensor-core path (one CTA per SM).  Splits that can
// run as co-resident clusters merge on chip, so among those the plan takes
// the one with the fewest tiles per split; it falls back to as few waves
// and splits as possible (with partials and a combine kernel) only when no
// cluster split fits or a plain split is clearly shorter.
void attn_tc_plan(const ddt_attn_args* a, int sms, int* qtiles, int* nsplit, int* tps) {
  const int g = a->hq / a->hkv;
  const long R = (long)a->n_max * g;
  *qtiles = (int)((R + tc::BM - 1) / tc::BM);
  const long base = (long)*qtiles * a->batch * a->hkv;
  const int tiles = (a->max_ctx + tc::BN - 1) / tc::BN + (a->n_max + tc::BN - 1) / tc::BN;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 16 && s <= tiles; ++s) {
    const long ctas = base * s;
    const long waves = (ctas + sms - 1) / sms;
    const double eff = (double)ctas / (double)(waves * sms);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = s;
    }
  }
  int t = (tiles + best - 1) / best;
  const long plain_waves = (base * ((tiles + t - 1) / t) + sms - 1) / sms;
  // the partials and their combine cost about as much as kMergeTiles tiles
  constexpr int kMergeTiles = 3;
  const long plain_cost = plain_waves * t + (best > 1 ? kMergeTiles : 0);
  int cbest = 0, ct = 0;
  for (int s = 2; s <= 8 && s <= tiles; ++s) {
    const int ts = (tiles + s - 1) / s;
    if (attn_tc_cluster(s, base) && (cbest == 0 || ts < ct)) {
      cbest = s;
      ct = ts;
    }
  }
  if (cbest > 0 && ct <= plain_cost) {
    *tps = ct;
    *nsplit = (tiles + ct - 1) / ct;
    return;
  }
  *tps = t;
  *nsplit = (tiles + t - 1) / t;
}
// Can the KV splits of one query tile run as a thread-block cluster (and
// merge on chip)?  Up to 8 splits (the portable cluster size), when the
// device can co-schedule such a cluster of these CTAs.
bool attn_tc_cluster(int nsplit, long clusters) {
  if (nsplit < 2 || nsplit > 8) return false;
  static std::mutex mu;
  static int known[9] = {0};  // co-resident clusters of each size; -1: none
  std::lock_guard<std::mutex> lock(mu);
  if (known[nsplit] == 0) {
    bool ok = ensure_smem_attr((const void*)tc::attn_tc_kernel, tc::smem_bytes()) == cudaSuccess;
    if (ok) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, nsplit, 1);
      cfg.blockDim = dim3(tc::kThreads, 1, 1);
      cfg.dynamicSmemBytes = tc::smem_bytes();
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 1;
      attr.val.clusterDim.y = nsplit;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      ok = cudaOccupancyMaxActiveClusters(&n, (void*)tc::attn_tc_kernel, &cfg) == cudaSuccess && n > 0;
      known[nsplit] = ok ? n : -1;
    } else {
      known[nsplit] = -1;
    }
    cudaGetLastError();  // a failed query must not leave a sticky error behind
  }
  // only when every cluster of the launch runs in the first wave
  return known[nsplit] > 0 && clusters <= known[nsplit];
}

// The two-query-tile kernel serves every call on a dense cache with at least
// two query tiles per kv head whose splits would not merge on chip.  Its KV-split plan
// minimises waves x tiles per split (plus the combine's cost when split).
bool attn_pair_plan(const ddt_attn_args* a, int sms, int* qtiles, int* nsplit, int* tps) {
  int qt, ns, t;
  attn_tc_plan(a, sms, &qt, &ns, &t);
  const int choice = attn_kernel_choice();
  if (qt < 2 || choice == 1) return false;
  if (choice == 0 && ns > 1 && attn_tc_cluster(ns, (long)qt * a->batch * a->hkv)) return false;
  // paged caches: the pair kernel's ring holds two K/V tiles (the one-tile
  // kernel's three), too shallow for page gathers in random order (measured
  // on a B200: 32 ragged sequences, 64-token pages, 2.27 ms against 1.85 ms)
  if (choice == 0 && a->page_table) return false;
  const long base = (long)((qt + 1) / 2) * a->batch * a->hkv;
  const int tiles = (a->max_ctx + tc::BN - 1) / tc::BN + (a->n_max + tc::BN - 1) / tc::BN;
  constexpr int kMergeTiles = 3;
  long best_cost = -1;
  int best_s = 1;
  for (int s = 1; s <= 16 && s <= tiles; ++s) {
    const int ts = (tiles + s - 1) / s;
    const int sp = (tiles + ts - 1) / ts;
    const long waves = (base * sp + sms - 1) / sms;
    const long cost = waves * ts + (sp > 1 ? kMergeTiles : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_s = s;
    }
  }
  *qtiles = qt;
  *tps = (tiles + best_s - 1) / best_s;
  *nsplit = (tiles + *tps - 1) / *tps;
  return true;
}

size_t attn_tc_workspace_size(const ddt_attn_args* a, int sms) {
  int qt, ns, tps;
  if (!attn_pair_plan(a, sms, &qt, &ns, &tps)) {
    attn_tc_plan(a, sms, &qt, &ns, &tps);
    if (ns <= 1 || attn_tc_cluster(ns, (long)qt * a->batch * a->hkv)) return 0;
  } else if (ns <= 1) {
    return 0;
  }
  const size_t rows = (size_t)a->batch * a->hkv * qt * ns * tc::BM;
  return ((rows * tc::D * sizeof(float) + 255) & ~(size_t)255) + rows * sizeof(float2);
}

ddt_status launch_attn_tc(const ddt_attn_args* a, void* ws, int sms, cudaStream_t stream) {
  using namespace tc;
  Params p;
  p.batch = a->batch;
  p.n_max = a->n_max;
  p.hq = a->hq;
  p.hkv = a->hkv;
  p.g = a->hq / a->hkv;
  p.W = (a->n_max + 31) / 32;
  p.max_ctx = a->max_ctx;
  p.paged = a->page_table != nullptr;
  p.page_size = a->page_size;
  p.max_pages = a->max_pages;
  p.rows_per_box = p.paged ? (a->page_size < 128 ? a->page_size : 128) : 128;
  p.boxes_per_tile = 128 / p.rows_per_box;
  p.t_max = a->t_max;
  p.scale_log2 = a->scale * kLog2e;
  p.ctx_len = a->ctx_len;
  p.n_nodes = a->n_nodes;
  p.mask = a->mask;
  p.page_table = a->page_table;
  p.out = (uint16_t*)a->out;
  p.lse_out = a->lse_out;
  p.status = a->dev_status;
  p.wait_cycles = wait_limit_cycles();
  const bool pairs = attn_pair_plan(a, sms, &p.qtiles, &p.nsplit, &p.tiles_per_split);
  if (!pairs) attn_tc_plan(a, sms, &p.qtiles, &p.nsplit, &p.tiles_per_split);
  p.cluster = !pairs && attn_tc_cluster(p.nsplit, (long)p.qtiles * a->batch * a->hkv) ? 1 : 0;
  if (p.nsplit > 1 && !p.cluster) {
    const size_t rows = (size_t)a->batch * a->hkv * p.qtiles * p.nsplit * BM;
    p.part_o = (float*)ws;
    p.part_ml = (float2*)((char*)ws + ((rows * D * sizeof(float) + 255) & ~(size_t)255));
  } else {
    p.part_o = nullptr;
    p.part_ml = nullptr;
  }
  const int g = p.g;
  const cuuint64_t hkv = (cuuint64_t)a->hkv;
  CUtensorMap mq, mk, mv, mkt, mvt;
  {
    cuuint64_t dims[3] = {D, (cuuint64_t)a->hq, (cuuint64_t)a->batch * a->n_max};
    cuuint64_t str[2] = {D * 2, (cuuint64_t)a->hq * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)(BM / g)};
    if (!encode(&mq, a->q, 3, dims, str, box)) return DDT_ERR_CUDA;
  }
  {
    cuuint64_t dims[3] = {D, hkv, (cuuint64_t)a->batch * a->n_max};
    cuuint64_t str[2] = {D * 2, hkv * D * 2};
    cuuint32_t box[3] = {64, 1, BN};
    if (!encode(&mkt, a->k_tree, 3, dims, str, box)) return DDT_ERR_CUDA;
    if (!encode(&mvt, a->v_tree, 3, dims, str, box)) return DDT_ERR_CUDA;
  }
  if (a->max_ctx > 0 && !p.paged) {
    cuuint64_t dims[3] = {D, hkv, (cuuint64_t)a->batch * a->t_max};
    cuuint64_t str[2] = {D * 2, hkv * D * 2};
    cuuint32_t box[3] = {64, 1, BN};
    if (!encode(&mk, a->k_cache, 3, dims, str, box)) return DDT_ERR_CUDA;
    if (!encode(&mv, a->v_cache, 3, dims, str, box)) return DDT_ERR_CUDA;
  } else if (a->max_ctx > 0) {
    cuuint64_t dims[4] = {D, hkv, (cuuint64_t)a->page_size, (cuuint64_t)a->num_pages};
    cuuint64_t str[3] = {D * 2, hkv * D * 2, (cuuint64_t)a->page_size * hkv * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)p.rows_per_box, 1};
    if (!encode(&mk, a->k_cache, 4, dims, str, box)) return DDT_ERR_CUDA;
    if (!encode(&mv, a->v_cache, 4, dims, str, box)) return DDT_ERR_CUDA;
  } else {
    mk = mkt;  // no context: never read
    mv = mvt;
  }
  if (pairs) {
    const size_t smem = pair_smem_bytes();
    if (ensure_smem_attr((const void*)attn_pair_kernel, smem) != cudaSuccess) return DDT_ERR_CUDA;
    dim3 grid((p.qtiles + 1) / 2, p.nsplit, a->batch * a->hkv);
    if (launch_pdl(attn_pair_kernel, grid, dim3(kPairThreads), smem, stream, 0, mq, mk, mv, mkt, mvt, p) !=
        cudaSuccess)
      return DDT_ERR_CUDA;
  } else {
    const size_t smem = smem_bytes();
    if (ensure_smem_attr((const void*)attn_tc_kernel, smem) != cudaSuccess) return DDT_ERR_CUDA;
    dim3 grid(p.qtiles, p.nsplit, a->batch * a->hkv);
    if (launch_pdl(attn_tc_kernel, grid, dim3(kThreads), smem, stream, p.cluster ? p.nsplit : 0, mq, mk, mv,
                   mkt, mvt, p) != cudaSuccess)
      return DDT_ERR_CUDA;
  }
  if (p.nsplit > 1 && !p.cluster) {
    if (launch_pdl(attn_tc_combine, dim3(p.qtiles * BM / 8, a->batch * a->hkv), dim3(256), 0, stream, 0, p) !=
        cudaSuccess)
      return DDT_ERR_CUDA;
  }
  return DDT_OK;
}

}  // namespace ddt
