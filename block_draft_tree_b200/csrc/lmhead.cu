// lmhead.cu -- stage 4 from the target's last hidden states: the LM head's
// logits of every tree row, their argmax and the walk, without ever storing
// the logits.
//
// DDTree page, section 運作流程 step 4: the target's greedy decision at each
// tree row is the argmax of its LM head, logits = h W^T over the vocabulary;
// the walk accepts a child carrying that token and continues, and the first
// token that matches no child is the bonus.  The logits of all rows are a
// dense contraction H[rows x K] W^T[K x V], so they run on the tensor cores
// and only the argmax leaves the chip:
//   * persistent CTAs (one per SM) over tiles of 128 rows x bn tokens (bn a
//     multiple of 16 up to 256, chosen per call so that the tiles fill whole
//     waves of SMs);
//     warp 0 streams 64-wide K slices of H and W by TMA (128-byte swizzle)
//     through a 4-deep shared-memory ring, warp 1 issues tcgen05 MMAs
//     (M 128, N bn, K 16; bf16 in, fp32 accumulate) into one of two TMEM
//     accumulators, so the next tile's MMAs overlap this tile's epilogue;
//   * warps 2-5 read the accumulator (one row per TMEM lane), take the
//     row's largest logit and its smallest column, and fold it into a 64-bit
//     key per row (ordered value, then smaller token id) with atomicMax: the
//     merge over vocabulary tiles is exact and independent of their order;
//   * the last CTA to finish (grid ticket) turns the keys into row tokens and
//     walks every sequence's tree with one warp, then clears the keys.
// Every mbarrier wait is bounded (about one second); a wait that gives up
// raises DDT_ERR_TIMEOUT in the status word and the CTA stops issuing work,
// lets its loads and MMAs in flight complete (again with bounded waits),
// frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "tcgen05.cuh"

namespace ddt {
namespace tc {
bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box);
}  // namespace tc

namespace lm {

constexpr int BM = 128;                 // rows per tile (MMA M)
constexpr int BN = 256;                 // largest vocabulary tile (MMA N); the launch picks bn <= BN
constexpr int BK = 64;                  // K slice per stage (128 bytes of bf16)
constexpr int kStages = 4;
constexpr int kThreads = 192;           // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t kTmemCols = 512;     // two 256-column fp32 accumulators
constexpr int kATile = BM * BK * 2;     // 16 KB
constexpr int kBTile = BN * BK * 2;     // 32 KB

struct Params {
  int M, K, V, m_tiles, total_tiles, kblocks;
  int bn;          // vocabulary entries per tile (multiple of 16, <= BN)
  uint32_t idesc;  // instruction descriptor for N = bn
  int batch, n_max, L;
  const int32_t *tok, *parent, *depth, *n_nodes;
  int32_t *acc_len, *acc_nodes, *acc_tok, *bonus, *row_token;
  unsigned long long* keys;  // [M], in the workspace's counter region
  unsigned* ticket;
  int32_t* status;
  long long wait_cycles;  // bound of every mbarrier wait
};

struct __align__(8) Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;  // after a wait gave up: completion of every MMA issued
  long long wait_cycles;
  uint32_t tmem_base;
  int abort;
  int last;
};

// ---------------------------------------------------------------- PTX helpers
// (the shared tcgen05 / TMA / mbarrier wrappers are in tcgen05.cuh)
// Bounded wait: false (and the CTA-wide abort flag set) if the phase does not
// complete within the launch's wait bound or another role already gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, Bars* bars) {
  return mbar_wait_bounded(b, parity, &bars->abort, bars->wait_cycles);
}
// K-major operand, 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_k(uint32_t saddr) { return sdesc(saddr, 16, 1024); }

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, A and B K-major,
// N = n, M = BM.
constexpr uint32_t idesc_for(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// The walk of sequence b by one warp over the row tokens in `rt`
// (this sequence's rows), reading the tree from global memory.
__device__ void walk_warp(const Params& p, int b, const int* rt) {
  const int lane = threadIdx.x & 31;
  int n = p.n_nodes[b];
  if (n < 1 || n > p.n_max) {
    if (lane == 0) raise_status(p.status, DDT_ERR_INVALID_ARG);
    n = min(max(n, 1), p.n_max);
  }
  const int64_t base = (int64_t)b * p.n_max;
  int x = 0, a = 0, bonus = 0;
#pragma unroll 1
  for (;;) {
    const int t = rt[x];
    int next = -1;
    if (a < p.L && p.depth[base + x] < p.L) {
      for (int c0 = x + 1; c0 < n; c0 += 32) {  // children come after their parent
        const int c = c0 + lane;
        const bool hit = c < n && p.parent[base + c] == x && p.tok[base + c] == t;
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

__global__ void __launch_bounds__(kThreads, 1)
    lmhead_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                  const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = smem;                      // [kStages][128 rows][128 B]
  unsigned char* sB = smem + kStages * kATile;   // [kStages][256 rows][128 B]
  Bars* bars = (Bars*)(sB + kStages * kBTile);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // set-up that reads no input runs before the wait for the previous kernel
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->acc_full[i], 1);
      mbar_init(&bars->acc_empty[i], 4 * 32);
    }
    mbar_init(&bars->drain, 1);
    bars->wait_cycles = p.wait_cycles;
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_h);
      prefetch_tmap(&tm_w);
    }
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int ntiles = (p.total_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        const int mt = t % p.m_tiles, nt = t / p.m_tiles;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&bars->empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, bars)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&bars->full[s], (uint32_t)(kATile + p.bn * BK * 2));
          tma_load_2d(sA + s * kATile, &tm_h, kb * BK, mt * BM, &bars->full[s]);
          tma_load_2d(sB + s * kBTile, &tm_w, kb * BK, nt * p.bn, &bars->full[s]);
        }
      }
      if (*(volatile int*)&bars->abort) {
        // a wait gave up: let the loads still in flight land before the CTA
        // (and its shared memory) goes away; the last kStages issued loads
        // are the only ones that can be outstanding
        int keep_going = 0;
        for (int q = it > kStages ? it - kStages : 0; q < it; ++q)
          mbar_wait_bounded(&bars->full[q % kStages], (uint32_t)(q / kStages) & 1u, &keep_going,
                            kDrainCycles);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int buf = i & 1;
        if (!mbar_wait(&bars->acc_empty[buf], ((uint32_t)(i >> 1) & 1u) ^ 1u, bars)) break;
        fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * BN);
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&bars->full[s], (uint32_t)(it / kStages) & 1u, bars)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t a = smem_u32(sA + s * kATile), b = smem_u32(sB + s * kBTile);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(d, sdesc_k(a + kk * 32), sdesc_k(b + kk * 32), p.idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars->empty[s]);
        }
        if (ok) mma_commit(&bars->acc_full[buf]);
      }
      if (*(volatile int*)&bars->abort) {
        // a wait gave up: every MMA issued completes before TMEM is freed
        int keep_going = 0;
        mma_commit(&bars->drain);
        mbar_wait_bounded(&bars->drain, 0u, &keep_going, kDrainCycles);
      }
    }
  } else {
    // ------------------------------------------------------------ argmax epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int i = 0; i < ntiles; ++i) {
      const int t = (int)blockIdx.x + i * (int)gridDim.x;
      const int mt = t % p.m_tiles, nt = t / p.m_tiles;
      const int buf = i & 1;
      if (!mbar_wait(&bars->acc_full[buf], (uint32_t)(i >> 1) & 1u, bars)) break;
      fence_after();
      const int n0 = nt * p.bn;
      const int ncols = min(p.bn, p.V - n0);
      float best = -INFINITY;
      int bcol = -1;
#pragma unroll 1
      for (int c = 0; c < p.bn; c += 32) {  // columns past bn are masked (c + e < ncols)
        uint32_t r[32];
        tmem_ld32(lane_base + (uint32_t)(buf * BN + c), r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float v = __uint_as_float(r[e]);
          if (c + e < ncols && (v > best || bcol < 0)) {  // ascending columns: ties keep the first
            best = v;
            bcol = c + e;
          }
        }
      }
      fence_before();
      mbar_arrive(&bars->acc_empty[buf]);
      const int m = mt * BM + row;
      if (m < p.M && bcol >= 0) atomicMax(&p.keys[m], (unsigned long long)cand_key(best, (uint32_t)(n0 + bcol)));
    }
    __threadfence();  // this thread's keys before the grid ticket
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  if (tid == 0 && bars->abort) raise_status(p.status, DDT_ERR_TIMEOUT);
  pdl_trigger();
  if (tid == 0) {
    __threadfence();
    bars->last = atomicAdd(p.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!bars->last) return;
  __threadfence();

  // ---------------------------------------------------------------- last CTA
  int* rt = (int*)smem;  // row tokens [M] (the ring is idle now; M * 4 <= its 192 KB)
  for (int m = tid; m < p.M; m += kThreads) {
    const unsigned long long k = atomicExch(&p.keys[m], 0ull);  // read and clear
    const int t = k ? (int)key_id(k) : 0;
    rt[m] = t;
    if (p.row_token) p.row_token[m] = t;
  }
  __syncthreads();
  for (int b = warp; b < p.batch; b += kThreads / 32) walk_warp(p, b, rt + (int64_t)b * p.n_max);
  if (tid == 0) *p.ticket = 0u;  // the counter region is left zero
}

size_t smem_bytes() { return 1024 + (size_t)kStages * (kATile + kBTile) + sizeof(Bars) + 64; }

}  // namespace lm

// Rows that fit the counter region (keys) beside the ticket.
constexpr int kLmHeadMaxRows = (int)(DDT_WS_COUNTER_BYTES / 8) - 16;

ddt_status launch_lm_head_walk(const ddt_lm_head_walk_args* a, void* ws, cudaStream_t stream) {
  using namespace lm;
  const int M = a->batch * a->n_max;
  if (a->batch == 0) return DDT_OK;
  CUtensorMap tm_h, tm_w;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a->K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)a->K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)BM};
    if (!tc::encode(&tm_h, a->hidden, 2, dims, strides, box)) return DDT_ERR_CUDA;
  }
  // Vocabulary tile width: with few waves, each CTA's time is about (tiles
  // it runs) x (tile width), so take the width (a multiple of 16) with the
  // fewest waves x width on this many SMs (a small per-tile cost favours
  // wider tiles on ties); with many waves the last one hardly matters and
  // the widest MMA is the most efficient.
  const int sms = device_sm_count();
  const int m_tiles = (M + BM - 1) / BM;
  int bn = BN;
  long best = -1;
  const long full_waves = ((long)m_tiles * ((a->V + BN - 1) / BN) + sms - 1) / sms;
  for (int w = BN; w >= 128 && full_waves < 16; w -= 16) {
    const long tiles = (long)m_tiles * ((a->V + w - 1) / w);
    const long waves = (tiles + sms - 1) / sms;
    const long cost = waves * (w + 16);
    if (best < 0 || cost < best) {
      best = cost;
      bn = w;
    }
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a->K, (cuuint64_t)a->V};
    const cuuint64_t strides[1] = {(cuuint64_t)a->K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)bn};
    if (!tc::encode(&tm_w, a->weight, 2, dims, strides, box)) return DDT_ERR_CUDA;
  }
  Params p;
  p.M = M;
  p.K = a->K;
  p.V = a->V;
  p.bn = bn;
  p.idesc = idesc_for(bn);
  p.m_tiles = m_tiles;
  const int n_tiles = (a->V + bn - 1) / bn;
  p.total_tiles = p.m_tiles * n_tiles;
  p.kblocks = (a->K + BK - 1) / BK;
  p.batch = a->batch;
  p.n_max = a->n_max;
  p.L = a->L;
  p.tok = a->tok;
  p.parent = a->parent;
  p.depth = a->depth;
  p.n_nodes = a->n_nodes;
  p.acc_len = a->acc_len;
  p.acc_nodes = a->acc_nodes;
  p.acc_tok = a->acc_tok;
  p.bonus = a->bonus;
  p.row_token = a->row_token;
  p.keys = (unsigned long long*)ws;
  p.ticket = (unsigned*)((unsigned long long*)ws + kLmHeadMaxRows + 8);
  p.status = a->dev_status;
  p.wait_cycles = wait_limit_cycles();
  const size_t smem = smem_bytes();
  if (ensure_smem_attr((const void*)lmhead_kernel, smem) != cudaSuccess) return DDT_ERR_CUDA;
  const int grid = p.total_tiles < sms ? p.total_tiles : sms;
  return launch_pdl(lmhead_kernel, dim3(grid), dim3(kThreads), smem, stream, 0, tm_h, tm_w, p) ==
                 cudaSuccess
             ? DDT_OK
             : DDT_ERR_CUDA;
}

int lm_head_max_rows() { return kLmHeadMaxRows; }

}  // namespace ddt
