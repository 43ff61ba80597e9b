// attn_common.cuh -- parameters and epilogues shared by the tree-attention paths.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace ddt {

struct AttnParams {
  const uint16_t *q, *kc, *vc, *kt, *vt;
  const int32_t* page_table;  // null: dense cache
  int page_size, max_pages;
  int64_t t_max;
  const int32_t* ctx_len;
  int max_ctx;
  const uint32_t* mask;
  const int32_t* n_nodes;
  int batch, n_max, hq, hkv, d, g, W;
  float scale_log2;           // softmax scale * log2(e)
  uint16_t* out;
  float* lse_out;
  int32_t* status;
  int nsplit, tok_per_split, row_tiles;
  float* part_o;              // [batch*hkv][nsplit][R][d]
  float2* part_ml;            // [batch*hkv][nsplit][R]: (running max, running sum), base 2
  unsigned* tickets;          // [batch*hkv][row_tiles]
};

// Row of the (dense or paged) context cache holding position t of sequence b.
__device__ __forceinline__ int64_t kv_row(const AttnParams& p, int b, int t) {
  if (p.page_table == nullptr) return (int64_t)b * p.t_max + t;
  const int pg = p.page_table[(int64_t)b * p.max_pages + t / p.page_size];
  return (int64_t)pg * p.page_size + (t % p.page_size);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Final normalisation of one query row held as DV values per lane
// (dims lane + 32*i).  A row that saw nothing (l == 0) is written as 0 / -inf.
template <int DV>
__device__ __forceinline__ void write_row_final(const AttnParams& p, int b, int kvh, int qr,
                                                const float* o, float m, float l, int lane) {
  const int j = qr / p.g, h = kvh * p.g + qr % p.g;
  const int D = DV * 32;
  uint16_t* dst = p.out + (((int64_t)b * p.n_max + j) * p.hq + h) * D;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < DV; ++i) dst[lane + 32 * i] = f32_to_bf16(o[i] * inv);
  if (p.lse_out && lane == 0)
    p.lse_out[((int64_t)b * p.n_max + j) * p.hq + h] =
        l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
}

// Combine the per-split partials of one query row and write it.
template <int DV>
__device__ void combine_row(const AttnParams& p, int64_t grp, int b, int kvh, int qr, int lane) {
  const int R = p.n_max * p.g;
  const int D = DV * 32;
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, ld_cg_f2(&p.part_ml[(grp * p.nsplit + s) * R + qr]).x);
  float o[DV];
#pragma unroll
  for (int i = 0; i < DV; ++i) o[i] = 0.f;
  float l = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.nsplit; ++s) {
      const float2 ml = ld_cg_f2(&p.part_ml[(grp * p.nsplit + s) * R + qr]);
      if (ml.x == -INFINITY) continue;
      const float w = ex2(ml.x - M);
      l += ml.y * w;
      const float* po = p.part_o + ((grp * p.nsplit + s) * R + qr) * D;
#pragma unroll
      for (int i = 0; i < DV; ++i) o[i] = fmaf(w, __ldcg(po + lane + 32 * i), o[i]);
    }
  }
  write_row_final<DV>(p, b, kvh, qr, o, M, l, lane);
}

}  // namespace ddt
