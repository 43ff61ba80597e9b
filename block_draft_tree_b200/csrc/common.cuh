// common.cuh -- small device helpers shared by the libddt kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ddt.h"

namespace ddt {

constexpr float kLog2e = 1.4426950408889634f;

// Order-preserving map of a float onto uint32 (larger float -> larger key).
// -0.0 is folded onto +0.0 so that equal values compare equal.
__device__ __forceinline__ uint32_t ord32(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_ord32(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}
// Same map on the 16 bits of a bf16 value.
__device__ __forceinline__ uint32_t ord16(uint32_t b) {
  b &= 0xFFFFu;
  if (b == 0x8000u) b = 0u;
  return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
}

// A candidate key: larger key = larger value, and among equal values the
// smaller token id.  Key 0 never belongs to a real element.
__device__ __forceinline__ uint64_t cand_key(float z, uint32_t id) {
  return ((uint64_t)ord32(z) << 32) | (uint64_t)(0xFFFFFFFFu - id);
}
__device__ __forceinline__ uint32_t key_id(uint64_t key) {
  return 0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull);
}
__device__ __forceinline__ float key_val(uint64_t key) { return from_ord32((uint32_t)(key >> 32)); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

// Streaming 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Hardware base-2 exponential (single MUFU instruction).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Merge two (max, sum-of-exp2((x-max)*c)) pairs.
__device__ __forceinline__ void ms_merge(float& m, float& s, float m2, float s2, float c) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float M = fmaxf(m, m2);
  s = s * ex2((m - M) * c) + s2 * ex2((m2 - M) * c);
  m = M;
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int lane_mask) {
  uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
  lo = __shfl_xor_sync(0xFFFFFFFFu, lo, lane_mask);
  hi = __shfl_xor_sync(0xFFFFFFFFu, hi, lane_mask);
  return ((uint64_t)hi << 32) | lo;
}

// Two fp32 values in one 64-bit register pair (lane 0 in the low word), and
// the sm_100 packed two-wide fp32 arithmetic on such pairs: one instruction
// for both lanes, each lane rounded exactly as the scalar instruction.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// x - y lane by lane, rounded once (y * -1 is exact).
__device__ __forceinline__ uint64_t fsub2(uint64_t x, uint64_t y) {
  return ffma2(y, pack2(-1.f, -1.f), x);
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Raise a device status word (never lowers it).
__device__ __forceinline__ void raise_status(int32_t* st, int code) {
  if (st) atomicMax(st, code);
}

// L2-coherent loads for data written by other CTAs of the same grid.
__device__ __forceinline__ uint64_t ld_cg_u64(const uint64_t* p) { return __ldcg((const unsigned long long*)p); }
// Atomic add, acquire-release at device scope (a ticket that publishes what
// the CTA wrote before its barrier and sees what earlier holders wrote).
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ float2 ld_cg_f2(const float2* p) { return __ldcg(p); }

// Programmatic dependent launch: every kernel of the library is launched
// with programmatic stream serialization, waits for the previous kernel's
// results before its first read of any input, and lets the next kernel be
// scheduled once its own main work is issued.  Without the launch attribute
// both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace ddt
