// Shared device helpers for the Q2 MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_q2.h"

namespace moe {

constexpr int kQBlock = 32;       // weights per Q2 block
constexpr int kCanonBlockBytes = 10;
constexpr int kBlocksPerGroup = 4;  // blocks per "block group" (128 weights along K)
// Packed unit: a 16-row m16 tile.  Per block group: 32 lanes x 16 B of codes, then
// 8 x 16 B of scales.
constexpr int kGroupCodeBytes = 512;
constexpr int kGroupScaleBytes = 128;
constexpr int kGroupBytes = kGroupCodeBytes + kGroupScaleBytes;  // 640

// Sticky device status bits (workspace word 0).
constexpr uint32_t kStatusBadIndex = 1u;
constexpr uint32_t kStatusTimeout = 2u;

struct PackedGeom {
  int H, I;
  int gu_units;      // I / 8: each unit = 8 gate rows + 8 up rows
  int dn_units;      // H / 16: each unit = 16 down rows
  int gu_groups;     // H / 128 block groups along K for gate/up
  int dn_groups;     // I / 128 block groups along K for down
  size_t gu_unit_bytes, dn_unit_bytes;
  size_t gu_bytes;   // offset of the down section inside an expert
  size_t expert_bytes;  // padded stride
};

__host__ __device__ inline PackedGeom packed_geom(int H, int I) {
  PackedGeom g;
  g.H = H;
  g.I = I;
  g.gu_units = I / 8;
  g.dn_units = H / 16;
  g.gu_groups = H / 128;
  g.dn_groups = I / 128;
  g.gu_unit_bytes = (size_t)g.gu_groups * kGroupBytes;
  g.dn_unit_bytes = (size_t)g.dn_groups * kGroupBytes;
  g.gu_bytes = (size_t)g.gu_units * g.gu_unit_bytes;
  size_t raw = g.gu_bytes + (size_t)g.dn_units * g.dn_unit_bytes;
  g.expert_bytes = (raw + 255) & ~(size_t)255;
  return g;
}

// ---- bf16 helpers -------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ---- Q2 fragment decode ----------------------------------------------------------
// A packed 32-bit code word holds the 16 codes one lane needs for the two
// m16n8k16 steps of a 32-weight block: 8 pairs, the even-k code of a pair in
// the low half-word and the odd-k code at the same offset in the high half.
// Pair (step s, fragment register P) sits at bit 8s + {0, 4, 2, 6}[P], so that
// P0/P1 (k pair 4c, 4c+1) are read with the mask 0x3 and P2/P3 (k pair 4c+2,
// 4c+3) with the mask 0xC after shifts of 0, 4, 8, 12.  OR-ing a masked code
// into the mantissa of bf16 128.0 gives 128 + q (mask 0x3) or 128 + 4q (mask
// 0xC), exactly.
// Bit offset of fragment register P (0..3) in step 0.
__host__ __device__ constexpr int pair_pos(int P) { return P == 0 ? 0 : (P == 1 ? 4 : (P == 2 ? 2 : 6)); }

// Biased decode: p[0..3] / p[4..7] are the A registers of steps 0 / 1 holding
// 128 + q (P0, P1) and 128 + 4q (P2, P3).  Used with the B registers of P2/P3
// scaled by 1/4 and the accumulator started at -sum_k c_k x_k with c_k = 129
// (k % 4 < 2) or 33 (k % 4 >= 2), which leaves sum_k (q_k - 1) x_k.
__device__ __forceinline__ void decode_q2_biased(uint32_t w, uint32_t (&p)[8]) {
  constexpr uint32_t kMagic = 0x43004300u;  // bf16 pair (128, 128)
  const uint32_t w4 = w >> 4, w8 = w >> 8, w12 = w >> 12;
  p[0] = (w & 0x00030003u) | kMagic;
  p[1] = (w4 & 0x00030003u) | kMagic;
  p[2] = (w & 0x000C000Cu) | kMagic;
  p[3] = (w4 & 0x000C000Cu) | kMagic;
  p[4] = (w8 & 0x00030003u) | kMagic;
  p[5] = (w12 & 0x00030003u) | kMagic;
  p[6] = (w8 & 0x000C000Cu) | kMagic;
  p[7] = (w12 & 0x000C000Cu) | kMagic;
}

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Exact decode: the same registers holding q - 1 (one bf16x2 FMA per pair, exact).
__device__ __forceinline__ void decode_q2_exact(uint32_t w, uint32_t (&p)[8]) {
  constexpr uint32_t kOne = 0x3F803F80u;      // (1, 1)
  constexpr uint32_t kQuarter = 0x3E803E80u;  // (1/4, 1/4)
  constexpr uint32_t kM129 = 0xC301C301u;     // (-129, -129)
  constexpr uint32_t kM33 = 0xC204C204u;      // (-33, -33)
  decode_q2_biased(w, p);
  p[0] = bf16x2_fma(p[0], kOne, kM129);
  p[1] = bf16x2_fma(p[1], kOne, kM129);
  p[2] = bf16x2_fma(p[2], kQuarter, kM33);
  p[3] = bf16x2_fma(p[3], kQuarter, kM33);
  p[4] = bf16x2_fma(p[4], kOne, kM129);
  p[5] = bf16x2_fma(p[5], kOne, kM129);
  p[6] = bf16x2_fma(p[6], kQuarter, kM33);
  p[7] = bf16x2_fma(p[7], kQuarter, kM33);
}

// D = A(16x16 bf16) * B(16x8 bf16) + C, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                               const float (&c)[4]) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

// (a0, a1) += (s, s) * (d0, d1): one packed fp32x2 FMA (sm_100), each lane rounded like fmaf.
__device__ __forceinline__ void fma2_bcast(float &a0, float &a1, float s, float d0, float d1) {
  uint64_t acc, dd, ss;
  asm("mov.b64 %0, {%1, %2};" : "=l"(acc) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(dd) : "f"(d0), "f"(d1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(s));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(ss), "l"(dd));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
}

// Read-only global load through the non-coherent path (weights, router).
__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

}  // namespace moe
