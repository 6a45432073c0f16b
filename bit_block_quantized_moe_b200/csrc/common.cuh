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
// One 32-bit code word holds 8 pairs; pair p keeps its even-k code at bits 2p and
// its odd-k code at bits 16+2p.  OR-ing the masked code into the mantissa of
// bf16 128.0 gives 128 + q*4^s exactly (s = 0,1,2); one bf16x2 FMA then yields
// q - 1 exactly.

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Decodes the 8 pairs of `w` into q-1 as bf16x2 (exact).
__device__ __forceinline__ void decode_q2_word(uint32_t w, uint32_t (&p)[8]) {
  constexpr uint32_t kMagic = 0x43004300u;  // (128, 128)
  constexpr uint32_t kOne = 0x3F803F80u;    // (1, 1)
  constexpr uint32_t kQuarter = 0x3E803E80u;
  constexpr uint32_t kSixteenth = 0x3D803D80u;
  constexpr uint32_t kM129 = 0xC301C301u;   // (-129, -129)
  constexpr uint32_t kM33 = 0xC204C204u;    // (-33, -33)
  constexpr uint32_t kM9 = 0xC110C110u;     // (-9, -9)
  uint32_t w6 = w >> 6, w12 = w >> 12;
  p[0] = bf16x2_fma((w & 0x00030003u) | kMagic, kOne, kM129);
  p[1] = bf16x2_fma((w & 0x000C000Cu) | kMagic, kQuarter, kM33);
  p[2] = bf16x2_fma((w & 0x00300030u) | kMagic, kSixteenth, kM9);
  p[3] = bf16x2_fma((w6 & 0x00030003u) | kMagic, kOne, kM129);
  p[4] = bf16x2_fma((w6 & 0x000C000Cu) | kMagic, kQuarter, kM33);
  p[5] = bf16x2_fma((w6 & 0x00300030u) | kMagic, kSixteenth, kM9);
  p[6] = bf16x2_fma((w12 & 0x00030003u) | kMagic, kOne, kM129);
  p[7] = bf16x2_fma((w12 & 0x000C000Cu) | kMagic, kQuarter, kM33);
}

// D = A(16x16 bf16) * B(16x8 bf16) + C, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                               const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

}  // namespace moe
