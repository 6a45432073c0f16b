// Grouped expert projections straight from packed Q2 units, on the tensor cores
// through register-resident dequantisation (sm_100a).
//
// Work item = (expert, up to 8 tokens that were routed to it, a chunk of
// 16-row units).  Each 16x32 block-tile is decoded in registers to exact
// bf16 (q - 1) values, multiplied by the 8 tokens on the tensor cores
// (m16n8k16, fp32 accumulate) and scaled by the fp16 block scale d in fp32:
//   acc += d * sum_k (q_k - 1) x_k,
// so every product is exact and only fp32 accumulation rounds.
#include "kernels.cuh"

namespace moe {

enum { kGateUp = 0, kDown = 1 };

struct ExpertArgs {
  const uint8_t *experts;
  const uint8_t *shared;
  PackedGeom G;
  int E;
  const uint16_t *act;       // gate/up: x [T, H]; down: h [positions, I]
  int act_stride;            // elements per activation row
  const int32_t *sorted_tok; // gate/up: token of each sorted position
  const int4 *items;
  const uint32_t *n_items;
  int chunks;                // unit chunks per item
  int units_per_chunk;
  uint16_t *h_out;           // gate/up output [positions, I] bf16
  float *y_out;              // down output [positions, H] fp32
};

template <int MODE>
__global__ void __launch_bounds__(256) expert_mma_kernel(ExpertArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int item_id = blockIdx.x / a.chunks, chunk = blockIdx.x % a.chunks;
  if (item_id >= (int)*a.n_items) return;
  const int4 it = a.items[item_id];
  const int e = it.x, pos0 = it.y, ntok = it.z;
  const uint8_t *ex = (e == a.E) ? a.shared : a.experts + (size_t)e * a.G.expert_bytes;
  const int groups = MODE == kGateUp ? a.G.gu_groups : a.G.dn_groups;
  const int units = MODE == kGateUp ? a.G.gu_units : a.G.dn_units;
  const size_t unit_bytes = MODE == kGateUp ? a.G.gu_unit_bytes : a.G.dn_unit_bytes;
  const uint8_t *sec = MODE == kGateUp ? ex : ex + a.G.gu_bytes;
  const int K = a.act_stride;
  const int row_elems = K + 16;  // +32 bytes of padding: conflict-free 8-byte fragment loads

  // Stage the (up to 8) activation rows of this item in shared memory.
  uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
  for (int i = threadIdx.x; i < 8 * (K / 8); i += blockDim.x) {
    const int r = i / (K / 8), c8 = i % (K / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < ntok) {
      const int row = MODE == kGateUp ? a.sorted_tok[pos0 + r] : pos0 + r;
      v = *reinterpret_cast<const uint4 *>(a.act + (size_t)row * K + c8 * 8);
    }
    *reinterpret_cast<uint4 *>(xs + r * row_elems + c8 * 8) = v;
  }
  float *red = reinterpret_cast<float *>(smem + 8 * row_elems * 2);  // [8 warps][32 lanes][4]
  __syncthreads();

  const int wk = groups >= 8 ? 8 : (groups >= 4 ? 4 : (groups >= 2 ? 2 : 1));  // warps along K
  const int wu = 8 / wk;                                                          // units in flight
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kw = warp % wk, uw = warp / wk;
  const int g = lane >> 2, c = lane & 3;
  const uint16_t *xrow = xs + g * row_elems + 4 * c;

  const int u_begin = chunk * a.units_per_chunk;
  const int u_end = min(units, u_begin + a.units_per_chunk);
  for (int u0 = u_begin; u0 < u_end; u0 += wu) {
    const int u = u0 + uw;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (u < u_end) {
      const uint8_t *up = sec + (size_t)u * unit_bytes;
      for (int grp = kw; grp < groups; grp += wk) {
        const uint8_t *gp = up + (size_t)grp * kGroupBytes;
        const uint4 cw = ldg_nc_v4(gp + lane * 16);
        const uint4 sw = ldg_nc_v4(gp + kGroupCodeBytes + g * 16);
        const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
        const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t p[8];
          decode_q2_exact(cws[blk], p);
          const int kb = 128 * grp + 32 * blk;
          const uint2 b0 = *reinterpret_cast<const uint2 *>(xrow + kb);
          const uint2 b1 = *reinterpret_cast<const uint2 *>(xrow + kb + 16);
          const uint32_t a0[4] = {p[0], p[1], p[2], p[3]};
          const uint32_t a1[4] = {p[4], p[5], p[6], p[7]};
          const float z[4] = {0.f, 0.f, 0.f, 0.f};
          float d[4];
          mma_bf16_16816(d, a0, b0.x, b0.y, z);
          mma_bf16_16816(d, a1, b1.x, b1.y, d);
          const float2 s2 = __half22float2(*reinterpret_cast<const __half2 *>(&sws[blk]));
          acc[0] = fmaf(s2.x, d[0], acc[0]);
          acc[1] = fmaf(s2.x, d[1], acc[1]);
          acc[2] = fmaf(s2.y, d[2], acc[2]);
          acc[3] = fmaf(s2.y, d[3], acc[3]);
        }
      }
    }
    *reinterpret_cast<float4 *>(red + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (kw == 0 && u < u_end) {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      for (int kk = 0; kk < wk; ++kk) {
        const float4 v = *reinterpret_cast<const float4 *>(red + ((uw * wk + kk) * 32 + lane) * 4);
        s[0] += v.x;
        s[1] += v.y;
        s[2] += v.z;
        s[3] += v.w;
      }
      const int n0 = 2 * c, n1 = 2 * c + 1;
      if (MODE == kGateUp) {
        const int I = a.G.I;
        const int i = 8 * u + g;  // tile rows g (gate) and g+8 (up) share intermediate row i
        if (n0 < ntok) a.h_out[(size_t)(pos0 + n0) * I + i] = float_to_bf16_bits(silu_f(s[0]) * s[2]);
        if (n1 < ntok) a.h_out[(size_t)(pos0 + n1) * I + i] = float_to_bf16_bits(silu_f(s[1]) * s[3]);
      } else {
        const int H = a.G.H;
        const int r0 = 16 * u + g, r1 = r0 + 8;
        if (n0 < ntok) {
          a.y_out[(size_t)(pos0 + n0) * H + r0] = s[0];
          a.y_out[(size_t)(pos0 + n0) * H + r1] = s[2];
        }
        if (n1 < ntok) {
          a.y_out[(size_t)(pos0 + n1) * H + r0] = s[1];
          a.y_out[(size_t)(pos0 + n1) * H + r1] = s[3];
        }
      }
    }
    __syncthreads();
  }
}

static size_t expert_smem_bytes(int K) { return (size_t)8 * (K + 16) * 2 + 8 * 32 * 4 * sizeof(float); }

cudaError_t launch_experts(const moe_dims &d, const PackedGeom &G, const uint8_t *experts, const uint8_t *shared,
                           const uint16_t *x, int T, const Workspace &ws, cudaStream_t s) {
  ExpertArgs a{};
  a.experts = experts;
  a.shared = shared;
  a.G = G;
  a.E = d.n_experts;
  a.items = ws.items;
  a.n_items = ws.n_items;
  a.sorted_tok = ws.sorted_tok;
  a.h_out = ws.h;
  a.y_out = ws.y;
  // gate/up + SwiGLU
  {
    a.act = x;
    a.act_stride = G.H;
    a.units_per_chunk = T <= 8 ? 8 : 16;
    a.chunks = (G.gu_units + a.units_per_chunk - 1) / a.units_per_chunk;
    const size_t smem = expert_smem_bytes(G.H);
    cudaError_t err = cudaFuncSetAttribute(expert_mma_kernel<kGateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    trace_mark(MOE_KERNEL_GATE_UP, false, s);
    expert_mma_kernel<kGateUp><<<ws.max_items * a.chunks, 256, smem, s>>>(a);
    trace_mark(MOE_KERNEL_GATE_UP, true, s);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  // down
  {
    a.act = ws.h;
    a.act_stride = G.I;
    a.units_per_chunk = T <= 8 ? 16 : 32;
    a.chunks = (G.dn_units + a.units_per_chunk - 1) / a.units_per_chunk;
    const size_t smem = expert_smem_bytes(G.I);
    cudaError_t err = cudaFuncSetAttribute(expert_mma_kernel<kDown>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    trace_mark(MOE_KERNEL_DOWN, false, s);
    expert_mma_kernel<kDown><<<ws.max_items * a.chunks, 256, smem, s>>>(a);
    trace_mark(MOE_KERNEL_DOWN, true, s);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace moe
