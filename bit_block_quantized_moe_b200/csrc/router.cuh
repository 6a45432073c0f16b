// Router arithmetic shared by the stand-alone routing kernels and the fused
// decode kernel, so that both take bit-identical routing decisions.
#pragma once

#include "common.cuh"

namespace moe {

// Router arithmetic for T <= 8 tokens.  The row is cut into 2 halves of H/2;
// half h is summed by one warp: lane l accumulates k = h*H/2 + 4l + 128 i in
// order, then a butterfly sum.  The logit is (p0 + p1) + b.  Both the routing
// kernel and the fused decode kernel use exactly this order, so they take
// identical routing decisions.  kT is the token count when it is fixed at
// compile time (0: T at run time); the arithmetic is the same either way, but a
// run-time T leaves all 8 token slots in the code behind predicates, about
// twice the cycles for T = 3 on B200 (router_part_any picks the instance: compile-time
// T for the decode window T <= 3, the 8-slot code for larger windows).
constexpr int kRouterParts = 2;
template <bool kWrShared, int kT = 0>
__device__ __forceinline__ void router_part(const uint16_t *x, int xstride, int T_, const float *wrow, int H,
                                            int part, int lane, float (&acc)[8]) {
  const int T = kT ? kT : T_;
#pragma unroll
  for (int t = 0; t < 8; ++t) acc[t] = 0.f;
  const int kq = H / kRouterParts;
#pragma unroll 4
  for (int k = part * kq + lane * 4; k < (part + 1) * kq; k += 128) {
    const uint4 wv = kWrShared ? *reinterpret_cast<const uint4 *>(wrow + k) : ldg_nc_v4(wrow + k);
    const float w0 = __uint_as_float(wv.x), w1 = __uint_as_float(wv.y), w2 = __uint_as_float(wv.z),
                w3 = __uint_as_float(wv.w);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (t < T) {
        const uint2 xv = *reinterpret_cast<const uint2 *>(x + (size_t)t * xstride + k);
        float a = acc[t];
        a = fmaf(__uint_as_float(xv.x << 16), w0, a);
        a = fmaf(__uint_as_float(xv.x & 0xffff0000u), w1, a);
        a = fmaf(__uint_as_float(xv.y << 16), w2, a);
        a = fmaf(__uint_as_float(xv.y & 0xffff0000u), w3, a);
        acc[t] = a;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    if (t < T) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    }
  }
}

template <bool kWrShared>
__device__ __forceinline__ void router_part_any(const uint16_t *x, int xstride, int T, const float *wrow, int H,
                                                int part, int lane, float (&acc)[8]) {
  switch (T) {
    case 1: router_part<kWrShared, 1>(x, xstride, T, wrow, H, part, lane, acc); break;
    case 2: router_part<kWrShared, 2>(x, xstride, T, wrow, H, part, lane, acc); break;
    case 3: router_part<kWrShared, 3>(x, xstride, T, wrow, H, part, lane, acc); break;
    default: router_part<kWrShared, 0>(x, xstride, T, wrow, H, part, lane, acc); break;
  }
}

__device__ __forceinline__ float router_combine(const float *parts, float b) { return (parts[0] + parts[1]) + b; }

// Grid-stride clear of n words (the routing step's first kernel clears the
// dispatch bit map and counters of the call).
__device__ __forceinline__ void clear_range(uint32_t *p, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = 0;
}

// Exact 3-way bf16 split of an fp32 router weight: w = hi + mid + lo, each a
// bf16 holding the next 8 significant bits of the remainder.  With bf16
// tokens every product token * part is exact in fp32, so a tensor-core dot
// product over the three parts rounds only in its fp32 accumulation.
__device__ __forceinline__ void split3_bf16(float w, uint16_t &hi, uint16_t &mid, uint16_t &lo) {
  hi = float_to_bf16_bits(w);
  const float r1 = w - bf16_bits_to_float(hi);
  mid = float_to_bf16_bits(r1);
  const float r2 = r1 - bf16_bits_to_float(mid);
  lo = float_to_bf16_bits(r2);
}

// fp32 softmax over the k winners held by lanes 0..k-1 (lane order = selection order).
__device__ __forceinline__ float topk_softmax(float myv, int lane, int k) {
  const float mx = __shfl_sync(0xffffffffu, myv, 0);
  const float ex = lane < k ? expf(myv - mx) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  return ex / sum;
}

// Warp arg-max of (value desc, index asc) over the lanes' candidates.
__device__ __forceinline__ void warp_argmax(float &bv, int &be) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oe = __shfl_xor_sync(0xffffffffu, be, off);
    if (ov > bv || (ov == bv && oe < be)) {
      bv = ov;
      be = oe;
    }
  }
}

// Top-k with the token's logits held in registers (E <= 32 * NPL): one read
// of the row, then k selection rounds in registers.  Same selection rule and
// softmax as warp_topk, hence the same result.
// Logit loads: from shared memory, or through L2 (.cg) so that values written
// by other CTAs of the same kernel are seen.
template <bool kSmem>
__device__ __forceinline__ float load_logit(const float *row, int e) {
  return kSmem ? row[e] : __ldcg(row + e);
}

template <int NPL, bool kSmem = false>
__device__ __forceinline__ void warp_topk_regs_sel(const float *row, int E, int k, int lane, int &e_out, float &v_out) {
  float v[NPL];
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int e = lane + 32 * j;
    float t = e < E ? load_logit<kSmem>(row, e) : -INFINITY;
    if (t != t) t = -INFINITY;
    v[j] = t;
  }
  float lastv = INFINITY;
  int laste = -1;
  float myv = -INFINITY;
  int mye = 0;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int e = lane + 32 * j;  // increasing in j: the first of equal values has the lower index
      const float t = v[j];
      const bool avail = e < E && ((t < lastv) || (t == lastv && e > laste));
      if (avail && (be == 0x7fffffff || t > bv)) {
        bv = t;
        be = e;
      }
    }
    warp_argmax(bv, be);
    lastv = bv;
    laste = be;
    if (lane == r) {
      myv = bv;
      mye = be;
    }
  }
  e_out = mye;
  v_out = myv;
}

template <int NPL, bool kSmem = false>
__device__ __forceinline__ void warp_topk_regs(const float *row, int E, int k, int lane, int &e_out, float &w_out) {
  float v;
  warp_topk_regs_sel<NPL, kSmem>(row, E, k, lane, e_out, v);
  w_out = topk_softmax(v, lane, k);
}

// Top-k of one token's logits (one warp): k rounds, each taking the largest
// logit strictly after the previous winner in the order (logit desc, index
// asc); NaN ranks as -inf.  Lane j < k returns winner j (e) and its weight,
// the fp32 softmax over the k winners.  Logits are read through L2 (.cg) so
// values written by other CTAs of the same kernel are seen.
__device__ __forceinline__ void warp_topk(const float *row, int E, int k, int lane, int &e_out, float &w_out) {
  float lastv = INFINITY;
  int laste = -1;
  float myv = -INFINITY;
  int mye = 0;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      float v = __ldcg(row + e);
      if (v != v) v = -INFINITY;
      const bool avail = (v < lastv) || (v == lastv && e > laste);
      if (avail && (v > bv || (v == bv && e < be))) {
        bv = v;
        be = e;
      }
    }
    warp_argmax(bv, be);
    lastv = bv;
    laste = be;
    if (lane == r) {
      myv = bv;
      mye = be;
    }
  }
  e_out = mye;
  w_out = topk_softmax(myv, lane, k);
}

// Monotonic 32-bit key of a float (larger float -> larger key); NaN ranks as -inf.
__device__ __forceinline__ uint32_t float_key(float v) {
  if (v != v) v = -INFINITY;
  if (v == 0.f) v = 0.f;  // -0 and +0 are equal logits (the index decides)
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-k by threshold, filter and rank (E <= 32 * NPL, one warp).  Every
// (logit, index) is ranked by the 64-bit key float_key(logit) << 32 | ~index,
// so that "larger" is the selection order (logit desc, index asc).  The k-th
// largest of the 32 lane maxima, L, bounds the k-th largest value from below;
// the values at or above it (usually a few more than k) are compacted into
// shared memory and ranked by counting.  Falls back to warp_topk_regs when
// more than 32 values pass.  Few dependent steps: shared-memory broadcasts
// instead of shuffle chains.  `scratch` is 64 uint64 of shared memory private
// to the warp.  Same selection and softmax as warp_topk, hence the same result.
// kFull: E == 32 * NPL, so every lane loads all its values with no bounds test
// (the run-time test around each load costs about 1.7k cycles per call on B200).
template <int NPL, bool kSmem = false, bool kFull = false>
__device__ __forceinline__ void warp_topk_fast_sel(const float *row, int E, int k, int lane, uint64_t *scratch,
                                                   int &e_out, float &v_out) {
  uint32_t kv[NPL];
  uint32_t mk = 0;
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int e = lane + 32 * j;
    kv[j] = (kFull || e < E) ? float_key(load_logit<kSmem>(row, e)) : 0u;
    mk = kv[j] > mk ? kv[j] : mk;
  }
  uint32_t *lmax = reinterpret_cast<uint32_t *>(scratch + 32);  // 32 lane maxima
  lmax[lane] = mk;
  __syncwarp();
  int ge = 0;  // lane maxima >= mine
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 q = reinterpret_cast<const uint4 *>(lmax)[i];
    ge += (q.x >= mk) + (q.y >= mk) + (q.z >= mk) + (q.w >= mk);
  }
  // L = the k-th largest lane maximum: the largest mk that at least k lane maxima reach
  const uint32_t L = __reduce_max_sync(0xffffffffu, ge >= k ? mk : 0u);
  int cnt = 0;
#pragma unroll
  for (int j = 0; j < NPL; ++j) cnt += kv[j] >= L;
  const int total = __reduce_add_sync(0xffffffffu, cnt);
  if (total > 32) {
    __syncwarp();
    warp_topk_regs_sel<NPL, kSmem>(row, E, k, lane, e_out, v_out);
    return;
  }
  int pos = cnt;  // exclusive prefix of the candidate counts
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, pos, off);
    if (lane >= off) pos += v;
  }
  pos -= cnt;
  __syncwarp();
#pragma unroll
  for (int j = 0; j < NPL; ++j)
    if (kv[j] >= L) scratch[pos++] = ((uint64_t)kv[j] << 32) | (uint32_t)~(lane + 32 * j);
  __syncwarp();
  const uint64_t cand = lane < total ? scratch[lane] : 0ull;
  int r = 0;
#pragma unroll
  for (int o = 0; o < 32; o += 2) {
    const ulonglong2 q = reinterpret_cast<const ulonglong2 *>(scratch)[o >> 1];
    r += (o < total && q.x > cand) + (o + 1 < total && q.y > cand);
  }
  __syncwarp();
  if (lane < total && r < k) scratch[32 + r] = cand;
  __syncwarp();
  const uint64_t mine = lane < k ? scratch[32 + lane] : 0ull;
  __syncwarp();
  e_out = (int)~(uint32_t)mine;
  v_out = key_float((uint32_t)(mine >> 32));
}

// Selection and weights (fp32 softmax over the k winners, lane j < k holding winner j).
template <int NPL, bool kSmem = false, bool kFull = false>
__device__ __forceinline__ void warp_topk_fast(const float *row, int E, int k, int lane, uint64_t *scratch,
                                               int &e_out, float &w_out) {
  float v;
  warp_topk_fast_sel<NPL, kSmem, kFull>(row, E, k, lane, scratch, e_out, v);
  w_out = topk_softmax(v, lane, k);
}

}  // namespace moe
