// Repacking, routing, dispatch, combine and the between-layer RMSNorm (sm_100a).
//
// Routing follows the problem statement of the pages: each token goes to
// top_k of n_experts routed experts plus one shared expert (Strata tuning
// page, section 2 model table; devlabs page, section 1).  The selection rule
// (largest logit, ties to the lower index), the fp32 softmax over the
// selected set and the bias placement are this library's stated readings.
#include <float.h>

#include <algorithm>

#include "kernels.cuh"
#include "router.cuh"
#include "sync.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// moe_pack_q2: canonical 10-byte blocks -> fragment-ordered units.
//
// A unit is a 16-row tile.  Gate/up unit u: tile rows 0-7 are gate rows
// 8u..8u+7, tile rows 8-15 are up rows 8u..8u+7.  Down unit u: tile rows are
// down rows 16u..16u+15.  Along K the unit is cut into groups of 4 blocks
// (128 weights); a group stores 32 lanes x 16 bytes of codes followed by
// 8 x 16 bytes of scales.  Lane (g = lane/4, c = lane%4) owns tile rows g and
// g+8; its word for block b holds, for k16 step s in {0,1}, the k pairs
// (4c, 4c+1) and (4c+2, 4c+3) of both rows, one pair per A-fragment register P:
// P = 0: row g, k 4c;  P = 1: row g+8, k 4c;  P = 2: row g, k 4c+2;  P = 3: row g+8, k 4c+2
// (k relative to 32b + 16s); the even-k code sits at bit 8s + {0,4,2,6}[P],
// the odd-k code 16 bits higher.  Scales: for g in 0..7, block 0..3:
// (d[row g], d[row g+8]).
__global__ void pack_q2_kernel(const uint8_t *__restrict__ canon, uint8_t *__restrict__ packed, int n_experts,
                               PackedGeom G, size_t canon_stride) {
  const int ug_per_expert = G.gu_units * G.gu_groups + G.dn_units * G.dn_groups;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)n_experts * ug_per_expert * 32;
  if (tid >= total) return;
  const int lane = (int)(tid & 31);
  const long long r = tid >> 5;
  const int ug = (int)(r % ug_per_expert);
  const int e = (int)(r / ug_per_expert);
  const uint8_t *ce = canon + (size_t)e * canon_stride;
  uint8_t *pe = packed + (size_t)e * G.expert_bytes;
  const size_t gu_mat_bytes = (size_t)G.I * G.H / kQBlock * kCanonBlockBytes;
  const bool is_gu = ug < G.gu_units * G.gu_groups;
  int unit, grp, ncols;
  uint8_t *dst;
  if (is_gu) {
    unit = ug / G.gu_groups;
    grp = ug % G.gu_groups;
    ncols = G.H;
    dst = pe + (size_t)unit * G.gu_unit_bytes + (size_t)grp * kGroupBytes;
  } else {
    const int v = ug - G.gu_units * G.gu_groups;
    unit = v / G.dn_groups;
    grp = v % G.dn_groups;
    ncols = G.I;
    dst = pe + G.gu_bytes + (size_t)unit * G.dn_unit_bytes + (size_t)grp * kGroupBytes;
  }
  const int nb = ncols / kQBlock;
  auto row_ptr = [&](int rho) -> const uint8_t * {
    if (is_gu) {
      return rho < 8 ? ce + (size_t)(8 * unit + rho) * nb * kCanonBlockBytes
                     : ce + gu_mat_bytes + (size_t)(8 * unit + rho - 8) * nb * kCanonBlockBytes;
    }
    return ce + 2 * gu_mat_bytes + (size_t)(16 * unit + rho) * nb * kCanonBlockBytes;
  };
  auto code = [&](int rho, int k) -> uint32_t {
    const uint8_t *blk = row_ptr(rho) + (size_t)(k / kQBlock) * kCanonBlockBytes;
    const int j = k % kQBlock;
    return (blk[2 + (j >> 2)] >> (2 * (j & 3))) & 3u;
  };
  const int g = lane >> 2, c = lane & 3;
  uint32_t words[4];
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const int b = grp * 4 + wi;
    uint32_t w = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const int s = p >> 2, P = p & 3;
      const int rho = g + 8 * (P & 1);
      const int k = 32 * b + 16 * s + 4 * c + 2 * (P >> 1);
      const int pos = 8 * s + pair_pos(P);
      w |= code(rho, k) << pos;
      w |= code(rho, k + 1) << (16 + pos);
    }
    words[wi] = w;
  }
  *reinterpret_cast<uint4 *>(dst + lane * 16) = make_uint4(words[0], words[1], words[2], words[3]);
  if (lane < 8) {
    uint32_t sc[4];
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const int b = grp * 4 + wi;
      const uint8_t *b0 = row_ptr(lane) + (size_t)b * kCanonBlockBytes;
      const uint8_t *b1 = row_ptr(lane + 8) + (size_t)b * kCanonBlockBytes;
      const uint32_t d0 = b0[0] | ((uint32_t)b0[1] << 8);
      const uint32_t d1 = b1[0] | ((uint32_t)b1[1] << 8);
      sc[wi] = d0 | (d1 << 16);
    }
    *reinterpret_cast<uint4 *>(dst + kGroupCodeBytes + lane * 16) = make_uint4(sc[0], sc[1], sc[2], sc[3]);
  }
}

cudaError_t launch_pack(const uint8_t *canon, uint8_t *packed, int n_experts, const PackedGeom &G,
                        size_t canon_stride, cudaStream_t s) {
  const long long ug = (long long)G.gu_units * G.gu_groups + (long long)G.dn_units * G.dn_groups;
  const long long threads = (long long)n_experts * ug * 32;
  const int bs = 256;
  const long long blocks = (threads + bs - 1) / bs;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  pack_q2_kernel<<<(unsigned)blocks, bs, 0, s>>>(canon, packed, n_experts, G, canon_stride);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Router logits, fp32 accumulation.  Also clears the dispatch bit map for this
// call (stream order puts the clear before the top-k kernel's atomics).

// Few tokens (T <= 8): one CTA of 2 warps per expert row, warp h summing the
// row's half h (router_part), combined in half order.
__global__ void __launch_bounds__(64) router_logits_small_kernel(const uint16_t *__restrict__ x,
                                                                  const float *__restrict__ Wr,
                                                                  const float *__restrict__ bias, int T, int H,
                                                                  int E, float *__restrict__ logits,
                                                                  uint32_t *zero_p, size_t zero_n) {
  clear_range(zero_p, zero_n);
  __shared__ float part[8][kRouterParts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x;
  float acc[8];
  router_part_any<false>(x, H, T, Wr + (size_t)e * H, H, warp, lane, acc);
  if (lane == 0) {
#pragma unroll
    for (int t = 0; t < 8; ++t) part[t][warp] = acc[t];
  }
  __syncthreads();
  if (threadIdx.x < T) logits[(size_t)threadIdx.x * E + e] = router_combine(part[threadIdx.x], bias ? bias[e] : 0.f);
}

// Many tokens without a split-weight workspace (the no-allocation routing
// entry point) or with a hidden size that is not a multiple of 256: legacy
// warp MMAs on the exact 3-way bf16 split of the fp32 router weights, split
// in registers (split3_bf16).  Each 256-wide K slice is accumulated in a fresh
// accumulator and then added to the running fp32 sum.  With a workspace the
// tcgen05 router (router_tc.cu) is used instead.
constexpr int kRbE = 64, kRbT = 32, kRbK = 64, kRbStages = 3;  // CTA tile: experts x tokens x K step
constexpr int kRwStride = kRbK + 8;                                // floats (bank spread for float2 reads)
constexpr int kRxStride = kRbK + 8;                                // bf16
constexpr int kRwBytes = kRbE * kRwStride * 4;
constexpr int kRxBytes = kRbT * kRxStride * 2;
constexpr int kRStageBytes = kRwBytes + kRxBytes;
constexpr int kRouterSmem = kRbStages * kRStageBytes;

__device__ __forceinline__ void cp_async16_zfill(void *dst_smem, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

// CTA tile 64 experts x 32 tokens, 4 warps of 16 experts x 32 tokens; K in
// steps of 64 through a 3-stage cp.async pipeline (rows past E or T read as 0).
__global__ void __launch_bounds__(128) router_logits_mma_kernel(const uint16_t *__restrict__ x,
                                                                 const float *__restrict__ Wr,
                                                                 const float *__restrict__ bias, int T, int H, int E,
                                                                 float *__restrict__ logits, uint32_t *zero_p,
                                                                 size_t zero_n) {
  clear_range(zero_p, zero_n);
  extern __shared__ __align__(16) uint8_t rsm[];
  const int e0 = blockIdx.x * kRbE, t0 = blockIdx.y * kRbT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int nk = H / kRbK;
  auto load_stage = [&](int st, int k0) {
    float *ws = reinterpret_cast<float *>(rsm + st * kRStageBytes);
    uint16_t *xs = reinterpret_cast<uint16_t *>(rsm + st * kRStageBytes + kRwBytes);
#pragma unroll
    for (int j = 0; j < (kRbE * kRbK / 4) / 128; ++j) {
      const int i = tid + 128 * j, r = i / (kRbK / 4), c4 = i % (kRbK / 4);
      const bool ok = e0 + r < E;
      cp_async16_zfill(ws + r * kRwStride + 4 * c4, Wr + (size_t)(ok ? e0 + r : 0) * H + k0 + 4 * c4, ok);
    }
#pragma unroll
    for (int j = 0; j < (kRbT * kRbK / 8) / 128; ++j) {
      const int i = tid + 128 * j, r = i / (kRbK / 8), c8 = i % (kRbK / 8);
      const bool ok = t0 + r < T;
      cp_async16_zfill(xs + r * kRxStride + 8 * c8, x + (size_t)(ok ? t0 + r : 0) * H + k0 + 8 * c8, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[4][4] = {};
  float part[4][4] = {};
  load_stage(0, 0);
  if (nk > 1) load_stage(1, kRbK);
  else asm volatile("cp.async.commit_group;" ::: "memory");
  for (int kt = 0; kt < nk; ++kt) {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();  // stage kt visible to all; stage (kt + 2) % 3 no longer read
    if (kt + 2 < nk) load_stage((kt + 2) % kRbStages, (kt + 2) * kRbK);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    const float *ws = reinterpret_cast<const float *>(rsm + (kt % kRbStages) * kRStageBytes);
    const uint16_t *xs = reinterpret_cast<const uint16_t *>(rsm + (kt % kRbStages) * kRStageBytes + kRwBytes);
#pragma unroll
    for (int kk = 0; kk < kRbK; kk += 16) {
      // A fragments of the three splits: rows 16 * warp + g (+8), k = kk + 2c (+1) and kk + 2c + 8 (+9)
      uint32_t ah[4], am[4], al[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = warp * 16 + g + 8 * (q & 1), col = kk + 2 * c + 8 * (q >> 1);
        const float2 w2 = *reinterpret_cast<const float2 *>(ws + row * kRwStride + col);
        uint16_t h0, m0, l0, h1, m1, l1;
        split3_bf16(w2.x, h0, m0, l0);
        split3_bf16(w2.y, h1, m1, l1);
        ah[q] = h0 | ((uint32_t)h1 << 16);
        am[q] = m0 | ((uint32_t)m1 << 16);
        al[q] = l0 | ((uint32_t)l1 << 16);
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const uint16_t *xr = xs + (nt * 8 + g) * kRxStride + kk + 2 * c;
        const uint32_t b0 = *reinterpret_cast<const uint32_t *>(xr);
        const uint32_t b1 = *reinterpret_cast<const uint32_t *>(xr + 8);
        mma_bf16_16816(part[nt], ah, b0, b1, part[nt]);
        mma_bf16_16816(part[nt], am, b0, b1, part[nt]);
        mma_bf16_16816(part[nt], al, b0, b1, part[nt]);
      }
    }
    if ((((kt + 1) * kRbK) & 255) == 0 || kt + 1 == nk) {  // end of a 256-wide K slice
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[nt][q] += part[nt][q];
          part[nt][q] = 0.f;
        }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // D fragment: (row g, cols 2c, 2c+1), (row g+8, cols 2c, 2c+1); rows = experts, cols = tokens
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = e0 + warp * 16 + g + 8 * (q >> 1);
      const int t = t0 + nt * 8 + 2 * c + (q & 1);
      if (e < E && t < T) logits[(size_t)t * E + e] = acc[nt][q] + (bias ? bias[e] : 0.f);
    }
}

// Top-k per token, one warp per token (see warp_topk); optionally marks the
// token in the expert's membership bit map for the dispatch step.
__global__ void __launch_bounds__(256) topk_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                   int32_t *__restrict__ idx, float *__restrict__ w,
                                                   uint32_t *bitmap, int words) {
  __shared__ __align__(16) uint64_t scratch[8][64];
  const int t = (int)(((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float wt;
  int e;
  const float *row = logits + (size_t)t * E;
  if (E == 512)
    warp_topk_fast<16, false, true>(row, E, k, lane, scratch[threadIdx.x >> 5], e, wt);
  else if (E < 512)
    warp_topk_fast<16>(row, E, k, lane, scratch[threadIdx.x >> 5], e, wt);
  else if (E <= 1024)
    warp_topk_fast<32>(row, E, k, lane, scratch[threadIdx.x >> 5], e, wt);
  else
    warp_topk(row, E, k, lane, e, wt);
  if (lane < k) {
    idx[(size_t)t * k + lane] = e;
    w[(size_t)t * k + lane] = wt;
    if (bitmap) atomicOr(&bitmap[(size_t)e * words + (t >> 5)], 1u << (t & 31));
  }
}

cudaError_t launch_route(const moe_dims &d, const uint16_t *x, const float *Wr, const float *bias, int T,
                         const Workspace &ws, bool with_dispatch_bits, cudaStream_t s) {
  const int H = d.hidden, E = d.n_experts, k = d.top_k;
  if (T <= 8) {
    trace_mark(MOE_KERNEL_ROUTER_LOGITS, false, s);
    router_logits_small_kernel<<<E, 32 * kRouterParts, 0, s>>>(x, Wr, bias, T, H, E, ws.logits, ws.zero_begin, ws.zero_words);
    trace_mark(MOE_KERNEL_ROUTER_LOGITS, true, s);
  } else if (ws.wsplit && router_tc_supported(d, T)) {
    const cudaError_t e0 = launch_router_tc(d, x, Wr, bias, T, ws, s);
    if (e0 != cudaSuccess) return e0;
  } else {
    dim3 grid((E + kRbE - 1) / kRbE, (T + kRbT - 1) / kRbT);
    cudaError_t e0 = cudaFuncSetAttribute(router_logits_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          kRouterSmem);
    if (e0 != cudaSuccess) return e0;
    trace_mark(MOE_KERNEL_ROUTER_LOGITS, false, s);
    router_logits_mma_kernel<<<grid, 128, kRouterSmem, s>>>(x, Wr, bias, T, H, E, ws.logits, ws.zero_begin,
                                                            ws.zero_words);
    trace_mark(MOE_KERNEL_ROUTER_LOGITS, true, s);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int blocks = (T * 32 + 255) / 256;
  trace_mark(MOE_KERNEL_TOPK, false, s);
  topk_kernel<<<blocks, 256, 0, s>>>(ws.logits, T, E, k, ws.idx, ws.w, with_dispatch_bits ? ws.bitmap : nullptr,
                                     ws.words);
  trace_mark(MOE_KERNEL_TOPK, true, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Dispatch: counts, offsets and a stable (expert, token)-ordered permutation.
// The sorted position of slot (t, j) routed to expert e is
//   offsets[e] + #{t' < t : t' routed to e},
// read off the expert's membership bit map with popcounts, so the result is
// independent of thread timing.  The shared expert's slots follow the routed
// ones: position T*k + t.

// One CTA of 1024 threads: per expert (one warp each, in turn) the popcount
// prefix of its membership words and its count; then a block-wide exclusive
// scan gives the offsets and the starts of each expert's work items: tiles of
// 8 tokens for the register-dequant path (experts with at most cold_max
// tokens) and of tc_n tokens for the tcgen05 path (the other experts); the
// shared expert's items follow the routed ones, on the register-dequant list
// when shared_cold, else on the tcgen05 list.
constexpr int kScanThreads = 1024;

__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_sums, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
    int wi = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += t;
    }
    warp_sums[lane] = wi - ws;  // exclusive over warps
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - v;
  total = warp_sums[32];
  __syncthreads();  // warp_sums is reused by the next scan
  return r;
}

// Per expert (one CTA each): exclusive popcount prefix of its membership words
// and its token count.
__global__ void __launch_bounds__(kScanThreads) dispatch_wscan_kernel(const uint32_t *__restrict__ bitmap, int words,
                                                                      uint32_t *__restrict__ wprefix,
                                                                      int32_t *__restrict__ counts) {
  __shared__ int warp_sums[33];
  const int e = blockIdx.x;
  int run = 0;
  for (int w0 = 0; w0 < words; w0 += blockDim.x) {
    const int wi = w0 + threadIdx.x;
    const uint32_t bits = wi < words ? bitmap[(size_t)e * words + wi] : 0u;
    int tot;
    const int ex = block_exclusive_scan(__popc(bits), warp_sums, tot);
    if (wi < words) wprefix[(size_t)e * words + wi] = (uint32_t)(run + ex);
    run += tot;
  }
  if (threadIdx.x == 0) counts[e] = run;
}

// Expert offsets and the work lists from the per-expert counts (one CTA).
__global__ void __launch_bounds__(kScanThreads) dispatch_scan_kernel(int E, int T, int k,
                                                                     const int32_t *__restrict__ counts,
                                                                     int32_t *offsets, int4 *items, uint32_t *n_items,
                                                                     int4 *tc_items, uint32_t *n_tc_items, int tc_n,
                                                                     int cold_max, int shared_cold) {
  __shared__ int warp_sums[33];
  // thread i owns experts [i * per, (i + 1) * per)
  const int per = (E + kScanThreads - 1) / kScanThreads;
  const int eb = threadIdx.x * per, ee = min(E, eb + per);
  int my_cnt = 0, my_items = 0, my_tc = 0;
  for (int i = eb; i < ee; ++i) {
    const int c = counts[i];
    my_cnt += c;
    if (c <= cold_max) my_items += (c + 7) >> 3;
    else my_tc += (c + tc_n - 1) / tc_n;
  }
  int tot_cnt, tot_items, tot_tc;
  int pos = block_exclusive_scan(my_cnt, warp_sums, tot_cnt);
  int it = block_exclusive_scan(my_items, warp_sums, tot_items);
  int itc = block_exclusive_scan(my_tc, warp_sums, tot_tc);
  for (int i = eb; i < ee; ++i) {
    const int c = counts[i];
    offsets[i] = pos;
    if (c <= cold_max)
      for (int j = 0; j < c; j += 8) items[it++] = make_int4(i, pos + j, min(8, c - j), 0);
    else
      for (int j = 0; j < c; j += tc_n) tc_items[itc++] = make_int4(i, pos + j, min(tc_n, c - j), 0);
    pos += c;
  }
  // the shared expert's items follow the routed ones
  const int shared_items = shared_cold ? (T + 7) >> 3 : 0, shared_tc = shared_cold ? 0 : (T + tc_n - 1) / tc_n;
  for (int i = threadIdx.x; i < shared_items; i += blockDim.x)
    items[tot_items + i] = make_int4(E, T * k + 8 * i, min(8, T - 8 * i), 0);
  for (int i = threadIdx.x; i < shared_tc; i += blockDim.x)
    tc_items[tot_tc + i] = make_int4(E, T * k + tc_n * i, min(tc_n, T - tc_n * i), 0);
  if (threadIdx.x == 0) {
    offsets[E] = tot_cnt;  // == T * k when every index was valid
    *n_items = (uint32_t)(tot_items + shared_items);
    *n_tc_items = (uint32_t)(tot_tc + shared_tc);
  }
}

__global__ void dispatch_place_kernel(const int32_t *__restrict__ idx, const float *__restrict__ w, int T, int k,
                                      int E, int words, const uint32_t *__restrict__ bitmap,
                                      const uint32_t *__restrict__ wprefix, const int32_t *__restrict__ offsets,
                                      int32_t *slot_pos, int32_t *sorted_tok, float *sorted_w, int32_t *perm,
                                      uint32_t *status) {
  const long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long routed = (long long)T * k;
  if (s >= routed + T) return;
  if (s < routed) {
    const int t = (int)(s / k);
    const int e = idx[s];
    if (e < 0 || e >= E) {
      set_status(status, kStatusBadIndex);
      slot_pos[s] = -1;  // the combine skips this slot
      return;
    }
    const uint32_t word = bitmap[(size_t)e * words + (t >> 5)];
    const int pos = offsets[e] + (int)wprefix[(size_t)e * words + (t >> 5)] + __popc(word & ((1u << (t & 31)) - 1u));
    slot_pos[s] = pos;
    sorted_tok[pos] = t;
    sorted_w[pos] = w[s];
    if (perm) perm[pos] = (int32_t)s;
  } else {
    const int t = (int)(s - routed);
    sorted_tok[routed + t] = t;
    sorted_w[routed + t] = 1.f;
  }
}

// Membership bits from a routing supplied by the caller (moe_experts_forward).
__global__ void dispatch_bits_kernel(const int32_t *__restrict__ idx, int T, int k, int E, int words,
                                     uint32_t *bitmap, uint32_t *status) {
  const long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= (long long)T * k) return;
  const int t = (int)(s / k);
  const int e = idx[s];
  if (e < 0 || e >= E) {
    set_status(status, kStatusBadIndex);
    return;
  }
  atomicOr(&bitmap[(size_t)e * words + (t >> 5)], 1u << (t & 31));
}

cudaError_t launch_dispatch_bits(const moe_dims &d, int T, const Workspace &ws, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(ws.zero_begin, 0, ws.zero_words * 4, s);
  if (err != cudaSuccess) return err;
  const long long n = (long long)T * d.top_k;
  trace_mark(MOE_KERNEL_DISPATCH_BITS, false, s);
  dispatch_bits_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(ws.idx, T, d.top_k, d.n_experts, ws.words,
                                                                    ws.bitmap, ws.status);
  trace_mark(MOE_KERNEL_DISPATCH_BITS, true, s);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const moe_dims &d, int T, const Workspace &ws, cudaStream_t s) {
  const int E = d.n_experts, k = d.top_k;
  trace_mark(MOE_KERNEL_DISPATCH_SCAN, false, s);
  const int wthreads = std::min(kScanThreads, (ws.words + 31) & ~31);
  dispatch_wscan_kernel<<<E, wthreads, 0, s>>>(ws.bitmap, ws.words, ws.wprefix, ws.counts);
  // few tokens: every expert on the register-dequant list; a prefill chunk: experts with at most
  // cold_expert_tokens(T) tokens there, the rest and the shared expert on the tcgen05 list
  const bool small = T <= 8;
  dispatch_scan_kernel<<<1, kScanThreads, 0, s>>>(E, T, k, ws.counts, ws.offsets, ws.items, ws.n_items, ws.tc_items,
                                                  ws.n_tc_items, ws.tc_item_tokens > 0 ? ws.tc_item_tokens : 64,
                                                  small ? 0x7fffffff : cold_expert_tokens(d, T), small ? 1 : 0);
  trace_mark(MOE_KERNEL_DISPATCH_SCAN, true, s);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const long long n = (long long)T * k + T;
  trace_mark(MOE_KERNEL_DISPATCH_PLACE, false, s);
  dispatch_place_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(ws.idx, ws.w, T, k, E, ws.words, ws.bitmap,
                                                                     ws.wprefix, ws.offsets, ws.slot_pos,
                                                                     ws.sorted_tok, ws.sorted_w, ws.perm, ws.status);
  trace_mark(MOE_KERNEL_DISPATCH_PLACE, true, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Combine: out[t] = Y_shared[t] + sum_j w[t,j] Y[slot(t,j)], fp32 in a fixed
// order (shared first, then j = 0..k-1), rounded once to bf16.
__global__ void combine_kernel(const float *__restrict__ Y, const int32_t *__restrict__ slot_pos,
                               const float *__restrict__ topk_w, int T, int k, int H, uint16_t *__restrict__ out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = H >> 2;
  if (i >= (long long)T * per_row) return;
  const int t = (int)(i / per_row), c4 = (int)(i % per_row);
  float4 acc = reinterpret_cast<const float4 *>(Y + ((size_t)T * k + t) * H)[c4];
  // four slots' rows in flight at a time, accumulated in slot order
  int j = 0;
  for (; j + 4 <= k; j += 4) {
    float4 v[4];
    float wj[4];
    bool ok[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int pos = slot_pos[(size_t)t * k + j + u];
      ok[u] = pos >= 0;  // an invalid slot adds nothing
      wj[u] = topk_w[(size_t)t * k + j + u];
      v[u] = reinterpret_cast<const float4 *>(Y + (size_t)(ok[u] ? pos : 0) * H)[c4];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!ok[u]) continue;
      acc.x = fmaf(wj[u], v[u].x, acc.x);
      acc.y = fmaf(wj[u], v[u].y, acc.y);
      acc.z = fmaf(wj[u], v[u].z, acc.z);
      acc.w = fmaf(wj[u], v[u].w, acc.w);
    }
  }
  for (; j < k; ++j) {
    const int pos = slot_pos[(size_t)t * k + j];
    if (pos < 0) continue;
    const float wj = topk_w[(size_t)t * k + j];
    const float4 v = reinterpret_cast<const float4 *>(Y + (size_t)pos * H)[c4];
    acc.x = fmaf(wj, v.x, acc.x);
    acc.y = fmaf(wj, v.y, acc.y);
    acc.z = fmaf(wj, v.z, acc.z);
    acc.w = fmaf(wj, v.w, acc.w);
  }
  uint2 o;
  o.x = pack_bf16x2(acc.x, acc.y);
  o.y = pack_bf16x2(acc.z, acc.w);
  reinterpret_cast<uint2 *>(out + (size_t)t * H)[c4] = o;
}

cudaError_t launch_combine(const moe_dims &d, int T, const Workspace &ws, uint16_t *out, cudaStream_t s) {
  const long long n = (long long)T * (d.hidden / 4);
  trace_mark(MOE_KERNEL_COMBINE, false, s);
  combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(ws.y, ws.slot_pos, ws.w, T, d.top_k, d.hidden, out);
  trace_mark(MOE_KERNEL_COMBINE, true, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Between layers: resid += y (optional); x_norm = bf16(resid * rsqrt(mean(resid^2) + eps)).  One CTA of 256
// threads per token; the sum of squares is reduced in a fixed order (deterministic).

// Sum over the CTA (blockDim.x a multiple of 32, at most 1024); every thread gets the total.
__device__ __forceinline__ float block_sum(float v, float *part) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    float u = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
    if (threadIdx.x == 0) part[32] = u;
  }
  __syncthreads();
  return part[32];
}

template <typename YT>  // layer output type: uint16_t (bf16 bits) or float
__global__ void __launch_bounds__(256) rmsnorm_residual_kernel(float *__restrict__ resid, const YT *__restrict__ y,
                                                               uint16_t *__restrict__ x_norm, int H, float eps) {
  const int t = blockIdx.x;
  float *r = resid + (size_t)t * H;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    float v = r[i];
    if (y) {
      const YT yv = y[(size_t)t * H + i];
      if constexpr (sizeof(YT) == 2) v += bf16_bits_to_float(yv);
      else v += yv;
      r[i] = v;
    }
    ss = fmaf(v, v, ss);
  }
  __shared__ float part[33];
  const float scale = 1.0f / sqrtf(block_sum(ss, part) / (float)H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x) x_norm[(size_t)t * H + i] = float_to_bf16_bits(r[i] * scale);
}

cudaError_t launch_rmsnorm_residual(float *resid, const uint16_t *y, uint16_t *x_norm, int T, int H, float eps,
                                    cudaStream_t s) {
  rmsnorm_residual_kernel<uint16_t><<<T, 256, 0, s>>>(resid, y, x_norm, H, eps);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_residual_f32(float *resid, const float *y, uint16_t *x_norm, int T, int H, float eps,
                                        cudaStream_t s) {
  rmsnorm_residual_kernel<float><<<T, 256, 0, s>>>(resid, y, x_norm, H, eps);
  return cudaGetLastError();
}

// Combine fused with the residual and the next layer's RMSNorm (one CTA per token): y = Y_shared[t] +
// sum_j w[t,j] Y[slot(t,j)] in the combine's fixed order (fp32, never rounded), resid += y, x_norm =
// bf16(resid / sqrt(mean(resid^2) + eps)).
__global__ void __launch_bounds__(256) combine_rmsnorm_kernel(const float *__restrict__ Y,
                                                              const int32_t *__restrict__ slot_pos,
                                                              const float *__restrict__ topk_w, int T, int k, int H,
                                                              float *__restrict__ resid, uint16_t *__restrict__ x_norm,
                                                              float eps) {
  const int t = blockIdx.x;
  float4 *r4 = reinterpret_cast<float4 *>(resid + (size_t)t * H);
  __shared__ int pos_s[32];
  __shared__ float w_s[32];
  __shared__ float part[33];
  if (threadIdx.x < k) {
    pos_s[threadIdx.x] = slot_pos[(size_t)t * k + threadIdx.x];
    w_s[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  float ss = 0.f;
  for (int c4 = threadIdx.x; c4 < H / 4; c4 += blockDim.x) {
    float4 acc = reinterpret_cast<const float4 *>(Y + ((size_t)T * k + t) * H)[c4];
    for (int j = 0; j < k; ++j) {
      const int pos = pos_s[j];
      if (pos < 0) continue;  // an invalid slot adds nothing
      const float wj = w_s[j];
      const float4 v = reinterpret_cast<const float4 *>(Y + (size_t)pos * H)[c4];
      acc.x = fmaf(wj, v.x, acc.x);
      acc.y = fmaf(wj, v.y, acc.y);
      acc.z = fmaf(wj, v.z, acc.z);
      acc.w = fmaf(wj, v.w, acc.w);
    }
    float4 rv = r4[c4];
    rv.x += acc.x;
    rv.y += acc.y;
    rv.z += acc.z;
    rv.w += acc.w;
    r4[c4] = rv;
    ss = fmaf(rv.x, rv.x, ss);
    ss = fmaf(rv.y, rv.y, ss);
    ss = fmaf(rv.z, rv.z, ss);
    ss = fmaf(rv.w, rv.w, ss);
  }
  const float scale = 1.0f / sqrtf(block_sum(ss, part) / (float)H + eps);
  for (int c4 = threadIdx.x; c4 < H / 4; c4 += blockDim.x) {
    const float4 rv = r4[c4];
    uint2 o;
    o.x = pack_bf16x2(rv.x * scale, rv.y * scale);
    o.y = pack_bf16x2(rv.z * scale, rv.w * scale);
    reinterpret_cast<uint2 *>(x_norm + (size_t)t * H)[c4] = o;
  }
}

cudaError_t launch_combine_rmsnorm(const moe_dims &d, int T, const Workspace &ws, float *resid, uint16_t *x_norm,
                                   float eps, cudaStream_t s) {
  trace_mark(MOE_KERNEL_COMBINE, false, s);
  combine_rmsnorm_kernel<<<T, 256, 0, s>>>(ws.y, ws.slot_pos, ws.w, T, d.top_k, d.hidden, resid, x_norm, eps);
  trace_mark(MOE_KERNEL_COMBINE, true, s);
  return cudaGetLastError();
}

}  // namespace moe
