// Fused decode/verify-window layer (T <= 8 tokens) in one persistent,
// cooperatively launched kernel (sm_100a).  One CTA per SM: 16 consumer
// warps and 1 producer warp.
//
//  A  The producer bulk-copies (TMA engine) the tokens and this CTA's router
//     rows into shared memory and prefetches its slice of the shared expert
//     into L2.  Consumers compute the router rows (4 warps per row, one
//     quarter of K each) and the correction sums of the biased decode.
//     -- grid barrier: all logits written --
//  B  Every CTA selects the top-k of every token (threshold + rank, one warp
//     per token) and builds the same sorted list of touched experts plus the
//     shared expert.
//  C  Work lists, expert-major, cut into equal contiguous ranges per CTA:
//     gate/up units (expert, 8 intermediate rows) and down pairs (expert, 16
//     output rows).  The producer streams the CTA's units into a ring of
//     shared-memory stages as stages free up.  Gate/up: K split over the 16
//     warps, partial sums reduced through a double-buffered shared slot by a
//     rotating epilogue warp (mbarrier hand-off, no CTA-wide barrier), which
//     writes h = silu(g) * u (bf16).  At the end the CTA publishes, per
//     expert, how many of its units are done.
//  D  Down pairs, 4 warps per pair (K split), once the expert's h is
//     complete (per-expert counter, bounded wait): partial = w[t, e] * (Wd_e
//     h_e) per (expert, tile).  The last CTA to contribute to a tile sums its
//     partials in expert order and writes out (bf16).
// Dequantisation happens in registers and feeds m16n8k16 tensor-core MMAs
// with the tokens as the 8 columns; gate/up uses the biased decode with the
// -1 offset folded into the accumulator start (decode_q2_biased), down the
// exact decode.  Every wait is bounded (sync.cuh).
#include "kernels.cuh"
#include "router.cuh"
#include "sync.cuh"

namespace moe {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxTok = 8;
constexpr int kMaxSel = 128;              // T * top_k
constexpr int kMaxEntries = kMaxSel + 1;  // touched experts + shared
constexpr int kMaxE = 1024;
constexpr int kNR = 2;                    // gate/up reduction slots
constexpr int kBarConsumers = 1;          // named barrier ids (0 = __syncthreads)
constexpr int kBarPairLane0 = 2;          // 2..5

struct DecodeArgs {
  const uint16_t *x;
  const float *Wr;
  const float *bias;
  const uint8_t *experts;
  const uint8_t *shared;
  PackedGeom G;
  int T, E, k;
  float *logits;       // [T][E]
  uint16_t *h;         // [T][k+1][I]
  float *partial;      // [entries][dn_units][32][4]
  uint32_t *tile_cnt;  // [dn_units] then ready[kMaxEntries]
  uint32_t *gbar;      // [0] count, [1] generation
  int32_t *idx_out;    // optional [T][k]
  float *w_out;        // optional [T][k]
  uint16_t *out;       // [T][H]
  uint32_t *status;
  int ns;              // ring stages
  uint32_t stage_bytes;
};

struct SmemLayout {
  uint32_t bars, xs, corr, rpart, red, sel_idx, sel_w, bitmap, wpre, ent, tokj, tokw, misc, ring, total;
};

__host__ __device__ inline uint32_t align_to(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout smem_layout(int T, int H, int ns, uint32_t stage_bytes) {
  SmemLayout L;
  uint32_t o = 0;
  L.bars = o;  // full[ns], empty[ns], rbar, xbar, rfull[kNR], rfree[kNR]
  o = align_to(o + 8u * (2 * ns + 2 + 2 * kNR), 16);
  L.xs = o;
  o = align_to(o + (uint32_t)T * (H + 16) * 2, 16);
  L.corr = o;
  o = align_to(o + (uint32_t)(H / 32) * kMaxTok * 4, 16);
  L.rpart = o;  // [4 rows][8 tokens][4 quarters]
  o += 4 * kMaxTok * 4 * 4;
  L.red = o;    // gate/up: [kNR][16 warps][32][4]; down: [2][4 lanes][4][32][4]; top-k scratch
  o += kNR * kConsumerWarps * 32 * 16;
  L.sel_idx = o;
  o += kMaxSel * 4;
  L.sel_w = o;
  o += kMaxSel * 4;
  L.bitmap = o;
  o += (kMaxE / 32) * 4;
  L.wpre = o;
  o += (kMaxE / 32) * 4;
  L.ent = o;
  o = align_to(o + kMaxEntries * 4, 16);
  L.tokj = o;
  o = align_to(o + kMaxEntries * kMaxTok, 16);
  L.tokw = o;
  o = align_to(o + kMaxEntries * kMaxTok * 4, 16);
  L.misc = o;
  o += 32;
  L.ring = align_to(o, 128);
  L.total = L.ring + (uint32_t)ns * stage_bytes;
  return L;
}

// B-operand scale 1/4 for the fragment registers of k pair (4c+2, 4c+3); exact.
__device__ __forceinline__ uint32_t bf16x2_quarter(uint32_t v) { return bf16x2_fma(v, 0x3E803E80u, 0x80008000u); }

template <int GPW>  // gate/up block groups per consumer warp (H / 128 / 16)
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const PackedGeom &G = a.G;
  const int T = a.T, E = a.E, K = a.k, H = G.H, I = G.I;
  const SmemLayout L = smem_layout(T, H, a.ns, a.stage_bytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *empty = full + a.ns;
  uint64_t *rbar = empty + a.ns;
  uint64_t *xbar = rbar + 1;
  uint64_t *rfull = xbar + 1;
  uint64_t *rfree = rfull + kNR;
  uint16_t *xs = reinterpret_cast<uint16_t *>(smem + L.xs);
  float *corr = reinterpret_cast<float *>(smem + L.corr);
  float *rpart = reinterpret_cast<float *>(smem + L.rpart);
  float *red = reinterpret_cast<float *>(smem + L.red);
  int *sel_idx = reinterpret_cast<int *>(smem + L.sel_idx);
  float *sel_w = reinterpret_cast<float *>(smem + L.sel_w);
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + L.bitmap);
  uint32_t *wpre = reinterpret_cast<uint32_t *>(smem + L.wpre);
  int *ent = reinterpret_cast<int *>(smem + L.ent);
  int8_t *tokj = reinterpret_cast<int8_t *>(smem + L.tokj);
  float *tokw = reinterpret_cast<float *>(smem + L.tokw);
  int *misc = reinterpret_cast<int *>(smem + L.misc);  // [0] entries [1] abort [2] barrier flag [3] done tiles
  uint8_t *ring = smem + L.ring;
  uint32_t *ready = a.tile_cnt + G.dn_units;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_producer = warp == kConsumerWarps;
  const int g = lane >> 2, c = lane & 3;
  const int xstride = H + 16;
  const int n_rrows = E > (int)blockIdx.x ? (E - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  float *wr_s = reinterpret_cast<float *>(ring);  // router rows live in the ring until phase C

  // A wait that hits its limit marks the CTA aborted; later waits are skipped
  // so every warp keeps the same control flow and the kernel ends in bounded
  // time with the timeout bit set.
  auto bounded_wait = [&](uint64_t *bar, uint32_t parity) {
    if (*reinterpret_cast<volatile int *>(&misc[1])) return;
    if (!mbar_wait(bar, parity)) {
      set_status(a.status, kStatusTimeout);
      misc[1] = 1;
    }
  };

  // ---------------- phase A: set-up, router ----------------
  if (tid == 0) {
    for (int i = 0; i < a.ns; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    mbar_init(rbar, 1);
    mbar_init(xbar, 1);
    for (int i = 0; i < kNR; ++i) {
      mbar_init(&rfull[i], kConsumerWarps);
      mbar_init(&rfree[i], 1);
    }
    mbar_fence_init();
    for (int i = 0; i < 8; ++i) misc[i] = 0;
  }
  __syncthreads();

  if (is_producer) {
    if (lane == 0) {
      mbar_arrive_expect_tx(xbar, (uint32_t)(T * H * 2));
      for (int t = 0; t < T; ++t) bulk_g2s(xs + t * xstride, a.x + (size_t)t * H, (uint32_t)(H * 2), xbar);
      if (n_rrows > 0) {
        mbar_arrive_expect_tx(rbar, (uint32_t)(n_rrows * H * 4));
        for (int r = 0; r < n_rrows; ++r)
          bulk_g2s(wr_s + (size_t)r * H, a.Wr + (size_t)(blockIdx.x + (size_t)gridDim.x * r) * H, (uint32_t)(H * 4),
                   rbar);
      }
      const size_t per = ((G.expert_bytes + gridDim.x - 1) / gridDim.x + 15) & ~(size_t)15;
      const size_t off = per * blockIdx.x;
      if (off < G.expert_bytes) {
        const size_t n = min(per, G.expert_bytes - off);
        for (size_t o = 0; o < n; o += 32768)
          bulk_prefetch_l2(a.shared + off + o, (uint32_t)min((size_t)32768, n - o));
      }
    }
  } else {
    if (blockIdx.x == 0)
      for (int i = tid; i < G.dn_units + kMaxEntries; i += kConsumers) a.tile_cnt[i] = 0u;
    bounded_wait(xbar, 0);
    // correction sums of the biased decode: C[b][t] = sum_j c_j x[t][32b + j], c_j = 129 (j%4 < 2) or 33
    for (int i = tid; i < (H / 32) * T; i += kConsumers) {
      const int b = i / T, t = i % T;
      const uint4 *xr = reinterpret_cast<const uint4 *>(xs + t * xstride + 32 * b);
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = xr[q];
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2) {  // elements j = 8q + 2h2 (even) and j + 1
          const float coef = (h2 & 1) ? 33.f : 129.f;
          s = fmaf(coef, __uint_as_float(wd[h2] << 16), s);
          s = fmaf(coef, __uint_as_float(wd[h2] & 0xffff0000u), s);
        }
      }
      corr[b * kMaxTok + t] = s;
    }
    bounded_wait(rbar, 0);
    for (int r0 = 0; r0 < n_rrows; r0 += 4) {
      const int r = r0 + (warp >> 2), q = warp & 3;
      if (r < n_rrows) {
        float acc[8];
        router_quarter<true>(xs, xstride, T, wr_s + (size_t)r * H, H, q, lane, acc);
        if (lane == 0) {
#pragma unroll
          for (int t = 0; t < 8; ++t) rpart[((r - r0) * kMaxTok + t) * 4 + q] = acc[t];
        }
      }
      named_bar(kBarConsumers, kConsumers);
      if (tid < 4 * T) {
        const int rr = tid / T, t = tid % T;
        if (r0 + rr < n_rrows) {
          const int e = blockIdx.x + gridDim.x * (r0 + rr);
          a.logits[(size_t)t * E + e] = router_combine(rpart + (rr * kMaxTok + t) * 4, a.bias ? a.bias[e] : 0.f);
        }
      }
      named_bar(kBarConsumers, kConsumers);
    }
    grid_barrier(&a.gbar[0], &a.gbar[1], kBarConsumers, kConsumers, tid == 0, a.status, &misc[2]);

    // ---------------- phase B: top-k and the touched-expert list ----------------
    if (warp < T) {
      int e;
      float wt;
      uint64_t *scratch = reinterpret_cast<uint64_t *>(red) + warp * 64;
      if (E <= 512)
        warp_topk_fast<16>(a.logits + (size_t)warp * E, E, K, lane, scratch, e, wt);
      else
        warp_topk_fast<32>(a.logits + (size_t)warp * E, E, K, lane, scratch, e, wt);
      if (lane < K) {
        sel_idx[warp * K + lane] = e;
        sel_w[warp * K + lane] = wt;
        if (blockIdx.x == 0 && a.idx_out) {
          a.idx_out[warp * K + lane] = e;
          a.w_out[warp * K + lane] = wt;
        }
      }
    }
    named_bar(kBarConsumers, kConsumers);
    if (warp == 0) {
      bitmap[lane] = 0u;
      __syncwarp();
      for (int i = lane; i < T * K; i += 32) atomicOr(&bitmap[sel_idx[i] >> 5], 1u << (sel_idx[i] & 31));
      __syncwarp();
      const uint32_t word = bitmap[lane];
      const uint32_t cnt = __popc(word);
      uint32_t incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const uint32_t pre = incl - cnt;
      wpre[lane] = pre;
      uint32_t wbits = word;
      for (uint32_t r = pre; wbits; ++r) {
        const int b = __ffs(wbits) - 1;
        wbits &= wbits - 1;
        ent[r] = lane * 32 + b;
      }
      const int U = __shfl_sync(0xffffffffu, (int)incl, 31);
      for (int i = lane; i < (U + 1) * kMaxTok; i += 32) {
        tokj[i] = -1;
        tokw[i] = 0.f;
      }
      __syncwarp();
      for (int i = lane; i < T * K; i += 32) {
        const int t = i / K, j = i % K, e = sel_idx[i];
        const int r = wpre[e >> 5] + __popc(bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
        tokj[r * kMaxTok + t] = (int8_t)j;
        tokw[r * kMaxTok + t] = sel_w[i];
      }
      if (lane < T) {
        tokj[U * kMaxTok + lane] = (int8_t)K;  // shared expert: slot k, weight 1
        tokw[U * kMaxTok + lane] = 1.f;
      }
      if (lane == 0) {
        ent[U] = E;
        misc[0] = U + 1;
      }
    }
  }
  __syncthreads();  // the list is visible to the producer as well

  const int nent = misc[0];
  const int n_gu = nent * G.gu_units, n_dn = nent * G.dn_units;
  const int g0 = (int)((long long)n_gu * blockIdx.x / gridDim.x);
  const int g1 = (int)((long long)n_gu * (blockIdx.x + 1) / gridDim.x);
  const int d0 = (int)((long long)n_dn * blockIdx.x / gridDim.x);
  const int d1 = (int)((long long)n_dn * (blockIdx.x + 1) / gridDim.x);
  const int pps = (int)(a.stage_bytes / G.dn_unit_bytes);  // down pairs per stage
  const int n_gu_st = g1 - g0;
  const int n_dn_st = (d1 - d0 + pps - 1) / pps;
  const int n_st = n_gu_st + n_dn_st;
  auto expert_ptr = [&](int entry) -> const uint8_t * {
    const int e = ent[entry];
    return e == E ? a.shared : a.experts + (size_t)e * G.expert_bytes;
  };

  if (is_producer) {
    // ---------------- producer: stream this CTA's units into the ring ----------------
    if (lane == 0) {
      int issued = 0;
      for (int s = 0; s < n_st; ++s) {
        const int slot = s % a.ns;
        if (*reinterpret_cast<volatile int *>(&misc[1]) || !mbar_wait(&empty[slot], ((s / a.ns) & 1) ^ 1)) {
          set_status(a.status, kStatusTimeout);
          misc[1] = 1;
          break;
        }
        uint8_t *dst = ring + (size_t)slot * a.stage_bytes;
        if (s < n_gu_st) {
          const int id = g0 + s;
          const uint8_t *src = expert_ptr(id / G.gu_units) + (size_t)(id % G.gu_units) * G.gu_unit_bytes;
          mbar_arrive_expect_tx(&full[slot], (uint32_t)G.gu_unit_bytes);
          bulk_g2s(dst, src, (uint32_t)G.gu_unit_bytes, &full[slot]);
        } else {
          const int q0 = d0 + (s - n_gu_st) * pps, q1 = min(d1, q0 + pps);
          mbar_arrive_expect_tx(&full[slot], (uint32_t)((q1 - q0) * G.dn_unit_bytes));
          for (int q = q0; q < q1; ++q) {
            const uint8_t *src =
                expert_ptr(q / G.dn_units) + G.gu_bytes + (size_t)(q % G.dn_units) * G.dn_unit_bytes;
            bulk_g2s(dst + (size_t)(q - q0) * G.dn_unit_bytes, src, (uint32_t)G.dn_unit_bytes, &full[slot]);
          }
        }
        issued = s + 1;
      }
      // Before the CTA may exit, every copy this thread issued must have landed.
      for (int s = max(0, issued - a.ns); s < issued; ++s)
        if (!mbar_wait(&full[s % a.ns], (s / a.ns) & 1)) set_status(a.status, kStatusTimeout);
    }
    return;
  }

  // ---------------- consumers, phase C: gate/up + SwiGLU ----------------
  const int kw = warp;  // K split over the 16 consumer warps
  uint32_t B[GPW][4][2][2];
  float negC[GPW][4][2];
#pragma unroll
  for (int gi = 0; gi < GPW; ++gi)
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      const int b = (kw * GPW + gi) * 4 + blk;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        uint2 v = make_uint2(0u, 0u);
        if (g < T) v = *reinterpret_cast<const uint2 *>(xs + g * xstride + 32 * b + 16 * s + 4 * c);
        B[gi][blk][s][0] = v.x;
        B[gi][blk][s][1] = bf16x2_quarter(v.y);
      }
      negC[gi][blk][0] = 2 * c < T ? -corr[b * kMaxTok + 2 * c] : 0.f;
      negC[gi][blk][1] = 2 * c + 1 < T ? -corr[b * kMaxTok + 2 * c + 1] : 0.f;
    }

  int s_idx = 0;
  for (; s_idx < n_gu_st; ++s_idx) {
    const int slot = s_idx % a.ns;
    bounded_wait(&full[slot], (s_idx / a.ns) & 1);
    const uint8_t *st = ring + (size_t)slot * a.stage_bytes;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int gi = 0; gi < GPW; ++gi) {
      const uint8_t *gp = st + (size_t)(kw * GPW + gi) * kGroupBytes;
      const uint4 cw = lds128(gp + lane * 16);
      const uint4 sw = lds128(gp + kGroupCodeBytes + g * 16);
      const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
      const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t p[8];
        decode_q2_biased(cws[blk], p);
        const uint32_t a0[4] = {p[0], p[1], p[2], p[3]};
        const uint32_t a1[4] = {p[4], p[5], p[6], p[7]};
        const float cin[4] = {negC[gi][blk][0], negC[gi][blk][1], negC[gi][blk][0], negC[gi][blk][1]};
        float d[4];
        mma_bf16_16816(d, a0, B[gi][blk][0][0], B[gi][blk][0][1], cin);
        mma_bf16_16816(d, a1, B[gi][blk][1][0], B[gi][blk][1][1], d);
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2 *>(&sws[blk]));
        acc[0] = fmaf(s2.x, d[0], acc[0]);
        acc[1] = fmaf(s2.x, d[1], acc[1]);
        acc[2] = fmaf(s2.y, d[2], acc[2]);
        acc[3] = fmaf(s2.y, d[3], acc[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    const int rs = s_idx % kNR, use = s_idx / kNR;
    if (use > 0) bounded_wait(&rfree[rs], (use - 1) & 1);  // epilogue of unit s_idx - kNR done
    float *rb = red + rs * (kConsumerWarps * 32 * 4);
    *reinterpret_cast<float4 *>(rb + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&rfull[rs]);
    if (warp == s_idx % kConsumerWarps) {
      // epilogue for this unit: sum the 16 partials (warp order), SwiGLU, store h
      bounded_wait(&rfull[rs], use & 1);
      float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float4 v = *reinterpret_cast<const float4 *>(rb + (w * 32 + lane) * 4);
        sm[0] += v.x;
        sm[1] += v.y;
        sm[2] += v.z;
        sm[3] += v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfree[rs]);
      const int id = g0 + s_idx;
      const int entry = id / G.gu_units, u = id % G.gu_units;
      const int i = 8 * u + g;  // tile rows g (gate) and g+8 (up) share intermediate row i
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int n = 2 * c + half;
        if (n < T) {
          const int j = tokj[entry * kMaxTok + n];
          if (j >= 0)
            a.h[((size_t)n * (K + 1) + j) * I + i] = float_to_bf16_bits(silu_f(sm[half]) * sm[2 + half]);
        }
      }
    }
  }

  // Publish this CTA's finished gate/up units per expert (one fence for all of them).
  named_bar(kBarConsumers, kConsumers);
  if (tid == 0 && g1 > g0) {
    __threadfence();
    for (int entry = g0 / G.gu_units; entry <= (g1 - 1) / G.gu_units; ++entry) {
      const int lo = max(g0, entry * G.gu_units), hi = min(g1, (entry + 1) * G.gu_units);
      atomicAdd(&ready[entry], (uint32_t)(hi - lo));
    }
  }

  // ---------------- consumers, phase D: down projection + combine ----------------
  const int pl = warp >> 2, kd = warp & 3;  // pair lane (0..3), K group (I / 128 == 4)
  int cur_entry = -1;
  uint32_t Bd[4][2][2];
  int dbuf = 0;
  for (int sd = 0; s_idx < n_st; ++s_idx, ++sd) {
    const int slot = s_idx % a.ns;
    bounded_wait(&full[slot], (s_idx / a.ns) & 1);
    const uint8_t *st = ring + (size_t)slot * a.stage_bytes;
    const int q0 = d0 + sd * pps, q1 = min(d1, q0 + pps);
    for (int q = q0 + pl; q < q1; q += 4) {
      const int entry = q / G.dn_units, tile = q % G.dn_units;
      if (entry != cur_entry) {
        cur_entry = entry;
        // wait until every gate/up unit of this expert is published
        if (lane == 0 && !*reinterpret_cast<volatile int *>(&misc[1])) {
          const uint64_t t0 = global_timer_ns();
          while (ld_acquire_gpu(&ready[entry]) < (uint32_t)G.gu_units) {
            if (global_timer_ns() - t0 > kWaitLimitNs) {
              set_status(a.status, kStatusTimeout);
              misc[1] = 1;
              break;
            }
          }
        }
        __syncwarp();
        const int j = g < T ? tokj[entry * kMaxTok + g] : -1;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk)
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            uint2 v = make_uint2(0u, 0u);
            if (j >= 0) v = ldg_cg_v2(a.h + ((size_t)g * (K + 1) + j) * I + 128 * kd + 32 * blk + 16 * s + 4 * c);
            Bd[blk][s][0] = v.x;
            Bd[blk][s][1] = v.y;
          }
      }
      const uint8_t *gp = st + (size_t)(q - q0) * G.dn_unit_bytes + (size_t)kd * kGroupBytes;
      const uint4 cw = lds128(gp + lane * 16);
      const uint4 sw = lds128(gp + kGroupCodeBytes + g * 16);
      const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
      const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t p[8];
        decode_q2_exact(cws[blk], p);
        const uint32_t a0[4] = {p[0], p[1], p[2], p[3]};
        const uint32_t a1[4] = {p[4], p[5], p[6], p[7]};
        const float z[4] = {0.f, 0.f, 0.f, 0.f};
        float d[4];
        mma_bf16_16816(d, a0, Bd[blk][0][0], Bd[blk][0][1], z);
        mma_bf16_16816(d, a1, Bd[blk][1][0], Bd[blk][1][1], d);
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2 *>(&sws[blk]));
        acc[0] = fmaf(s2.x, d[0], acc[0]);
        acc[1] = fmaf(s2.x, d[1], acc[1]);
        acc[2] = fmaf(s2.y, d[2], acc[2]);
        acc[3] = fmaf(s2.y, d[3], acc[3]);
      }
      float *rb = red + ((dbuf * 4 + pl) * 4) * 32 * 4;
      *reinterpret_cast<float4 *>(rb + (kd * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      named_bar(kBarPairLane0 + pl, 128);
      if (kd == 0) {
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 v = *reinterpret_cast<const float4 *>(rb + (w * 32 + lane) * 4);
          sm[0] += v.x;
          sm[1] += v.y;
          sm[2] += v.z;
          sm[3] += v.w;
        }
        const float w0 = tokw[entry * kMaxTok + 2 * c], w1 = tokw[entry * kMaxTok + 2 * c + 1];
        float *pp = a.partial + ((size_t)entry * G.dn_units + tile) * 128;
        *reinterpret_cast<float4 *>(pp + lane * 4) = make_float4(sm[0] * w0, sm[1] * w1, sm[2] * w0, sm[3] * w1);
      }
      dbuf ^= 1;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }

  // Count this CTA's contributions per output tile (one fence per writer
  // warp); the last contributor of a tile sums its partials in expert order.
  int *done_tiles = sel_idx;  // phase-B scratch, free now
  if (kd == 0) __threadfence();
  named_bar(kBarConsumers, kConsumers);
  for (int i = tid; i < d1 - d0; i += kConsumers) {
    const int tile = (d0 + i) % G.dn_units;
    if (atomicAdd(&a.tile_cnt[tile], 1u) == (uint32_t)(nent - 1)) {
      __threadfence();
      done_tiles[atomicAdd(&misc[3], 1)] = tile;
    }
  }
  named_bar(kBarConsumers, kConsumers);
  const int n_done = misc[3];
  for (int i = warp; i < n_done; i += kConsumerWarps) {
    const int tile = done_tiles[i];
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    const float *pp = a.partial + (size_t)tile * 128 + lane * 4;
    int e2 = 0;
    for (; e2 + 4 <= nent; e2 += 4) {  // four loads in flight, summed in expert order
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ldg_cg_f4(pp + (size_t)(e2 + u) * G.dn_units * 128);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        o[0] += v[u].x;
        o[1] += v[u].y;
        o[2] += v[u].z;
        o[3] += v[u].w;
      }
    }
    for (; e2 < nent; ++e2) {
      const float4 v = ldg_cg_f4(pp + (size_t)e2 * G.dn_units * 128);
      o[0] += v.x;
      o[1] += v.y;
      o[2] += v.z;
      o[3] += v.w;
    }
    const int r0 = 16 * tile + g;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int n = 2 * c + half;
      if (n < T) {
        a.out[(size_t)n * H + r0] = float_to_bf16_bits(o[half]);
        a.out[(size_t)n * H + r0 + 8] = float_to_bf16_bits(o[2 + half]);
      }
    }
  }
}

}  // namespace

bool decode_fused_supported(const moe_dims &d, int T) {
  const PackedGeom G = packed_geom(d.hidden, d.inter);
  if (T < 1 || T > kMaxTok || T * d.top_k > kMaxSel || d.n_experts > kMaxE) return false;
  if (G.dn_groups != 4) return false;                         // down: 4 warps x 1 group (inter 512)
  if (G.gu_groups != 16 && G.gu_groups != 32) return false;  // gate/up: 16 warps x 1 or 2 groups
  return true;
}

size_t decode_partial_floats(const moe_dims &d, int T) {
  const PackedGeom G = packed_geom(d.hidden, d.inter);
  const int entries = min(T * d.top_k, d.n_experts) + 1;
  return (size_t)entries * G.dn_units * 128;
}

size_t decode_counter_words(const moe_dims &d) { return (size_t)d.hidden / 16 + kMaxEntries; }

cudaError_t launch_decode_fused(const moe_dims &d, const uint16_t *x, const float *Wr, const float *bias,
                                const uint8_t *experts, const uint8_t *shared, int T, const Workspace &ws,
                                int32_t *idx_out, float *w_out, uint16_t *out, cudaStream_t s) {
  const PackedGeom G = packed_geom(d.hidden, d.inter);
  int dev = 0, n_sm = 0, max_smem = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const uint32_t stage_bytes = (uint32_t)max(G.gu_unit_bytes, 4 * G.dn_unit_bytes);
  const SmemLayout L0 = smem_layout(T, G.H, 0, stage_bytes);
  int ns = (int)((max_smem - (int)L0.ring - 128) / (int)(stage_bytes + 16));
  ns = min(ns, 32);
  if (ns < 2) return cudaErrorInvalidConfiguration;
  const SmemLayout L = smem_layout(T, G.H, ns, stage_bytes);
  if (L.total > (uint32_t)max_smem) return cudaErrorInvalidConfiguration;
  // the per-CTA down range must fit the 128-entry completed-tile list
  const int max_entries = min(T * d.top_k, d.n_experts) + 1;
  if ((max_entries * G.dn_units + n_sm - 1) / n_sm > kMaxSel) return cudaErrorInvalidConfiguration;
  const int rrows = (d.n_experts + n_sm - 1) / n_sm;  // router rows per CTA, staged in the ring
  if ((size_t)rrows * d.hidden * 4 > (size_t)ns * stage_bytes) return cudaErrorInvalidConfiguration;

  DecodeArgs a{};
  a.x = x;
  a.Wr = Wr;
  a.bias = bias;
  a.experts = experts;
  a.shared = shared;
  a.G = G;
  a.T = T;
  a.E = d.n_experts;
  a.k = d.top_k;
  a.logits = ws.logits;
  a.h = ws.h;
  a.partial = ws.partial;
  a.tile_cnt = ws.tile_cnt;
  a.gbar = ws.gbar;
  a.idx_out = idx_out;
  a.w_out = w_out;
  a.out = out;
  a.status = ws.status;
  a.ns = ns;
  a.stage_bytes = stage_bytes;

  void (*kern)(DecodeArgs) = nullptr;
  switch (G.gu_groups / 16) {
    case 1: kern = decode_fused_kernel<1>; break;
    case 2: kern = decode_fused_kernel<2>; break;
    default: return cudaErrorInvalidValue;
  }
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, L.total);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  trace_mark(MOE_KERNEL_DECODE_FUSED, false, s);
  err = cudaLaunchKernelEx(&cfg, kern, a);
  trace_mark(MOE_KERNEL_DECODE_FUSED, true, s);
  return err;
}

}  // namespace moe
