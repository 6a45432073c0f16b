// Fused decode/verify-window layer (T <= 8 tokens) in one persistent,
// cooperatively launched kernel (sm_100a).  One CTA per SM: 14 consumer
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
//     shared-memory stages as stages free up; stage s belongs to consumer
//     warp s % 14, which computes the whole unit (full K) with no cross-warp
//     reduction and writes h = silu(g) * u (bf16) straight from its
//     accumulators.  At the end the CTA publishes, per expert, how many of
//     its units are done.
//  D  Once the h of the (at most two) experts in the CTA's down range is
//     complete (per-expert counter, bounded wait) it is copied into shared
//     memory; each down stage (up to 4 pairs) again belongs to one warp:
//     partial = w[t, e] * (Wd_e h_e) per (expert, tile).  The last CTA to
//     contribute to a tile sums its partials in expert order and writes out
//     (bf16).
// Dequantisation happens in registers and feeds m16n8k16 tensor-core MMAs
// with the tokens as the 8 columns; gate/up uses the biased decode with the
// -1 offset folded into the accumulator start (decode_q2_biased), down the
// exact decode.  Every wait is bounded (sync.cuh).
#include "kernels.cuh"
#include "router.cuh"
#include "sync.cuh"

namespace moe {

namespace {

constexpr int kConsumerWarps = 14;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxTok = 8;
constexpr int kMaxSel = 128;              // T * top_k
constexpr int kMaxEntries = kMaxSel + 1;  // touched experts + shared
constexpr int kMaxE = 1024;
constexpr int kMaxI = 512;                // down K handled by the h cache
constexpr int kBarConsumers = 1;          // named barrier id (0 = __syncthreads)

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
  L.bars = o;  // full[ns], empty[ns], rbar, xbar
  o = align_to(o + 8u * (2 * ns + 2), 16);
  L.xs = o;
  o = align_to(o + (uint32_t)T * (H + 16) * 2, 16);
  L.corr = o;
  o = align_to(o + (uint32_t)(H / 32) * kMaxTok * 4, 16);
  L.rpart = o;  // [rows per pass <= 4][8 tokens][4 quarters]
  o += 4 * kMaxTok * 4 * 4;
  L.red = o;    // top-k scratch (phase B), then the h cache of phase D: [2 entries][8 tokens][I + 16]
  o += align_to(2u * kMaxTok * (kMaxI + 16) * 2, 16);
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

__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const PackedGeom &G = a.G;
  const int T = a.T, E = a.E, K = a.k, H = G.H, I = G.I;
  const SmemLayout L = smem_layout(T, H, a.ns, a.stage_bytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *empty = full + a.ns;
  uint64_t *rbar = empty + a.ns;
  uint64_t *xbar = rbar + 1;
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
      mbar_init(&empty[i], 1);  // each stage is consumed by one warp
    }
    mbar_init(rbar, 1);
    mbar_init(xbar, 1);
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
    constexpr int kRowsPerPass = kConsumerWarps / 4;  // 4 warps (quarters) per router row
    for (int r0 = 0; r0 < n_rrows; r0 += kRowsPerPass) {
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
      if (tid < kRowsPerPass * T) {
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
  // B fragments read the tokens from shared memory: scale the k pair (4c+2,
  // 4c+3) of every 4 by 1/4 in place (exact) and negate the correction sums.
  for (int i = tid; i < T * (H / 4); i += kConsumers) {
    uint32_t *p2 = reinterpret_cast<uint32_t *>(xs + (i / (H / 4)) * xstride + 4 * (i % (H / 4)) + 2);
    *p2 = bf16x2_quarter(*p2);
  }
  for (int i = tid; i < (H / 32) * kMaxTok; i += kConsumers) corr[i] = (i % kMaxTok) < T ? -corr[i] : 0.f;
  named_bar(kBarConsumers, kConsumers);

  const uint16_t *xrow = xs + (g < T ? g : 0) * xstride + 4 * c;
  const bool row_ok = g < T;
  for (int s_idx = warp; s_idx < n_gu_st; s_idx += kConsumerWarps) {
    const int slot = s_idx % a.ns;
    bounded_wait(&full[slot], (s_idx / a.ns) & 1);
    const uint8_t *st = ring + (size_t)slot * a.stage_bytes;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int grp = 0; grp < G.gu_groups; ++grp) {
      // one block group: 4 independent block tiles, staged load -> decode -> MMA -> scale
      const uint8_t *gp = st + (size_t)grp * kGroupBytes;
      const uint4 cw = lds128(gp + lane * 16);
      const uint4 sw = lds128(gp + kGroupCodeBytes + g * 16);
      const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
      const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
      uint2 b0[4], b1[4];
      float2 nc[4];
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        const int b = grp * 4 + blk;
        b0[blk] = *reinterpret_cast<const uint2 *>(xrow + 32 * b);
        b1[blk] = *reinterpret_cast<const uint2 *>(xrow + 32 * b + 16);
        if (!row_ok) b0[blk] = b1[blk] = make_uint2(0u, 0u);
        nc[blk] = *reinterpret_cast<const float2 *>(corr + b * kMaxTok + 2 * c);
      }
      uint32_t p[4][8];
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) decode_q2_biased(cws[blk], p[blk]);
      float d[4][4];
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        const uint32_t a0[4] = {p[blk][0], p[blk][1], p[blk][2], p[blk][3]};
        const float cin[4] = {nc[blk].x, nc[blk].y, nc[blk].x, nc[blk].y};
        mma_bf16_16816(d[blk], a0, b0[blk].x, b0[blk].y, cin);
      }
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        const uint32_t a1[4] = {p[blk][4], p[blk][5], p[blk][6], p[blk][7]};
        mma_bf16_16816(d[blk], a1, b1[blk].x, b1[blk].y, d[blk]);
      }
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2 *>(&sws[blk]));
        acc[0] = fmaf(s2.x, d[blk][0], acc[0]);
        acc[1] = fmaf(s2.x, d[blk][1], acc[1]);
        acc[2] = fmaf(s2.y, d[blk][2], acc[2]);
        acc[3] = fmaf(s2.y, d[blk][3], acc[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    const int id = g0 + s_idx;
    const int entry = id / G.gu_units, u = id % G.gu_units;
    const int i = 8 * u + g;  // tile rows g (gate) and g+8 (up) share intermediate row i
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int n = 2 * c + half;
      if (n < T) {
        const int j = tokj[entry * kMaxTok + n];
        if (j >= 0) a.h[((size_t)n * (K + 1) + j) * I + i] = float_to_bf16_bits(silu_f(acc[half]) * acc[2 + half]);
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
  // h of the experts in this CTA's down range (at most two) into shared memory.
  uint16_t *hc = reinterpret_cast<uint16_t *>(red);
  const int hstride = I + 16;
  const int e_lo = d1 > d0 ? d0 / G.dn_units : 0;
  const int n_hc = d1 > d0 ? (d1 - 1) / G.dn_units - e_lo + 1 : 0;
  if (tid < n_hc && !*reinterpret_cast<volatile int *>(&misc[1])) {
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_gpu(&ready[e_lo + tid]) < (uint32_t)G.gu_units) {
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        set_status(a.status, kStatusTimeout);
        misc[1] = 1;
        break;
      }
    }
  }
  named_bar(kBarConsumers, kConsumers);
  for (int i = tid; i < n_hc * kMaxTok * (I / 8); i += kConsumers) {
    const int he = i / (kMaxTok * (I / 8)), r = i % (kMaxTok * (I / 8));
    const int t = r / (I / 8), c8 = r % (I / 8);
    const int j = t < T ? tokj[(e_lo + he) * kMaxTok + t] : -1;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j >= 0) v = __ldcg(reinterpret_cast<const uint4 *>(a.h + ((size_t)t * (K + 1) + j) * I + c8 * 8));
    *reinterpret_cast<uint4 *>(hc + (he * kMaxTok + t) * hstride + c8 * 8) = v;
  }
  named_bar(kBarConsumers, kConsumers);

  for (int s_idx = n_gu_st + ((warp - n_gu_st % kConsumerWarps + kConsumerWarps) % kConsumerWarps); s_idx < n_st;
       s_idx += kConsumerWarps) {
    const int sd = s_idx - n_gu_st;
    const int slot = s_idx % a.ns;
    bounded_wait(&full[slot], (s_idx / a.ns) & 1);
    const uint8_t *st = ring + (size_t)slot * a.stage_bytes;
    const int q0 = d0 + sd * pps, q1 = min(d1, q0 + pps);
    for (int q = q0; q < q1; ++q) {
      const int entry = q / G.dn_units, tile = q % G.dn_units;
      const uint16_t *hrow = hc + ((entry - e_lo) * kMaxTok + g) * hstride + 4 * c;
      const uint8_t *pp_st = st + (size_t)(q - q0) * G.dn_unit_bytes;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int grp = 0; grp < 4; ++grp) {
        const uint8_t *gp = pp_st + (size_t)grp * kGroupBytes;
        const uint4 cw = lds128(gp + lane * 16);
        const uint4 sw = lds128(gp + kGroupCodeBytes + g * 16);
        const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
        const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
        uint2 b0[4], b1[4];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const int b = grp * 4 + blk;
          b0[blk] = *reinterpret_cast<const uint2 *>(hrow + 32 * b);
          b1[blk] = *reinterpret_cast<const uint2 *>(hrow + 32 * b + 16);
        }
        uint32_t p[4][8];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) decode_q2_exact(cws[blk], p[blk]);
        float d[4][4];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const uint32_t a0[4] = {p[blk][0], p[blk][1], p[blk][2], p[blk][3]};
          const float z[4] = {0.f, 0.f, 0.f, 0.f};
          mma_bf16_16816(d[blk], a0, b0[blk].x, b0[blk].y, z);
        }
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const uint32_t a1[4] = {p[blk][4], p[blk][5], p[blk][6], p[blk][7]};
          mma_bf16_16816(d[blk], a1, b1[blk].x, b1[blk].y, d[blk]);
        }
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const float2 s2 = __half22float2(*reinterpret_cast<const __half2 *>(&sws[blk]));
          acc[0] = fmaf(s2.x, d[blk][0], acc[0]);
          acc[1] = fmaf(s2.x, d[blk][1], acc[1]);
          acc[2] = fmaf(s2.y, d[blk][2], acc[2]);
          acc[3] = fmaf(s2.y, d[blk][3], acc[3]);
        }
      }
      const float w0 = tokw[entry * kMaxTok + 2 * c], w1 = tokw[entry * kMaxTok + 2 * c + 1];
      float *pp = a.partial + ((size_t)entry * G.dn_units + tile) * 128;
      *reinterpret_cast<float4 *>(pp + lane * 4) = make_float4(acc[0] * w0, acc[1] * w1, acc[2] * w0, acc[3] * w1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }

  // Count this CTA's contributions per output tile (one fence per writer
  // warp); the last contributor of a tile sums its partials in expert order.
  int *done_tiles = sel_idx;  // phase-B scratch, free now
  __threadfence();
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
  if (G.dn_groups != 4) return false;  // down: 4 groups of 128 (inter 512, the h cache size)
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

  void (*kern)(DecodeArgs) = decode_fused_kernel;
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
