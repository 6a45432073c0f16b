// Fused decode/verify-window layer (T <= 8 tokens) in one persistent,
// cooperatively launched kernel (sm_100a).  One CTA per SM, 14 warps, each of
// which both streams and computes.
//
//  A  Every thread copies (cp.async, 16 B) its pieces of this CTA's router
//     rows into shared memory and one thread prefetches the CTA's slice of the
//     shared expert into L2; launched as a programmatic dependent of the
//     previous decode launch, the CTA does this while that launch finishes and
//     only then (griddepcontrol.wait) copies the tokens.  2 warps per router
//     row (one half of K each) write the logits.
//     -- grid barrier: all logits written.  Between arriving and waiting the
//        CTA prepares its token rows as the MMA B operand (block correction
//        sums, the (4c+2, 4c+3) pairs scaled by 1/4) --
//  B  One warp per token reads its logits from L2 and selects the top-k
//     (threshold + rank); its weights are the softmax over its winners.
//     Work entries: for T <= 3 one per (token, slot), fixed in advance, plus
//     the shared expert (an expert two tokens chose is streamed twice; the
//     weights are computed while phase D waits for h); for
//     larger T the sorted list of touched experts plus the shared expert,
//     built by a spare warp from a bit map of the winners while the token
//     warps fill their table entries (the tables were cleared while waiting
//     on the barrier).  Every CTA builds the same entries.
//  C  Work lists, expert-major, cut into equal contiguous ranges per CTA:
//     gate/up units (expert, 8 intermediate rows) and down stages (expert, two
//     16-row units).  Stage s belongs to warp s % 14, which copies it into its
//     own shared-memory slot in four cp.async groups, keeps the next two
//     quarters in flight while it computes, runs the whole unit (full K) with
//     no cross-warp reduction and writes h = silu(g) * u (bf16) straight from
//     its accumulators.  For one token (fewer units than warps) the kernel
//     instance <2, 1> splits each unit's K over two warps, whose sums meet in
//     shared memory in part order, and gives each down stage one unit.  At the
//     end the CTA publishes, per expert, how many of its units are done.
//  D  Once the h of the (at most two) experts in the CTA's down range is
//     complete (per-expert counter, bounded wait) it is copied into shared
//     memory; each down stage (two 16-row units) again belongs to one warp:
//     partial = w[t, e] * (Wd_e h_e) per (entry, tile).
//     -- second grid barrier: all partials written --
//     One warp per output tile sums its partials in a fixed order and writes
//     out (bf16, or fp32).
// Dequantisation happens in registers: the 2-bit codes of a row OR into the
// mantissa of bf16 128.0 (128 + q, or 128 + 4q with the matching activation
// pair pre-scaled by 1/4), one logic op per pair of weights, and feed
// m16n8k16 tensor-core MMAs with the tokens as the 8 columns.  The -1 of
// d * (q - 1) and the 128 bias start the accumulator at minus the weighted
// block sum of the token; the fp16 block scale d multiplies each block's fp32
// result.  All products are exact.  Every wait is bounded (sync.cuh).
#include <atomic>
#include <mutex>

#include "kernels.cuh"
#include "router.cuh"
#include "sync.cuh"

namespace moe {

namespace {

constexpr int kConsumerWarps = 14;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers;  // every warp computes and streams its own stages
constexpr int kMaxTok = 8;
constexpr int kMaxSel = 128;              // T * top_k
constexpr int kMaxEntries = kMaxSel + 1;  // touched experts + shared
constexpr int kSlotTokens = 3;            // up to this many tokens: one work entry per (token, slot)
constexpr int kMaxE = 1024;
constexpr int kMaxI = 512;                // down K handled by the h cache
constexpr int kBarConsumers = 1;          // named barrier id (0 = __syncthreads)
constexpr int kMaxParts = 40;             // gate/up K parts a CTA may hold in shared memory (128 floats each)

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
  uint32_t *ready;     // [kMaxEntries] per-entry count of finished gate/up units
  uint64_t *gbar;      // monotonic grid-barrier arrival counter
  int32_t *idx_out;    // optional [T][k]
  float *w_out;        // optional [T][k]
  uint16_t *out;       // [T][H] bf16, or
  float *out_f32;      // [T][H] fp32 (when set: the layer output is not rounded)
  uint32_t *status;
  int ns;              // ring stages: nw warps x (ns / nw) private slots each
  int nw;              // warps that stream and compute expert stages
  uint32_t stage_bytes;
};

struct SmemLayout {
  uint32_t xs, corr, hcorr, rpart, red, bitmap, slv, ent, tokj, tokw, misc, ring, total;
};

__host__ __device__ inline uint32_t align_to(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout smem_layout(int T, int H, int ns, uint32_t stage_bytes, int kp) {
  SmemLayout L;
  uint32_t o = 0;
  L.xs = o;  // [T + 1][H + 16] bf16 token rows (the B operand once prepared); row T stays zero
  o = align_to(o + (uint32_t)(T + 1) * (H + 16) * 2, 16);
  L.corr = o;  // [H/32 blocks][8 tokens] accumulator starts of the biased decode
  o = align_to(o + (uint32_t)(H / 32) * kMaxTok * 4, 16);
  L.hcorr = o;  // [2 cached experts][I/32][8]
  o = align_to(o + 2u * (kMaxI / 32) * kMaxTok * 4, 16);
  L.rpart = o;  // [rows per pass][8 tokens][router parts]
  o += (kConsumerWarps / kRouterParts) * kMaxTok * kRouterParts * 4;
  o = align_to(o, 16);
  // top-k scratch (phase B: 64 uint64 per token), the gate/up K parts at the end of phase C (kp > 1:
  // [unit][part][32 lanes][4] floats), then the h staging of phase D: [2][T][I + 16] bf16
  L.red = o;
  const uint32_t parts_bytes = kp > 1 ? (uint32_t)kMaxParts * 128 * 4 : 0u;
  o += align_to(max(max((uint32_t)kMaxTok * 64 * 8, 2u * T * (kMaxI + 16) * 2), parts_bytes), 16);
  L.bitmap = o;
  o += (kMaxE / 32) * 4;
  L.slv = o;  // slot entries: the winners' logits, token-major
  o += kMaxSel * 4;
  L.ent = o;
  o = align_to(o + kMaxEntries * 4, 16);
  L.tokj = o;
  o = align_to(o + kMaxEntries * kMaxTok, 16);
  L.tokw = o;
  o = align_to(o + kMaxEntries * kMaxTok * 4, 16);
  L.misc = o;  // [0] entries [1] abort [2] grid-barrier flag
  o += 64;
  L.ring = align_to(o, 128);
  L.total = L.ring + (uint32_t)ns * stage_bytes;
  return L;
}

// Prepares T bf16 rows v[t][0..K) (`stride` elements apart, t < T) in shared
// memory as the B operand of the biased decode (decode_q2_biased): for every
// 32-wide block b, corr[b][t] = -(129 * sum_{k%4<2} v[t][k] + 33 * sum_{k%4>=2}
// v[t][k]), then the pairs (4c+2, 4c+3) of every four are scaled by 1/4 in place
// (exact).  The MMA of codes 128 + q / 128 + 4q against these rows, started at
// corr, gives sum_k (q_k - 1) v[t][k].  One thread per (block, token).
__device__ __forceinline__ void prep_rows(uint16_t *v, int stride, int K, int T, float *corr, int tid) {
  for (int i = tid; i < (K / 32) * T; i += kConsumers) {
    const int b = i / T, t = i % T;
    uint4 *xr = reinterpret_cast<uint4 *>(v + t * stride + 32 * b);
    float s129 = 0.f, s33 = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w = xr[q];
      s129 += __uint_as_float(w.x << 16) + __uint_as_float(w.x & 0xffff0000u);
      s33 += __uint_as_float(w.y << 16) + __uint_as_float(w.y & 0xffff0000u);
      s129 += __uint_as_float(w.z << 16) + __uint_as_float(w.z & 0xffff0000u);
      s33 += __uint_as_float(w.w << 16) + __uint_as_float(w.w & 0xffff0000u);
      w.y = bf16x2_fma(w.y, 0x3E803E80u, 0x80008000u);
      w.w = bf16x2_fma(w.w, 0x3E803E80u, 0x80008000u);
      xr[q] = w;
    }
    corr[b * kMaxTok + t] = -(129.f * s129 + 33.f * s33);
  }
}

// Block groups [grp0, grp1) of one 16-row unit against the (at most 8) token
// rows `rows` (row g of this lane's B column; tokens >= T read the zero row `zrow`); adds
// to acc = (row g, token 2c), (row g, token 2c+1), (row g+8, token 2c),
// (row g+8, token 2c+1).  Per block: the codes decode to bf16 128 + q /
// 128 + 4q (decode_q2_biased), two m16n8k16 MMAs with the accumulator started
// at the block's corr, then the fp16 block scales.
__device__ __forceinline__ void unit_gemv(const uint8_t *st, int grp0, int grp1, const uint16_t *rows, int stride,
                                          int T, const uint16_t *zrow, const float *corr, int lane, float (&acc)[4]) {
  const int g = lane >> 2, c = lane & 3;
  const uint16_t *xrow = (g < T ? rows + g * stride : zrow) + 4 * c;
  for (int grp = grp0; grp < grp1; ++grp) {
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
      fma2_bcast(acc[0], acc[1], s2.x, d[blk][0], d[blk][1]);
      fma2_bcast(acc[2], acc[3], s2.y, d[blk][2], d[blk][3]);
    }
  }
}

template <int KP, int PPS>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(DecodeArgs a) {
  static_assert((KP == 1 || KP == 2 || KP == 4) && (PPS == 1 || PPS == 2), "work granularity");
  extern __shared__ __align__(128) uint8_t smem[];
  const PackedGeom &G = a.G;
  const int T = a.T, E = a.E, K = a.k, H = G.H, I = G.I;
  const SmemLayout L = smem_layout(T, H, a.ns, a.stage_bytes, KP);
  uint16_t *xs = reinterpret_cast<uint16_t *>(smem + L.xs);
  float *corr = reinterpret_cast<float *>(smem + L.corr);
  float *hcorr = reinterpret_cast<float *>(smem + L.hcorr);
  float *rpart = reinterpret_cast<float *>(smem + L.rpart);
  float *red = reinterpret_cast<float *>(smem + L.red);
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + L.bitmap);
  float *slv = reinterpret_cast<float *>(smem + L.slv);
  int *ent = reinterpret_cast<int *>(smem + L.ent);
  int8_t *tokj = reinterpret_cast<int8_t *>(smem + L.tokj);
  float *tokw = reinterpret_cast<float *>(smem + L.tokw);
  int *misc = reinterpret_cast<int *>(smem + L.misc);
  uint8_t *ring = smem + L.ring;
  uint32_t *ready = a.ready;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int xstride = H + 16;
  const uint16_t *zrow = xs + T * xstride;  // zeros: the B column of tokens >= T
  const int n_rrows = E > (int)blockIdx.x ? (E - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  float *wr_s = reinterpret_cast<float *>(ring);  // router rows live in the ring until phase C

  // ---------------- phase A: set-up, router ----------------
  // The next launch on this stream may start its own set-up on the SMs this grid frees: it reads nothing
  // that this grid writes before its griddepcontrol.wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0)
    for (int i = 0; i < 16; ++i) misc[i] = 0;
  // This CTA's router rows (weights: no earlier launch writes them), cp.async pieces from every thread, and
  // an L2 prefetch of this CTA's slice of the shared expert.
  for (int i = tid; i < n_rrows * (H / 4); i += kConsumers) {
    const int r = i / (H / 4), c4 = i % (H / 4);
    cp_async16(wr_s + (size_t)r * H + c4 * 4, a.Wr + (size_t)(blockIdx.x + (size_t)gridDim.x * r) * H + c4 * 4);
  }
  cp_async_commit();
  if (tid == 0) {
    const size_t per = ((G.expert_bytes + gridDim.x - 1) / gridDim.x + 15) & ~(size_t)15;
    const size_t off = per * blockIdx.x;
    if (off < G.expert_bytes) {
      const size_t n = min(per, G.expert_bytes - off);
      for (size_t o = 0; o < n; o += 32768) bulk_prefetch_l2(a.shared + off + o, (uint32_t)min((size_t)32768, n - o));
    }
  }
  // Everything below may depend on the previous launch on this stream (its outputs, the workspace).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint64_t bar_target = 0;  // the grid barriers' leader (the last thread) reads the arrival counter now
  if (tid == kConsumers - 1) {
    const uint64_t c0 = *reinterpret_cast<volatile uint64_t *>(a.gbar);
    bar_target = (c0 / gridDim.x + 1) * gridDim.x;
  }
  for (int i = tid; i < T * (H / 8); i += kConsumers) {
    const int t = i / (H / 8), c8 = i % (H / 8);
    cp_async16(xs + t * xstride + c8 * 8, a.x + (size_t)t * H + c8 * 8);
  }
  cp_async_commit();
  for (int i = tid; i < xstride / 8; i += kConsumers)
    reinterpret_cast<uint4 *>(xs + T * xstride)[i] = make_uint4(0u, 0u, 0u, 0u);
  {
    if (blockIdx.x == 0)
      for (int i = tid; i < kMaxEntries; i += kConsumers) ready[i] = 0u;
    constexpr int kRowsPerPass = kConsumerWarps / kRouterParts;  // one warp per router row part
    // the bias of the logit this thread finishes in the first pass, loaded while the copies land
    float bias0 = 0.f;
    if (a.bias && tid < kRowsPerPass * T && tid / T < n_rrows) bias0 = __ldg(a.bias + blockIdx.x + gridDim.x * (tid / T));
    cp_async_wait_group<0>();  // this thread's pieces of the tokens and router rows have landed
    named_bar(kBarConsumers, kConsumers);
    for (int r0 = 0; r0 < n_rrows; r0 += kRowsPerPass) {
      const int r = r0 + warp / kRouterParts, q = warp % kRouterParts;
      if (r < n_rrows) {
        float acc[8];
        router_part_any<true>(xs, xstride, T, wr_s + (size_t)r * H, H, q, lane, acc);
        if (lane == 0) {
#pragma unroll
          for (int t = 0; t < 8; ++t) rpart[((r - r0) * kMaxTok + t) * kRouterParts + q] = acc[t];
        }
      }
      named_bar(kBarConsumers, kConsumers);
      if (tid < kRowsPerPass * T) {
        const int rr = tid / T, t = tid % T;
        if (r0 + rr < n_rrows) {
          const int e = blockIdx.x + gridDim.x * (r0 + rr);
          a.logits[(size_t)t * E + e] = router_combine(rpart + (rr * kMaxTok + t) * kRouterParts,
                                                       r0 == 0 ? bias0 : (a.bias ? a.bias[e] : 0.f));
        }
      }
      named_bar(kBarConsumers, kConsumers);
    }
    // Arrive on the grid barrier, prepare the token rows as the B operand while the other CTAs finish
    // their logits (the router is done with them), then wait.  The barrier's leader (the last thread,
    // which has the fewest token-row pieces to prepare) read the arrival counter at the start.
    const bool leader = tid == kConsumers - 1;
    grid_arrive_release(a.gbar, kBarConsumers, kConsumers, leader);
    prep_rows(xs, xstride, H, T, corr, tid);
    // the touched-expert tables start empty (filled once the top-k is known)
    for (int i = tid; i < kMaxEntries * kMaxTok; i += kConsumers) {
      tokj[i] = -1;
      tokw[i] = 0.f;
    }
    if (tid < kMaxE / 32) bitmap[tid] = 0u;
    grid_wait(a.gbar, bar_target, kBarConsumers, kConsumers, leader, a.status, &misc[2]);

    // ---------------- phase B: top-k and the touched-expert list ----------------
    // One warp per token reads its token's logits straight from L2 (other CTAs wrote them).
    int e = 0;
    float lv = 0.f;
    if (warp < T) {
      uint64_t *scratch = reinterpret_cast<uint64_t *>(red) + warp * 64;
      const float *row = a.logits + (size_t)warp * E;
      if (E == 512)
        warp_topk_fast_sel<16, false, true>(row, E, K, lane, scratch, e, lv);
      else if (E < 512)
        warp_topk_fast_sel<16, false>(row, E, K, lane, scratch, e, lv);
      else
        warp_topk_fast_sel<32, false>(row, E, K, lane, scratch, e, lv);
      if (lane < K) atomicOr(&bitmap[e >> 5], 1u << (e & 31));
    }
    if (T <= kSlotTokens && T * K <= E) {
      // Slot entries: entry t * k + j is token t's j-th winner and the shared expert comes last, so the
      // work split is fixed before the routing is known and no list is built; an expert that two tokens
      // chose is streamed once per token.  The weights are computed later, while the CTA waits for h.
      if (warp < T && lane < K) {
        const int entry = warp * K + lane;
        ent[entry] = e;
        tokj[entry * kMaxTok + warp] = (int8_t)lane;
        slv[entry] = lv;
      }
      if (warp == kConsumerWarps - 1 && lane < T) {
        tokj[T * K * kMaxTok + lane] = (int8_t)K;  // shared expert: slot k, weight 1
        tokw[T * K * kMaxTok + lane] = 1.f;
        if (lane == 0) {
          ent[T * K] = E;
          misc[0] = T * K + 1;
        }
      }
    } else {
      named_bar(kBarConsumers, kConsumers);  // every selected expert is in the bit map
      if (warp < T) {
        // While a spare warp builds the list: the token's weights (fp32 softmax over its winners) and its
        // table entries, each lane ranking its expert among the touched ones from the bit map.
        const float wt = topk_softmax(lv, lane, K);
        if (lane < K) {
          const int wq = e >> 5;
          int r = __popc(bitmap[wq] & ((1u << (e & 31)) - 1u));
          for (int w2 = 0; w2 < wq; ++w2) r += __popc(bitmap[w2]);
          tokj[r * kMaxTok + warp] = (int8_t)lane;
          tokw[r * kMaxTok + warp] = wt;
          if (blockIdx.x == 0 && a.idx_out) {
            a.idx_out[warp * K + lane] = e;
            a.w_out[warp * K + lane] = wt;
          }
        }
      }
      if (warp == kConsumerWarps - 1) {
        const uint32_t word = bitmap[lane];
        const uint32_t cnt = __popc(word);
        uint32_t incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += v;
        }
        const uint32_t pre = incl - cnt;
        uint32_t wbits = word;
        for (uint32_t r = pre; wbits; ++r) {
          const int b = __ffs(wbits) - 1;
          wbits &= wbits - 1;
          ent[r] = lane * 32 + b;
        }
        const int U = __shfl_sync(0xffffffffu, (int)incl, 31);
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
  }
  __syncthreads();  // the list is visible to every warp

  const int nent = misc[0];
  const int nw = a.nw;
  const int n_gu = nent * G.gu_units, n_dn = nent * G.dn_units;
  // contiguous shares of the units (32-bit products: at most 129 entries x 256 units x the grid)
  const int g0 = (int)((uint32_t)n_gu * blockIdx.x / gridDim.x);
  const int g1 = (int)((uint32_t)n_gu * (blockIdx.x + 1) / gridDim.x);
  const int d0 = (int)((uint32_t)n_dn * blockIdx.x / gridDim.x);
  const int d1 = (int)((uint32_t)n_dn * (blockIdx.x + 1) / gridDim.x);
  // Granularity (compile-time, chosen by the launcher): a gate/up unit's K is split into kp parts on
  // different warps (stages of a quarter of the part each), summed in part order before SwiGLU, and a down
  // stage holds pps units (quarters of half or a quarter of a unit).
  constexpr int kp = KP, pps = PPS;
  constexpr int qpu = 4 / pps;  // quarters per down unit
  const int n_gu_st = (g1 - g0) * kp;
  const int n_dn_st = (d1 - d0 + pps - 1) / pps;
  const int n_st = n_gu_st + n_dn_st;
  // Stage s belongs to warp s % nw, which copies it (cp.async) into its own
  // ring slot, waits for its own copies, computes it and refills the slot with
  // its next stage s + nw.  No other warp touches the slot.
  auto expert_ptr = [&](int entry) -> const uint8_t * {
    const int e = ent[entry];
    return e == E ? a.shared : a.experts + (size_t)e * G.expert_bytes;
  };
  auto stage_ptr = [&](int) { return ring + (size_t)warp * a.stage_bytes; };
  // A stage is copied as 4 commit groups (its quarters): gate/up = one unit, or
  // one of its kp K parts (quarter = 4 / kp block groups), down = pps units of
  // 16 rows (quarter = half a unit, or a quarter with one unit).  A warp walks
  // the quarters of its stages in order and keeps the next two in flight:
  // quarter i is computed after quarter i + 1 was issued, and quarter i + 2 goes
  // into a slot region that overlaps none of quarter i + 1's (the region
  // quarter i used, or for the first down quarters the first gate/up ones').
  // Past the last stage the groups are empty.
  auto issue_quarter = [&](int qi) {
    const int s = warp + (qi >> 2) * nw, qt = qi & 3;
    if (s < n_st) {
      uint8_t *dst = stage_ptr(s);
      if (s < n_gu_st) {
        const int id = g0 + s / kp, part = s % kp;
        const size_t qb = G.gu_unit_bytes / (4 * kp);
        warp_cp_async(dst + qt * qb,
                      expert_ptr(id / G.gu_units) + (size_t)(id % G.gu_units) * G.gu_unit_bytes +
                          (size_t)(4 * part + qt) * qb,
                      (uint32_t)qb, lane);
      } else {
        const int q = d0 + (s - n_gu_st) * pps + qt / qpu, piece = qt % qpu;
        const size_t pb = G.dn_unit_bytes / qpu;
        if (q < d1)
          warp_cp_async(dst + (size_t)(qt / qpu) * G.dn_unit_bytes + piece * pb,
                        expert_ptr(q / G.dn_units) + G.gu_bytes + (size_t)(q % G.dn_units) * G.dn_unit_bytes +
                            piece * pb,
                        (uint32_t)pb, lane);
      }
    }
    cp_async_commit();
  };
  // Quarter qi has landed (only quarter qi + 1 may still be in flight), then queue quarter qi + 2.
  int qi = 0;
  auto next_quarter = [&]() {
    cp_async_wait_group<1>();
    __syncwarp();
  };
  auto done_quarter = [&]() {
    __syncwarp();  // every lane has read the quarter before its region is refilled
    issue_quarter(qi + 2);
    ++qi;
  };
  if (warp < nw) {
    issue_quarter(0);
    issue_quarter(1);
  }

  // ---------------- consumers, phase C: gate/up + SwiGLU ----------------
  // h = silu(gate) * up of unit id from its accumulators (rows g and g+8, tokens 2c and 2c + 1).
  auto write_h = [&](int id, const float (&acc)[4]) {
    const int entry = id / G.gu_units, u = id % G.gu_units;
    const int i = 8 * u + g;  // tile rows g (gate) and g+8 (up) share intermediate row i
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int n = 2 * c + hf;  // this lane's tokens: 2c, 2c + 1
      if (n < T) {
        const int j = tokj[entry * kMaxTok + n];
        if (j >= 0) a.h[((size_t)n * (K + 1) + j) * I + i] = float_to_bf16_bits(silu_f(acc[hf]) * acc[2 + hf]);
      }
    }
  };
  for (int s_idx = warp; warp < nw && s_idx < n_gu_st; s_idx += nw) {
    const uint8_t *st = stage_ptr(s_idx);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int gq = G.gu_groups / (4 * kp);     // block groups per quarter
    const int k0 = (s_idx % kp) * 4 * gq;      // the part's first block group along K
    for (int qt = 0; qt < 4; ++qt) {
      next_quarter();
      unit_gemv(st - (size_t)k0 * kGroupBytes, k0 + qt * gq, k0 + (qt + 1) * gq, xs, xstride, T, zrow, corr, lane,
                acc);
      done_quarter();
    }
    if constexpr (kp == 1)
      write_h(g0 + s_idx, acc);
    else  // the part's sums into [unit][part][32 lanes][4] (the top-k scratch is free, the h cache not yet used)
      *reinterpret_cast<float4 *>(red + (size_t)s_idx * 128 + lane * 4) =
          make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
  if constexpr (kp > 1) {
    named_bar(kBarConsumers, kConsumers);
    for (int ul = warp; ul < g1 - g0; ul += kConsumerWarps) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int p = 0; p < kp; ++p) {
        const float4 v = *reinterpret_cast<const float4 *>(red + (size_t)(ul * kp + p) * 128 + lane * 4);
        acc[0] += v.x;
        acc[1] += v.y;
        acc[2] += v.z;
        acc[3] += v.w;
      }
      write_h(g0 + ul, acc);
    }
  }

  // Publish this CTA's finished gate/up units per expert (one fence for all of them).
  named_bar(kBarConsumers, kConsumers);
  if (tid == 0 && g1 > g0) {
    // release: the CTA's h stores (ordered before by the barrier) before the counts; no value returned
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    for (int entry = g0 / G.gu_units; entry <= (g1 - 1) / G.gu_units; ++entry) {
      const int lo = max(g0, entry * G.gu_units), hi = min(g1, (entry + 1) * G.gu_units);
      asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(&ready[entry]), "r"((uint32_t)(hi - lo)) : "memory");
    }
  }

  // ---------------- consumers, phase D: down projection + combine ----------------
  // h of the experts in this CTA's down range (at most two) into shared memory.
  uint16_t *hc = reinterpret_cast<uint16_t *>(red);
  const int hstride = I + 16;
  const int e_lo = d1 > d0 ? d0 / G.dn_units : 0;
  const int n_hc = d1 > d0 ? (d1 - 1) / G.dn_units - e_lo + 1 : 0;
  if (T <= kSlotTokens && T * K <= E && warp < T) {
    // slot entries: the token's weights, fp32 softmax over its winners (the down stages read them)
    const float wt = topk_softmax(lane < K ? slv[warp * K + lane] : 0.f, lane, K);
    if (lane < K) {
      tokw[(warp * K + lane) * kMaxTok + warp] = wt;
      if (blockIdx.x == 0 && a.idx_out) {
        a.idx_out[warp * K + lane] = ent[warp * K + lane];
        a.w_out[warp * K + lane] = wt;
      }
    }
  }
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
  for (int i = tid; i < n_hc * T * (I / 8); i += kConsumers) {
    const int he = i / (T * (I / 8)), r = i % (T * (I / 8));
    const int t = r / (I / 8), c8 = r % (I / 8);
    const int j = tokj[(e_lo + he) * kMaxTok + t];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j >= 0) v = __ldcg(reinterpret_cast<const uint4 *>(a.h + ((size_t)t * (K + 1) + j) * I + c8 * 8));
    *reinterpret_cast<uint4 *>(hc + (he * T + t) * hstride + c8 * 8) = v;
  }
  named_bar(kBarConsumers, kConsumers);
  for (int he = 0; he < n_hc; ++he) prep_rows(hc + he * T * hstride, hstride, I, T, hcorr + he * (kMaxI / 32) * kMaxTok, tid);
  named_bar(kBarConsumers, kConsumers);

  // Sums a finished output tile's partials in a fixed order (deterministic) and writes its rows.
  // A lane's column c holds tokens 2c, 2c + 1, so only ceil(T / 2) columns carry tokens: the
  // lanes of the other columns take a share of the entries instead.  cu columns (a power of
  // two) are summed, each by 4 / cu lanes over the entries e = sub (mod 4 / cu) in order, and
  // the lanes' sums are added in a fixed butterfly (every lane ends with the same bits).
  auto reduce_tile = [&](int tile) {
    const int cu = T <= 2 ? 1 : (T <= 4 ? 2 : 4), nsub = 4 / cu, sub = c / cu, cc = c % cu;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    const float *pp = a.partial + (size_t)tile * 128 + (4 * g + cc) * 4;
    const size_t est = (size_t)G.dn_units * 128;
    for (int e2 = sub; e2 < nent; e2 += 16 * nsub) {  // up to sixteen loads in flight per lane
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        v[u] = e2 + u * nsub < nent ? ldg_cg_f4(pp + (size_t)(e2 + u * nsub) * est) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        o[0] += v[u].x;
        o[1] += v[u].y;
        o[2] += v[u].z;
        o[3] += v[u].w;
      }
    }
    for (int m = cu; m < 4; m <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] += __shfl_xor_sync(0xffffffffu, o[i], m);
    const int r0 = 16 * tile + g;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int n = 2 * c + hf;
      if (sub == 0 && n < T) {
        if (a.out_f32) {
          a.out_f32[(size_t)n * H + r0] = o[hf];
          a.out_f32[(size_t)n * H + r0 + 8] = o[2 + hf];
        } else {
          a.out[(size_t)n * H + r0] = float_to_bf16_bits(o[hf]);
          a.out[(size_t)n * H + r0 + 8] = float_to_bf16_bits(o[2 + hf]);
        }
      }
    }
  };

  for (int s_idx = n_gu_st + ((warp - n_gu_st % nw + nw) % nw); warp < nw && s_idx < n_st; s_idx += nw) {
    const int sd = s_idx - n_gu_st;
    const uint8_t *st = stage_ptr(s_idx);
    const int q0 = d0 + sd * pps, q1 = min(d1, q0 + pps);
    for (int q = q0; q < q0 + pps; ++q) {  // a stage always spans 4 quarters, the last one may hold one unit
      const bool live = q < q1;
      const int entry = q / G.dn_units, tile = q % G.dn_units, he = entry - e_lo;
      const uint8_t *pp_st = st + (size_t)(q - q0) * G.dn_unit_bytes;
      const uint16_t *hrows = hc + he * T * hstride;
      const float *hce = hcorr + he * (kMaxI / 32) * kMaxTok;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const int hg = G.dn_groups / qpu;  // block groups per quarter
      for (int hq = 0; hq < qpu; ++hq) {
        next_quarter();
        if (live) unit_gemv(pp_st, hq * hg, (hq + 1) * hg, hrows, hstride, T, zrow, hce, lane, acc);
        done_quarter();
      }
      if (!live) continue;
      // partial tile layout: lane (g, c) -> {row g tok 2c, row g tok 2c+1, row g+8 tok 2c, row g+8 tok 2c+1}
      const float w0 = 2 * c < T ? tokw[entry * kMaxTok + 2 * c] : 0.f;
      const float w1 = 2 * c + 1 < T ? tokw[entry * kMaxTok + 2 * c + 1] : 0.f;
      const float o4[4] = {acc[0] * w0, acc[1] * w1, acc[2] * w0, acc[3] * w1};
      float *pp = a.partial + ((size_t)entry * G.dn_units + tile) * 128;
      *reinterpret_cast<float4 *>(pp + lane * 4) = make_float4(o4[0], o4[1], o4[2], o4[3]);
    }
  }

  // Second grid barrier: once every CTA has passed it, every partial of this launch is written
  // (the arrival's release add publishes the CTA's partial stores).  Then the output tiles are
  // shared out, the CTA's k-th tile to warp k mod 14.  One arrival per CTA replaces a counted,
  // acquire-release atomic per unit (two per warp, about 1 us each on the warp's path).
  {
    const bool leader = tid == kConsumers - 1;
    grid_arrive_release(a.gbar, kBarConsumers, kConsumers, leader);
    if (grid_wait(a.gbar, bar_target + gridDim.x, kBarConsumers, kConsumers, leader, a.status, &misc[2]))
      for (int k = 0, tile = blockIdx.x; tile < G.dn_units; ++k, tile += gridDim.x)
        if (warp == k % kConsumerWarps) reduce_tile(tile);
  }
  cp_async_wait_all();  // nothing of this thread's may still be landing when the CTA ends
}

// Per-device launch facts of the fused decode kernel.
constexpr int kMaxDevices = 64;
struct LaunchCache {
  std::atomic<int> n_sm{0}, max_smem{0};
  // per kernel instance (0: <1, 2>, 1: <2, 1>)
  std::atomic<uint32_t> checked_smem[2] = {{0u}, {0u}};  // shared-memory size whose residency was checked (0: none)
  uint32_t smem_attr[2] = {0u, 0u};                        // largest dynamic shared memory opted into (under mu)
  std::mutex mu;
};
LaunchCache g_launch_cache[kMaxDevices];

}  // namespace

bool decode_fused_supported(const moe_dims &d, int T) {
  const PackedGeom G = packed_geom(d.hidden, d.inter);
  if (T < 1 || T > kMaxTok || T * d.top_k > kMaxSel || d.n_experts > kMaxE) return false;
  if (G.dn_groups != 4) return false;  // down: 4 groups of 128 (inter 512, the h cache size)
  if (G.gu_groups % 4) return false;   // gate/up units stream in quarters of whole block groups
  return true;
}

size_t decode_partial_floats(const moe_dims &d, int T) {
  const PackedGeom G = packed_geom(d.hidden, d.inter);
  const int entries = min(T * d.top_k, d.n_experts) + 1;
  return (size_t)entries * G.dn_units * 128;
}

size_t decode_counter_words(const moe_dims &) { return kMaxEntries; }

cudaError_t launch_decode_fused(const moe_dims &d, const uint16_t *x, const float *Wr, const float *bias,
                                const uint8_t *experts, const uint8_t *shared, int T, const Workspace &ws,
                                int32_t *idx_out, float *w_out, uint16_t *out, float *out_f32, cudaStream_t s) {
  const PackedGeom G = packed_geom(d.hidden, d.inter);
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  LaunchCache &lc = g_launch_cache[dev];
  int n_sm = lc.n_sm.load(std::memory_order_acquire), max_smem = lc.max_smem.load(std::memory_order_acquire);
  if (n_sm == 0) {  // device properties, queried once per device
    if ((err = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess ||
        (err = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return err;
    lc.max_smem.store(max_smem, std::memory_order_release);
    lc.n_sm.store(n_sm, std::memory_order_release);
  }
  const uint32_t stage_bytes = (uint32_t)max(G.gu_unit_bytes, 4 * G.dn_unit_bytes);
  // Work granularity.  One token gives a CTA fewer gate/up units than warps (4.75 of 14 at the pages' shape): that
  // instance splits each unit's K over two warps and gives each down stage one unit (21.2 -> 19.6 us per step on
  // B200); every other window keeps whole units and two-unit down stages.
  const int gu_cta = ((min(T * d.top_k, d.n_experts) + 1) * G.gu_units + n_sm - 1) / n_sm;
  const int inst = (T == 1 && G.gu_groups % 8 == 0 && gu_cta * 2 <= kMaxParts) ? 1 : 0;
  const int kp = inst ? 2 : 1;
  const SmemLayout L0 = smem_layout(T, G.H, 0, stage_bytes, kp);
  const int slots = (int)((max_smem - (int)L0.ring - 128) / (int)stage_bytes);
  if (slots < 1) return cudaErrorInvalidConfiguration;
  const int nw = min(kConsumerWarps, slots);  // warps streaming and computing stages, one slot each
  const int ns = nw;
  const SmemLayout L = smem_layout(T, G.H, ns, stage_bytes, kp);
  if (L.total > (uint32_t)max_smem) return cudaErrorInvalidConfiguration;
  // a CTA's down range spans at most two entries (the h cache of phase D holds two): at most dn_units units
  const int max_entries = min(T * d.top_k, d.n_experts) + 1;
  if ((max_entries * G.dn_units + n_sm - 1) / n_sm > G.dn_units) return cudaErrorInvalidConfiguration;
  const int rrows = (d.n_experts + n_sm - 1) / n_sm;  // router rows per CTA, staged in the ring
  if ((size_t)rrows * d.hidden * 4 > (size_t)ns * stage_bytes) return cudaErrorInvalidConfiguration;
  if ((size_t)T * d.n_experts * 4 > (size_t)ns * stage_bytes) return cudaErrorInvalidConfiguration;  // logits

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
  a.ready = ws.ready;
  a.gbar = ws.gbar;
  a.idx_out = idx_out;
  a.w_out = w_out;
  a.out = out;
  a.out_f32 = out_f32;
  a.status = ws.status;
  a.ns = ns;
  a.nw = nw;
  a.stage_bytes = stage_bytes;

  void (*kern)(DecodeArgs) = inst ? decode_fused_kernel<2, 1> : decode_fused_kernel<1, 2>;
  // The shared-memory opt-in and the residency check are done once per device, instance and shared-memory
  // size (they depend on nothing else), not on every call.
  if (lc.checked_smem[inst].load(std::memory_order_acquire) != L.total) {
    std::lock_guard<std::mutex> lock(lc.mu);
    if (L.total > lc.smem_attr[inst]) {
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
      if (err != cudaSuccess) return err;
      lc.smem_attr[inst] = L.total;
    }
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, L.total);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    lc.checked_smem[inst].store(L.total, std::memory_order_release);
  }

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  trace_mark(MOE_KERNEL_DECODE_FUSED, false, s);
  err = cudaLaunchKernelEx(&cfg, kern, a);
  trace_mark(MOE_KERNEL_DECODE_FUSED, true, s);
  return err;
}

}  // namespace moe
