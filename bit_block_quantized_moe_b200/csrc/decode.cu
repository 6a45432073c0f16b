// Fused decode/verify-window layer (T <= 8 tokens) in one persistent,
// cooperatively launched kernel (sm_100a).  One CTA per SM: 14 consumer
// warps and 1 producer warp.
//
//  A  The producer warp copies (cp.async, 16 B per lane) the tokens and this
//     CTA's router rows into shared memory and prefetches its slice of the
//     shared expert into L2.  Consumers compute the router rows (2 warps per row, one
//     half of K each) and the correction sums of the biased decode.
//     -- grid barrier: all logits written --
//  B  Every CTA selects the top-k of every token (threshold + rank, one warp
//     per token) and builds the same sorted list of touched experts plus the
//     shared expert.
//  C  Work lists, expert-major, cut into equal contiguous ranges per CTA:
//     gate/up units (expert, 8 intermediate rows) and down pairs (expert, 16
//     output rows).  The producer streams the CTA's units into a ring of
//     shared-memory stages as stages free up; stage s belongs to consumer
//     warp s % min(14, stages), which computes the whole unit (full K) with no cross-warp
//     reduction and writes h = silu(g) * u (bf16) straight from its
//     accumulators.  At the end the CTA publishes, per expert, how many of
//     its units are done.
//  D  Once the h of the (at most two) experts in the CTA's down range is
//     complete (per-expert counter, bounded wait) it is copied into shared
//     memory; each down stage (up to 4 pairs) again belongs to one warp:
//     partial = w[t, e] * (Wd_e h_e) per (expert, tile).  The last CTA to
//     contribute to a tile sums its partials in expert order and writes out
//     (bf16).
// Weights reach the tensor cores with no arithmetic: the 2-bit codes of a
// row are masked into e4m3 bytes (value q * 2^-9) that form the A fragment of
// an m16n8k32 fp8 MMA.  The tokens form the B fragment: each token vector is
// scaled by a power of two and split into two e4m3 terms (columns 2t and
// 2t+1, 4 tokens per MMA), exact for every element above 2^-8 of the
// vector's largest.  The -1 of d * (q - 1) starts the accumulator at minus the
// block sum of the token, and the fp16 block scale d multiplies each block's
// fp32 result.  Every wait is bounded (sync.cuh).
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
  uint64_t *gbar;      // monotonic grid-barrier arrival counter
  int32_t *idx_out;    // optional [T][k]
  float *w_out;        // optional [T][k]
  uint16_t *out;       // [T][H]
  uint32_t *status;
  int ns;              // ring stages: nw warps x (ns / nw) private slots each
  int nw;              // warps that stream and compute expert stages
  uint32_t stage_bytes;
};

struct SmemLayout {
  uint32_t xs, corr, xb, xsc, hb, hcorr, hsc, rpart, red, sel_idx, sel_w, bitmap, wpre, ent, tokj, tokw, misc,
      ring, total;
};

// Token quads: the 8 columns of an m16n8k32 MMA hold 4 tokens x 2 split terms.
__host__ __device__ inline int token_quads(int T) { return (T + 3) / 4; }

__host__ __device__ inline uint32_t align_to(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout smem_layout(int T, int H, int ns, uint32_t stage_bytes) {
  SmemLayout L;
  uint32_t o = 0;
  // xs: the tokens (bf16 rows, phase A).  The same bytes hold the h fragments of phase D.
  const uint32_t hb_bytes = 2u * token_quads(T) * (kMaxI / 32) * 256;
  const uint32_t hcorr_bytes = 2u * (kMaxI / 32) * kMaxTok * 4;
  const uint32_t xs_bytes = (uint32_t)T * (H + 16) * 2;
  L.xs = o;
  L.hb = o;  // [2 cached experts][quads][I/32][32] B fragments of h
  L.hcorr = o + hb_bytes;  // [2][I/32][8]
  L.hsc = L.hcorr + hcorr_bytes;  // [2][8]
  o = align_to(o + max(xs_bytes, hb_bytes + hcorr_bytes + 2u * kMaxTok * 4), 16);
  L.corr = o;  // [H/32 blocks][8 tokens]: -2^-9 * sum of the scaled tokens over the block
  o = align_to(o + (uint32_t)(H / 32) * kMaxTok * 4, 16);
  L.xb = o;  // [quads][H/32 blocks][32 lanes] B fragments (uint2) of the scaled, split tokens
  o = align_to(o + (uint32_t)token_quads(T) * (H / 32) * 256, 16);
  L.xsc = o;  // [8] 2^(9 - s_t): undoes the token scale and the 2^-9 of the A bytes
  o += kMaxTok * 4;
  L.rpart = o;  // [rows per pass][8 tokens][router parts]
  o += (kConsumerWarps / kRouterParts) * kMaxTok * kRouterParts * 4;
  L.red = o;  // top-k scratch (phase B: 64 uint64 per token), then the h staging of phase D: [2][T][I + 16] bf16
  o += align_to(max((uint32_t)kMaxTok * 64 * 8, 2u * T * (kMaxI + 16) * 2), 16);
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
  L.misc = o;  // [0] entries [1] abort [2] barrier flag [3] done tiles [8..15] token scale exponents
  o += 64;
  L.ring = align_to(o, 128);
  L.total = L.ring + (uint32_t)ns * stage_bytes;
  return L;
}

// Per-token power-of-two scales, block correction sums and e4m3 B fragments of
// the vectors v[t][0..K) (bf16 rows `stride` elements apart), t < T.  All
// consumer threads call it (it holds named barriers).
//   unscale[t] = 2^(9 - s_t), with max_k |v[t][k]| * 2^s_t in [128, 256);
//   corr[b][t] = -2^-9 * sum_{k in block b} v[t][k] * 2^s_t  (the -1 of q - 1);
//   frag[(quad * nb + b) * 32 + lane]: lane (g, c) holds column g = 2 * (t % 4)
//   + split term, rows k in block order e4m3_k_lo (x) / e4m3_k_hi (x, times 1/4).
__device__ void build_b_fragments(const uint16_t *v, int stride, int K, int T, int nq, uint2 *frag, float *corr,
                                  float *unscale, int *sexp, int warp, int lane, int tid) {
  const int nb = K / 32;
  if (warp < T) {
    uint32_t m = 0;  // largest |v| as a bf16 bit pattern (ordered like the magnitudes)
    for (int i = lane; i < K / 8; i += 32) {
      const uint4 u = *reinterpret_cast<const uint4 *>(v + warp * stride + 8 * i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) m = max(m, max(w[h] & 0x7FFFu, (w[h] >> 16) & 0x7FFFu));
    }
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == 0) {
      const int sx = e4m3_scale_exp(__uint_as_float(m << 16));
      sexp[warp] = sx;
      unscale[warp] = 512.f * exp2_int(-sx);
    }
  }
  named_bar(kBarConsumers, kConsumers);
  for (int i = tid; i < nb * kMaxTok; i += kConsumers) {
    const int b = i / kMaxTok, t = i % kMaxTok;
    float sum = 0.f;
    if (t < T) {
      const float sc = exp2_int(sexp[t]);
      const uint4 *row = reinterpret_cast<const uint4 *>(v + t * stride + 32 * b);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 u = row[q];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          sum = fmaf(__uint_as_float(w[h] << 16), sc, sum);
          sum = fmaf(__uint_as_float(w[h] & 0xffff0000u), sc, sum);
        }
      }
    }
    corr[b * kMaxTok + t] = -sum * (1.f / 512.f);
  }
  for (int i = tid; i < nq * nb * 32; i += kConsumers) {
    const int qd = i / (nb * 32), r = i % (nb * 32), b = r / 32, ln = r % 32;
    const int gq = ln >> 2, cq = ln & 3, t = 4 * qd + (gq >> 1), part = gq & 1;
    uint2 f = make_uint2(0u, 0u);
    if (t < T) {
      const float sc = exp2_int(sexp[t]);
      const uint16_t *row = v + t * stride + 32 * b;
      float lo[4], hi[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float vl = bf16_bits_to_float(row[e4m3_k_lo(cq, j)]) * sc;
        const float vh = bf16_bits_to_float(row[e4m3_k_hi(cq, j)]) * sc * 0.25f;
        const float hl = e4m3_split_hi(vl), hh = e4m3_split_hi(vh);
        lo[j] = part ? vl - hl : hl;
        hi[j] = part ? vh - hh : hh;
      }
      f.x = pack_e4m3x4(lo[0], lo[1], lo[2], lo[3]);
      f.y = pack_e4m3x4(hi[0], hi[1], hi[2], hi[3]);
    }
    frag[i] = f;
  }
  named_bar(kBarConsumers, kConsumers);
}

// One 16-row unit over n_groups block groups: acc[quad][r] with r = (row g,
// split 0), (row g, split 1), (row g+8, split 0), (row g+8, split 1) of token
// 4 * quad + c, in units of 2^(s_t - 9).  Four block tiles per group are
// staged: loads, code masking, one m16n8k32 MMA per quad (accumulator started
// at the block's correction), then the fp16 block scales.
// Block groups [grp0, grp1) of a unit whose K spans n_groups groups; adds to acc.
template <int NQ>
__device__ __forceinline__ void unit_gemv(const uint8_t *st, int grp0, int grp1, int n_groups, const uint2 *frag,
                                          const float *corr, int lane, float (&acc)[2][4]) {
  const int g = lane >> 2, c = lane & 3;
  const int nb = n_groups * 4;
  for (int grp = grp0; grp < grp1; ++grp) {
    const uint8_t *gp = st + (size_t)grp * kGroupBytes;
    const uint4 cw = lds128(gp + lane * 16);
    const uint4 sw = lds128(gp + kGroupCodeBytes + g * 16);
    const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
    const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
    uint2 bf[NQ][4];
    float cn[NQ][4];
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      const int b = grp * 4 + blk;
#pragma unroll
      for (int qd = 0; qd < NQ; ++qd) {
        bf[qd][blk] = frag[(qd * nb + b) * 32 + lane];
        cn[qd][blk] = corr[b * kMaxTok + 4 * qd + c];
      }
    }
    float d[NQ][4][4];
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      uint32_t am[4];
      decode_q2_e4m3(cws[blk], am);
#pragma unroll
      for (int qd = 0; qd < NQ; ++qd) {
        const float cin[4] = {cn[qd][blk], 0.f, cn[qd][blk], 0.f};
        mma_e4m3_16832(d[qd][blk], am, bf[qd][blk].x, bf[qd][blk].y, cin);
      }
    }
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      const float2 s2 = __half22float2(*reinterpret_cast<const __half2 *>(&sws[blk]));
#pragma unroll
      for (int qd = 0; qd < NQ; ++qd) {
        fma2_bcast(acc[qd][0], acc[qd][1], s2.x, d[qd][blk][0], d[qd][blk][1]);
        fma2_bcast(acc[qd][2], acc[qd][3], s2.y, d[qd][blk][2], d[qd][blk][3]);
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const PackedGeom &G = a.G;
  const int T = a.T, E = a.E, K = a.k, H = G.H, I = G.I;
  const SmemLayout L = smem_layout(T, H, a.ns, a.stage_bytes);
  uint16_t *xs = reinterpret_cast<uint16_t *>(smem + L.xs);
  float *corr = reinterpret_cast<float *>(smem + L.corr);
  uint2 *xb = reinterpret_cast<uint2 *>(smem + L.xb);
  float *xsc = reinterpret_cast<float *>(smem + L.xsc);
  uint2 *hb = reinterpret_cast<uint2 *>(smem + L.hb);
  float *hcorr = reinterpret_cast<float *>(smem + L.hcorr);
  float *hsc = reinterpret_cast<float *>(smem + L.hsc);
  const int nq = token_quads(T);
  float *rpart = reinterpret_cast<float *>(smem + L.rpart);
  float *red = reinterpret_cast<float *>(smem + L.red);
  int *sel_idx = reinterpret_cast<int *>(smem + L.sel_idx);
  float *sel_w = reinterpret_cast<float *>(smem + L.sel_w);
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + L.bitmap);
  uint32_t *wpre = reinterpret_cast<uint32_t *>(smem + L.wpre);
  int *ent = reinterpret_cast<int *>(smem + L.ent);
  int8_t *tokj = reinterpret_cast<int8_t *>(smem + L.tokj);
  float *tokw = reinterpret_cast<float *>(smem + L.tokw);
  int *misc = reinterpret_cast<int *>(smem + L.misc);
  uint8_t *ring = smem + L.ring;
  uint32_t *ready = a.tile_cnt + G.dn_units;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int xstride = H + 16;
  const int n_rrows = E > (int)blockIdx.x ? (E - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  float *wr_s = reinterpret_cast<float *>(ring);  // router rows live in the ring until phase C

  // ---------------- phase A: set-up, router ----------------
  if (tid == 0)
    for (int i = 0; i < 16; ++i) misc[i] = 0;
  // The tokens, then this CTA's router rows: cp.async pieces from every thread
  // (two commit groups), and an L2 prefetch of this CTA's slice of the shared expert.
  for (int i = tid; i < T * (H / 8); i += kConsumers) {
    const int t = i / (H / 8), c8 = i % (H / 8);
    cp_async16(xs + t * xstride + c8 * 8, a.x + (size_t)t * H + c8 * 8);
  }
  cp_async_commit();
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
  {
    if (blockIdx.x == 0)
      for (int i = tid; i < G.dn_units + kMaxEntries; i += kConsumers) a.tile_cnt[i] = 0u;
    cp_async_wait_group<1>();  // this thread's token pieces have landed
    named_bar(kBarConsumers, kConsumers);
    // Tokens as e4m3 B fragments: per-token power-of-two scale, two split terms.
    build_b_fragments(xs, xstride, H, T, nq, xb, corr, xsc, misc + 8, warp, lane, tid);
    cp_async_wait_group<0>();  // router rows
    named_bar(kBarConsumers, kConsumers);
    constexpr int kRowsPerPass = kConsumerWarps / kRouterParts;  // one warp per router row part
    for (int r0 = 0; r0 < n_rrows; r0 += kRowsPerPass) {
      const int r = r0 + warp / kRouterParts, q = warp % kRouterParts;
      if (r < n_rrows) {
        float acc[8];
        router_part<true>(xs, xstride, T, wr_s + (size_t)r * H, H, q, lane, acc);
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
          a.logits[(size_t)t * E + e] =
              router_combine(rpart + (rr * kMaxTok + t) * kRouterParts, a.bias ? a.bias[e] : 0.f);
        }
      }
      named_bar(kBarConsumers, kConsumers);
    }
    grid_barrier(a.gbar, kBarConsumers, kConsumers, tid == 0, a.status, &misc[2]);

    // ---------------- phase B: top-k and the touched-expert list ----------------
    // All logits into shared memory first (one coalesced pass through L2), then one warp per token.
    float *lg = reinterpret_cast<float *>(ring);  // the ring is free until the stages start
    for (int i = tid; i < T * E / 4; i += kConsumers)
      reinterpret_cast<float4 *>(lg)[i] = ldg_cg_f4(a.logits + 4 * (size_t)i);
    for (int i = (T * E / 4) * 4 + tid; i < T * E; i += kConsumers) lg[i] = __ldcg(a.logits + i);
    named_bar(kBarConsumers, kConsumers);
    if (warp < T) {
      int e;
      float wt;
      uint64_t *scratch = reinterpret_cast<uint64_t *>(red) + warp * 64;
      if (E <= 512)
        warp_topk_fast<16, true>(lg + (size_t)warp * E, E, K, lane, scratch, e, wt);
      else
        warp_topk_fast<32, true>(lg + (size_t)warp * E, E, K, lane, scratch, e, wt);
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
  __syncthreads();  // the list is visible to every warp

  const int nent = misc[0];
  const int n_gu = nent * G.gu_units, n_dn = nent * G.dn_units;
  const int g0 = (int)((long long)n_gu * blockIdx.x / gridDim.x);
  const int g1 = (int)((long long)n_gu * (blockIdx.x + 1) / gridDim.x);
  const int d0 = (int)((long long)n_dn * blockIdx.x / gridDim.x);
  const int d1 = (int)((long long)n_dn * (blockIdx.x + 1) / gridDim.x);
  const int pps = 2;  // down units (16 rows) per stage: enough stages to keep every warp busy
  const int n_gu_st = g1 - g0;
  const int n_dn_st = (d1 - d0 + pps - 1) / pps;
  const int n_st = n_gu_st + n_dn_st;
  // Stage s belongs to warp s % nw, which copies it (cp.async) into its own
  // ring slot, waits for its own copies, computes it and refills the slot with
  // its next stage s + nw.  No other warp touches the slot.
  const int nw = a.nw, spw = 1;
  auto expert_ptr = [&](int entry) -> const uint8_t * {
    const int e = ent[entry];
    return e == E ? a.shared : a.experts + (size_t)e * G.expert_bytes;
  };
  auto stage_ptr = [&](int s) { return ring + (size_t)(warp * spw + (s / nw) % spw) * a.stage_bytes; };
  // A stage is copied as 4 commit groups (its quarters, in order) so that the
  // warp can start on the first quarter while the rest is still arriving:
  // gate/up = one unit (quarter = 4 block groups), down = 2 units of 16 rows
  // (quarter = half a unit).  Past the last stage the groups are empty.
  auto issue_stage = [&](int s) {
    for (int qt = 0; qt < 4; ++qt) {
      if (s < n_st) {
        uint8_t *dst = stage_ptr(s);
        if (s < n_gu_st) {
          const int id = g0 + s;
          const size_t qb = G.gu_unit_bytes / 4;
          warp_cp_async(dst + qt * qb,
                        expert_ptr(id / G.gu_units) + (size_t)(id % G.gu_units) * G.gu_unit_bytes + qt * qb,
                        (uint32_t)qb, lane);
        } else {
          const int q = d0 + (s - n_gu_st) * pps + (qt >> 1);
          const size_t hb2 = G.dn_unit_bytes / 2;
          if (q < d1)
            warp_cp_async(dst + (size_t)(qt >> 1) * G.dn_unit_bytes + (qt & 1) * hb2,
                          expert_ptr(q / G.dn_units) + G.gu_bytes + (size_t)(q % G.dn_units) * G.dn_unit_bytes +
                              (qt & 1) * hb2,
                          (uint32_t)hb2, lane);
        }
      }
      cp_async_commit();
    }
  };
  // quarter qt of the warp's current stage has landed (spw == 1: nothing newer is in flight)
  auto wait_quarter = [&](int qt) {
    if (qt == 0)
      cp_async_wait_group<3>();
    else if (qt == 1)
      cp_async_wait_group<2>();
    else if (qt == 2)
      cp_async_wait_group<1>();
    else
      cp_async_wait_group<0>();
    __syncwarp();
  };
  if (warp < nw) issue_stage(warp);

  // ---------------- consumers, phase C: gate/up + SwiGLU ----------------
  for (int s_idx = warp; warp < nw && s_idx < n_gu_st; s_idx += nw) {
    const uint8_t *st = stage_ptr(s_idx);
    float acc[2][4] = {};
    const int gq = G.gu_groups / 4;  // block groups per quarter
    for (int qt = 0; qt < 4; ++qt) {
      wait_quarter(qt);
      if (nq == 1)
        unit_gemv<1>(st, qt * gq, (qt + 1) * gq, G.gu_groups, xb, corr, lane, acc);
      else
        unit_gemv<2>(st, qt * gq, (qt + 1) * gq, G.gu_groups, xb, corr, lane, acc);
    }
    __syncwarp();
    issue_stage(s_idx + spw * nw);
    const int id = g0 + s_idx;
    const int entry = id / G.gu_units, u = id % G.gu_units;
    const int i = 8 * u + g;  // tile rows g (gate) and g+8 (up) share intermediate row i
#pragma unroll
    for (int qd = 0; qd < 2; ++qd) {
      const int n = 4 * qd + c;  // this lane's token
      if (qd < nq && n < T) {
        const int j = tokj[entry * kMaxTok + n];
        const float gate = (acc[qd][0] + acc[qd][1]) * xsc[n], up = (acc[qd][2] + acc[qd][3]) * xsc[n];
        if (j >= 0) a.h[((size_t)n * (K + 1) + j) * I + i] = float_to_bf16_bits(silu_f(gate) * up);
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
  for (int i = tid; i < n_hc * T * (I / 8); i += kConsumers) {
    const int he = i / (T * (I / 8)), r = i % (T * (I / 8));
    const int t = r / (I / 8), c8 = r % (I / 8);
    const int j = tokj[(e_lo + he) * kMaxTok + t];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j >= 0) v = __ldcg(reinterpret_cast<const uint4 *>(a.h + ((size_t)t * (K + 1) + j) * I + c8 * 8));
    *reinterpret_cast<uint4 *>(hc + (he * T + t) * hstride + c8 * 8) = v;
  }
  named_bar(kBarConsumers, kConsumers);
  for (int he = 0; he < n_hc; ++he)
    build_b_fragments(hc + he * T * hstride, hstride, I, T, nq, hb + he * nq * (kMaxI / 32) * 32,
                      hcorr + he * (kMaxI / 32) * kMaxTok, hsc + he * kMaxTok, misc + 8, warp, lane, tid);

  for (int s_idx = n_gu_st + ((warp - n_gu_st % nw + nw) % nw); warp < nw && s_idx < n_st; s_idx += nw) {
    const int sd = s_idx - n_gu_st;
    const uint8_t *st = stage_ptr(s_idx);
    const int q0 = d0 + sd * pps, q1 = min(d1, q0 + pps);
    for (int q = q0; q < q1; ++q) {
      const int entry = q / G.dn_units, tile = q % G.dn_units, he = entry - e_lo;
      const uint8_t *pp_st = st + (size_t)(q - q0) * G.dn_unit_bytes;
      const uint2 *hbe = hb + he * nq * (kMaxI / 32) * 32;
      const float *hce = hcorr + he * (kMaxI / 32) * kMaxTok;
      float acc[2][4] = {};
      const int hg = G.dn_groups / 2;  // block groups per half unit
      for (int h2 = 0; h2 < 2; ++h2) {
        wait_quarter(2 * (q - q0) + h2);
        if (nq == 1)
          unit_gemv<1>(pp_st, h2 * hg, (h2 + 1) * hg, G.dn_groups, hbe, hce, lane, acc);
        else
          unit_gemv<2>(pp_st, h2 * hg, (h2 + 1) * hg, G.dn_groups, hbe, hce, lane, acc);
      }
      // partial tile layout: lane (g, c) -> {row g tok c, row g+8 tok c, row g tok c+4, row g+8 tok c+4}
      float o4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int qd = 0; qd < 2; ++qd) {
        if (qd >= nq) break;
        const int n = 4 * qd + c;
        const float f = hsc[he * kMaxTok + n] * tokw[entry * kMaxTok + n];
        o4[2 * qd] = (acc[qd][0] + acc[qd][1]) * f;
        o4[2 * qd + 1] = (acc[qd][2] + acc[qd][3]) * f;
      }
      float *pp = a.partial + ((size_t)entry * G.dn_units + tile) * 128;
      *reinterpret_cast<float4 *>(pp + lane * 4) = make_float4(o4[0], o4[1], o4[2], o4[3]);
    }
    __syncwarp();
    issue_stage(s_idx + spw * nw);
  }
  cp_async_wait_all();  // nothing of this thread's may still be landing when the CTA ends

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
    for (int qd = 0; qd < 2; ++qd) {
      const int n = 4 * qd + c;
      if (n < T) {
        a.out[(size_t)n * H + r0] = float_to_bf16_bits(o[2 * qd]);
        a.out[(size_t)n * H + r0 + 8] = float_to_bf16_bits(o[2 * qd + 1]);
      }
    }
  }
}

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
  const int slots = (int)((max_smem - (int)L0.ring - 128) / (int)stage_bytes);
  if (slots < 1) return cudaErrorInvalidConfiguration;
  const int nw = min(kConsumerWarps, slots);  // warps streaming and computing stages, one slot each
  const int ns = nw;
  const SmemLayout L = smem_layout(T, G.H, ns, stage_bytes);
  if (L.total > (uint32_t)max_smem) return cudaErrorInvalidConfiguration;
  // the per-CTA down range must fit the 128-entry completed-tile list
  const int max_entries = min(T * d.top_k, d.n_experts) + 1;
  if ((max_entries * G.dn_units + n_sm - 1) / n_sm > kMaxSel) return cudaErrorInvalidConfiguration;
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
  a.tile_cnt = ws.tile_cnt;
  a.gbar = ws.gbar;
  a.idx_out = idx_out;
  a.w_out = w_out;
  a.out = out;
  a.status = ws.status;
  a.ns = ns;
  a.nw = nw;
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
