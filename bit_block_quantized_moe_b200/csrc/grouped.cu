// Grouped expert GEMMs for many tokens (T > 8) on m16n8k32 e4m3 tensor-core
// MMAs (sm_100a).
//
// Per call, after routing and dispatch:
//   frag_prep (x)  one warp per token: power-of-two scale, block correction
//                  sums and the two-term e4m3 split of the token, stored in
//                  MMA B-fragment order: per 128-wide K chunk, four 64-byte
//                  block records and the four block corrections (272 B);
//   grouped<0>     gate/up + SwiGLU -> h (bf16) per sorted position;
//   frag_prep (h)  the same for every h row;
//   grouped<1>     down -> fp32 expert output per sorted position, summed by
//                  the combine kernel.
// grouped<MODE> runs one persistent CTA per SM with 16 warps.  A work item is a token tile (<= 32 sorted positions of one
// expert) times a group of 16 units (16-row tiles of the projection).  For
// every 128-wide K chunk the warps copy (cp.async, 16 B per lane; warp u takes
// unit u and every 16th token) the 16 units' packed codes and scales of that
// chunk (640 B each) and each token's 272-byte chunk record into a
// shared-memory stage, ns stages ahead of use; warp u runs unit
// u's 4 block tiles against every token quad of the tile (one m16n8k32 MMA per
// block and quad, accumulator started at the block correction), scales each
// block result by its fp16 d and keeps the sums in registers across chunks.
// The codes enter the MMA as masked bytes (decode_q2_e4m3); every wait is
// bounded (sync.cuh).
#include "kernels.cuh"
#include "sync.cuh"

namespace moe {

namespace {

constexpr int kGW = 16;                   // consumer warps = units per work item
constexpr int kGThreads = kGW * 32;
constexpr int kTileTok = 32;              // sorted positions per work item (8 token quads)
constexpr int kChunkRec = 4 * 64 + 16;     // per token and K chunk: 4 block records + 4 corrections
constexpr int kTokStride = 320;            // shared-memory stride of a token's chunk record (bank spread)
constexpr int kStageA = kGW * kGroupBytes;               // 10240: one block group of 16 units
constexpr int kStageB = kTileTok * kTokStride;           // 10240
constexpr int kStageBytes = kStageA + kStageB;           // 20480
constexpr int kMaxStages = 16;
static_assert(kStageBytes % 128 == 0, "stages keep 128-byte alignment");

struct GArgs {
  const uint8_t *experts;
  const uint8_t *shared;
  PackedGeom G;
  int E;
  const int4 *tiles;          // (expert or E for the shared expert, first sorted position, tokens <= 32, 0)
  const uint32_t *n_tiles;
  int units;                  // 16-row units per expert in this projection
  int ugroups;                // ceil(units / 16)
  int kchunks;                // 128-wide K chunks
  size_t unit_bytes;
  size_t sec_off;             // section offset inside a packed expert
  const uint8_t *frag;        // [rows][K/128][272 B] chunk records
  const float *unscale;       // [rows]
  const int32_t *row_of_pos;  // gate/up: token of each sorted position; down: null (row = position)
  uint16_t *h_out;            // gate/up: [positions][I] bf16
  float *y_out;               // down: [positions][H] fp32
  uint32_t *status;
  int ns;
};

// One block group (4 block tiles) of one unit against NQ token quads.
template <int NQ>
__device__ __forceinline__ void chunk_mma(const uint8_t *st, int u, int lane, float (&acc)[8][4]) {
  const int g = lane >> 2, c = lane & 3;
  const uint8_t *gp = st + u * kGroupBytes;
  const uint4 cw = lds128(gp + lane * 16);
  const uint4 sw = lds128(gp + kGroupCodeBytes + g * 16);
  const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
  const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
  // lane (g, c) reads column g = 2 * (token in quad) + split term: token g / 2 of the quad
  const uint8_t *bq = st + kStageA + (g >> 1) * kTokStride + (g & 1) * 32 + c * 8;
  const uint8_t *cq = st + kStageA + c * kTokStride + 4 * 64;  // corrections of token c of each quad
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    uint32_t am[4];
    decode_q2_e4m3(cws[blk], am);
    const float2 s2 = __half22float2(*reinterpret_cast<const __half2 *>(&sws[blk]));
#pragma unroll
    for (int qd = 0; qd < NQ; ++qd) {
      const uint2 bf = *reinterpret_cast<const uint2 *>(bq + qd * 4 * kTokStride + blk * 64);
      const float cn = *reinterpret_cast<const float *>(cq + qd * 4 * kTokStride + blk * 4);
      const float cin[4] = {cn, 0.f, cn, 0.f};
      float d[4];
      mma_e4m3_16832(d, am, bf.x, bf.y, cin);
      fma2_bcast(acc[qd][0], acc[qd][1], s2.x, d[0], d[1]);
      fma2_bcast(acc[qd][2], acc[qd][3], s2.y, d[2], d[3]);
    }
  }
}

template <int MODE>  // 0: gate/up + SwiGLU -> h; 1: down -> y
__global__ void __launch_bounds__(kGThreads, 1) grouped_kernel(const GArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)a.ns * kStageBytes);
  uint64_t *empty = full + a.ns;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + a.ns);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_work = (int)*a.n_tiles * a.ugroups;

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.ns; ++i) {
      mbar_init(&full[i], kGThreads);  // one cp.async arrival per thread
      mbar_init(&empty[i], kGW);       // one arrival per warp once it has read the stage
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  const int u = warp, g = lane >> 2, c = lane & 3;
  const int n_stages = ((n_work - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * a.kchunks;
  // Every warp copies its share of stage q (this CTA's q-th K chunk): unit u's
  // 640-byte piece and the chunk records of tokens u and u + 16; then each
  // thread arrives on the stage's full barrier once its copies have landed.
  auto issue = [&](int q) {
    const int w = (int)blockIdx.x + (q / a.kchunks) * (int)gridDim.x, kc = q % a.kchunks;
    const int4 tile = a.tiles[w / a.ugroups];
    const int u0 = (w % a.ugroups) * kGW, nu = min(kGW, a.units - u0);
    uint8_t *st = smem + (size_t)(q % a.ns) * kStageBytes;
    if (u < nu) {
      const uint8_t *src = (tile.x == a.E ? a.shared : a.experts + (size_t)tile.x * a.G.expert_bytes) + a.sec_off +
                           (size_t)(u0 + u) * a.unit_bytes + (size_t)kc * kGroupBytes;
      for (int i = lane; i < kGroupBytes / 16; i += 32) cp_async16(st + u * kGroupBytes + i * 16, src + i * 16);
    }
    for (int tk = u; tk < tile.z; tk += kGW) {
      const int r = a.row_of_pos ? a.row_of_pos[tile.y + tk] : tile.y + tk;
      if (lane < kChunkRec / 16)
        cp_async16(st + kStageA + tk * kTokStride + lane * 16,
                   a.frag + ((size_t)r * a.kchunks + kc) * kChunkRec + lane * 16);
    }
    cp_async_arrive(&full[q % a.ns]);
  };
  for (int q = 0; q < min(a.ns, n_stages); ++q) issue(q);

  int cnt = 0;
  for (int w = blockIdx.x; w < n_work; w += gridDim.x) {
    const int4 tile = a.tiles[w / a.ugroups];
    const int unit = (w % a.ugroups) * kGW + u;
    const bool active = unit < a.units;
    const int nq = (tile.z + 3) >> 2;
    float acc[8][4];
#pragma unroll
    for (int qd = 0; qd < 8; ++qd)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[qd][r] = 0.f;
    for (int kc = 0; kc < a.kchunks; ++kc, ++cnt) {
      const int s = cnt % a.ns;
      if (!*abort_flag && !mbar_wait(&full[s], (cnt / a.ns) & 1)) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      if (!*abort_flag && active) {
        const uint8_t *st = smem + (size_t)s * kStageBytes;
        switch (nq) {
          case 1: chunk_mma<1>(st, u, lane, acc); break;
          case 2: chunk_mma<2>(st, u, lane, acc); break;
          case 3: chunk_mma<3>(st, u, lane, acc); break;
          case 4: chunk_mma<4>(st, u, lane, acc); break;
          case 5: chunk_mma<5>(st, u, lane, acc); break;
          case 6: chunk_mma<6>(st, u, lane, acc); break;
          case 7: chunk_mma<7>(st, u, lane, acc); break;
          default: chunk_mma<8>(st, u, lane, acc); break;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      // refill this slot with stage cnt + ns once every warp has read it
      if (cnt + a.ns < n_stages) {
        if (!*abort_flag && !mbar_wait(&empty[s], (cnt / a.ns) & 1)) {
          set_status(a.status, kStatusTimeout);
          *abort_flag = 1;
        }
        if (!*abort_flag) issue(cnt + a.ns);
      }
    }
    if (!active || *abort_flag) continue;
#pragma unroll
    for (int qd = 0; qd < 8; ++qd) {
      const int n = 4 * qd + c;
      if (qd < nq && n < tile.z) {
        const int p = tile.y + n;
        if (MODE == 0) {
          const float us = a.unscale[a.row_of_pos[p]];
          const float gate = (acc[qd][0] + acc[qd][1]) * us, up = (acc[qd][2] + acc[qd][3]) * us;
          a.h_out[(size_t)p * a.G.I + 8 * unit + g] = float_to_bf16_bits(silu_f(gate) * up);
        } else {
          const float us = a.unscale[p];
          float *yr = a.y_out + (size_t)p * a.G.H + 16 * unit + g;
          yr[0] = (acc[qd][0] + acc[qd][1]) * us;
          yr[8] = (acc[qd][2] + acc[qd][3]) * us;
        }
      }
    }
  }
  cp_async_wait_all();  // nothing of this thread's may still be landing when the CTA ends
}

// One warp per row of v ([rows][K] bf16): the row's unscale factor 2^(9 - s),
// with max |v| * 2^s in [128, 256), and per 128-wide K chunk a 272-byte record:
// for each of its 4 blocks b a 64-byte record of B-fragment words (for split
// term t (0: high 4 bits, 1: the rest) and lane column c, the pair (lo, hi) at
// byte (4t + c) * 8, lo holding block positions e4m3_k_lo(c, 0..3), hi
// positions e4m3_k_hi(c, 0..3) times 1/4), then the 4 block corrections
// -2^-9 * sum_k v[k] * 2^s.
__global__ void __launch_bounds__(256) frag_prep_kernel(const uint16_t *__restrict__ v, int rows, int K,
                                                        uint8_t *__restrict__ frag, float *__restrict__ unscale) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int nb = K / 32;
  const uint4 *src = reinterpret_cast<const uint4 *>(v + (size_t)row * K);
  uint32_t m = 0;
  for (int i = lane; i < K / 8; i += 32) {
    const uint4 q = src[i];
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) m = max(m, max(wv[h] & 0x7FFFu, (wv[h] >> 16) & 0x7FFFu));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  const int sx = e4m3_scale_exp(__uint_as_float(m << 16));
  const float sc = exp2_int(sx);
  if (lane == 0) unscale[row] = 512.f * exp2_int(-sx);
  for (int b = lane; b < nb; b += 32) {
    uint32_t wv[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u4 = src[b * 4 + q];
      wv[4 * q] = u4.x;
      wv[4 * q + 1] = u4.y;
      wv[4 * q + 2] = u4.z;
      wv[4 * q + 3] = u4.w;
    }
    auto val = [&](int k) {
      return __uint_as_float((k & 1) ? (wv[k >> 1] & 0xffff0000u) : (wv[k >> 1] << 16)) * sc;
    };
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) sum += val(k);
    uint8_t *chunk = frag + ((size_t)row * (nb / 4) + b / 4) * kChunkRec;
    reinterpret_cast<float *>(chunk + 4 * 64)[b % 4] = -sum * (1.f / 512.f);
    uint32_t rec[16];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float lo[4], hi[4], lo2[4], hi2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float vl = val(e4m3_k_lo(c, i)), vh = val(e4m3_k_hi(c, i)) * 0.25f;
        lo[i] = e4m3_split_hi(vl);
        lo2[i] = vl - lo[i];
        hi[i] = e4m3_split_hi(vh);
        hi2[i] = vh - hi[i];
      }
      rec[c * 2] = pack_e4m3x4(lo[0], lo[1], lo[2], lo[3]);
      rec[c * 2 + 1] = pack_e4m3x4(hi[0], hi[1], hi[2], hi[3]);
      rec[8 + c * 2] = pack_e4m3x4(lo2[0], lo2[1], lo2[2], lo2[3]);
      rec[8 + c * 2 + 1] = pack_e4m3x4(hi2[0], hi2[1], hi2[2], hi2[3]);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(chunk + (b % 4) * 64);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(rec[4 * q], rec[4 * q + 1], rec[4 * q + 2], rec[4 * q + 3]);
  }
}

size_t grouped_smem_bytes(int ns) { return (size_t)ns * kStageBytes + 2 * ns * 8 + 16; }

template <int MODE>
cudaError_t launch_grouped(const GArgs &a0, int n_sm, int max_smem, cudaStream_t s) {
  GArgs a = a0;
  a.ns = min(kMaxStages, (int)((max_smem - 64) / (kStageBytes + 16)));
  if (a.ns < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = grouped_smem_bytes(a.ns);
  cudaError_t err = cudaFuncSetAttribute(grouped_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, grouped_kernel<MODE>, kGThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  grouped_kernel<MODE><<<n_sm, kGThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_experts(const moe_dims &d, const PackedGeom &G, const uint8_t *experts,
                                   const uint8_t *shared, const uint16_t *x, int T, const Workspace &ws,
                                   cudaStream_t s) {
  const int P = T * d.top_k + T;  // sorted positions (routed + shared)
  int dev = 0, n_sm = 0, max_smem = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);

  trace_mark(MOE_KERNEL_FRAG_X, false, s);
  frag_prep_kernel<<<(unsigned)((T + 7) / 8), 256, 0, s>>>(x, T, G.H, ws.xf, ws.xunscale);
  trace_mark(MOE_KERNEL_FRAG_X, true, s);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  GArgs a{};
  a.experts = experts;
  a.shared = shared;
  a.G = G;
  a.E = d.n_experts;
  a.tiles = ws.g_tiles;
  a.n_tiles = ws.n_g_tiles;
  a.status = ws.status;
  a.h_out = ws.h;
  a.y_out = ws.y;

  // gate/up + SwiGLU: units of 8 gate + 8 up rows, K = H
  a.units = G.gu_units;
  a.ugroups = (G.gu_units + kGW - 1) / kGW;
  a.kchunks = G.gu_groups;
  a.unit_bytes = G.gu_unit_bytes;
  a.sec_off = 0;
  a.frag = ws.xf;
  a.unscale = ws.xunscale;
  a.row_of_pos = ws.sorted_tok;
  trace_mark(MOE_KERNEL_GATE_UP, false, s);
  err = launch_grouped<0>(a, n_sm, max_smem, s);
  trace_mark(MOE_KERNEL_GATE_UP, true, s);
  if (err != cudaSuccess) return err;

  trace_mark(MOE_KERNEL_FRAG_H, false, s);
  frag_prep_kernel<<<(unsigned)((P + 7) / 8), 256, 0, s>>>(ws.h, P, G.I, ws.hf, ws.hunscale);
  trace_mark(MOE_KERNEL_FRAG_H, true, s);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  // down: units of 16 output rows, K = I
  a.units = G.dn_units;
  a.ugroups = (G.dn_units + kGW - 1) / kGW;
  a.kchunks = G.dn_groups;
  a.unit_bytes = G.dn_unit_bytes;
  a.sec_off = G.gu_bytes;
  a.frag = ws.hf;
  a.unscale = ws.hunscale;
  a.row_of_pos = nullptr;
  trace_mark(MOE_KERNEL_DOWN, false, s);
  err = launch_grouped<1>(a, n_sm, max_smem, s);
  trace_mark(MOE_KERNEL_DOWN, true, s);
  return err;
}

}  // namespace moe
