// Router logits for many tokens on the 5th-generation tensor cores (tcgen05,
// sm_100a).
//
// logits[t][e] = sum_k x[t][k] * Wr[e][k] + b[e] with bf16 tokens and fp32
// router weights.  A first kernel splits the weights into three bf16 planes,
// w = hi + mid + lo exactly (split3_bf16); every product token * plane is then
// exact in the fp32 accumulator.  One CTA tile is 128 experts (tensor-memory
// lanes) x 64 tokens.  K runs in 256-wide slices: each slice, 3 planes x 16 K
// steps of tcgen05.mma into a fresh tensor-memory accumulator, is added in
// fp32 to a running sum in the epilogue threads' registers, slice after slice
// in K order.  When the tiles alone would leave SMs idle, K is also split
// across CTAs; a last kernel adds the partial sums in split order plus the
// bias.  The result is deterministic.
//   producer warp    : per 64-wide K chunk, TMA loads of the three planes'
//                      128 x 64 boxes (rows past E read as zeros) and of the
//                      64 x 64 token box (rows past T read as zeros), 128-byte
//                      swizzle, into one of 3 shared-memory stages;
//   MMA warp         : 12 tcgen05.mma per chunk, both operands in shared
//                      memory, double-buffered slice accumulators;
//   4 epilogue warps : tcgen05.ld of each finished slice, fp32 add to the
//                      running sums, then the tile (plus bias) or its K-split
//                      partial, one coalesced 128-byte row per token.
// Every wait is bounded (sync.cuh).
#include <algorithm>

#include "kernels.cuh"
#include "router.cuh"
#include "tc.cuh"

namespace moe {

namespace {

constexpr int kRtM = 128;                                     // experts per tile
constexpr int kRtN = 64;                                      // tokens per tile
constexpr int kRtK = 64;                                      // K per chunk: one 128-byte swizzle row of bf16
constexpr int kRtSlice = 256;                                 // K per fresh accumulator
constexpr int kRtStages = 3;
constexpr int kRtPlaneBytes = kRtM * kRtK * 2;                // 16 KB
constexpr int kRtBBytes = kRtN * kRtK * 2;                    // 8 KB
constexpr int kRtStageBytes = 3 * kRtPlaneBytes + kRtBBytes;  // 56 KB
constexpr int kRtThreads = 6 * 32;                            // producer, MMA, 4 epilogue warps
constexpr int kRtWave = 148;                                  // work units aimed at per wave (one per SM)
constexpr uint32_t kRtTmemCols = 2 * kRtN;
static_assert(kRtStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the 128-byte swizzle");

struct RtBars {
  uint64_t full[kRtStages], empty[kRtStages], dfull[2], dempty[2], done;
  uint32_t tmem;
  int abort;
};

struct RtArgs {
  int T, E, H;
  int ks;            // K splits
  int n_et, n_units;
  const float *bias;  // applied here when ks == 1
  float *out;         // logits [T][E] when ks == 1, else partials [ks][T][E]
  uint32_t *status;
};

__device__ __forceinline__ bool rt_wait(uint64_t *bar, uint32_t parity, RtBars &B, uint32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*reinterpret_cast<volatile int *>(&B.abort)) return false;
  if (!mbar_wait(bar, parity)) {
    set_status(status, kStatusTimeout);
    B.abort = 1;
    return false;
  }
  return true;
}

__global__ void router_split_kernel(const float4 *__restrict__ w, size_t n4, uint2 *__restrict__ planes,
                                    uint32_t *zero_p, size_t zero_n) {
  clear_range(zero_p, zero_n);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = w[i];
    uint16_t h[4], m[4], l[4];
    split3_bf16(v.x, h[0], m[0], l[0]);
    split3_bf16(v.y, h[1], m[1], l[1]);
    split3_bf16(v.z, h[2], m[2], l[2]);
    split3_bf16(v.w, h[3], m[3], l[3]);
    planes[i] = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
    planes[n4 + i] = make_uint2(m[0] | ((uint32_t)m[1] << 16), m[2] | ((uint32_t)m[3] << 16));
    planes[2 * n4 + i] = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
  }
}

__global__ void __launch_bounds__(kRtThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, RtArgs a) {
  extern __shared__ __align__(1024) uint8_t rt_raw[];
  uint8_t *smem = rt_raw + ((1024u - (smem_u32(rt_raw) & 1023u)) & 1023u);
  RtBars &B = *reinterpret_cast<RtBars *>(smem + kRtStages * kRtStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kper = a.H / a.ks, slices = kper / kRtSlice;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRtStages; ++i) {
      mbar_init(&B.full[i], 1);
      mbar_init(&B.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.dfull[i], 1);
      mbar_init(&B.dempty[i], 4);
    }
    mbar_init(&B.done, 1);
    B.abort = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&B.tmem, kRtTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = B.tmem;

  if (warp == 0) {
    // The whole warp runs the loop on warp-uniform values; one elected lane issues the copies.  After a wait
    // gives up no further copy is issued, so the copies in flight are those of counts [issued - stages, issued).
    int cnt = 0, issued = 0;
    bool live = true;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
      const int ks = u % a.ks, tile = u / a.ks, et = tile % a.n_et, tt = tile / a.n_et;
      for (int c = 0; c < kper / kRtK; ++c, ++cnt) {
        const int s = cnt % kRtStages;
        if (live && !rt_wait(&B.empty[s], ((cnt / kRtStages) & 1) ^ 1, B, a.status)) live = false;
        if (!live) continue;
        issued = cnt + 1;
        if (elect_one()) {
          uint8_t *st = smem + s * kRtStageBytes;
          mbar_arrive_expect_tx(&B.full[s], (uint32_t)kRtStageBytes);
          const int k0 = ks * kper + c * kRtK;
          for (int p = 0; p < 3; ++p) tma_load_3d(st + p * kRtPlaneBytes, &wmap, k0, et * kRtM, p, &B.full[s]);
          tma_load_2d(st + 3 * kRtPlaneBytes, &xmap, k0, tt * kRtN, &B.full[s]);
        }
        __syncwarp();
      }
    }
    // Every copy issued must land before the CTA exits, also after an abort: a bounded wait of its own
    // (the shared abort flag would end it at once), the phase of count c2 being the last one its stage had.
    for (int c2 = max(0, issued - kRtStages); c2 < issued; ++c2)
      if (!mbar_wait(&B.full[c2 % kRtStages], (c2 / kRtStages) & 1)) set_status(a.status, kStatusTimeout);
  } else if (warp == 1) {
    // The whole warp runs the loop on warp-uniform values; one elected lane issues the MMAs and commits (a
    // lane-0-only loop issues them about 20% slower).
    const uint32_t idesc = umma_idesc_bf16(kRtM, kRtN);
    int cnt = 0, sc = 0;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
      for (int sl = 0; sl < slices; ++sl, ++sc) {
        const int db = sc & 1;
        rt_wait(&B.dempty[db], ((sc >> 1) & 1) ^ 1, B, a.status);
        tc_fence_after();
        const uint32_t dcol = tbase + db * kRtN;
        for (int c = 0; c < kRtSlice / kRtK; ++c, ++cnt) {
          const int s = cnt % kRtStages;
          rt_wait(&B.full[s], (cnt / kRtStages) & 1, B, a.status);
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * kRtStageBytes);
          const uint64_t bdesc0 = umma_sdesc_sw128(st + 3 * kRtPlaneBytes);
          if (elect_one()) {
#pragma unroll
            for (int p = 0; p < 3; ++p) {
              const uint64_t adesc0 = umma_sdesc_sw128(st + p * kRtPlaneBytes);
              // K step j: 32 bytes further along the swizzled 128-byte rows (2 in the 16-byte address field)
#pragma unroll
              for (int j = 0; j < kRtK / 16; ++j)
                umma_ss(dcol, adesc0 + 2 * j, bdesc0 + 2 * j, idesc, (c | p | j) != 0);
            }
            umma_commit(&B.empty[s]);
          }
          __syncwarp();
        }
        if (elect_one()) umma_commit(&B.dfull[db]);
        __syncwarp();
      }
    }
    // all MMAs issued by this warp have completed before tensor memory is released
    if (elect_one()) {
      umma_commit(&B.done);
      if (!mbar_wait(&B.done, 0)) set_status(a.status, kStatusTimeout);
    }
    __syncwarp();
  } else {
    // ---- epilogue: TMEM lane quadrant q = rows 32q .. 32q + 31 of the tile ----
    const int q = warp & 3;
    int sc = 0;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
      const int ks = u % a.ks, tile = u / a.ks, et = tile % a.n_et, tt = tile / a.n_et;
      float run[kRtN];
#pragma unroll
      for (int n = 0; n < kRtN; ++n) run[n] = 0.f;
      for (int sl = 0; sl < slices; ++sl, ++sc) {
        const int db = sc & 1;
        rt_wait(&B.dfull[db], (sc >> 1) & 1, B, a.status);
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < kRtN / 32; ++h) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + ((uint32_t)(32 * q) << 16) + db * kRtN + 32 * h, v);
          tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < 32; ++n) run[32 * h + n] += __uint_as_float(v[n]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.dempty[db]);
      }
      const int e = et * kRtM + 32 * q + lane;
      if (e < a.E) {
        const float b = (a.ks == 1 && a.bias) ? a.bias[e] : 0.f;
        float *o = a.out + (size_t)ks * a.T * a.E;
#pragma unroll
        for (int n = 0; n < kRtN; ++n) {
          const int t = tt * kRtN + n;
          if (t < a.T) o[(size_t)t * a.E + e] = run[n] + b;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kRtTmemCols);
  }
}

// logits = ((p_0 + p_1) + ...) + b, the K-split partials in split order.
__global__ void router_ksum_kernel(const float *__restrict__ part, int ks, size_t TE, int E,
                                   const float *__restrict__ bias, float *__restrict__ logits) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < TE; i += (size_t)gridDim.x * blockDim.x) {
    float s = part[i];
    for (int j = 1; j < ks; ++j) s += part[(size_t)j * TE + i];
    logits[i] = s + (bias ? bias[i % E] : 0.f);
  }
}

// 3-D map over the weight planes [3][E][H] bf16: boxes of 128 rows x 64 columns, 128-byte swizzle.
bool make_planes_map(CUtensorMap *map, const void *base, int E, int H) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)H, (cuuint64_t)E, 3};
  const cuuint64_t strides[2] = {(cuuint64_t)H * 2, (cuuint64_t)E * H * 2};
  const cuuint32_t box[3] = {kRtK, kRtM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool router_tc_supported(const moe_dims &d, int T) { return T > 8 && d.hidden % kRtSlice == 0; }

int router_tc_ksplit(const moe_dims &d, int T) {
  const int tiles = ((d.n_experts + kRtM - 1) / kRtM) * ((T + kRtN - 1) / kRtN);
  const int slices = d.hidden / kRtSlice;
  int ks = 1;
  while (ks * 2 <= slices && slices % (ks * 2) == 0 && tiles * ks * 2 <= kRtWave) ks *= 2;
  return ks;
}

// K-split partials never exceed one wave of tiles: ksplit x tiles <= kRtWave, so ksplit x T x E <= kRtWave x
// kRtM x kRtN.  Sizing the workspace with this bound keeps moe_workspace_bytes(max_T) valid for every T <= max_T.
size_t router_tc_partial_bytes_max() { return (size_t)kRtWave * kRtM * kRtN * 4; }

size_t router_tc_smem_bytes() { return (size_t)kRtStages * kRtStageBytes + sizeof(RtBars) + 1024; }

cudaError_t launch_router_tc(const moe_dims &d, const uint16_t *x, const float *Wr, const float *bias, int T,
                             const Workspace &ws, cudaStream_t s) {
  const int E = d.n_experts, H = d.hidden;
  const size_t n4 = (size_t)E * H / 4;
  const int ks = router_tc_ksplit(d, T);
  trace_mark(MOE_KERNEL_ROUTER_LOGITS, false, s);
  router_split_kernel<<<(unsigned)std::min<size_t>((n4 + 255) / 256, 1184), 256, 0, s>>>(
      reinterpret_cast<const float4 *>(Wr), n4, reinterpret_cast<uint2 *>(ws.wsplit), ws.zero_begin, ws.zero_words);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  CUtensorMap wmap, xmap;
  if (!make_planes_map(&wmap, ws.wsplit, E, H) || !make_rows_map(&xmap, x, T, H, kRtN)) return cudaErrorInvalidValue;
  RtArgs a{};
  a.T = T;
  a.E = E;
  a.H = H;
  a.ks = ks;
  a.n_et = (E + kRtM - 1) / kRtM;
  a.n_units = a.n_et * ((T + kRtN - 1) / kRtN) * ks;
  a.bias = bias;
  a.out = ks == 1 ? ws.logits : ws.rpart;
  a.status = ws.status;
  int dev = 0, n_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = router_tc_smem_bytes();
  err = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  router_tc_kernel<<<min(n_sm, a.n_units), kRtThreads, smem, s>>>(wmap, xmap, a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (ks > 1) {
    const size_t TE = (size_t)T * E;
    router_ksum_kernel<<<(unsigned)std::min<size_t>((TE + 255) / 256, 1184), 256, 0, s>>>(ws.rpart, ks, TE, E, bias,
                                                                                    ws.logits);
    err = cudaGetLastError();
  }
  trace_mark(MOE_KERNEL_ROUTER_LOGITS, true, s);
  return err;
}

}  // namespace moe
