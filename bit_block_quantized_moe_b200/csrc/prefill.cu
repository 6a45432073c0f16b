// Grouped expert GEMMs for prefill chunks on the 5th-generation tensor cores
// (tcgen05, sm_100a).
//
// One persistent CTA per SM walks a list of work items (expert, two 128-row
// M tiles, up to 64 tokens; or, once experts average 64 tokens, one M tile and
// up to 128 tokens): the tiles of an item share every load of the expert's
// token rows.  For each 128-wide K chunk:
//   producer warp    : one TMA load of the tiles' packed Q2 codes + scales
//                      (8 units x 640 B per tile, a 4-D tensor map over the
//                      experts; units past the expert's last tile read as
//                      zeros) and two of the expert's token rows (slot-sorted
//                      activations, 128-byte swizzle, 16/32/64/128-row boxes)
//                      into one of 8 (5) shared-memory stages;
//   16 dequant warps : two groups of 8 on alternate chunks (one group's
//                      waits and stores overlap the other's decode); each
//                      warp decodes one 16-row unit (4 blocks) of every M
//                      tile in registers to bf16 d * (q - 1) while the tensor
//                      core still reads the A stage it will fill, then stores
//                      them (tcgen05.st); once the MMAs of the group's
//                      previous chunk have completed it also releases that
//                      chunk's shared-memory stage to the producer;
//   MMA warp        : 8 tcgen05.mma per M tile and chunk (A from tensor memory, B
//                     from shared memory), fp32 accumulators in tensor
//                     memory, one commit per chunk.  It waits only on the A
//                     stage: the dequant warps passed the chunk's TMA barrier
//                     before filling it, which orders the B rows too.  The
//                     whole warp runs the loop on warp-uniform values and one
//                     elected lane issues (a lane-0-only loop issues the same
//                     MMAs about 20% slower; the producer warp likewise);
//   4 epilogue warps: tcgen05.ld the accumulators; gate/up writes
//                     h = silu(g) * u (bf16, each lane one SiLU per pair of
//                     token columns), down writes the fp32 expert output rows
//                     for the combine.
// The issuing thread of the MMAs is the pipeline's pace: everything it waits
// on is taken off its path.  Accumulators are double-buffered so the epilogue
// of one item overlaps the MMAs of the next.  Every wait is bounded (sync.cuh).
#include <algorithm>

#include "kernels.cuh"
#include "tc.cuh"

namespace moe {

namespace {

constexpr int kTileUnits = 8;      // 16-row units per 128-row M tile

constexpr int kWarpProducer = 0, kWarpMMA = 1, kWarpDequant0 = 2, kNumDequant = 16, kWarpEpi0 = 18, kNumEpi = 4;
constexpr int kThreadsTC = (kWarpEpi0 + kNumEpi) * 32;  // 704
constexpr uint32_t kTmemCols = 512;

// Two shapes of work item.  Few tokens per expert (the 1024-token chunk: about 20): two 128-row M tiles and
// at most 64 tokens, so that both tiles share every token-row load.  Many tokens per expert: one M tile and
// at most 128 tokens, so that each expert's codes are decoded half as often and every MMA covers twice the
// tokens for about the same issue cost.
template <int MT, int MAXN>
struct TcCfg {
  static constexpr int kMT = MT;                                  // 128-row M tiles per work item
  static constexpr int kMaxN = MAXN;                              // tokens per work item
  static constexpr int kABytes = MT * kTileUnits * kGroupBytes;   // codes + scales of one K chunk
  static constexpr int kBSub = MAXN * 128;                        // one 64-wide K half of the token rows
  static constexpr int kStageBytes = kABytes + 2 * kBSub;
  static constexpr int kStages = MT == 2 ? 8 : 5;                 // shared-memory stages (A codes + B rows)
  static constexpr int kAStages = 2;                              // tensor-memory A stages (MT x 64 columns)
  static constexpr uint32_t kDCols = MT * MAXN;                   // one accumulator buffer
  static constexpr uint32_t kTmemA0 = 2 * kDCols;                 // D buffers at 0 and kDCols, A stages after
  static_assert(kTmemA0 + kAStages * MT * 64 <= kTmemCols, "tensor memory columns");
  static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment for the 128-byte swizzle");
  static_assert(kAStages == 2 && kNumDequant == 16, "two dequant groups of 8, one per A stage");
};
using CfgFew = TcCfg<2, 64>;
using CfgMany = TcCfg<1, 128>;

struct TcArgs {
  const uint8_t *experts;
  const uint8_t *shared;
  PackedGeom G;
  int E;
  const int4 *items;          // (expert or E for shared, first sorted position, tokens <= kMaxN, 0)
  const uint32_t *n_items;
  int mtiles;                 // 128-row tiles per expert for this projection
  int mgroups;                // ceil(mtiles / kMT): work items per token item
  int kchunks;                // 128-wide K chunks (block groups)
  size_t unit_bytes;
  size_t sec_off;             // section offset inside a packed expert
  uint16_t *h_out;            // gate/up output [positions][I]
  float *y_out;               // down output [positions][H]
  uint32_t *status;
};

template <class C>
struct Bars {
  uint64_t full[C::kStages], empty[C::kStages], afull[C::kAStages], aempty[C::kAStages], dfull[2], dempty[2], done;
  uint32_t tmem;
  int abort;
};

template <class BarsT>
__device__ __forceinline__ bool waitb(uint64_t *bar, uint32_t parity, BarsT &B, uint32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*reinterpret_cast<volatile int *>(&B.abort)) return false;
  if (!mbar_wait(bar, parity)) {
    set_status(status, kStatusTimeout);
    B.abort = 1;
    return false;
  }
  return true;
}

// Scales pair (d_g, d_g8) fp16 -> bf16 pairs (d, d) for the two rows.
__device__ __forceinline__ void scale_pairs(uint32_t sh2, uint32_t &sg, uint32_t &sg8) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&sh2));
  sg = pack_bf16x2(f.x, f.x);
  sg8 = pack_bf16x2(f.y, f.y);
}

// silu(z) = z / (1 + e^-z) with the fast division (h is rounded to bf16 right after).
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

struct TcMaps {
  CUtensorMap a_routed;  // packed units of the routed experts, 4-D (u32 in unit group, group, unit, expert)
  CUtensorMap a_shared;  // the shared expert, same shape with one expert
  CUtensorMap b[4];      // token rows [positions][K] bf16, boxes of 16 / 32 / 64 / 128 rows x 64 columns
};

template <int MODE, class C>  // MODE 0: gate/up + SwiGLU -> h (bf16); 1: down -> y (fp32)
__global__ void __launch_bounds__(kThreadsTC, 1) tc_expert_kernel(const __grid_constant__ TcMaps maps, TcArgs a) {
  constexpr int kMT = C::kMT, kMaxN = C::kMaxN, kABytes = C::kABytes, kBSub = C::kBSub;
  constexpr int kStageBytes = C::kStageBytes, kStages = C::kStages, kAStages = C::kAStages;
  constexpr uint32_t kDCols = C::kDCols, kTmemA0 = C::kTmemA0;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned start (pointer arithmetic on the shared array keeps shared-memory addressing)
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars<C> &B = *reinterpret_cast<Bars<C> *>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = (int)*a.n_items;
  const int n_work = n_items * a.mgroups;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&B.full[i], 1);
      mbar_init(&B.empty[i], kNumDequant / 2);  // each warp of the group that read it, once its MMAs completed
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&B.afull[i], kNumDequant / 2);  // the warps of the group filling it
      mbar_init(&B.aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.dfull[i], 1);
      mbar_init(&B.dempty[i], kNumEpi);
    }
    mbar_init(&B.done, 1);
    B.abort = 0;
    mbar_fence_init();
  }
  if (warp == kWarpProducer) tmem_alloc(&B.tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = B.tmem;

  if (warp == kWarpProducer) {
    // The whole warp runs the loop; one elected lane issues the copies.  After a wait gives up no further
    // copy is issued, so the copies in flight are those of counts [issued - kStages, issued).
    int cnt = 0, issued = 0;
    bool live = true;
    for (int w = blockIdx.x; w < n_work; w += gridDim.x) {
      const int4 it = a.items[w / a.mgroups];
      const int mt0 = (w % a.mgroups) * kMT;
      const int bsel = it.z <= 16 ? 0 : (it.z <= 32 ? 1 : (it.z <= 64 ? 2 : 3));
      const int nrows = 16 << bsel;
      const CUtensorMap *amap = it.x == a.E ? &maps.a_shared : &maps.a_routed;
      const int ae = it.x == a.E ? 0 : it.x;
      for (int kc = 0; kc < a.kchunks; ++kc, ++cnt) {
        const int s = cnt % kStages;
        if (live && !waitb(&B.empty[s], ((cnt / kStages) & 1) ^ 1, B, a.status)) live = false;
        if (!live) continue;
        issued = cnt + 1;
        if (elect_one()) {
          uint8_t *st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&B.full[s], (uint32_t)(kABytes + 2 * nrows * 128));
          // kMT x 8 units; units past the expert's last tile read as zeros (tensor-map bounds)
          tma_load_4d(st, amap, 0, kc, mt0 * kTileUnits, ae, &B.full[s]);
          for (int sub = 0; sub < 2; ++sub)
            tma_load_2d(st + kABytes + sub * kBSub, &maps.b[bsel], kc * 128 + sub * 64, it.y, &B.full[s]);
        }
        __syncwarp();
      }
    }
    // Every copy issued must land before the CTA exits, also after an abort: a bounded wait of its own
    // (the shared abort flag would end it at once), the phase of count c2 being the last one its stage had.
    for (int c2 = max(0, issued - kStages); c2 < issued; ++c2)
      if (!mbar_wait(&B.full[c2 % kStages], (c2 / kStages) & 1)) set_status(a.status, kStatusTimeout);
  } else if (warp == kWarpMMA) {
    // The whole warp runs the loop on warp-uniform values; one elected lane issues the MMAs and commits.
    int cnt = 0, dcnt = 0;
    for (int w = blockIdx.x; w < n_work; w += gridDim.x) {
      const int4 it = a.items[w / a.mgroups];
      const int N = max(16, (it.z + 15) & ~15);
      const uint32_t idesc = umma_idesc_bf16(128, N);
      const int db = dcnt & 1;
      waitb(&B.dempty[db], ((dcnt >> 1) & 1) ^ 1, B, a.status);
      tc_fence_after();
      const uint32_t dcol = tbase + db * kDCols;
      for (int kc = 0; kc < a.kchunks; ++kc, ++cnt) {
        const int s = cnt % kStages, sa = cnt % kAStages;
        waitb(&B.afull[sa], (cnt / kAStages) & 1, B, a.status);
        tc_fence_after();
        const uint64_t bdesc0 = umma_sdesc_sw128(smem_u32(smem + s * kStageBytes + kABytes));
        const uint32_t acol = tbase + kTmemA0 + sa * kMT * 64;
        if (elect_one()) {
#pragma unroll
          for (int m = 0; m < kMT; ++m)
#pragma unroll
            for (int j = 0; j < 8; ++j)
              umma_ts(dcol + m * kMaxN, acol + m * 64 + 8 * j,
                      bdesc0 + (uint64_t)((j >> 2) * (kBSub >> 4) + (j & 3) * 2), idesc, (kc | j) != 0);
          umma_commit(&B.aempty[sa]);
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(&B.dfull[db]);
      __syncwarp();
      ++dcnt;
    }
    // all MMAs issued by this warp have completed before tensor memory is released
    if (elect_one()) {
      umma_commit(&B.done);
      if (!mbar_wait(&B.done, 0)) set_status(a.status, kStatusTimeout);
    }
    __syncwarp();
  } else if (warp < kWarpEpi0) {
    // ---- dequant warps: two groups of 8 take alternate K chunks, so that one group's barrier waits and
    // tensor-memory stores overlap the other group's decode.  In a group, 2 warps per TMEM lane quadrant (the
    // quadrant holds units 2q, 2q + 1 of each M tile), each decoding its unit in every M tile of the chunk ----
    const int dw = warp - kWarpDequant0;
    const int grp = dw >> 3, q = warp & 3, uq = (dw >> 2) & 1;
    const int unit = 2 * q + uq;
    const uint32_t lane_base = (uint32_t)(32 * q + 16 * uq) << 16;
    const int g = lane >> 2;
    int cnt = 0;
    for (int w = blockIdx.x; w < n_work; w += gridDim.x) {
      for (int kc = 0; kc < a.kchunks; ++kc, ++cnt) {
        if ((cnt & 1) != grp) continue;
        const int s = cnt % kStages, sa = cnt % kAStages;
        waitb(&B.full[s], (cnt / kStages) & 1, B, a.status);
        const uint32_t acol = tbase + lane_base + kTmemA0 + sa * kMT * 64;
#pragma unroll 1
        for (int m = 0; m < kMT; ++m) {
          const uint8_t *gp = smem + s * kStageBytes + (m * kTileUnits + unit) * kGroupBytes;
          const uint4 cw = *reinterpret_cast<const uint4 *>(gp + lane * 16);
          const uint4 sw = *reinterpret_cast<const uint4 *>(gp + kGroupCodeBytes + g * 16);
          const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
          const uint32_t sws[4] = {sw.x, sw.y, sw.z, sw.w};
          // registers P0, P2 belong to row g, P1, P3 to row g+8
          uint32_t av[4][8];
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            uint32_t p[8];
            decode_q2_exact(cws[bb], p);
            uint32_t sg, sg8;
            scale_pairs(sws[bb], sg, sg8);
            av[bb][0] = bf16x2_mul(p[0], sg);
            av[bb][1] = bf16x2_mul(p[2], sg);
            av[bb][2] = bf16x2_mul(p[1], sg8);
            av[bb][3] = bf16x2_mul(p[3], sg8);
            av[bb][4] = bf16x2_mul(p[4], sg);
            av[bb][5] = bf16x2_mul(p[6], sg);
            av[bb][6] = bf16x2_mul(p[5], sg8);
            av[bb][7] = bf16x2_mul(p[7], sg8);
          }
          if (m == 0) {
            waitb(&B.aempty[sa], ((cnt / kAStages) & 1) ^ 1, B, a.status);
            // The MMAs of chunk cnt - kAStages (this group's previous chunk) have completed (the commit that
            // freed this A stage follows them): their shared-memory stage, whose codes this group read, is free.
            if (cnt >= kAStages) {
              __syncwarp();
              if (lane == 0) mbar_arrive(&B.empty[(cnt - kAStages) % kStages]);
            }
            tc_fence_after();
          }
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            tmem_st_16x256b(acol + m * 64 + 16 * bb, av[bb][0], av[bb][1], av[bb][2], av[bb][3]);
            tmem_st_16x256b(acol + m * 64 + 16 * bb + 8, av[bb][4], av[bb][5], av[bb][6], av[bb][7]);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.afull[sa]);
      }
    }
  } else {
    // ---- epilogue warps: one TMEM lane quadrant each ----
    const int q = warp & 3;
    int dcnt = 0;
    for (int w = blockIdx.x; w < n_work; w += gridDim.x) {
      const int4 it = a.items[w / a.mgroups];
      const int mt0 = (w % a.mgroups) * kMT;
      const int db = dcnt & 1;
      waitb(&B.dfull[db], (dcnt >> 1) & 1, B, a.status);
      tc_fence_after();
      const int ntok = it.z;
      for (int m = 0; m < kMT; ++m) {
      const int mt = mt0 + m;
      if (mt >= a.mtiles) break;  // the zero-filled tile past the expert's last one
      for (int col0 = 0; col0 < ntok; col0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + ((uint32_t)(32 * q) << 16) + db * kDCols + m * kMaxN + col0, v);
        tmem_wait_ld();
        const int nmax = min(32, ntok - col0);
        if (MODE == 0) {
          // Lane rho < 8 holds gate row i of its unit, lane rho + 8 the up row of the same i.  For each
          // pair of token columns (n, n + 1) the gate lane finishes column n and the up lane column n + 1.
          const int r = 32 * q + lane, tu = r >> 4, rho = r & 15;
          const bool gate_lane = rho < 8;
          const int i = (mt * kTileUnits + tu) * 8 + (rho & 7);
          const int I = a.G.I;
#pragma unroll
          for (int n = 0; n < 32; n += 2) {
            const float mine0 = __uint_as_float(v[n]), mine1 = __uint_as_float(v[n + 1]);
            const float other = __shfl_xor_sync(0xffffffffu, gate_lane ? mine1 : mine0, 8);
            const float gv = gate_lane ? mine0 : other, uv = gate_lane ? other : mine1;
            const int nn = gate_lane ? n : n + 1;
            if (nn < nmax) a.h_out[(size_t)(it.y + col0 + nn) * I + i] = float_to_bf16_bits(silu_fast(gv) * uv);
          }
        } else {
          const int H = a.G.H;
          const int row = mt * 128 + 32 * q + lane;
#pragma unroll
          for (int n = 0; n < 32; ++n)
            if (n < nmax) a.y_out[(size_t)(it.y + col0 + n) * H + row] = __uint_as_float(v[n]);
        }
      }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.dempty[db]);
      ++dcnt;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpProducer) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Token rows in slot order: xs[p] = x[sorted_tok[p]] (one warp per position).
__global__ void gather_rows_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ sorted_tok, int P, int H,
                                   uint16_t *__restrict__ xs) {
  const long long wg = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wg >= P) return;
  const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)sorted_tok[wg] * H);
  uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)wg * H);
  for (int i = lane; i < H / 8; i += 32) dst[i] = src[i];
}

// 4-D map over packed units: (32-bit word within a 640-byte block group, group, unit, expert);
// one box is one group of box_units consecutive units (640 bytes each, no swizzle).
bool make_units_map(CUtensorMap *map, const void *base, int groups, int units, int experts, size_t unit_bytes,
                    size_t expert_bytes, int box_units) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {kGroupBytes / 4, (cuuint64_t)groups, (cuuint64_t)units, (cuuint64_t)experts};
  const cuuint64_t strides[3] = {kGroupBytes, unit_bytes, expert_bytes};
  const cuuint32_t box[4] = {kGroupBytes / 4, 1, (cuuint32_t)box_units, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_maps(TcMaps *m, const uint8_t *experts, const uint8_t *shared, const PackedGeom &G, int E, bool down,
               const void *rows, int P, int mt) {
  const int groups = down ? G.dn_groups : G.gu_groups;
  const int units = down ? G.dn_units : G.gu_units;
  const size_t ub = down ? G.dn_unit_bytes : G.gu_unit_bytes;
  const size_t off = down ? G.gu_bytes : 0;
  const int K = down ? G.I : G.H;
  bool ok = make_units_map(&m->a_routed, experts + off, groups, units, E, ub, G.expert_bytes, kTileUnits * mt) &&
            make_units_map(&m->a_shared, shared + off, groups, units, 1, ub, G.expert_bytes, kTileUnits * mt);
  for (int i = 0; i < 4 && ok; ++i) ok = make_rows_map(&m->b[i], rows, P, K, 16 << i);
  return ok;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_rows_map(CUtensorMap *map, const void *base, int rows, int cols, int box_rows) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <class C>
size_t tc_smem_bytes() {
  return (size_t)C::kStages * C::kStageBytes + sizeof(Bars<C>) + 1024;
}

template <class C>
cudaError_t launch_tc_pair(const moe_dims &d, const PackedGeom &G, const uint8_t *experts, const uint8_t *shared,
                           int P, const Workspace &ws, cudaStream_t s) {
  int dev = 0, n_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = tc_smem_bytes<C>();
  TcArgs a{};
  a.experts = experts;
  a.shared = shared;
  a.G = G;
  a.E = d.n_experts;
  a.items = ws.tc_items;
  a.n_items = ws.n_tc_items;
  a.status = ws.status;
  a.h_out = ws.h;
  a.y_out = ws.y;

  TcMaps maps_gu, maps_dn;
  if (!make_maps(&maps_gu, experts, shared, G, d.n_experts, false, ws.xs, P, C::kMT) ||
      !make_maps(&maps_dn, experts, shared, G, d.n_experts, true, ws.h, P, C::kMT))
    return cudaErrorInvalidValue;

  // gate/up + SwiGLU: M = 2I interleaved rows (8 gate + 8 up per unit), K = H
  a.mtiles = G.gu_units / kTileUnits;
  a.mgroups = (a.mtiles + C::kMT - 1) / C::kMT;
  a.kchunks = G.gu_groups;
  a.unit_bytes = G.gu_unit_bytes;
  a.sec_off = 0;
  cudaError_t err = cudaFuncSetAttribute(tc_expert_kernel<0, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  trace_mark(MOE_KERNEL_GATE_UP, false, s);
  tc_expert_kernel<0, C><<<n_sm, kThreadsTC, smem, s>>>(maps_gu, a);
  trace_mark(MOE_KERNEL_GATE_UP, true, s);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  // down: M = H rows, K = I
  a.mtiles = G.dn_units / kTileUnits;
  a.mgroups = (a.mtiles + C::kMT - 1) / C::kMT;
  a.kchunks = G.dn_groups;
  a.unit_bytes = G.dn_unit_bytes;
  a.sec_off = G.gu_bytes;
  err = cudaFuncSetAttribute(tc_expert_kernel<1, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  trace_mark(MOE_KERNEL_DOWN, false, s);
  tc_expert_kernel<1, C><<<n_sm, kThreadsTC, smem, s>>>(maps_dn, a);
  trace_mark(MOE_KERNEL_DOWN, true, s);
  return cudaGetLastError();
}

}  // namespace

int tc_item_tokens(const moe_dims &d, int T) {
  // one M tile and 128-token items once an expert averages at least 64 tokens
  return (long long)T * d.top_k >= 64LL * d.n_experts ? CfgMany::kMaxN : CfgFew::kMaxN;
}

// Experts of a prefill chunk with at most this many tokens go to the register-dequant kernels (one 8-token
// item each), the rest to the tcgen05 kernels; set per host thread by moe_set_cold_expert_tokens.  0 (none) by
// default: on B200 the tcgen05 path was faster for every expert, down to one token.
static thread_local int g_cold_expert_tokens = 0;

void set_cold_expert_tokens(int n) { g_cold_expert_tokens = n; }

int cold_expert_tokens(const moe_dims &d, int T) {
  (void)d;
  (void)T;
  return g_cold_expert_tokens;
}

cudaError_t launch_tc_experts(const moe_dims &d, const PackedGeom &G, const uint8_t *experts, const uint8_t *shared,
                              const uint16_t *x, int T, const Workspace &ws, cudaStream_t s) {
  const int cold = cold_expert_tokens(d, T);
  if (cold > 0) {  // the cold experts' items on the register-dequant kernels first
    Workspace wc = ws;  // grid sized by the cold list's bound: at most ceil(cold / 8) items per expert
    wc.max_items = (int)std::min<long long>(ws.max_items, (long long)d.n_experts * ((cold + 7) / 8));
    const cudaError_t e0 = launch_experts(d, G, experts, shared, x, T, wc, s);
    if (e0 != cudaSuccess) return e0;
  }
  const int P = T * d.top_k + T;  // sorted positions (routed + shared)
  trace_mark(MOE_KERNEL_GATHER, false, s);
  gather_rows_kernel<<<(unsigned)(((long long)P * 32 + 255) / 256), 256, 0, s>>>(x, ws.sorted_tok, P, G.H, ws.xs);
  trace_mark(MOE_KERNEL_GATHER, true, s);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  return tc_item_tokens(d, T) == CfgMany::kMaxN ? launch_tc_pair<CfgMany>(d, G, experts, shared, P, ws, s)
                                                : launch_tc_pair<CfgFew>(d, G, experts, shared, P, ws, s);
}

}  // namespace moe
