// gemm_tc.cu — persistent, warp-specialised bf16 GEMM engine for sm_100a.
//
// Every contraction of the tensor-parallel layers runs through this kernel:
// the column-parallel GEMM with its bias + GeLU epilogue, the row-parallel
// GEMM whose shard sum (the g operator's all-reduce, and the f operator's in
// backward) is fused into the accumulator or into an ordered split
// reduction, the dGeLU GEMM, the two weight-gradient GEMMs and the
// output-embedding logits GEMM.
//
// Two tile configurations share one kernel template:
//   CG = 2  a pair of CTAs (a 2-CTA cluster on neighbouring SMs) computes a
//           256 x 256 output tile with tcgen05.mma.cta_group::2: each CTA
//           stages 128 rows of A and 128 columns of B per k-block, and each
//           CTA's tensor memory holds its 128 rows x 256 fp32 columns;
//   CG = 1  one CTA computes a 128 x 256 tile (problems one tile high).
// Roles inside each CTA (persistent over output tiles):
//   warp 0    TMA producer: one elected lane streams k-blocks of 64 bf16
//             into a ring of shared-memory stages (no cluster multicast);
//   warp 1    owns tensor memory (512 columns = two accumulators); in the
//             pair leader one elected lane issues the MMAs;
//   warps 2-9 epilogue: tcgen05.ld of the finished accumulator (two warps per
//             TMEM lane quadrant, 128 columns each), fused element-wise
//             work, then each warp's 32 x 32 chunk out through a 64-byte-
//             swizzled staging buffer and a TMA store (bf16 and fp32
//             outputs), or stores from registers (split partials, outputs
//             a tensor map cannot describe).
// The accumulator is double buffered, so the epilogue of one tile overlaps
// the main loop of the next.
//
// Operands may be K-major or MN-major in global memory; both are loaded by
// TMA with 128-byte swizzle and described to the tensor core by matching
// shared-memory descriptors, so no operand is ever transposed in memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "sm100_ptx.cuh"

// per-SM throughput of the tall tile relative to the 256 x 256 pair tile when
// it is forced (alone on the h = 4096 MLP GEMMs: 1.0-1.05)
#ifndef TP_GEMM_TALL_EFF
#define TP_GEMM_TALL_EFF 1.0
#endif

#ifndef TP_GEMM_STAGE_BUDGET
#define TP_GEMM_STAGE_BUDGET 196608u
#endif

namespace tpl {

namespace {

constexpr int BM = 128;              // rows of A per CTA row half
constexpr double kTallEfficiency = TP_GEMM_TALL_EFF;
constexpr int BN = 256;              // output columns of the widest tile
constexpr int BK = 64;               // bf16 elements per k-block (one 128-byte swizzle row)
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 64 + kEpiThreads;

struct GemmArgs {
  int M, N, K;
  int a_mn, b_mn;
  int tiles_m, tiles_n, splits, group_m;
  int group_n;                      // > 0: bands of group_n tile columns instead of group_m rows
  int full_tiles;                   // split-sum GEMMs: the first full_tiles tiles (raster
                                    // order) take their whole K range, the rest are split
  int num_units;
  int split_kb[kMaxSplits + 1];     // k-block boundaries of the splits
  int act;
  void* out0;
  void* out1;
  int64_t ldo;
  const __nv_bfloat16* bias;
  const __nv_bfloat16* aux;
  int64_t ld_aux;
  float* dbias_part;
  float* part;                      // split partials: zpart [splits,M,N] or tile-chunk buffer
  int part_is_zpart;
  int* counters;
  int32_t* dev_status;
  uint64_t wait_ns;
  const int64_t* targets;           // EPI_XENT_*
  float* stat_m;
  float* stat_s;
  int32_t* stat_i;
  float* tgt_logit;
  const float* row_lse;
  float grad_scale;
  int inject_unit, inject_kb;       // debug: the producer stops before this k-block (-1: never)
  int tma_out;                      // bf16 outputs leave through tensor maps (tmO)
};

// One launch runs one problem, or two independent problems with the same
// tile shape and epilogue one after the other in its unit order (a grouped
// launch: the units of the second fill the first one's last wave).
struct __align__(64) GemmParams {
  CUtensorMap tmA[2];
  CUtensorMap tmB[2];
  CUtensorMap tmO[2][2];            // [problem][out0, out1]: 32 x 32 boxes, 64-byte swizzle
  GemmArgs a[2];
  int units0;                       // units of problem 0
  int total_units;                  // units of both problems
};

// Tile configurations: CG CTAs (1 or 2, a cluster pair with cta_group::2)
// compute a (128·RH·CG) x BNT output tile, BNT = 256 or 128 columns.  RH = 1:
// each CTA holds 128 rows and tensor memory holds two accumulators, so one
// tile's epilogue overlaps the next tile's main loop.  RH = 2 (the tall
// tile, pairs of 256-column tiles only): each CTA holds 256 rows as two
// halves that share every B stage, which halves the operand bytes per MMA;
// the two halves fill tensor memory, so the epilogue does not overlap.
template <int CG, int BNT, int RH>
struct Cfg {
  static constexpr int kRowsCTA = BM * RH;       // output rows per CTA
  static constexpr int kRows = kRowsCTA * CG;    // output rows per tile
  static constexpr int kBCols = BNT / CG;        // B columns staged per CTA
  static constexpr uint32_t kABytes = kRowsCTA * BK * 2;
  static constexpr uint32_t kBBytes = kBCols * BK * 2;
  // TP_GEMM_STAGE_BUDGET bytes of operand stages (default 192 KB: 6 stages of
  // the 2 x 256 tile, 4 of 1 x 256 and of the tall tile, 8 of 2 x 128, 6 of
  // 1 x 128; a seventh stage measured no faster)
  static constexpr int kStages = static_cast<int>(TP_GEMM_STAGE_BUDGET / (kABytes + kBBytes));
  static constexpr uint32_t kOffB = kStages * kABytes;
  static constexpr uint32_t kOffBar = kOffB + kStages * kBBytes;
  static constexpr uint32_t kNumBars = 2 * kStages + 5;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kOffRed = (kOffMisc + 16 + 15) & ~15u;   // dbias quadrant sums
  // per epilogue warp, one 32 x 32 bf16 chunk on its way to a TMA store
  static constexpr uint32_t kOffStage = (kOffRed + 4 * BNT * 4 + 1023) & ~1023u;
  static constexpr uint32_t kStageBytes = 32 * 32 * 2;
  static constexpr uint32_t kBytes = kOffStage + 8 * kStageBytes;
  static constexpr uint32_t kAlloc = kBytes + 1024;   // slack for 1024-byte alignment
  static constexpr uint32_t kTmemCols = 2 * BNT;      // two accumulators, or two row halves
  static constexpr int kAccBufs = RH == 2 ? 1 : 2;    // accumulator buffers in tensor memory
  static constexpr int kChunks = BNT / 64;            // 32-column chunks per epilogue warp
};

// -------------------------------------------------------------------------
// activation (no page gives a formula: tanh closed form by default)
// 0.5·u·(1 + tanh(z)) is written as u·σ(2z), which stays accurate in the
// negative tail where 1 + tanh(z) cancels.
// -------------------------------------------------------------------------
// The activation is a template argument: the epilogues branch once per
// 32-column chunk on the (uniform) runtime code and run straight-line code
// for the one form, instead of carrying every form's arithmetic per element.
template <int ACT>
__device__ __forceinline__ float act_apply(float u) {
  if constexpr (ACT == TP_ACT_GELU_TANH) {
    const float z = 0.7978845608028654f * (u + 0.044715f * u * u * u);
    return __fdividef(u, 1.0f + __expf(-2.0f * z));
  } else if constexpr (ACT == TP_ACT_GELU_ERF) {
    return 0.5f * u * (1.0f + erff(u * 0.7071067811865476f));
  } else {
    return u;
  }
}

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GeLU'(u) of the tanh form, 0.5·(1 + t) + 0.5·u·(1 − t²)·c·(1 + 3a·u²) with
// t = tanh(c·(u + a·u³)), from one hardware tanh (absolute error of GeLU'
// about 2.5e-4, below the bf16 rounding of the dU it scales).
template <int ACT>
__device__ __forceinline__ float act_deriv(float u) {
  if constexpr (ACT == TP_ACT_GELU_TANH) {
    constexpr float c = 0.7978845608028654f, a = 0.044715f;
    const float u2 = u * u;
    const float t = tanh_approx(u * fmaf(c * a, u2, c));
    const float half_dz = fmaf(1.5f * c * a, u2, 0.5f * c);   // 0.5·c·(1 + 3a·u²)
    return fmaf(u * half_dz, fmaf(-t, t, 1.0f), fmaf(0.5f, t, 0.5f));
  } else if constexpr (ACT == TP_ACT_GELU_ERF) {   // explicit fmaf: the same bits as act_deriv_value
    const float cdf = fmaf(0.5f, erff(u * 0.7071067811865476f), 0.5f);
    return fmaf(u * 0.3989422804014327f, __expf(-0.5f * u * u), cdf);
  } else {
    return 1.0f;
  }
}

// act'(u) and act(u) together.  For the tanh form the value 0.5·u·(1 + t)
// reuses the derivative's t; where 1 + t cancels (u < 0) its absolute
// error stays below 2.5e-4·|u|, the size of a bf16 rounding step of values
// near 0.1.
template <int ACT>
__device__ __forceinline__ float act_deriv_value(float u, float& y) {
  if constexpr (ACT == TP_ACT_GELU_TANH) {
    constexpr float c = 0.7978845608028654f, a = 0.044715f;
    const float u2 = u * u;
    const float t = tanh_approx(u * fmaf(c * a, u2, c));
    const float half_dz = fmaf(1.5f * c * a, u2, 0.5f * c);
    const float hu = 0.5f * u;
    y = fmaf(hu, t, hu);
    return fmaf(u * half_dz, fmaf(-t, t, 1.0f), fmaf(0.5f, t, 0.5f));
  } else if constexpr (ACT == TP_ACT_GELU_ERF) {
    const float cdf = fmaf(0.5f, erff(u * 0.7071067811865476f), 0.5f);
    y = u * cdf;
    return fmaf(u * 0.3989422804014327f, __expf(-0.5f * u * u), cdf);
  } else {
    y = u;
    return 1.0f;
  }
}

// One 32-column chunk through the activation / its derivative.
template <int ACT>
__device__ __forceinline__ void act_chunk(float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = act_apply<ACT>(v[j]);
}
template <int ACT>
__device__ __forceinline__ void dact_chunk(float (&v)[32], const float (&u)[32], bool ok) {
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = ok ? v[j] * act_deriv<ACT>(u[j]) : 0.0f;
}
// dU = dY·act'(U) and, in place of U, Y = act(U)
template <int ACT>
__device__ __forceinline__ void dact_value_chunk(float (&v)[32], float (&u)[32], bool ok) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    float y;
    const float d = act_deriv_value<ACT>(u[j], y);
    v[j] = ok ? v[j] * d : 0.0f;
    u[j] = y;
  }
}

// -------------------------------------------------------------------------
// tile scheduling: unit -> (tile row, tile column, split)
// Tiles are visited in bands of group_m tile rows, column by column inside a
// band, so that one wave of CTAs shares A rows and B columns through L2 and
// B is read once per band; or, when B is the larger operand and a band of
// its columns fits in L2, in bands of group_n tile columns, row by row
// inside a band, so that A is the one read once per band.
// Split-sum GEMMs: the first full_tiles tiles take their whole K range
// (s = −1, stored directly); the tiles of the last, partial wave are split,
// split-major (every tile's first K range, then every tile's second), and
// the last split of a tile sums the partials the earlier splits left
// behind.  Without full tiles every tile is split.
// -------------------------------------------------------------------------
__device__ __forceinline__ void unit_map(const GemmArgs& a, int unit, int& tm, int& tn, int& s,
                                         int& tile) {
  const int tiles = a.tiles_m * a.tiles_n;
  if (unit < a.full_tiles) {
    s = -1;
    tile = unit;
  } else {
    const int rem = tiles - a.full_tiles;
    const int u = unit - a.full_tiles;
    s = u / rem;
    tile = a.full_tiles + (u - s * rem);
  }
  if (a.group_n > 0) {
    const int per_group = a.group_n * a.tiles_m;
    const int g = tile / per_group;
    const int first_n = g * a.group_n;
    const int gn = min(a.tiles_n - first_n, a.group_n);
    const int r = tile - g * per_group;
    tn = first_n + r % gn;
    tm = r / gn;
    return;
  }
  const int per_group = a.group_m * a.tiles_n;
  const int g = tile / per_group;
  const int first_m = g * a.group_m;
  const int gm = min(a.tiles_m - first_m, a.group_m);
  const int r = tile - g * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
}

__device__ __forceinline__ void flag_timeout(const GemmArgs& a, volatile int* abort_flag) {
  *abort_flag = 1;
  if (a.dev_status) atomicOr(a.dev_status, TP_DEVERR_TIMEOUT);
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v, int ncols_left) {
  // ncols_left is a multiple of 8 (row lengths are multiples of 8)
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (8 * j < ncols_left) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
      w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
      w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
      w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
      *reinterpret_cast<uint4*>(dst + 8 * j) = w;
    }
  }
}

__device__ __forceinline__ void load_raw_bf16x32(const __nv_bfloat16* src, uint4 (&w)[4],
                                                 int ncols_left) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[j] = make_uint4(0, 0, 0, 0);
    if (8 * j < ncols_left) w[j] = __ldg(reinterpret_cast<const uint4*>(src + 8 * j));
  }
}

// bf16 -> fp32 is exact as a 16-bit shift of the bit pattern: two integer
// ops per pair, which keeps the conversions off the transcendental unit the
// epilogues' exp / tanh already load.
__device__ __forceinline__ void unpack_bf16x32(const uint4 (&w)[4], float* v) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[8 * j + 2 * q] = __uint_as_float(ww[q] << 16);
      v[8 * j + 2 * q + 1] = __uint_as_float(ww[q] & 0xffff0000u);
    }
  }
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLog2e = 1.4426950408889634f;

// Transpose-reduce across the warp: lane l ends with Σ_lanes v[l].
__device__ __forceinline__ float warp_column_sums(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

// One warp's 32 x 32 chunk (lane = row, 32 columns each) out through a TMA
// store: the rows go to the warp's staging buffer as 64-byte lines in the
// 64-byte swizzle (16-byte granule g of row r at g ^ ((r >> 1) & 3): the
// eight lanes of each store phase hit eight different bank groups), then
// one lane stores the box at (col0, row0).  Each store instruction of the
// direct path touches 32 rows; this writes whole lines.  The previous
// chunk's store must have read the buffer first.
__device__ __forceinline__ void stage_store_bf16x32(const CUtensorMap* tm, uint8_t* stg,
                                                    const float (&v)[32], int lane, int col0,
                                                    int row0) {
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * g + 0], v[8 * g + 1]);
    w.y = pack_bf16x2(v[8 * g + 2], v[8 * g + 3]);
    w.z = pack_bf16x2(v[8 * g + 4], v[8 * g + 5]);
    w.w = pack_bf16x2(v[8 * g + 6], v[8 * g + 7]);
    *reinterpret_cast<uint4*>(stg + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) = w;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm, stg, col0, row0);
    bulk_commit_group();
  }
}

// fp32 outputs: half h (16 of the chunk's 32 columns, 64-byte lines) of the
// chunk through the same staging buffer and a TMA store with an evict-first
// hint (the logits are written once and read by a later kernel).
__device__ __forceinline__ void stage_store_f32x16(const CUtensorMap* tm, uint8_t* stg,
                                                   const float (&v)[32], int h, int lane, int col0,
                                                   int row0) {
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
#pragma unroll
  for (int g = 0; g < 4; ++g)
    *reinterpret_cast<float4*>(stg + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) =
        make_float4(v[16 * h + 4 * g], v[16 * h + 4 * g + 1], v[16 * h + 4 * g + 2],
                    v[16 * h + 4 * g + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d_evict_first(tm, stg, col0 + 16 * h, row0);
    bulk_commit_group();
  }
}

template <int CG, int BNT, int RH, int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams P) {
  using C = Cfg<CG, BNT, RH>;
  static_assert(RH == 1 || (CG == 2 && BNT == 256), "tall tiles are 2-CTA 256-column tiles");
  static_assert(BNT == 256 || (EPI != EPI_XENT_STATS && EPI != EPI_XENT_GRAD),
                "the cross-entropy epilogues take 128-column slices of a 256-column tile");
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const GemmArgs& a0 = P.a[0];   // wait limit and status word (the same in both problems)

  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kOffB;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* bcast = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;   // 0 = pair leader
  const int slot0 = CG == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nslots = CG == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kEpiWarps * CG);   // one arrival per epilogue warp of the pair
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc_cg<CG>(tmem_slot, C::kTmemCols);
    tmem_relinquish_cg<CG>();
  }
  tc_fence_before_sync();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();   // peer barriers initialised before any signal
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  // launched as a programmatic dependent of the previous kernel in the
  // stream: the set-up above overlapped its tail; nothing below touches
  // global memory before that kernel has completed
  grid_dependency_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one_sync()) {
      tma_prefetch_desc(&P.tmA[0]);
      tma_prefetch_desc(&P.tmB[0]);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int unit = slot0; ok && unit < P.total_units; unit += nslots) {
        const int prob = unit >= P.units0 ? 1 : 0;
        const GemmArgs& a = P.a[prob];
        const CUtensorMap* tmA = &P.tmA[prob];
        const CUtensorMap* tmB = &P.tmB[prob];
        int tm, tn, s, tile;
        unit_map(a, unit - prob * P.units0, tm, tn, s, tile);
        const int a_row = tm * C::kRows + static_cast<int>(rank) * C::kRowsCTA;
        const int b_col = tn * BNT + static_cast<int>(rank) * C::kBCols;
        const int kb_lo = s < 0 ? a.split_kb[0] : a.split_kb[s];
        const int kb_hi = s < 0 ? a.split_kb[a.splits] : a.split_kb[s + 1];
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (unit == a0.inject_unit && kb == a0.inject_kb) {
            // debug injection: stop issuing without a word, as a producer
            // that died would; the MMA issuer's bounded wait runs out
            ok = false;
            break;
          }
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a0.wait_ns, abort_flag)) {
            if (!*abort_flag) flag_timeout(a0, abort_flag);
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], CG * (C::kABytes + C::kBBytes));
          const int k0 = kb * BK;
          uint8_t* dA = sA + stage * C::kABytes;
          uint8_t* dB = sB + stage * C::kBBytes;
          if constexpr (CG == 2) {
            const uint32_t bar = mapa_shared(&full[stage], 0);
            if (!a.a_mn) {
              tma_load_2d_cg2(dA, tmA, bar, k0, a_row);
            } else {
#pragma unroll
              for (int j = 0; j < C::kRowsCTA / 64; ++j)
                tma_load_2d_cg2(dA + j * 8192, tmA, bar, a_row + j * 64, k0);
            }
            if (!a.b_mn) {
              tma_load_2d_cg2(dB, tmB, bar, k0, b_col);
            } else {
#pragma unroll
              for (int j = 0; j < C::kBCols / 64; ++j)
                tma_load_2d_cg2(dB + j * 8192, tmB, bar, b_col + j * 64, k0);
            }
          } else {
            if (!a.a_mn) {
              tma_load_2d(dA, tmA, &full[stage], k0, a_row);
            } else {
#pragma unroll
              for (int j = 0; j < C::kRowsCTA / 64; ++j)
                tma_load_2d(dA + j * 8192, tmA, &full[stage], a_row + j * 64, k0);
            }
            if (!a.b_mn) {
              tma_load_2d(dB, tmB, &full[stage], k0, b_col);
            } else {
#pragma unroll
              for (int j = 0; j < C::kBCols / 64; ++j)
                tma_load_2d(dB + j * 8192, tmB, &full[stage], b_col + j * 64, k0);
            }
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Let every copy started by this pair land before the CTAs can exit
      // (bounded in time, not cut short by the abort flag).  The stage
      // barriers live in the leader and count both CTAs' bytes.
      if (rank == 0) {
        volatile int keep_waiting = 0;
        const int inflight = issued < STAGES ? issued : STAGES;
        for (int i = 0; i < inflight; ++i) {
          if (--stage < 0) {
            stage = STAGES - 1;
            phase ^= 1u;
          }
          mbar_wait_bounded(&full[stage], phase, a0.wait_ns, &keep_waiting);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (pair leader)
    if (rank == 0 && elect_one_sync()) {
      const uint16_t pair_mask = CG == 2 ? 0x3 : 0x1;
      int stage = 0;
      uint32_t phase = 0;
      int t = 0;
      bool ok = true, any = false;
      for (int unit = slot0; ok && unit < P.total_units; unit += nslots, ++t) {
        const int prob = unit >= P.units0 ? 1 : 0;
        const GemmArgs& a = P.a[prob];
        // one MMA covers 128 rows per CTA (256 for the pair); the tall tile
        // issues one per row half
        const uint32_t idesc = idesc_bf16_f32(BM * CG, BNT, a.a_mn != 0, a.b_mn != 0);
        const uint32_t a_lbo = a.a_mn ? 8192u : 16u;
        const uint32_t b_lbo = a.b_mn ? 8192u : 16u;
        const uint32_t a_kstep = a.a_mn ? 2048u : 32u;   // bytes per 16-element K step
        const uint32_t b_kstep = a.b_mn ? 2048u : 32u;
        int tm, tn, s, tile;
        unit_map(a, unit - prob * P.units0, tm, tn, s, tile);
        const int acc = t % C::kAccBufs;
        const uint32_t use = static_cast<uint32_t>(t / C::kAccBufs);
        if (!mbar_wait_bounded(&tempty[acc], (use & 1u) ^ 1u, a0.wait_ns, abort_flag)) {
          if (!*abort_flag) flag_timeout(a0, abort_flag);
          break;
        }
        tc_fence_after_sync();
        // RH = 1: accumulator buffer acc; RH = 2: row half h at column h·BNT
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BNT);
        const int kb0 = s < 0 ? a.split_kb[0] : a.split_kb[s];
        const int kb1 = s < 0 ? a.split_kb[a.splits] : a.split_kb[s + 1];
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, a0.wait_ns, abort_flag)) {
            if (!*abort_flag) flag_timeout(a0, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_base = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_base = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t bdesc = smem_desc_sw128(b_base + k * b_kstep, b_lbo, 1024);
#pragma unroll
            for (int h = 0; h < RH; ++h) {   // the row halves share the B stage
              // a row half is 128 rows: 16 KB of the A stage in either layout
              const uint64_t adesc =
                  smem_desc_sw128(a_base + h * (BM * 128) + k * a_kstep, a_lbo, 1024);
              tc_mma_bf16_cg<CG>(d_tmem + static_cast<uint32_t>(h * BNT), adesc, bdesc, idesc,
                                 (kb > kb0 || k > 0) ? 1u : 0u);
            }
          }
          any = true;
          tc_commit_mc<CG>(&empty[stage], pair_mask);   // frees the stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit_mc<CG>(&tfull[acc], pair_mask);   // accumulators ready
      }
      if (any) {   // every issued MMA must finish before tensor memory is freed
        volatile int keep_waiting = 0;
        tc_commit_local<CG>(mma_done);
        mbar_wait_bounded(mma_done, 0, a0.wait_ns, &keep_waiting);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;              // 0..7
    const int q = warp & 3;               // TMEM lane quadrant this warp may access
    const int half = ew >> 2;             // which 128 of the 256 accumulator columns
    const int row_in_tile = q * 32 + lane;
    const int et = threadIdx.x - 64;      // 0..255 among the epilogue threads
    const uint32_t tempty_addr0 = CG == 2 ? mapa_shared(&tempty[0], 0) : smem_u32(&tempty[0]);
    int t = 0;
    for (int unit = slot0; unit < P.total_units; unit += nslots, ++t) {
      const int prob = unit >= P.units0 ? 1 : 0;
      const GemmArgs& a = P.a[prob];
      int tm, tn, s, tile;
      unit_map(a, unit - prob * P.units0, tm, tn, s, tile);
      const int acc = t % C::kAccBufs;
      const uint32_t use = static_cast<uint32_t>(t / C::kAccBufs);
      const bool got = mbar_wait_bounded<true>(&tfull[acc], use & 1u, a0.wait_ns, abort_flag);
      // all epilogue threads leave together or go on together, so no warp
      // can be left waiting in a later named barrier
      if (!named_barrier_and(1, kEpiThreads, got)) {
        if (et == 0 && !*abort_flag) flag_timeout(a0, abort_flag);
        break;
      }
      tc_fence_after_sync();
#pragma unroll 1
      for (int hr = 0; hr < RH; ++hr) {   // the CTA's 128-row halves (one unless tall)
      const int row =
          tm * C::kRows + static_cast<int>(rank) * C::kRowsCTA + hr * BM + row_in_tile;
      const bool row_ok = row < a.M;
      // this CTA's 128-row piece of the tile: the unit of the split partials,
      // the arrival counters and (times four) the dbias partial rows
      const int htile = (tile * CG + static_cast<int>(rank)) * RH + hr;
      const uint32_t t_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                              static_cast<uint32_t>((acc + hr) * BNT);
      const int c0 = half * C::kChunks;   // this warp's first 32-column chunk

      if constexpr (EPI == EPI_SPLIT_SUM) {
       if (s < 0) {
        // a whole tile: the accumulator is the sum over every shard
#pragma unroll 1
        for (int c = c0; c < c0 + C::kChunks; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_base + c * 32, r);
          tc_wait_ld();
          const int col0 = tn * BNT + c * 32;
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          if (row_ok && col0 < a.N)
            store_bf16x32(static_cast<__nv_bfloat16*>(a.out0) + row * a.ldo + col0, v, a.N - col0);
        }
       } else {
        // 1) publish this split's fp32 partial
#pragma unroll 1
        for (int c = c0; c < c0 + C::kChunks; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_base + c * 32, r);
          tc_wait_ld();
          const int col0 = tn * BNT + c * 32;
          if (a.part_is_zpart) {
            if (row_ok) {
              float* dst = a.part + (static_cast<int64_t>(s) * a.M + row) * a.N + col0;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (col0 + 4 * j < a.N)
                  __stcg(reinterpret_cast<float4*>(dst + 4 * j),
                         make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                     __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
            }
          } else {
            float* dst = a.part +
                         ((static_cast<int64_t>(htile) * a.splits + s) * (BNT / 32) + c) * (BM * 32) +
                         row_in_tile * 32;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              __stcg(reinterpret_cast<float4*>(dst + 4 * j),
                     make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
          }
        }
        __threadfence();
        named_barrier_sync(1, kEpiThreads);
        if (et == 0) {
          const int prev = atomicAdd(&a.counters[htile], 1);
          const int last = (prev == a.splits - 1);
          if (last) a.counters[htile] = 0;   // ready for the next call
          *bcast = last;
        }
        named_barrier_sync(1, kEpiThreads);
        const bool last = *bcast != 0;
        if (last) {
          __threadfence();
          // 2) the last split of this half tile sums all partials in split order
#pragma unroll 1
          for (int c = c0; c < c0 + C::kChunks; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_base + c * 32, r);
            tc_wait_ld();
            const int col0 = tn * BNT + c * 32;
            float sum[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) sum[j] = 0.0f;
            for (int ss = 0; ss < a.splits; ++ss) {
              float p[32];
              if (ss == s) {
#pragma unroll
                for (int j = 0; j < 32; ++j) p[j] = __uint_as_float(r[j]);
              } else if (a.part_is_zpart) {
#pragma unroll
                for (int j = 0; j < 32; ++j) p[j] = 0.0f;
                if (row_ok) {
                  const float* src = a.part + (static_cast<int64_t>(ss) * a.M + row) * a.N + col0;
#pragma unroll
                  for (int j = 0; j < 8; ++j)
                    if (col0 + 4 * j < a.N) {
                      const float4 f = __ldcg(reinterpret_cast<const float4*>(src + 4 * j));
                      p[4 * j] = f.x; p[4 * j + 1] = f.y; p[4 * j + 2] = f.z; p[4 * j + 3] = f.w;
                    }
                }
              } else {
                const float* src =
                    a.part +
                    ((static_cast<int64_t>(htile) * a.splits + ss) * (BNT / 32) + c) * (BM * 32) +
                    row_in_tile * 32;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float4 f = __ldcg(reinterpret_cast<const float4*>(src + 4 * j));
                  p[4 * j] = f.x; p[4 * j + 1] = f.y; p[4 * j + 2] = f.z; p[4 * j + 3] = f.w;
                }
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) sum[j] += p[j];
            }
            if (row_ok && col0 < a.N)
              store_bf16x32(static_cast<__nv_bfloat16*>(a.out0) + row * a.ldo + col0, sum,
                            a.N - col0);
          }
        }
       }
      } else if constexpr (EPI == EPI_XENT_STATS) {
        // Softmax statistics of this warp's 128-column slice of each row: the
        // maximum m, s = Σ exp(acc − m) (rescaled whenever m grows) and the
        // first column holding m; the thread whose slice holds the row's
        // target keeps that accumulator.  Columns past the vocabulary are
        // left out.  Nothing of the logits matrix is written.
        const int slice = tn * (BNT / kXentSlice) + half;
        if (slice * kXentSlice < a.N) {   // warp-uniform
          const int64_t tgt = row_ok ? a.targets[row] : -1;
          float m = -INFINITY, ssum = 0.0f;
          int arg = 0;
#pragma unroll 1
          for (int c = c0; c < c0 + C::kChunks; ++c) {
            const int col0 = tn * BNT + c * 32;
            if (col0 >= a.N) break;        // warp-uniform
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_base + c * 32, r);
            tc_wait_ld();
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            if (col0 + 32 > a.N) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j >= a.N) v[j] = -INFINITY;
            }
            if (tgt >= col0 && tgt < col0 + 32) {
              float tl = 0.0f;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j == tgt) tl = v[j];
              a.tgt_logit[row] = tl;
            }
            float cm[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              cm[j] = fmaxf(fmaxf(v[4 * j], v[4 * j + 1]), fmaxf(v[4 * j + 2], v[4 * j + 3]));
            const float cmax = fmaxf(fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3])),
                                     fmaxf(fmaxf(cm[4], cm[5]), fmaxf(cm[6], cm[7])));
            int ci = 31;
#pragma unroll
            for (int j = 31; j >= 0; --j)
              if (v[j] == cmax) ci = j;
            if (cmax > m) arg = col0 + ci;
            const float mn = fmaxf(m, cmax);
            const float mn_l2 = mn * kLog2e;
            float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int j = 0; j < 32; ++j) ps[j & 3] += ex2_approx(fmaf(v[j], kLog2e, -mn_l2));
            // m = −inf before the first chunk: the old sum (0) is scaled by 0
            ssum = fmaf(ssum, ex2_approx((m - mn) * kLog2e), (ps[0] + ps[1]) + (ps[2] + ps[3]));
            m = mn;
          }
          if (row_ok) {
            const int64_t o = static_cast<int64_t>(slice) * a.M + row;
            a.stat_m[o] = m;
            a.stat_s[o] = ssum;
            a.stat_i[o] = arg;
          }
        }
      } else if constexpr (EPI == EPI_XENT_GRAD) {
        // grad_scale·(softmax − onehot) from the recomputed logits and the
        // row's log-sum-exp; a row whose target lies outside the vocabulary
        // gets NaN (its loss is undefined)
        float lse_l2 = 0.0f;
        int64_t tgt = -1;
        bool tgt_ok = false;
        if (row_ok) {
          lse_l2 = a.row_lse[row] * kLog2e;
          tgt = a.targets[row];
          tgt_ok = tgt >= 0 && tgt < a.N;
          if (!tgt_ok && tn == 0 && half == 0 && a.dev_status) atomicOr(a.dev_status, TP_DEVERR_RANGE);
        }
        const float gs = tgt_ok ? a.grad_scale : __int_as_float(0x7fc00000);
#pragma unroll 1
        for (int c = c0; c < c0 + C::kChunks; ++c) {
          const int col0 = tn * BNT + c * 32;
          if (col0 >= a.N) break;          // warp-uniform
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_base + c * 32, r);
          tc_wait_ld();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float p = ex2_approx(fmaf(__uint_as_float(r[j]), kLog2e, -lse_l2));
            v[j] = gs * (col0 + j == tgt ? p - 1.0f : p);
          }
          if (row_ok)
            store_bf16x32(static_cast<__nv_bfloat16*>(a.out0) + row * a.ldo + col0, v, a.N - col0);
        }
      } else {
        uint4 aux_w[4];
        constexpr bool kDact = EPI == EPI_DACT || EPI == EPI_DACT_Y;
        // bf16 outputs through this warp's staging buffer and a TMA store
        // when the outputs have tensor maps, else stored from registers
        uint8_t* stg = smem + C::kOffStage + ew * C::kStageBytes;
        const int row_w = row - lane;   // the warp's first row
        auto put = [&](int o, void* out, const float (&vals)[32], int col0) {
          if (a.tma_out)
            stage_store_bf16x32(&P.tmO[prob][o], stg, vals, lane, col0, row_w);
          else if (row_ok)
            store_bf16x32(static_cast<__nv_bfloat16*>(out) + row * a.ldo + col0, vals, a.N - col0);
        };
        if constexpr (kDact) {   // U for the first chunk
          const int col0 = tn * BNT + c0 * 32;
          if (row_ok && col0 < a.N) {
            load_raw_bf16x32(a.aux + row * a.ld_aux + col0, aux_w, a.N - col0);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) aux_w[j] = make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll 1
        for (int c = c0; c < c0 + C::kChunks; ++c) {
          const int col0 = tn * BNT + c * 32;
          const bool store_ok = row_ok && col0 < a.N;
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_base + c * 32, r);
          float aux_v[32];
          if constexpr (kDact) {
            unpack_bf16x32(aux_w, aux_v);
            const int coln = col0 + 32;   // prefetch U of the next chunk while this one runs
            if (c + 1 < c0 + C::kChunks && row_ok && coln < a.N) {
              load_raw_bf16x32(a.aux + row * a.ld_aux + coln, aux_w, a.N - coln);
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j) aux_w[j] = make_uint4(0, 0, 0, 0);
            }
          }
          tc_wait_ld();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);

          if constexpr (EPI == EPI_STORE_BF16) {
            if (col0 < a.N) put(0, a.out0, v, col0);
          } else if constexpr (EPI == EPI_STORE_F32) {
            if (a.tma_out) {
              if (col0 < a.N) {
                stage_store_f32x16(&P.tmO[prob][0], stg, v, 0, lane, col0, row_w);
                if (col0 + 16 < a.N) stage_store_f32x16(&P.tmO[prob][0], stg, v, 1, lane, col0, row_w);
              }
            } else if (store_ok) {
              float* dst = static_cast<float*>(a.out0) + row * a.ldo + col0;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (col0 + 4 * j < a.N)
                  *reinterpret_cast<float4*>(dst + 4 * j) =
                      make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            }
          } else if constexpr (EPI == EPI_BIAS_ACT) {
            if (a.bias != nullptr && col0 < a.N) {
              uint4 bw[4];
              float b[32];
              load_raw_bf16x32(a.bias + col0, bw, a.N - col0);
              unpack_bf16x32(bw, b);
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += b[j];
            }
            if (col0 < a.N && a.out0 != nullptr) put(0, a.out0, v, col0);
            if (a.act == TP_ACT_GELU_TANH)
              act_chunk<TP_ACT_GELU_TANH>(v);
            else if (a.act == TP_ACT_GELU_ERF)
              act_chunk<TP_ACT_GELU_ERF>(v);
            if (col0 < a.N) put(1, a.out1, v, col0);
          } else {  // EPI_DACT, EPI_DACT_Y
            if constexpr (EPI == EPI_DACT_Y) {
              // U is dead after its derivative: its registers take Y = act(U)
              if (a.act == TP_ACT_GELU_TANH)
                dact_value_chunk<TP_ACT_GELU_TANH>(v, aux_v, store_ok);
              else if (a.act == TP_ACT_GELU_ERF)
                dact_value_chunk<TP_ACT_GELU_ERF>(v, aux_v, store_ok);
              else
                dact_value_chunk<TP_ACT_NONE>(v, aux_v, store_ok);
            } else {
              if (a.act == TP_ACT_GELU_TANH)
                dact_chunk<TP_ACT_GELU_TANH>(v, aux_v, store_ok);
              else if (a.act == TP_ACT_GELU_ERF)
                dact_chunk<TP_ACT_GELU_ERF>(v, aux_v, store_ok);
              else
                dact_chunk<TP_ACT_NONE>(v, aux_v, store_ok);
            }
            if (col0 < a.N) put(0, a.out0, v, col0);
            if constexpr (EPI == EPI_DACT_Y) {
              if (col0 < a.N) put(1, a.out1, aux_v, col0);
            }
            if (a.dbias_part != nullptr) {
              const float colsum = warp_column_sums(v, lane);
              red[q * BNT + c * 32 + lane] = colsum;
            }
          }
        }
        if constexpr (kDact) {
          if (a.dbias_part != nullptr) {
            // one partial row per 128-row piece: the four lane quadrants'
            // column sums added in a fixed order
            named_barrier_sync(1, kEpiThreads);
            const int cc = et;   // one column per epilogue thread (BNT <= 256 columns)
            const int col = tn * BNT + cc;
            const int prow = (tm * CG + static_cast<int>(rank)) * RH + hr;
            if (cc < BNT && col < a.N && prow * BM < a.M) {   // pieces past M hold no rows
              const float sum = ((red[cc] + red[BNT + cc]) + red[2 * BNT + cc]) + red[3 * BNT + cc];
              a.dbias_part[static_cast<int64_t>(prow) * a.N + col] = sum;
            }
            named_barrier_sync(1, kEpiThreads);
          }
        }
      }
      }   // row halves
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {   // release the accumulator to the pair leader's MMA
        if constexpr (CG == 2)
          mbar_arrive_cluster(tempty_addr0 + static_cast<uint32_t>(acc * 8));
        else
          mbar_arrive(&tempty[acc]);
      }
    }
    if (lane == 0) bulk_wait_group0();   // this warp's TMA stores have landed
  }

  tc_fence_before_sync();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();   // no CTA leaves while its peer may touch it
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_cg<CG>(tmem_base, C::kTmemCols);
  }
}

// -------------------------------------------------------------------------
// host side
// -------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major bf16 matrix [outer, inner] with row stride ld (elements); box of
// box_inner x box_outer elements, 128-byte swizzle, zero fill outside.
bool make_tmap(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
               uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// TP_GEMM_BAND_MB=<MB> sizes the rasterisation bands by the bytes of their
// A rows instead (sweeps); 0 when unset.
double band_budget_bytes() {
  static double bytes = [] {
    double mb = 0.0;
    if (const char* e = std::getenv("TP_GEMM_BAND_MB")) {
      const double v = std::atof(e);
      if (v > 0.0) mb = v;
    }
    return mb * 1024.0 * 1024.0;
  }();
  return bytes;
}

// Row-major fp32 matrix [outer, inner], row stride ld elements.
bool make_tmap_f32(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                   uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// TP_GEMM_NO_COLUMN_BANDS=1 keeps row bands for every GEMM (sweeps).
bool column_bands_enabled() {
  const char* e = std::getenv("TP_GEMM_NO_COLUMN_BANDS");
  return !(e && e[0] == '1');
}

// TP_GEMM_SPLIT_ALL=1: split-sum GEMMs split every tile (sweeps).
bool split_all_tiles() {
  const char* e = std::getenv("TP_GEMM_SPLIT_ALL");
  return e && e[0] == '1';
}

// TP_GEMM_NO_TMA_STORE=1 stores the bf16 outputs from registers (sweeps).
bool tma_store_disabled() {
  const char* e = std::getenv("TP_GEMM_NO_TMA_STORE");
  return e && e[0] == '1';
}

// Programmatic dependent launch of the GEMMs; TP_GEMM_NO_PDL=1 turns it off
// (sweeps).
bool pdl_enabled() {
  const char* e = std::getenv("TP_GEMM_NO_PDL");
  return !(e && e[0] == '1');
}

// Launch with `slots` persistent CTAs (CG = 1) or CTA pairs (CG = 2), capped
// at the number that can be resident at once, so that no persistent slot
// starts only after another has finished.
template <int CG, int BNT, int RH, int EPI>
tp_status launch_impl(const GemmParams& prm, int slots, cudaStream_t stream) {
  using C = Cfg<CG, BNT, RH>;
  static_assert(C::kAlloc <= 232448, "shared memory budget");
  static int max_resident[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the CTAs may be set up while the previous
  // kernel drains (the kernel waits for it before any global access)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  if (!max_resident[dev & 63]) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<CG, BNT, RH, EPI>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kAlloc) != cudaSuccess)
      return TP_ERR_CUDA;
    int clusters = 0;
    cfg.gridDim = dim3(static_cast<unsigned>(CG * num_sms()));
    if (cudaOccupancyMaxActiveClusters(&clusters, gemm_tc_kernel<CG, BNT, RH, EPI>, &cfg) !=
            cudaSuccess ||
        clusters <= 0) {
      cudaGetLastError();
      clusters = num_sms() / CG;
    }
    max_resident[dev & 63] = clusters;
  }
  if (slots > max_resident[dev & 63]) slots = max_resident[dev & 63];
  const int grid = CG * slots;
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  if (cudaLaunchKernelEx(&cfg, gemm_tc_kernel<CG, BNT, RH, EPI>, prm) != cudaSuccess)
    return TP_ERR_CUDA;
  note_launches(1);
  return TP_OK;
}

template <int CG, int BNT, int RH>
tp_status launch_epi(const GemmParams& prm, int epi, int slots, cudaStream_t stream) {
  switch (epi) {
    case EPI_STORE_BF16: return launch_impl<CG, BNT, RH, EPI_STORE_BF16>(prm, slots, stream);
    case EPI_BIAS_ACT: return launch_impl<CG, BNT, RH, EPI_BIAS_ACT>(prm, slots, stream);
    case EPI_DACT: return launch_impl<CG, BNT, RH, EPI_DACT>(prm, slots, stream);
    case EPI_DACT_Y: return launch_impl<CG, BNT, RH, EPI_DACT_Y>(prm, slots, stream);
    case EPI_STORE_F32: return launch_impl<CG, BNT, RH, EPI_STORE_F32>(prm, slots, stream);
    case EPI_SPLIT_SUM: return launch_impl<CG, BNT, RH, EPI_SPLIT_SUM>(prm, slots, stream);
    case EPI_XENT_STATS:
      if constexpr (BNT == 256) return launch_impl<CG, BNT, RH, EPI_XENT_STATS>(prm, slots, stream);
      break;
    case EPI_XENT_GRAD:
      if constexpr (BNT == 256) return launch_impl<CG, BNT, RH, EPI_XENT_GRAD>(prm, slots, stream);
      break;
  }
  return TP_ERR_UNSUPPORTED;
}

// One-shot debug injection (tp_debug_stall_next_gemm): the next launch's
// producers stop before k-block `kb` of unit `unit`, and that launch's
// bounded waits give up after `wait_ns`.
std::mutex g_inject_mu;
bool g_inject_armed = false;
int g_inject_unit = -1, g_inject_kb = -1;
uint64_t g_inject_wait_ns = 0;

void take_injection(int& unit, int& kb, uint64_t& wait_ns) {
  std::lock_guard<std::mutex> lk(g_inject_mu);
  if (!g_inject_armed) return;
  unit = g_inject_unit;
  kb = g_inject_kb;
  wait_ns = g_inject_wait_ns;
  g_inject_armed = false;
}

struct TileChoice {
  int cg;    // CTAs per tile (1, or a cluster pair with cta_group::2)
  int bn;    // output columns per tile (256 or 128)
  int rh;    // 128-row halves per CTA (2: the tall 512 x 256 pair tile)
};

// Relative throughput of each tile shape per SM (the 256 x 256 pair tile is
// the reference): narrower or single-CTA tiles read more operand bytes per
// MMA and keep the tensor pipe a little less busy.
double tile_efficiency(const TileChoice& t) {
  // measured per SM against the 256 x 256 pair tile on the layer's shapes
  // (h = 4096 MLP, h = 1600 projections, logits): 0.60-0.75 for 256 x 128,
  // 0.90-1.0 for 128 x 256, 0.55-0.70 for 128 x 128
  if (t.cg == 2) return t.bn == 256 ? (t.rh == 2 ? kTallEfficiency : 1.0) : 0.70;
  return t.bn == 256 ? 0.92 : 0.60;
}

// Tile shape of a GEMM: the one with the least estimated time, counting
// whole waves of units (tiles x splits) over the resident slots, each wave
// costing one tile's work per SM.  Problems one 128-row tile high use
// single-CTA tiles; the cross-entropy epilogues need 256-column tiles.
// TP_GEMM_TILE=2x256|2x256t|2x128|1x256|1x128 forces a shape (tests, sweeps).
TileChoice choose_tile(int M, int N, int K, int splits, int epi) {
  const bool xent = epi == EPI_XENT_STATS || epi == EPI_XENT_GRAD;
  // the tall tile's epilogue does not overlap its main loop: only for long
  // main loops (K per split >= 4096) with bf16 outputs (the fp32 logits and
  // the cross-entropy epilogues stay on the overlapped tile)
  const bool tall_ok = K / splits >= 4096 && !xent && epi != EPI_STORE_F32;
  if (const char* e = std::getenv("TP_GEMM_TILE")) {
    TileChoice t{0, 0, 1};
    if (!std::strcmp(e, "2x256")) t = {2, 256, 1};
    else if (!std::strcmp(e, "2x256t")) t = {2, 256, 2};
    else if (!std::strcmp(e, "2x128")) t = {2, 128, 1};
    else if (!std::strcmp(e, "1x256")) t = {1, 256, 1};
    else if (!std::strcmp(e, "1x128")) t = {1, 128, 1};
    if (t.cg && !(xent && t.bn != 256)) return t;
  }
  // The tall tile is not among the automatic choices: in the whole layer
  // step (after the logits and the cross-entropy have filled L2 with their
  // write-backs) its non-overlapped epilogue made the MLP about 19 % slower,
  // although alone it ties or beats the 256 x 256 pair tile.
  const TileChoice cands[4] = {{2, 256, 1}, {2, 128, 1}, {1, 256, 1}, {1, 128, 1}};
  TileChoice best{M > BM ? 2 : 1, 256, 1};
  double best_cost = 0.0;
  bool have = false;
  for (const TileChoice& t : cands) {
    if (xent && t.bn != 256) continue;
    if (M <= BM && t.cg == 2) continue;
    if (t.rh == 2 && !tall_ok) continue;
    const int rows = BM * t.rh * t.cg;
    const long long tiles = static_cast<long long>((M + rows - 1) / rows) * ((N + t.bn - 1) / t.bn);
    const long long slots = num_sms() / t.cg;
    const long long waves = (tiles * splits + slots - 1) / slots;
    const double cost = static_cast<double>(waves) * t.rh * t.bn / tile_efficiency(t);
    if (!have || cost < best_cost * 0.999) {
      best = t;
      best_cost = cost;
      have = true;
    }
  }
  return best;
}

}  // namespace

bool make_tmap_bf16_sw128(void* tmap, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                          uint32_t box_inner, uint32_t box_outer) {
  return make_tmap(static_cast<CUtensorMap*>(tmap), ptr, inner, outer, ld, box_inner, box_outer);
}

bool make_tmap_f32_sw128(void* tmap, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                         uint32_t box_inner, uint32_t box_outer) {
  return make_tmap_f32(static_cast<CUtensorMap*>(tmap), ptr, inner, outer, ld, box_inner, box_outer,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t gemm_split_ws_bytes(int M, int N, int splits, bool with_zpart) {
  if (splits <= 1 && !with_zpart) return 0;
  // 128-row pieces of the 512-row tall tiling (covers the 256- and 128-row
  // tilings too); the partial bytes of 256-column tiles bound those of
  // 128-column tiles, whose counters are twice as many
  const size_t hrows = static_cast<size_t>((M + 4 * BM - 1) / (4 * BM)) * 4;
  size_t bytes = with_zpart ? 0 : hrows * ((N + BN - 1) / BN) * splits * BM * BN * sizeof(float);
  bytes += hrows * ((N + 127) / 128) * sizeof(int);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

double gemm_tc_estimate_s(int M, int N, int K, int splits, int epi) {
  const TileChoice t = choose_tile(M, N, K, splits, epi);
  const int rows = BM * t.rh * t.cg;
  const long long tiles = static_cast<long long>((M + rows - 1) / rows) * ((N + t.bn - 1) / t.bn);
  const long long slots = num_sms() / t.cg;
  const long long waves = (tiles * splits + slots - 1) / slots;
  const double k_split = static_cast<double>(K) / splits;
  const double per_sm_flops = 1.5e15 / 148.0;   // bf16 dense, sustained
  return static_cast<double>(waves) * 2.0 * BM * t.rh * t.bn * k_split /
         (per_sm_flops * tile_efficiency(t));
}

namespace {

// Kernel arguments, operand maps and (split epilogue) workspace of one
// problem with the given tile shape.
tp_status setup_problem(const GemmProblem& p, const TileChoice& tile, GemmArgs& a,
                        CUtensorMap* tmA, CUtensorMap* tmB, CUtensorMap* tmO, cudaStream_t stream) {
  if (p.M <= 0 || p.N <= 0 || p.K <= 0) return TP_ERR_SHAPE;
  if (p.splits < 1 || p.splits > kMaxSplits) return TP_ERR_SHAPE;
  const bool split_epi = p.splits > 1 || p.zpart != nullptr;
  const int CG = tile.cg, BNT = tile.bn, RH = tile.rh;
  const int rows = BM * RH * CG;
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.a_mn = p.a_mn;
  a.b_mn = p.b_mn;
  a.tiles_m = (p.M + rows - 1) / rows;
  a.tiles_n = (p.N + BNT - 1) / BNT;
  a.splits = p.splits;
  // bands of 2048 rows (inside a band the B columns are read once, so B is
  // read once per band and A once in all).  Taller bands read less in
  // principle but measured slower with more DRAM reads (the logits GEMM:
  // 7.3 GB read with 32-tile-row bands against 6.5 GB with 8); the byte
  // budget rule stays as a sweep switch
  a.group_m = CG == 2 ? 8 : 16;
  // Column bands when B is more than twice A, a band of 16 B panels (its
  // columns over the whole K range of a split) fits in a third of L2, and
  // there are enough tile rows for a band to hold several waves: A is then
  // re-read once per band instead of B once per row band (the logits GEMM:
  // 13 reads of H, 134 MB, instead of 8 of the 412 MB table; 5.9 against
  // 9.1 GB read in one capture).  The MLP's shapes (16 tile rows) read more
  // with column bands, so they keep row bands.
  a.group_n = 0;
  {
    const double kspan = static_cast<double>((p.K + p.splits - 1) / p.splits);
    const double panel = static_cast<double>(BNT) * kspan * 2.0;
    if (column_bands_enabled() && static_cast<int64_t>(p.N) > 2 * static_cast<int64_t>(p.M) &&
        16.0 * panel <= 42.0 * 1024.0 * 1024.0 && a.tiles_n > 16 && a.tiles_m >= 32)
      a.group_n = 16;
  }
  if (band_budget_bytes() > 0.0) {
    a.group_n = 0;
    const double row_bytes = static_cast<double>(rows) * ((p.K + p.splits - 1) / p.splits) * 2.0;
    const int band = static_cast<int>(band_budget_bytes() / row_bytes);
    a.group_m = band < 1 ? 1 : (band > a.tiles_m ? a.tiles_m : band);
  }
  const int kblocks = (p.K + BK - 1) / BK;
  if (p.splits == 1) {
    a.split_kb[0] = 0;
    a.split_kb[1] = kblocks;
  } else {
    for (int s = 0; s <= p.splits; ++s) {
      const int k = p.split_k[s];
      if (s > 0 && s < p.splits && (k % BK) != 0) return TP_ERR_UNSUPPORTED;
      a.split_kb[s] = (k + BK - 1) / BK;
      if (s > 0 && a.split_kb[s] <= a.split_kb[s - 1]) return TP_ERR_SHAPE;
    }
    if (p.split_k[0] != 0 || p.split_k[p.splits] != p.K) return TP_ERR_SHAPE;
  }
  // split-sum GEMMs split only the tiles of the last, partial wave (the
  // others run their whole K range in the accumulator); per-shard partials
  // (Zpart) split every tile.  TP_GEMM_SPLIT_ALL=1 splits every tile (sweeps).
  a.full_tiles = 0;
  if (p.splits > 1 && p.zpart == nullptr && !split_all_tiles()) {
    const int tiles = a.tiles_m * a.tiles_n;
    const int slots = num_sms() / CG;
    a.full_tiles = tiles - tiles % slots;
  }
  a.num_units = a.full_tiles + (a.tiles_m * a.tiles_n - a.full_tiles) * a.splits;
  // partials requested (Zpart) go through the split epilogue even for a
  // single split: it publishes the partial and stores the (one-term) sum
  if (p.zpart != nullptr && p.epi != EPI_STORE_BF16) return TP_ERR_UNSUPPORTED;
  a.act = p.act;
  a.out0 = p.out0;
  a.out1 = p.out1;
  a.ldo = p.ldo;
  a.bias = static_cast<const __nv_bfloat16*>(p.bias);
  a.aux = static_cast<const __nv_bfloat16*>(p.aux);
  a.ld_aux = p.ld_aux;
  a.dbias_part = p.dbias_part;
  a.dev_status = p.dev_status;
  a.wait_ns = wait_limit_ns();
  a.targets = p.targets;
  a.stat_m = p.stat_m;
  a.stat_s = p.stat_s;
  a.stat_i = p.stat_i;
  a.tgt_logit = p.tgt_logit;
  a.row_lse = p.row_lse;
  a.grad_scale = p.grad_scale;
  a.inject_unit = -1;
  a.inject_kb = -1;
  if ((p.epi == EPI_XENT_STATS || p.epi == EPI_XENT_GRAD) && p.splits != 1) return TP_ERR_UNSUPPORTED;
  if (split_epi) {
    const size_t need = gemm_split_ws_bytes(p.M, p.N, p.splits, p.zpart != nullptr);
    if (p.ws == nullptr || p.ws_bytes < need) return TP_ERR_WORKSPACE;
    const size_t htiles = static_cast<size_t>(a.tiles_m) * CG * RH * a.tiles_n;
    if (p.zpart) {
      a.part = p.zpart;
      a.part_is_zpart = 1;
      a.counters = static_cast<int*>(p.ws);
    } else {
      a.part = static_cast<float*>(p.ws);
      a.part_is_zpart = 0;
      a.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(p.ws) +
                                          htiles * p.splits * BM * BNT * sizeof(float));
    }
    if (cudaMemsetAsync(a.counters, 0, htiles * sizeof(int), stream) != cudaSuccess)
      return TP_ERR_CUDA;
  }
  // operand maps: A boxes of 128·RH rows (K-major) or 64 x 64 blocks
  // (MN-major); B boxes of BNT / CG rows (K-major) or 64 x 64 blocks (MN-major)
  const uint32_t b_rows = static_cast<uint32_t>(BNT / CG);
  bool ok;
  if (!p.a_mn)
    ok = make_tmap(tmA, p.A, p.K, p.M, p.lda, BK, static_cast<uint32_t>(BM * RH));
  else
    ok = make_tmap(tmA, p.A, p.M, p.K, p.lda, 64, BK);
  if (!ok) return TP_ERR_CUDA;
  if (!p.b_mn)
    ok = make_tmap(tmB, p.B, p.K, p.N, p.ldb, BK, b_rows);
  else
    ok = make_tmap(tmB, p.B, p.N, p.K, p.ldb, 64, BK);
  if (!ok) return TP_ERR_CUDA;
  // the bf16 outputs of the plain, bias + activation and dGeLU epilogues
  // leave through 32 x 32 TMA stores when both can be described (16-byte
  // aligned base, row stride a multiple of 16 bytes); otherwise from
  // registers
  a.tma_out = 0;
  const bool staged = !split_epi && (p.epi == EPI_STORE_BF16 || p.epi == EPI_BIAS_ACT ||
                                     p.epi == EPI_DACT || p.epi == EPI_DACT_Y);
  if (staged && !(tma_store_disabled())) {
    bool mk = true;
    void* outs[2] = {p.out0, p.out1};
    for (int o = 0; o < 2 && mk; ++o)
      if (outs[o] != nullptr)
        mk = (reinterpret_cast<uintptr_t>(outs[o]) & 15) == 0 && (p.ldo * 2) % 16 == 0 &&
             make_tmap(&tmO[o], outs[o], p.N, p.M, p.ldo, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    a.tma_out = mk ? 1 : 0;
  } else if (!split_epi && p.epi == EPI_STORE_F32 && !tma_store_disabled()) {
    // fp32: boxes of 16 columns (64-byte lines) x 32 rows
    a.tma_out = (reinterpret_cast<uintptr_t>(p.out0) & 15) == 0 && (p.ldo * 4) % 16 == 0 &&
                make_tmap_f32(&tmO[0], p.out0, p.N, p.M, p.ldo, 16, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  return TP_OK;
}

tp_status dispatch(GemmParams& prm, const TileChoice& tile, int epi, cudaStream_t stream) {
  take_injection(prm.a[0].inject_unit, prm.a[0].inject_kb, prm.a[0].wait_ns);
  prm.a[1].wait_ns = prm.a[0].wait_ns;
  const int slots = tile.cg == 2 ? num_sms() / 2 : num_sms();
  const int used = prm.total_units < slots ? prm.total_units : slots;
  if (tile.cg == 2) {
    if (tile.rh == 2) return launch_epi<2, 256, 2>(prm, epi, used, stream);
    return tile.bn == 256 ? launch_epi<2, 256, 1>(prm, epi, used, stream)
                          : launch_epi<2, 128, 1>(prm, epi, used, stream);
  }
  return tile.bn == 256 ? launch_epi<1, 256, 1>(prm, epi, used, stream)
                        : launch_epi<1, 128, 1>(prm, epi, used, stream);
}

}  // namespace

tp_status gemm_tc_launch(const GemmProblem& p, cudaStream_t stream) {
  const bool split_epi = p.splits > 1 || p.zpart != nullptr;
  const int epi = split_epi ? EPI_SPLIT_SUM : p.epi;
  const TileChoice tile = choose_tile(p.M, p.N, p.K, p.splits, epi);
  GemmParams prm;
  memset(&prm, 0, sizeof(prm));
  if (tp_status st = setup_problem(p, tile, prm.a[0], &prm.tmA[0], &prm.tmB[0], prm.tmO[0], stream))
    return st;
  prm.a[1] = prm.a[0];
  prm.tmA[1] = prm.tmA[0];
  prm.tmB[1] = prm.tmB[0];
  prm.tmO[1][0] = prm.tmO[0][0];
  prm.tmO[1][1] = prm.tmO[0][1];
  prm.units0 = prm.a[0].num_units;
  prm.total_units = prm.units0;
  return dispatch(prm, tile, epi, stream);
}

tp_status gemm_tc_launch_pair(const GemmProblem& p0, const GemmProblem& p1, cudaStream_t stream) {
  // TP_GEMM_NO_PAIR=1 runs the two problems as two launches (sweeps)
  if (const char* e = std::getenv("TP_GEMM_NO_PAIR"))
    if (e[0] == '1') {
      if (tp_status st = gemm_tc_launch(p0, stream)) return st;
      return gemm_tc_launch(p1, stream);
    }
  // two independent problems of one epilogue, no split, no partials: one launch
  if (p0.splits != 1 || p1.splits != 1 || p0.zpart || p1.zpart || p0.epi != p1.epi ||
      p0.epi == EPI_XENT_STATS || p0.epi == EPI_XENT_GRAD || p0.dbias_part || p1.dbias_part)
    return TP_ERR_UNSUPPORTED;
  // the tile shape of the larger problem, and pairs of CTAs only when both
  // are more than one 128-row tile high
  const bool first_larger = static_cast<double>(p0.M) * p0.N >= static_cast<double>(p1.M) * p1.N;
  const GemmProblem& big = first_larger ? p0 : p1;
  TileChoice tile = choose_tile(big.M, big.N, big.K, 1, p0.epi);
  if ((p0.M <= BM || p1.M <= BM) && tile.cg == 2) tile = TileChoice{1, 256, 1};
  GemmParams prm;
  memset(&prm, 0, sizeof(prm));
  if (tp_status st = setup_problem(p0, tile, prm.a[0], &prm.tmA[0], &prm.tmB[0], prm.tmO[0], stream))
    return st;
  if (tp_status st = setup_problem(p1, tile, prm.a[1], &prm.tmA[1], &prm.tmB[1], prm.tmO[1], stream))
    return st;
  prm.units0 = prm.a[0].num_units;
  prm.total_units = prm.units0 + prm.a[1].num_units;
  return dispatch(prm, tile, p0.epi, stream);
}

void arm_gemm_injection(int unit, int kb, uint64_t wait_ns) {
  std::lock_guard<std::mutex> lk(g_inject_mu);
  g_inject_unit = unit;
  g_inject_kb = kb;
  g_inject_wait_ns = wait_ns;
  g_inject_armed = true;
}

}  // namespace tpl
