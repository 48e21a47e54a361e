// attn.cu — attention core between the tensor-parallel projections, sm_100a.
//
// Each shard owns whole heads, so the core needs no communication: every head
// of every sequence is computed independently from the column-parallel QKV
// projection (shard-major columns: a shard's Q heads, then its K heads, then
// its V heads), and the context is written with the heads in order, which
// makes shard i's block of columns the input of its rows of the row-parallel
// output projection.
//
//   O = softmax(Q·Kᵀ·scale + causal mask)·V,  head_dim 64, bf16 in and out
//
// One CTA computes one 128-query tile of one head of one sequence, streaming
// 64-key blocks (flash-style online softmax); two or three CTAs share an SM,
// each with its own pipeline, so one CTA's MMAs run while another's softmax
// does and the uneven causal tiles (launched heaviest first) balance:
//   warp 0    TMA: the Q tile once, K and V blocks into a two-stage ring;
//   warp 1    owns 128 tensor-memory columns; one lane issues S = Q·Kᵀ
//             (128 x 64 fp32) as soon as the softmax has read the previous
//             S into registers, and O += P·V (128 x 64 fp32, accumulated in
//             tensor memory) once the softmax has written P;
//   warps 2-5 the softmax, one query row per thread (its TMEM lane): the
//             block's scores read in one round trip and released, row
//             maximum, p = 2^(x − m) in the log2 domain as bf16 into shared
//             memory in the 128-byte-swizzled K-major layout the MMA reads,
//             the running sum; O is rescaled in tensor memory only when a
//             row's maximum grows by more than 2^8.
// Every wait is bounded: on a timeout the kernel sets TP_DEVERR_TIMEOUT,
// lets its copies and MMAs finish and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace tpl {

namespace {

constexpr int kBQ = 128;                       // queries per tile (TMEM lanes)
constexpr int kFK = 64;                        // keys per forward block
constexpr int kHD = 64;                        // head dimension: one 128-byte row
constexpr int kFwdThreads = 192;               // 6 warps
constexpr int kSoftmaxThreads = 128;           // one warpgroup per query tile
constexpr int kMaxHeads = 256;
constexpr uint32_t kTile = kBQ * kHD * 2;      // 16 KB: 128 rows of 128 bytes
constexpr uint32_t kKVTile = kFK * kHD * 2;    // 8 KB: 64 rows of 128 bytes
constexpr int kFStages = 3;                    // K/V ring depth
constexpr uint32_t kPTileF = kBQ * kFK * 2;    // 16 KB: P of one block, bf16
// forward shared memory: Q, K and V in a ring, P double buffered
constexpr uint32_t kFOffQ = 0;
constexpr uint32_t kFOffK = kFOffQ + kTile;
constexpr uint32_t kFOffV = kFOffK + kFStages * kKVTile;
constexpr uint32_t kFOffP = kFOffV + kFStages * kKVTile;
constexpr uint32_t kFOffBar = kFOffP + 2 * kPTileF;
constexpr int kFNumBars = 4 + 2 * kFStages + 4;
constexpr uint32_t kFOffMisc = kFOffBar + kFNumBars * 8;
constexpr uint32_t kFwdAlloc = kFOffMisc + 16 + 1024;     // slack for 1024-byte alignment
static_assert(kFOffK % 1024 == 0 && kFOffV % 1024 == 0 && kFOffP % 1024 == 0 &&
                  kKVTile % 1024 == 0 && kPTileF % 1024 == 0,
              "forward shared-memory layout: swizzled tiles on 1024-byte boundaries");
constexpr uint32_t kFwdTmemCols = 128;                     // S: 64, O: 64
constexpr uint32_t kFTmemO = 64;
constexpr uint32_t kTmemCols = 512;                        // backward
constexpr float kLn2 = 0.6931471805599453f;

struct AttnArgs {
  int b, s, heads, nqb;
  int causal;
  float scale_log2;          // scale · log2(e)
  __nv_bfloat16* ctx;
  int64_t ldc;
  float* lse;                // [b, heads, s], nullable
  int32_t* dev_status;
  uint64_t wait_ns;
  int2 head_cols[kMaxHeads]; // (first Q column of the head, width of its shard's Q block)
};

struct __align__(64) AttnParams {
  CUtensorMap tm;            // QKV [b·s, 3h], boxes of 64 columns x 128 rows (Q)
  CUtensorMap tm_kv;         // QKV, boxes of 64 columns x 64 rows (K and V blocks)
  AttnArgs a;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// The running maximum only moves when a block's maximum exceeds it by more
// than 2^kTau (log2 units): p = 2^(x·sl − m) then stays below 2^kTau = 256,
// exact enough in bf16 and far from fp32 overflow, and O in tensor memory is
// rescaled only on those rare moves instead of after every block.
constexpr float kTau = 8.0f;

// All 64 scores of this thread's row of one block, read from tensor memory
// in one round trip (two 32-column loads, one wait).  With kMask, keys at
// positions >= klim become −inf.  Returns the row maximum.
template <bool kMask>
__device__ __forceinline__ float load_block_row(uint32_t sbase, int kpos0, int klim,
                                                uint32_t (&x)[kFK]) {
#pragma unroll
  for (int c = 0; c < kFK / 32; ++c)
    tmem_ld_32x32b_x32(sbase + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&x[c * 32]));
  tc_wait_ld();
  if (kMask) {
#pragma unroll
    for (int t = 0; t < kFK; ++t)
      if (kpos0 + t >= klim) x[t] = 0xff800000u;   // −inf
  }
  float acc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int t = 0; t < kFK; t += 8) {
    float& a = acc[(t >> 3) & 3];
    a = fmax3(a, __uint_as_float(x[t]), __uint_as_float(x[t + 1]));
    a = fmax3(a, __uint_as_float(x[t + 2]), __uint_as_float(x[t + 3]));
    a = fmax3(a, __uint_as_float(x[t + 4]), __uint_as_float(x[t + 5]));
    a = fmax3(a, __uint_as_float(x[t + 6]), __uint_as_float(x[t + 7]));
  }
  return fmaxf(fmax3(acc[0], acc[1], acc[2]), acc[3]);
}

// p = 2^(x·sl − m) of the row, stored as bf16 into this row of the P tile
// (one 128-byte row of 64 keys, 16-byte granule g at g ^ (row & 7): the
// 128-byte swizzle the MMA's descriptor names).  Returns Σ p.
// The scaling and the sums run on pairs (f32x2 FMA and add).
__device__ __forceinline__ float exp_store_row(const uint32_t (&x)[kFK], float sl, float m,
                                               uint8_t* prow, int r) {
  const float2 sl2 = make_float2(sl, sl);
  const float2 nm2 = make_float2(-m, -m);
  float2 ps[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
  for (int gr = 0; gr < 8; ++gr) {            // 16-byte granule of the 128-byte row
    float p[8];
#pragma unroll
    for (int t = 0; t < 8; t += 2) {
      const float2 y = __ffma2_rn(make_float2(__uint_as_float(x[gr * 8 + t]),
                                              __uint_as_float(x[gr * 8 + t + 1])), sl2, nm2);
      p[t] = ex2f(y.x);
      p[t + 1] = ex2f(y.y);
      ps[(t >> 1) & 1] = __fadd2_rn(ps[(t >> 1) & 1], make_float2(p[t], p[t + 1]));
    }
    uint4 w;
    w.x = pack_bf16x2(p[0], p[1]);
    w.y = pack_bf16x2(p[2], p[3]);
    w.z = pack_bf16x2(p[4], p[5]);
    w.w = pack_bf16x2(p[6], p[7]);
    *reinterpret_cast<uint4*>(prow + ((gr ^ (r & 7)) << 4)) = w;
  }
  return (ps[0].x + ps[1].x) + (ps[0].y + ps[1].y);
}

__device__ __forceinline__ void attn_timeout(const AttnArgs& a, volatile int* abort_flag) {
  if (!*abort_flag) {
    *abort_flag = 1;
    if (a.dev_status) atomicOr(a.dev_status, TP_DEVERR_TIMEOUT);
  }
}

__global__ void __launch_bounds__(kFwdThreads, 2) attn_fwd_kernel(const __grid_constant__ AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const AttnArgs& a = P.a;
  uint8_t* sQ = smem + kFOffQ;
  uint8_t* sK = smem + kFOffK;
  uint8_t* sV = smem + kFOffV;
  uint8_t* sP = smem + kFOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kFOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                    // [stage]
  uint64_t* kv_empty = kv_full + kFStages;         // [stage]
  uint64_t* s_full = kv_empty + kFStages;          // S(j) in tensor memory
  uint64_t* s_free = s_full + 1;                   // S(j) read into the softmax's registers
  uint64_t* p_full = s_free + 1;                   // [j & 1] P(j) written, O rescaled
  uint64_t* o_full = p_full + 2;                   // [j & 1] P·V(j) done: O current, P(j) free
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kFOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the last query tiles (the longest under the causal mask) first
  const int bh = a.b * a.heads;
  const int qb = a.nqb - 1 - static_cast<int>(blockIdx.x) / bh;
  const int rem = static_cast<int>(blockIdx.x) % bh;
  const int head = rem / a.b;
  const int batch = rem % a.b;
  const int row0 = batch * a.s;                         // first token row of the sequence
  const int nkb_all = (a.s + kFK - 1) / kFK;
  // key blocks of this tile: up to the tile's last query under the causal mask
  const int nk = a.causal ? min((qb + 1) * (kBQ / kFK), nkb_all) : nkb_all;
  const int qcol = a.head_cols[head].x;
  const int kcol = qcol + a.head_cols[head].y;
  const int vcol = kcol + a.head_cols[head].y;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kFStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftmaxThreads);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], kSoftmaxThreads);
      mbar_init(&o_full[i], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kFwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (elect_one_sync()) {
      tma_prefetch_desc(&P.tm);
      tma_prefetch_desc(&P.tm_kv);
      mbar_arrive_expect_tx(q_full, kTile);
      tma_load_2d(sQ, &P.tm, q_full, qcol, row0 + qb * kBQ);
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int st = j % kFStages;
        const uint32_t ph = static_cast<uint32_t>(j / kFStages) & 1u;
        if (!mbar_wait_bounded(&kv_empty[st], ph ^ 1u, a.wait_ns, abort_flag)) {
          attn_timeout(a, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(&kv_full[st], 2 * kKVTile);
        tma_load_2d(sK + st * kKVTile, &P.tm_kv, &kv_full[st], kcol, row0 + j * kFK);
        tma_load_2d(sV + st * kKVTile, &P.tm_kv, &kv_full[st], vcol, row0 + j * kFK);
        ++issued;
      }
      // every copy lands before the CTA can exit (bounded, not cut short by
      // the abort flag): the Q tile and the last stages of the ring
      volatile int keep_waiting = 0;
      mbar_wait_bounded(q_full, 0, a.wait_ns, &keep_waiting);
      for (int j = issued > kFStages ? issued - kFStages : 0; j < issued; ++j)
        mbar_wait_bounded(&kv_full[j % kFStages], static_cast<uint32_t>(j / kFStages) & 1u,
                          a.wait_ns, &keep_waiting);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one_sync()) {
      constexpr uint32_t idS = idesc_bf16_f32(kBQ, kFK, false, false);   // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16_f32(kBQ, kHD, false, true);    // P K-major, V MN-major
      bool any = false;
      const uint32_t qa = smem_u32(sQ);
      // S(j) = Q·K_jᵀ into the S columns
      auto issue_s = [&](int j) -> bool {
        const int st = j % kFStages;
        if (!mbar_wait_bounded(&kv_full[st], static_cast<uint32_t>(j / kFStages) & 1u, a.wait_ns,
                               abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t kb = smem_u32(sK + st * kKVTile);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)
          tc_mma_bf16(tmem, smem_desc_sw128(qa + k * 32, 16, 1024),
                      smem_desc_sw128(kb + k * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
        any = true;
        tc_commit(s_full);
        return true;
      };
      bool ok = mbar_wait_bounded(q_full, 0, a.wait_ns, abort_flag);
      if (ok && nk > 0) ok = issue_s(0);
      for (int j = 0; ok && j < nk; ++j) {
        // the next S as soon as the softmax holds S(j) in registers
        if (j + 1 < nk) {
          ok = mbar_wait_bounded(s_free, static_cast<uint32_t>(j & 1), a.wait_ns, abort_flag) &&
               issue_s(j + 1);
          if (!ok) break;
        }
        // O += P(j)·V_j once the softmax has written P(j) (and rescaled O)
        if (!mbar_wait_bounded(&p_full[j & 1], static_cast<uint32_t>(j >> 1) & 1u, a.wait_ns,
                               abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t vb = smem_u32(sV + (j % kFStages) * kKVTile);
        const uint32_t pa = smem_u32(sP + (j & 1) * kPTileF);
#pragma unroll
        for (int k = 0; k < kFK / 16; ++k)   // 16 keys per step
          tc_mma_bf16(tmem + kFTmemO, smem_desc_sw128(pa + k * 32, 16, 1024),
                      smem_desc_sw128(vb + k * 2048, 8192, 1024), idO,
                      (j > 0 || k > 0) ? 1u : 0u);
        tc_commit(&o_full[j & 1]);
        tc_commit(&kv_empty[j % kFStages]);   // K_j and V_j read by every MMA issued so far
      }
      if (!ok) attn_timeout(a, abort_flag);
      if (any) {   // every issued MMA completes before tensor memory is freed
        volatile int keep_waiting = 0;
        tc_commit(mma_done);
        mbar_wait_bounded(mma_done, 0, a.wait_ns, &keep_waiting);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int qd = warp & 3;                        // TMEM lane quadrant of this warp
    const int r = qd * 32 + lane;                   // row of the query tile
    const int qpos = qb * kBQ + r;                  // position in the sequence
    const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t sbase = tmem + lane_off;
    const uint32_t obase = tmem + lane_off + kFTmemO;
    const float sl = a.scale_log2;
    const int klim = a.causal ? min(qpos + 1, a.s) : a.s;   // keys [0, klim) are visible
    float m = -INFINITY;                            // running maximum (log2 units)
    float l = 0.0f;                                 // running sum of 2^(x − m)
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      // the warp's lanes agree before the warp-collective tensor-memory loads
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full, static_cast<uint32_t>(j & 1),
                                                     a.wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const int kpos0 = j * kFK;
      const bool need_mask = (a.causal && kpos0 + kFK > qb * kBQ) || kpos0 + kFK > a.s;
      uint32_t x[kFK];
      const float mx = need_mask ? load_block_row<true>(sbase, kpos0, klim, x)
                                 : load_block_row<false>(sbase, kpos0, klim, x);
      tc_fence_before_sync();
      mbar_arrive(s_free);                          // S read: the MMA may compute S(j+1)
      // finite at j = 0 (key 0 is visible to every row); a later block that
      // is wholly masked for this row gives −inf and moves nothing
      const float m_blk = mx * sl;
      const bool move = j == 0 || m_blk > m + kTau;
      const float alpha = (j > 0 && move) ? ex2f(m - m_blk) : 1.0f;
      if (move) m = m_blk;
      // P(j) reuses the buffer of P(j-2): P·V(j-2) must have finished
      if (j > 1 && !__all_sync(0xffffffffu, mbar_wait_bounded(&o_full[j & 1],
                                                                static_cast<uint32_t>((j - 2) >> 1) & 1u,
                                                                a.wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      // p = 2^(x·sl − m), bf16 into the swizzled P tile, and the row sum
      l = fmaf(l, alpha, exp_store_row(x, sl, m, sP + (j & 1) * kPTileF + r * 128, r));
      if (j > 0 && __any_sync(0xffffffffu, move)) {
        // rescale the rows whose maximum moved (the others by 1) once
        // P·V(j-1) has finished, before the P·V of this block adds to O
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&o_full[(j - 1) & 1],
                                                       static_cast<uint32_t>((j - 1) >> 1) & 1u,
                                                       a.wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < kHD / 32; ++c) {
          uint32_t rr[32];
          tmem_ld_32x32b_x32(obase + c * 32, rr);
          tc_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; t += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(rr[t]), __uint_as_float(rr[t + 1])), a2);
            rr[t] = __float_as_uint(v.x);
            rr[t + 1] = __float_as_uint(v.y);
          }
          tmem_st_32x32b_x32(obase + c * 32, rr);
        }
        tc_wait_st();
      }
      tc_fence_before_sync();                      // O written before the arrival
      fence_proxy_async_smem();                    // P visible to the tensor core
      mbar_arrive(&p_full[j & 1]);
    }
    // the last P·V's commit covers every MMA before it
    if (ok && nk > 0)
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_full[(nk - 1) & 1],
                                                     static_cast<uint32_t>((nk - 1) >> 1) & 1u,
                                                     a.wait_ns, abort_flag));
    if (!ok) {
      if (lane == 0) attn_timeout(a, abort_flag);
    } else if (nk > 0) {
      tc_fence_after_sync();
      const float inv = 1.0f / l;
      __nv_bfloat16* dst = a.ctx + static_cast<int64_t>(row0 + qpos) * a.ldc + head * kHD;
#pragma unroll
      for (int c = 0; c < kHD / 32; ++c) {
        uint32_t rr[32];
        tmem_ld_32x32b_x32(obase + c * 32, rr);   // every lane loads; rows past s store nothing
        tc_wait_ld();
#pragma unroll
        for (int gr = 0; gr < 4; ++gr) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(rr[8 * gr + 0]) * inv, __uint_as_float(rr[8 * gr + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(rr[8 * gr + 2]) * inv, __uint_as_float(rr[8 * gr + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(rr[8 * gr + 4]) * inv, __uint_as_float(rr[8 * gr + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(rr[8 * gr + 6]) * inv, __uint_as_float(rr[8 * gr + 7]) * inv);
          if (qpos < a.s) reinterpret_cast<uint4*>(dst + c * 32)[gr] = w;
        }
      }
      if (a.lse && qpos < a.s)
        a.lse[(static_cast<int64_t>(batch) * a.heads + head) * a.s + qpos] = m * kLn2 + logf(l);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}


// ===========================================================================
// Backward.  A prep kernel computes D = rowsum(dO ⊙ O) and zeroes the fp32
// dQ accumulator; then one CTA per 128-key tile of a head streams the queries
// in tiles of 64:
//   Sᵀ = K·Qᵀ and dPᵀ = V·dOᵀ in tensor memory,
//   Pᵀ = exp(Sᵀ·scale − lse) and dSᵀ = Pᵀ ⊙ (dPᵀ − D) per key row,
//   dV += Pᵀ·dO and dK += dSᵀ·Q accumulated in tensor memory,
//   dQ_pair = dS·K for every two streamed tiles (one 128-row MMA over the two
//   dS tiles, MN-major), staged in shared memory and added into the fp32
//   accumulator in global memory by a TMA reduce (the adds happen in L2, off
//   the load/store path the element-wise warps use);
// a finish kernel scales the accumulated dQ and writes it as bf16.  dK and dV
// of a key row come from exactly one CTA (reproducible bit for bit); dQ sums
// the key tiles' contributions in fp32 in whatever order they arrive, so its
// last bits may differ between runs.
//
// Roles (11 warps): warp 0 TMA (the fixed K and V tiles once, the streamed
// Q and dO tiles through a three-stage ring), warp 1 the MMA issuer, warps 2-5
// and 6-9 two element-wise warpgroups taking the streamed tiles in turn,
// warp 10 the dQ reduces.  S/dP and the bf16 P tiles are double buffered and
// the dS tiles quadruple buffered (a pair of them is read by the dQ MMA), so
// the MMAs of one tile run while the other warpgroup evaluates its
// exponentials.  Warpgroup w also reads out and stages the dQ of the pairs
// p ≡ w (mod 2), two streamed tiles later; warp 10 issues each pair's TMA
// reduce and alone waits for it to have read the staging buffer.
// ===========================================================================
constexpr int kBG = 64;                                // streamed rows per tile
constexpr int kGStages = 3;
constexpr int kBwdThreads = 352;                       // 11 warps
constexpr int kRedWarp = 10;                           // issues the dQ reduces
constexpr int kDSBufs = 4;
constexpr uint32_t kGTile = kBG * kHD * 2;             // 8 KB: 64 rows of 128 bytes
constexpr uint32_t kPTile = kBQ * kBG * 2;             // 16 KB: 128 keys x 64 queries
constexpr uint32_t kBOffF1 = 0;                        // fixed tiles: K, V
constexpr uint32_t kBOffF2 = kTile;
constexpr uint32_t kBOffG1 = 2 * kTile;                // streamed tiles Q, dO, kGStages each
constexpr uint32_t kBOffG2 = kBOffG1 + kGStages * kGTile;
constexpr uint32_t kBOffP = kBOffG2 + kGStages * kGTile;   // Pᵀ [2 buffers]
constexpr uint32_t kBOffDS = kBOffP + 2 * kPTile;          // dSᵀ [kDSBufs buffers]
constexpr uint32_t kBOffStage = kBOffDS + kDSBufs * kPTile;   // dQ of a pair, fp32, 2 x 16 KB
constexpr uint32_t kStageHalf = kBQ * 32 * 4;                    // 128 rows x 32 columns
constexpr uint32_t kBOffVec = kBOffStage + 2 * kStageHalf;      // [warpgroup][2][−lse·log2e | −D][64]
constexpr uint32_t kBOffBar = kBOffVec + 2 * 2 * 2 * kBG * 4;
// every swizzled tile and TMA box starts on a 1024-byte boundary
static_assert(kBOffG1 % 1024 == 0 && kBOffG2 % 1024 == 0 && kBOffP % 1024 == 0 &&
                  kBOffDS % 1024 == 0 && kBOffStage % 1024 == 0 && kGTile % 1024 == 0 &&
                  kPTile % 1024 == 0 && kStageHalf % 1024 == 0,
              "backward shared-memory layout");
constexpr int kBNumBars = 2 * kGStages + 16;
constexpr uint32_t kBOffMisc = kBOffBar + kBNumBars * 8;
constexpr uint32_t kBAlloc = kBOffMisc + 16 + 1024;
// tensor memory columns: Sᵀ (X) and dPᵀ (Y) double buffered, the
// accumulators dV (A1) and dK (A2), the dQ of a pair double buffered (Q)
constexpr uint32_t kTX = 0, kTY = 128, kTA1 = 256, kTA2 = 320, kTQ = 384;

struct AttnBwdArgs {
  int b, s, heads, nqb, ng;  // ng: streamed 64-row tiles of a sequence
  int causal;
  float scale, scale_log2;
  const float* lse;          // [b, heads, s] natural log
  const float* D;            // [b, heads, s]
  float* dq_acc;             // [b·s, heads·64] fp32, zeroed by the prep kernel
  __nv_bfloat16* dqkv;       // [b·s, 3h], the QKV layout
  int64_t ldq;               // 3h
  int32_t* dev_status;
  uint64_t wait_ns;
  int2 head_cols[kMaxHeads];
};

struct __align__(64) AttnBwdParams {
  CUtensorMap tm_qkv;        // QKV [b·s, 3h], boxes of 64 columns x 128 rows (fixed tiles)
  CUtensorMap tm_qkv_g;      // QKV, boxes of 64 columns x 64 rows (streamed tiles)
  CUtensorMap tm_do_g;       // dO [b·s, h], boxes of 64 columns x 64 rows
  CUtensorMap tm_dq;         // dQ accumulator [b·s, h] fp32, boxes of 32 columns x 128 rows
  AttnBwdArgs a;
};

// D = rowsum(dO ⊙ O) per (token, head), and the dQ accumulator of that
// (token, head) set to zero.  Eight lanes per (token, head): lane j takes
// columns 8j..8j+7 (one 16-byte word of O and of dO, 32 bytes of the
// accumulator), so a warp's loads and stores cover four heads' contiguous
// bytes; the eight partial sums meet by shuffles.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const uint4* __restrict__ O,
                                                            const uint4* __restrict__ dO,
                                                            int64_t rows, int heads, int s,
                                                            float* __restrict__ D,
                                                            float4* __restrict__ dq_acc) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t rh = i >> 3;                           // (row, head)
  const int j = static_cast<int>(i & 7);
  const bool live = rh < rows * heads;                 // whole groups of 8 share it
  float acc = 0.0f;
  if (live) {
    const uint4 a = __ldg(O + rh * 8 + j), c = __ldg(dO + rh * 8 + j);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      acc = fmaf(__uint_as_float(aw[w] << 16), __uint_as_float(cw[w] << 16), acc);
      acc = fmaf(__uint_as_float(aw[w] & 0xffff0000u), __uint_as_float(cw[w] & 0xffff0000u), acc);
    }
    dq_acc[rh * 16 + 2 * j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    dq_acc[rh * 16 + 2 * j + 1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (live && j == 0) {
    const int64_t row = rh / heads;
    const int head = static_cast<int>(rh - row * heads);
    const int64_t bb = row / s, pos = row - bb * s;
    D[(bb * heads + head) * s + pos] = acc;
  }
}

// dQ = scale · (accumulated dS·K), bf16, into this head's Q columns of dQKV.
// One thread per 8 columns of a (token, head).
__global__ void __launch_bounds__(256) attn_dq_finish_kernel(const __grid_constant__ AttnBwdArgs a) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t rows = static_cast<int64_t>(a.b) * a.s;
  if (i >= rows * a.heads * 8) return;
  const int64_t rh = i >> 3;                           // (row, head)
  const int g = static_cast<int>(i & 7);
  const int64_t row = rh / a.heads;
  const int head = static_cast<int>(rh - row * a.heads);
  const float4* src = reinterpret_cast<const float4*>(a.dq_acc) + rh * 16 + g * 2;
  const float4 v0 = src[0], v1 = src[1];
  const float f = a.scale;
  uint4 w;
  w.x = pack_bf16x2(v0.x * f, v0.y * f);
  w.y = pack_bf16x2(v0.z * f, v0.w * f);
  w.z = pack_bf16x2(v1.x * f, v1.y * f);
  w.w = pack_bf16x2(v1.z * f, v1.w * f);
  *reinterpret_cast<uint4*>(a.dqkv + row * a.ldq + a.head_cols[head].x + g * 8) = w;
}

__device__ __forceinline__ void bwd_timeout(const AttnBwdArgs& a, volatile int* abort_flag) {
  if (!*abort_flag) {
    *abort_flag = 1;
    if (a.dev_status) atomicOr(a.dev_status, TP_DEVERR_TIMEOUT);
  }
}

// Half h (32 query columns) of one key row of a streamed tile:
// p = 2^(x·sl − l) (zero where masked) and dS = p·(y − D), written as bf16
// into the row's 128-byte lines of the P and dS tiles, granule g at
// g ^ (row & 7).  −l and −D come per query column from shared memory, four
// at a time; the arithmetic runs on f32x2 pairs.
template <bool kMask>
__device__ __forceinline__ void bwd_half_rows(const uint32_t (&xr)[32], const uint32_t (&yr)[32],
                                              const float* vNL, const float* vND, float sl, int t0,
                                              int kpos, int s, int causal, uint8_t* prow,
                                              uint8_t* drow, int r, int h) {
  const float2 sl2 = make_float2(sl, sl);
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {             // 16-byte granule gr of the 128-byte row
    const int gr = h * 4 + g4;
    const float4 l0 = reinterpret_cast<const float4*>(vNL)[2 * gr];
    const float4 l1 = reinterpret_cast<const float4*>(vNL)[2 * gr + 1];
    const float4 d0 = reinterpret_cast<const float4*>(vND)[2 * gr];
    const float4 d1 = reinterpret_cast<const float4*>(vND)[2 * gr + 1];
    const float2 nl[4] = {make_float2(l0.x, l0.y), make_float2(l0.z, l0.w),
                          make_float2(l1.x, l1.y), make_float2(l1.z, l1.w)};
    const float2 nd[4] = {make_float2(d0.x, d0.y), make_float2(d0.z, d0.w),
                          make_float2(d1.x, d1.y), make_float2(d1.z, d1.w)};
    uint32_t pw[4], dw[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int j = g4 * 8 + 2 * t;            // column within the half
      const float2 e = __ffma2_rn(make_float2(__uint_as_float(xr[j]), __uint_as_float(xr[j + 1])),
                                  sl2, nl[t]);
      float p0 = ex2f(e.x), p1 = ex2f(e.y);
      if constexpr (kMask) {
        const int q0 = t0 + h * 32 + j;        // query positions of the two columns
        p0 = (q0 >= s || kpos >= s || (causal && q0 < kpos)) ? 0.0f : p0;
        p1 = (q0 + 1 >= s || kpos >= s || (causal && q0 + 1 < kpos)) ? 0.0f : p1;
      }
      const float2 dy = __fadd2_rn(make_float2(__uint_as_float(yr[j]), __uint_as_float(yr[j + 1])),
                                   nd[t]);
      const float2 ds = __fmul2_rn(make_float2(p0, p1), dy);
      pw[t] = pack_bf16x2(p0, p1);
      dw[t] = pack_bf16x2(ds.x, ds.y);
    }
    const int off = (gr ^ (r & 7)) << 4;
    *reinterpret_cast<uint4*>(prow + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
    *reinterpret_cast<uint4*>(drow + off) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
  }
}

__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_kernel(const __grid_constant__ AttnBwdParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const AttnBwdArgs& a = P.a;
  uint8_t* sF1 = smem + kBOffF1;
  uint8_t* sF2 = smem + kBOffF2;
  uint8_t* sG1 = smem + kBOffG1;
  uint8_t* sG2 = smem + kBOffG2;
  uint8_t* sP = smem + kBOffP;
  uint8_t* sDS = smem + kBOffDS;
  uint8_t* sStage = smem + kBOffStage;
  float* vec = reinterpret_cast<float*>(smem + kBOffVec);   // [warpgroup][buffer][−lse | −D][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBOffBar);
  uint64_t* f_full = bars;
  uint64_t* g_full = bars + 1;                   // [stage]
  uint64_t* g_empty = g_full + kGStages;         // [stage]
  uint64_t* x_full = g_empty + kGStages;         // [buffer]: Sᵀ and dPᵀ of a tile in tensor memory
  uint64_t* x_empty = x_full + 2;                // [buffer]: read out by the warpgroup
  uint64_t* pd_full = x_empty + 2;               // [warpgroup]: P and dS tiles written
  uint64_t* pd_empty = pd_full + 2;              // [warpgroup]: its buffers free again
  uint64_t* q_full = pd_empty + 2;               // [pair & 1]: dQ of a pair in tensor memory
  uint64_t* q_empty = q_full + 2;                // [pair & 1]: read out
  uint64_t* acc_done = q_empty + 2;
  uint64_t* stage_full = acc_done + 1;           // the dQ of a pair staged in shared memory
  uint64_t* stage_free = stage_full + 1;         // ... and read by its TMA reduce
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = a.b * a.heads;
  // fixed 128-key tile, longest first: under the causal mask key tile t
  // streams the queries from 128·t on
  const int ft = static_cast<int>(blockIdx.x) / bh;
  const int rem = static_cast<int>(blockIdx.x) % bh;
  const int head = rem / a.b;
  const int batch = rem % a.b;
  const int row0 = batch * a.s;
  const int t_begin = a.causal ? 2 * ft : 0;           // in 64-row tiles
  const int nt = a.ng - t_begin;
  const int npairs = (nt + 1) >> 1;
  const int qcol = a.head_cols[head].x;
  const int kcol = qcol + a.head_cols[head].y;
  const int vcol = kcol + a.head_cols[head].y;
  const int ocol = head * kHD;                         // this head's columns of dO

  if (threadIdx.x == 0) {
    mbar_init(f_full, 1);
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&g_full[i], 1);
      mbar_init(&g_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], kSoftmaxThreads);
      mbar_init(&pd_full[i], kSoftmaxThreads);
      mbar_init(&pd_empty[i], 1);
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], kSoftmaxThreads);
    }
    mbar_init(acc_done, 1);
    mbar_init(stage_full, kSoftmaxThreads);
    mbar_init(stage_free, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (elect_one_sync()) {
      tma_prefetch_desc(&P.tm_qkv);
      tma_prefetch_desc(&P.tm_qkv_g);
      tma_prefetch_desc(&P.tm_do_g);
      mbar_arrive_expect_tx(f_full, 2 * kTile);
      tma_load_2d(sF1, &P.tm_qkv, f_full, kcol, row0 + ft * kBQ);
      tma_load_2d(sF2, &P.tm_qkv, f_full, vcol, row0 + ft * kBQ);
      int issued = 0;
      for (int it = 0; it < nt; ++it) {
        const int st = it % kGStages;
        if (!mbar_wait_bounded(&g_empty[st], (static_cast<uint32_t>(it / kGStages) & 1u) ^ 1u,
                               a.wait_ns, abort_flag)) {
          bwd_timeout(a, abort_flag);
          break;
        }
        const int r = row0 + (t_begin + it) * kBG;
        mbar_arrive_expect_tx(&g_full[st], 2 * kGTile);
        tma_load_2d(sG1 + st * kGTile, &P.tm_qkv_g, &g_full[st], qcol, r);
        tma_load_2d(sG2 + st * kGTile, &P.tm_do_g, &g_full[st], ocol, r);
        ++issued;
      }
      volatile int keep_waiting = 0;   // every copy lands before the CTA can exit
      mbar_wait_bounded(f_full, 0, a.wait_ns, &keep_waiting);
      for (int it = issued > kGStages ? issued - kGStages : 0; it < issued; ++it)
        mbar_wait_bounded(&g_full[it % kGStages], static_cast<uint32_t>(it / kGStages) & 1u,
                          a.wait_ns, &keep_waiting);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one_sync()) {
      constexpr uint32_t idS = idesc_bf16_f32(kBQ, kBG, false, false);   // both K-major
      constexpr uint32_t idA = idesc_bf16_f32(kBQ, kHD, false, true);    // P K-major, G MN-major
      constexpr uint32_t idQ = idesc_bf16_f32(kBQ, kHD, true, true);     // dS MN-major, K MN-major
      bool ok = mbar_wait_bounded(f_full, 0, a.wait_ns, abort_flag);
      bool any = false;
      const uint32_t f1 = smem_u32(sF1), f2 = smem_u32(sF2);
      // X_b = K·Qᵀ (Sᵀ) and Y_b = V·dOᵀ (dPᵀ) of streamed tile it
      auto issue_xy = [&](int it) -> bool {
        const int st = it % kGStages, b = it & 1;
        if (!mbar_wait_bounded(&g_full[st], static_cast<uint32_t>(it / kGStages) & 1u, a.wait_ns,
                               abort_flag) ||
            !mbar_wait_bounded(&x_empty[b], (static_cast<uint32_t>(it >> 1) & 1u) ^ 1u, a.wait_ns,
                               abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t g1 = smem_u32(sG1 + st * kGTile), g2 = smem_u32(sG2 + st * kGTile);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k) {
          tc_mma_bf16(tmem + kTX + b * kBG, smem_desc_sw128(f1 + k * 32, 16, 1024),
                      smem_desc_sw128(g1 + k * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          tc_mma_bf16(tmem + kTY + b * kBG, smem_desc_sw128(f2 + k * 32, 16, 1024),
                      smem_desc_sw128(g2 + k * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
        }
        any = true;
        tc_commit(&x_full[b]);
        return true;
      };
      if (ok && nt > 0) ok = issue_xy(0);
      if (ok && nt > 1) ok = issue_xy(1);
      for (int it = 0; ok && it < nt; ++it) {
        const int st = it % kGStages, b = it & 1;
        // Sᵀ and dPᵀ of tile it+2 as soon as the warpgroup has read those of
        // tile it, ahead of tile it's gradient MMAs: their commit then does
        // not wait for those
        if (it + 2 < nt && !issue_xy(it + 2)) {
          ok = false;
          break;
        }
        if (!mbar_wait_bounded(&pd_full[b], static_cast<uint32_t>(it >> 1) & 1u, a.wait_ns,
                               abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t g1 = smem_u32(sG1 + st * kGTile), g2 = smem_u32(sG2 + st * kGTile);
        const uint32_t pa = smem_u32(sP + b * kPTile);
        const uint32_t da = smem_u32(sDS + (it % kDSBufs) * kPTile);
#pragma unroll
        for (int k = 0; k < kBG / 16; ++k) {   // K = the streamed tile's 64 queries
          const uint32_t acc = (it > 0 || k > 0) ? 1u : 0u;
          // dV += Pᵀ·dO
          tc_mma_bf16(tmem + kTA1, smem_desc_sw128(pa + k * 32, 16, 1024),
                      smem_desc_sw128(g2 + k * 2048, 8192, 1024), idA, acc);
          // dK += dSᵀ·Q
          tc_mma_bf16(tmem + kTA2, smem_desc_sw128(da + k * 32, 16, 1024),
                      smem_desc_sw128(g1 + k * 2048, 8192, 1024), idA, acc);
        }
        if ((it & 1) || it + 1 == nt) {
          // dQ of the pair (tiles it & ~1 and it & ~1 | 1) = dS·K: M = the
          // pair's 128 queries (two MN-major 64-query dS tiles, kPTile apart),
          // K = the 128 keys of this CTA, N = 64 (K tile MN-major)
          const int pr = it >> 1;
          if (!mbar_wait_bounded(&q_empty[pr & 1], (static_cast<uint32_t>(pr >> 1) & 1u) ^ 1u,
                                 a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t qa = smem_u32(sDS + ((2 * pr) % kDSBufs) * kPTile);
#pragma unroll
          for (int k = 0; k < kBQ / 16; ++k)
            tc_mma_bf16(tmem + kTQ + (pr & 1) * kHD, smem_desc_sw128(qa + k * 2048, kPTile, 1024),
                        smem_desc_sw128(f1 + k * 2048, 8192, 1024), idQ, k > 0 ? 1u : 0u);
          tc_commit(&q_full[pr & 1]);
        }
        tc_commit(&pd_empty[b]);
        tc_commit(&g_empty[st]);
      }
      if (!ok) bwd_timeout(a, abort_flag);
      if (any) {
        tc_commit(acc_done);   // completes once every MMA above has
        volatile int keep_waiting = 0;   // and this thread sees them done before teardown
        mbar_wait_bounded(acc_done, 0, a.wait_ns, &keep_waiting);
      } else {
        mbar_arrive(acc_done);
      }
    }
  } else if (warp == kRedWarp) {
    // ------------------------------------------------------------ dQ reduces
    // each pair's staged dQ goes to L2 as two TMA reduce-adds; the buffer is
    // handed back once they have read it (this thread alone waits for that)
    if (elect_one_sync()) {
      for (int pr = 0; pr < npairs; ++pr) {
        if (!mbar_wait_bounded(stage_full, static_cast<uint32_t>(pr) & 1u, a.wait_ns, abort_flag)) {
          bwd_timeout(a, abort_flag);
          break;
        }
        const int y = row0 + (t_begin + 2 * pr) * kBG;
        tma_reduce_add_2d(&P.tm_dq, sStage, head * kHD, y);
        tma_reduce_add_2d(&P.tm_dq, sStage + kStageHalf, head * kHD + 32, y);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(stage_free);
      }
      bulk_wait_group0();              // the reduces have landed
    }
  } else {
    // ------------------------------------------------------------ element-wise
    const int wg = (warp - 2) >> 2;                // warpgroup: streamed tiles wg, wg + 2, ...
    const int qd = warp & 3;
    const int r = qd * 32 + lane;                  // key row = TMEM lane
    const int et = threadIdx.x - 64 - wg * kSoftmaxThreads;   // 0..127 in the warpgroup
    const int kpos = ft * kBQ + r;                 // its position in the sequence
    const int sbase = (batch * a.heads + head) * a.s;
    const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
    const float sl = a.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    uint8_t* prow = sP + wg * kPTile + r * 128;
    bool ok = true;
    // dQ of pair pr (queries of streamed tiles 2pr, 2pr+1 = TMEM lanes): read
    // out and staged as two 128-byte-swizzled fp32 boxes of 32 columns (rows
    // past s as zeros) for the reduce warp.  `in` is the thread's state so
    // far; the answer is uniform across the warp, and a warp that gives up
    // does not arrive, so the reduce warp's bounded wait ends the pair.
    auto drain_pair = [&](int pr, bool in) -> bool {
      // the pair's dQ is in tensor memory and the staging buffer is free
      // once the previous pair's reduce has read it
      if (!__all_sync(0xffffffffu,
                      in &&
                          mbar_wait_bounded(&q_full[pr & 1], static_cast<uint32_t>(pr >> 1) & 1u,
                                            a.wait_ns, abort_flag) &&
                          (pr == 0 || mbar_wait_bounded(stage_free, static_cast<uint32_t>(pr - 1) & 1u,
                                                        a.wait_ns, abort_flag))))
        return false;
      tc_fence_after_sync();
      const bool valid = (t_begin + 2 * pr) * kBG + r < a.s;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t qr[32];
        tmem_ld_32x32b_x32(tmem + lane_off + kTQ + (pr & 1) * kHD + h * 32, qr);
        tc_wait_ld();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 v = valid ? make_float4(__uint_as_float(qr[4 * g]), __uint_as_float(qr[4 * g + 1]),
                                               __uint_as_float(qr[4 * g + 2]), __uint_as_float(qr[4 * g + 3]))
                                 : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          *reinterpret_cast<float4*>(sStage + h * kStageHalf + r * 128 + ((g ^ (r & 7)) << 4)) = v;
        }
      }
      tc_fence_before_sync();
      mbar_arrive(&q_empty[pr & 1]);               // dQ read: the MMA may reuse its columns
      fence_proxy_async_smem();                    // staged dQ visible to the TMA unit
      mbar_arrive(stage_full);
      return true;
    };
    // −lse·log2e and −D of the streamed queries: thread et < 64 loads those of
    // query et of a tile one tile ahead of its use, so the global loads are
    // in flight while the warpgroup works on a tile
    float nl = 0.0f, nd = 0.0f;
    auto fetch_vec = [&](int tile) {   // −lse·log2e and −D
      const int q = (t_begin + tile) * kBG + et;
      nl = q < a.s ? -a.lse[sbase + q] * kLog2e : 0.0f;
      nd = q < a.s ? -a.D[sbase + q] : 0.0f;
    };
    if (et < kBG && wg < nt) fetch_vec(wg);
    for (int it = wg; it < nt; it += 2) {
      const uint32_t use = static_cast<uint32_t>(it >> 1);   // this warpgroup's tile count
      const int t0 = (t_begin + it) * kBG;         // first query of the streamed tile
      const float* vL = vec + ((wg * 2 + (use & 1)) * 2) * kBG;
      const float* vD = vL + kBG;
      if (et < kBG) {
        float* w = vec + ((wg * 2 + (use & 1)) * 2) * kBG;
        w[et] = nl;
        w[kBG + et] = nd;
        if (it + 2 < nt) fetch_vec(it + 2);
      }
      // one barrier per tile that also carries every thread's state, so all
      // 128 threads of the warpgroup leave together and none is left in it
      ok = __all_sync(0xffffffffu, ok);
      if (!named_barrier_and(1 + wg, kSoftmaxThreads, ok)) {
        ok = false;
        break;
      }
      // the warp's lanes agree before the warp-collective tensor-memory
      // loads; a warp that gives up skips the tile's work but still reaches
      // the warpgroup's barriers (the dQ drain's, the next tile's), where
      // the others learn of it
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&x_full[wg], use & 1u, a.wait_ns, abort_flag));
      // this warpgroup's P buffer and dS buffer it % 4 are free once the
      // MMAs issued up to its previous tile (its dV/dK and the dQ of the
      // pair before) have completed
      if (ok)
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&pd_empty[wg], (use & 1u) ^ 1u, a.wait_ns,
                                                       abort_flag));
      if (ok) {
        tc_fence_after_sync();
        uint8_t* drow = sDS + (it % kDSBufs) * kPTile + r * 128;
        // the mask can only cut the tiles that meet the diagonal or the end
        // (of the queries, or of the keys: key rows past s must add nothing
        // to dQ)
        const bool need_mask =
            (a.causal && t0 < ft * kBQ + kBQ) || t0 + kBG > a.s || ft * kBQ + kBQ > a.s;
        // the two 32-column halves one after the other (half the registers
        // in flight); Sᵀ and dPᵀ are released after the second half's loads
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t xr[32], yr[32];
          tmem_ld_32x32b_x32(tmem + lane_off + kTX + wg * kBG + h * 32, xr);
          tmem_ld_32x32b_x32(tmem + lane_off + kTY + wg * kBG + h * 32, yr);
          tc_wait_ld();
          if (h == 1) {
            tc_fence_before_sync();
            mbar_arrive(&x_empty[wg]);           // Sᵀ and dPᵀ read: the MMA may refill them
          }
          if (need_mask)
            bwd_half_rows<true>(xr, yr, vL, vD, sl, t0, kpos, a.s, a.causal, prow, drow, r, h);
          else
            bwd_half_rows<false>(xr, yr, vL, vD, sl, t0, kpos, a.s, a.causal, prow, drow, r, h);
        }
        fence_proxy_async_smem();                // P and dS visible to the tensor core
        mbar_arrive(&pd_full[wg]);
      }
      // the dQ of pair (it − 2 − wg) / 2 when it belongs to this warpgroup:
      // issued after the other warpgroup's tile, it is done by now
      if (it >= 2 + wg && (((it - 2 - wg) >> 1) & 1) == wg)
        ok = drain_pair((it - 2 - wg) >> 1, ok);
    }
    // every thread of the warpgroup agrees on the state, then drains this
    // warpgroup's pairs not drained in the loop
    ok = named_barrier_and(1 + wg, kSoftmaxThreads, __all_sync(0xffffffffu, ok));
    for (int pr = wg; pr < npairs; pr += 2)
      if (2 * pr + 2 + wg >= nt) ok = drain_pair(pr, ok);
    // the accumulated gradients of the key rows: every lane takes part in
    // the warp-collective tensor-memory loads, only rows inside the sequence
    // are stored.  Warpgroup 0 stores dK, warpgroup 1 dV.
    const bool done =
        __all_sync(0xffffffffu, ok && mbar_wait_bounded<true>(acc_done, 0, a.wait_ns, abort_flag));
    if (!done) {
      if (lane == 0) bwd_timeout(a, abort_flag);
    } else {
      tc_fence_after_sync();
      const uint32_t col = wg == 1 ? kTA1 : kTA2;
      const float f = wg == 1 ? 1.0f : a.scale;
      __nv_bfloat16* dst = a.dqkv + static_cast<int64_t>(row0 + kpos) * a.ldq + (wg == 0 ? kcol : vcol);
#pragma unroll 1
      for (int c = 0; c < kHD / 32; ++c) {
        uint32_t rr[32];
        tmem_ld_32x32b_x32(tmem + lane_off + col + c * 32, rr);
        tc_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(rr[8 * g + 0]) * f, __uint_as_float(rr[8 * g + 1]) * f);
          w.y = pack_bf16x2(__uint_as_float(rr[8 * g + 2]) * f, __uint_as_float(rr[8 * g + 3]) * f);
          w.z = pack_bf16x2(__uint_as_float(rr[8 * g + 4]) * f, __uint_as_float(rr[8 * g + 5]) * f);
          w.w = pack_bf16x2(__uint_as_float(rr[8 * g + 6]) * f, __uint_as_float(rr[8 * g + 7]) * f);
          if (kpos < a.s) reinterpret_cast<uint4*>(dst + c * 32)[g] = w;
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

tp_status attention_fwd_launch(const void* QKV, int64_t b, int64_t s, int heads,
                               const int64_t* head_offsets, int N, bool causal, float scale,
                               void* ctx, float* lse, int32_t* dev_status, cudaStream_t stream) {
  if (heads > kMaxHeads) return TP_ERR_UNSUPPORTED;
  AttnParams prm;
  memset(&prm, 0, sizeof(prm));
  AttnArgs& a = prm.a;
  a.b = static_cast<int>(b);
  a.s = static_cast<int>(s);
  a.heads = heads;
  a.nqb = static_cast<int>((s + kBQ - 1) / kBQ);
  a.causal = causal ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.ctx = static_cast<__nv_bfloat16*>(ctx);
  a.ldc = static_cast<int64_t>(heads) * kHD;
  a.lse = lse;
  a.dev_status = dev_status;
  a.wait_ns = wait_limit_ns();
  for (int i = 0; i < N; ++i) {   // shard i: [Q heads | K heads | V heads] from column 3·64·first
    const int first = static_cast<int>(head_offsets[i]);
    const int nh = static_cast<int>(head_offsets[i + 1] - head_offsets[i]);
    for (int hh = 0; hh < nh; ++hh)
      a.head_cols[first + hh] = make_int2(3 * kHD * first + hh * kHD, nh * kHD);
  }
  const uint64_t ncols = static_cast<uint64_t>(3) * heads * kHD;
  if (!make_tmap_bf16_sw128(&prm.tm, QKV, ncols, static_cast<uint64_t>(b * s), ncols, kHD, kBQ) ||
      !make_tmap_bf16_sw128(&prm.tm_kv, QKV, ncols, static_cast<uint64_t>(b * s), ncols, kHD, kFK))
    return TP_ERR_CUDA;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!configured[dev & 63]) {
    // two CTAs per SM: the largest shared-memory carveout
    if (cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kFwdAlloc)) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return TP_ERR_CUDA;
    configured[dev & 63] = true;
  }
  // one CTA per (sequence, head, query tile), the longest causal tiles first
  const int64_t grid = b * heads * a.nqb;
  attn_fwd_kernel<<<static_cast<unsigned>(grid), kFwdThreads, kFwdAlloc, stream>>>(prm);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

size_t attention_bwd_ws_bytes(int64_t b, int64_t s, int heads) {
  // D [b·s·heads] fp32, then the dQ accumulator [b·s, heads·64] fp32
  const size_t d_bytes = (static_cast<size_t>(b * s) * heads * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return d_bytes + static_cast<size_t>(b * s) * heads * kHD * sizeof(float);
}

tp_status attention_bwd_launch(const void* QKV, const void* O, const void* dO, const float* lse,
                               int64_t b, int64_t s, int heads, const int64_t* head_offsets, int N,
                               bool causal, float scale, void* dQKV, void* ws, int32_t* dev_status,
                               cudaStream_t stream) {
  if (heads > kMaxHeads) return TP_ERR_UNSUPPORTED;
  float* D = static_cast<float*>(ws);
  float* dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                           ((static_cast<size_t>(b * s) * heads * sizeof(float) + 255) &
                                            ~static_cast<size_t>(255)));
  {
    const int64_t n = b * s * heads * 8;   // eight lanes per (token, head)
    attn_bwd_prep_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
        static_cast<const uint4*>(O), static_cast<const uint4*>(dO), b * s, heads,
        static_cast<int>(s), D, reinterpret_cast<float4*>(dq_acc));
    note_launches(1);
    if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  }
  AttnBwdParams prm;
  memset(&prm, 0, sizeof(prm));
  AttnBwdArgs& a = prm.a;
  a.b = static_cast<int>(b);
  a.s = static_cast<int>(s);
  a.heads = heads;
  a.nqb = static_cast<int>((s + kBQ - 1) / kBQ);
  a.ng = static_cast<int>((s + kBG - 1) / kBG);
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.lse = lse;
  a.D = D;
  a.dq_acc = dq_acc;
  a.dqkv = static_cast<__nv_bfloat16*>(dQKV);
  a.ldq = static_cast<int64_t>(3) * heads * kHD;
  a.dev_status = dev_status;
  a.wait_ns = wait_limit_ns();
  for (int i = 0; i < N; ++i) {
    const int first = static_cast<int>(head_offsets[i]);
    const int nh = static_cast<int>(head_offsets[i + 1] - head_offsets[i]);
    for (int hh = 0; hh < nh; ++hh)
      a.head_cols[first + hh] = make_int2(3 * kHD * first + hh * kHD, nh * kHD);
  }
  const uint64_t rows = static_cast<uint64_t>(b * s);
  const uint64_t ncols = static_cast<uint64_t>(3) * heads * kHD;
  const uint64_t hcols = static_cast<uint64_t>(heads) * kHD;
  if (!make_tmap_bf16_sw128(&prm.tm_qkv, QKV, ncols, rows, ncols, kHD, kBQ) ||
      !make_tmap_bf16_sw128(&prm.tm_qkv_g, QKV, ncols, rows, ncols, kHD, kBG) ||
      !make_tmap_bf16_sw128(&prm.tm_do_g, dO, hcols, rows, hcols, kHD, kBG) ||
      !make_tmap_f32_sw128(&prm.tm_dq, dq_acc, hcols, rows, hcols, 32, kBQ))
    return TP_ERR_CUDA;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!configured[dev & 63]) {
    if (cudaFuncSetAttribute(attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kBAlloc)) != cudaSuccess)
      return TP_ERR_CUDA;
    configured[dev & 63] = true;
  }
  // one CTA per (sequence, head, key tile), the longest causal tiles first
  const int64_t grid = b * heads * a.nqb;
  attn_bwd_kernel<<<static_cast<unsigned>(grid), kBwdThreads, kBAlloc, stream>>>(prm);
  note_launches(1);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  const int64_t nfin = b * s * heads * 8;
  attn_dq_finish_kernel<<<static_cast<unsigned>((nfin + 255) / 256), 256, 0, stream>>>(a);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

}  // namespace tpl
