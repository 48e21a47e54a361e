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
// One CTA computes two 128-query tiles (2p and 2p+1) of one head of one
// sequence, streaming 128-key blocks shared by both (flash-style online
// softmax), in the ping-pong order that keeps the tensor core busy while
// either tile's softmax runs:
//   warp 0    TMA: both Q tiles once, K and V blocks into a two-stage ring;
//   warp 1    owns tensor memory; one lane issues, per tile g, S_g = Q_g·Kᵀ
//             (128 x 128 fp32) and O_g = P_g·V (128 x 64 fp32) with
//             tcgen05.mma: P·V of block j and S of block j+1 for one tile as
//             soon as its softmax has released block j, then the other's;
//   warps 2-5 and 6-9, one warpgroup per tile, one query row per thread (its
//             TMEM lane): row maximum, p = 2^(x − m) in the log2 domain, P
//             as bf16 written into shared memory in the 128-byte-swizzled
//             K-major layout the MMA reads, the running sum, and O
//             accumulated in registers as O = O·2^(m_old − m_new) + O_blk,
//             so O never goes back to tensor memory.
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
constexpr int kBK = 128;                       // keys per block
constexpr int kHD = 64;                        // head dimension: one 128-byte row
constexpr int kAttnThreads = 320;              // 10 warps
constexpr int kSoftmaxThreads = 128;           // one warpgroup per query tile
constexpr int kMaxHeads = 256;
constexpr uint32_t kTile = kBQ * kHD * 2;      // 16 KB: 128 rows of 128 bytes
constexpr uint32_t kOffQ = 0;                          // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTile;          // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;          // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTile;          // per tile: 2 chunks of 64 keys
constexpr uint32_t kPBytes = 2 * kTile;
constexpr uint32_t kOffBar = kOffP + 2 * kPBytes;
constexpr int kNumBars = 18;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kAttnBytes = kOffMisc + 16;
constexpr uint32_t kAttnAlloc = kAttnBytes + 1024;     // slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 512;                    // S: 2 x 128, O_blk: 2 x 64
constexpr uint32_t kTmemO = 256;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnArgs {
  int b, s, heads, nqb, npairs;
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
  CUtensorMap tm;            // QKV [b·s, 3h], boxes of 64 columns x 128 rows
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

// Row maximum of one 128-key block of S (TMEM, this thread's lane), 64
// columns per tensor-memory round trip.  With kMask, keys at positions >=
// klim are left out.
template <bool kMask>
__device__ __forceinline__ float block_row_max(uint32_t sbase, int kpos0, int klim) {
  float acc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
  for (int c = 0; c < kBK / 32; c += 2) {
    uint32_t rr[64];
    tmem_ld_32x32b_x32(sbase + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&rr[0]));
    tmem_ld_32x32b_x32(sbase + c * 32 + 32, *reinterpret_cast<uint32_t(*)[32]>(&rr[32]));
    tc_wait_ld();
    float x[64];
#pragma unroll
    for (int t = 0; t < 64; ++t) {
      x[t] = __uint_as_float(rr[t]);
      if (kMask && kpos0 + c * 32 + t >= klim) x[t] = -INFINITY;
    }
#pragma unroll
    for (int t = 0; t < 64; t += 8) {
      float& a = acc[(t >> 3) & 3];
      a = fmax3(a, x[t], x[t + 1]);
      a = fmax3(a, x[t + 2], x[t + 3]);
      a = fmax3(a, x[t + 4], x[t + 5]);
      a = fmax3(a, x[t + 6], x[t + 7]);
    }
  }
  return fmaxf(fmax3(acc[0], acc[1], acc[2]), acc[3]);
}

// p = 2^(x·sl − m) of one block, stored as bf16 into this row of the P tile
// (two 64-key chunks of 128-byte rows, 16-byte granule g at g ^ (row & 7):
// the 128-byte swizzle the MMA's descriptor names).  One 64-key chunk per
// tensor-memory round trip.  Returns Σ p.
template <bool kMask>
__device__ __forceinline__ float block_exp_store(uint32_t sbase, int kpos0, int klim, float sl,
                                                 float m_use, uint8_t* prow, int r) {
  float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
  for (int h = 0; h < kBK / 64; ++h) {
    uint32_t rr[64];
    tmem_ld_32x32b_x32(sbase + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&rr[0]));
    tmem_ld_32x32b_x32(sbase + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&rr[32]));
    tc_wait_ld();
    float p[64];
#pragma unroll
    for (int t = 0; t < 64; ++t) {
      float x = __uint_as_float(rr[t]);
      if (kMask && kpos0 + h * 64 + t >= klim) x = -INFINITY;
      p[t] = ex2f(fmaf(x, sl, -m_use));
      ps[t & 3] += p[t];
    }
    uint8_t* chunk = prow + h * kTile;
#pragma unroll
    for (int gr = 0; gr < 8; ++gr) {            // 16-byte granule of the 128-byte row
      uint4 w;
      w.x = pack_bf16x2(p[8 * gr + 0], p[8 * gr + 1]);
      w.y = pack_bf16x2(p[8 * gr + 2], p[8 * gr + 3]);
      w.z = pack_bf16x2(p[8 * gr + 4], p[8 * gr + 5]);
      w.w = pack_bf16x2(p[8 * gr + 6], p[8 * gr + 7]);
      *reinterpret_cast<uint4*>(chunk + ((gr ^ (r & 7)) << 4)) = w;
    }
  }
  return (ps[0] + ps[1]) + (ps[2] + ps[3]);
}

__device__ __forceinline__ void attn_timeout(const AttnArgs& a, volatile int* abort_flag) {
  if (!*abort_flag) {
    *abort_flag = 1;
    if (a.dev_status) atomicOr(a.dev_status, TP_DEVERR_TIMEOUT);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const AttnArgs& a = P.a;
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;
  uint8_t* sP = smem + kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;        // [stage]
  uint64_t* kv_empty = bars + 3;       // [stage]
  uint64_t* s_full = bars + 5;         // [tile]
  uint64_t* s_empty = bars + 7;        // [tile]
  uint64_t* p_full = bars + 9;         // [tile]
  uint64_t* p_empty = bars + 11;       // [tile]
  uint64_t* o_full = bars + 13;        // [tile]
  uint64_t* o_empty = bars + 15;       // [tile]
  uint64_t* mma_done = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the pairs of the last query tiles (the longest under the causal mask) first
  const int bh = a.b * a.heads;
  const int pair = a.npairs - 1 - static_cast<int>(blockIdx.x) / bh;
  const int rem = static_cast<int>(blockIdx.x) % bh;
  const int head = rem / a.b;
  const int batch = rem % a.b;
  const int row0 = batch * a.s;                         // first token row of the sequence
  const int nkb_all = (a.s + kBK - 1) / kBK;
  int nkb[2];                                           // key blocks of each tile (0: absent)
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const int qb = 2 * pair + g;
    nkb[g] = qb >= a.nqb ? 0 : (a.causal ? min(qb + 1, nkb_all) : nkb_all);
  }
  const int nkb_max = max(nkb[0], nkb[1]);
  const int qcol = a.head_cols[head].x;
  const int kcol = qcol + a.head_cols[head].y;
  const int vcol = kcol + a.head_cols[head].y;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kSoftmaxThreads);
      mbar_init(&p_full[i], kSoftmaxThreads);
      mbar_init(&p_empty[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], kSoftmaxThreads);
    }
    mbar_init(mma_done, 1);
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
      tma_prefetch_desc(&P.tm);
      mbar_arrive_expect_tx(q_full, nkb[1] > 0 ? 2 * kTile : kTile);
      tma_load_2d(sQ, &P.tm, q_full, qcol, row0 + 2 * pair * kBQ);
      if (nkb[1] > 0) tma_load_2d(sQ + kTile, &P.tm, q_full, qcol, row0 + (2 * pair + 1) * kBQ);
      int issued = 0;
      for (int j = 0; j < nkb_max; ++j) {
        const int st = j & 1;
        const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
        if (!mbar_wait_bounded(&kv_empty[st], ph ^ 1u, a.wait_ns, abort_flag)) {
          attn_timeout(a, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(&kv_full[st], 2 * kTile);
        tma_load_2d(sK + st * kTile, &P.tm, &kv_full[st], kcol, row0 + j * kBK);
        tma_load_2d(sV + st * kTile, &P.tm, &kv_full[st], vcol, row0 + j * kBK);
        ++issued;
      }
      // every copy lands before the CTA can exit (bounded, not cut short by
      // the abort flag): the Q tiles and the last two K/V stages
      volatile int keep_waiting = 0;
      mbar_wait_bounded(q_full, 0, a.wait_ns, &keep_waiting);
      for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j)
        mbar_wait_bounded(&kv_full[j & 1], static_cast<uint32_t>(j >> 1) & 1u, a.wait_ns,
                          &keep_waiting);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one_sync()) {
      constexpr uint32_t idS = idesc_bf16_f32(kBQ, kBK, false, false);   // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16_f32(kBQ, kHD, false, true);    // P K-major, V MN-major
      bool any = false;
      // S_g(j) = Q_g·K_jᵀ into tile g's S buffer, once its softmax has read S_g(j-1)
      auto issue_s = [&](int g, int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait_bounded(&kv_full[st], static_cast<uint32_t>(j >> 1) & 1u, a.wait_ns,
                               abort_flag))
          return false;
        if (!mbar_wait_bounded(&s_empty[g], static_cast<uint32_t>(j & 1) ^ 1u, a.wait_ns,
                               abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t qa = smem_u32(sQ + g * kTile), kb = smem_u32(sK + st * kTile);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)
          tc_mma_bf16(tmem + g * kBK, smem_desc_sw128(qa + k * 32, 16, 1024),
                      smem_desc_sw128(kb + k * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
        any = true;
        tc_commit(&s_full[g]);
        return true;
      };
      // O_g = P_g(j)·V_j, once the softmax has written P_g(j) and taken O_g(j-1)
      auto issue_pv = [&](int g, int j) -> bool {
        const uint32_t ph = static_cast<uint32_t>(j & 1);
        if (!mbar_wait_bounded(&p_full[g], ph, a.wait_ns, abort_flag) ||
            !mbar_wait_bounded(&o_empty[g], ph ^ 1u, a.wait_ns, abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t pa = smem_u32(sP + g * kPBytes), vb = smem_u32(sV + (j & 1) * kTile);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)   // 16 keys per step; chunk of 64 keys = 16 KB
          tc_mma_bf16(tmem + kTmemO + g * kHD,
                      smem_desc_sw128(pa + (k >> 2) * kTile + (k & 3) * 32, 16, 1024),
                      smem_desc_sw128(vb + k * 2048, 8192, 1024), idO, k > 0 ? 1u : 0u);
        tc_commit(&o_full[g]);
        tc_commit(&p_empty[g]);
        return true;
      };
      bool ok = mbar_wait_bounded(q_full, 0, a.wait_ns, abort_flag);
      for (int g = 0; ok && g < 2; ++g)
        if (nkb[g] > 0) ok = issue_s(g, 0);
      for (int j = 0; ok && j < nkb_max; ++j) {
        for (int g = 0; ok && g < 2; ++g) {
          if (j >= nkb[g]) continue;
          ok = issue_pv(g, j);
          if (ok && j + 1 < nkb[g]) ok = issue_s(g, j + 1);
        }
        if (ok) tc_commit(&kv_empty[j & 1]);   // K_j and V_j read by every MMA issued so far
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
    const int g = (warp - 2) >> 2;                  // query tile of this warpgroup
    const int qd = warp & 3;                        // TMEM lane quadrant of this warp
    const int r = qd * 32 + lane;                   // row of the query tile
    const int qb = 2 * pair + g;
    const int qpos = qb * kBQ + r;                  // position in the sequence
    const int nk = nkb[g];
    const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t sbase = tmem + lane_off + static_cast<uint32_t>(g * kBK);
    const uint32_t obase = tmem + lane_off + kTmemO + static_cast<uint32_t>(g * kHD);
    uint8_t* prow = sP + g * kPBytes + r * 128;
    const float sl = a.scale_log2;
    const int klim = a.causal ? min(qpos + 1, a.s) : a.s;   // keys [0, klim) are visible
    float m = -INFINITY;                            // running maximum (log2 units)
    float l = 0.0f;                                 // running sum of 2^(x − m)
    float alpha_prev = 1.0f;
    float o[kHD];
#pragma unroll
    for (int i = 0; i < kHD; ++i) o[i] = 0.0f;
    bool ok = true;
    // O = O·2^(m_{j-2} − m_{j-1}) + P_{j-1}·V_{j-1}
    auto take_o = [&](int jb) -> bool {
      // the warp's lanes agree before the warp-collective tensor-memory loads
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&o_full[g], static_cast<uint32_t>(jb & 1),
                                                     a.wait_ns, abort_flag)))
        return false;
      tc_fence_after_sync();
#pragma unroll
      for (int c = 0; c < kHD / 32; ++c) {
        uint32_t rr[32];
        tmem_ld_32x32b_x32(obase + c * 32, rr);
        tc_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) o[c * 32 + t] = fmaf(o[c * 32 + t], alpha_prev, __uint_as_float(rr[t]));
      }
      tc_fence_before_sync();
      mbar_arrive(&o_empty[g]);
      return true;
    };
    for (int j = 0; j < nk; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[g], static_cast<uint32_t>(j & 1),
                                                     a.wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const int kpos0 = j * kBK;
      const bool need_mask = (a.causal && j == qb) || kpos0 + kBK > a.s;
      // pass 1: the row maximum of this block (the mask only where it cuts)
      const float mx = need_mask ? block_row_max<true>(sbase, kpos0, klim)
                                 : block_row_max<false>(sbase, kpos0, klim);
      const float m_new = fmaxf(m, mx * sl);
      const float m_use = m_new == -INFINITY ? 0.0f : m_new;
      const float alpha_j = ex2f(m - m_use);        // 0 before the first block
      // block j-1's P·V has finished (O taken, P buffer free) before P_j is written
      if (j >= 1 && !take_o(j - 1)) {
        ok = false;
        break;
      }
      alpha_prev = alpha_j;
      // pass 2: p = 2^(x·sl − m), bf16 into the swizzled P tile, row sum
      const float rs = need_mask ? block_exp_store<true>(sbase, kpos0, klim, sl, m_use, prow, r)
                                 : block_exp_store<false>(sbase, kpos0, klim, sl, m_use, prow, r);
      tc_fence_before_sync();
      mbar_arrive(&s_empty[g]);                    // S buffer read out
      fence_proxy_async_smem();                    // P visible to the tensor core
      mbar_arrive(&p_full[g]);
      l = fmaf(l, alpha_j, rs);
      m = m_new;
    }
    if (ok && nk > 0) ok = take_o(nk - 1);
    if (!ok) {
      if (lane == 0) attn_timeout(a, abort_flag);
    } else if (nk > 0 && qpos < a.s) {
      const float inv = 1.0f / l;
      __nv_bfloat16* dst = a.ctx + static_cast<int64_t>(row0 + qpos) * a.ldc + head * kHD;
#pragma unroll
      for (int gr = 0; gr < kHD / 8; ++gr) {
        uint4 w;
        w.x = pack_bf16x2(o[8 * gr + 0] * inv, o[8 * gr + 1] * inv);
        w.y = pack_bf16x2(o[8 * gr + 2] * inv, o[8 * gr + 3] * inv);
        w.z = pack_bf16x2(o[8 * gr + 4] * inv, o[8 * gr + 5] * inv);
        w.w = pack_bf16x2(o[8 * gr + 6] * inv, o[8 * gr + 7] * inv);
        reinterpret_cast<uint4*>(dst)[gr] = w;
      }
      if (a.lse)
        a.lse[(static_cast<int64_t>(batch) * a.heads + head) * a.s + qpos] = m * kLn2 + logf(l);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}


// ===========================================================================
// Backward.  D = rowsum(dO ⊙ O) first; then two kernels of one template:
//   kKV = true   one CTA per 128-key tile of a head: streams the query tiles,
//                Sᵀ = K·Qᵀ and dPᵀ = V·dOᵀ in tensor memory, Pᵀ = exp(Sᵀ·scale
//                − lse) and dSᵀ = Pᵀ ⊙ (dPᵀ − D) per key row, then
//                dV += Pᵀ·dO and dK += dSᵀ·Q accumulated in tensor memory;
//   kKV = false  one CTA per 128-query tile: streams the key tiles, S, dP,
//                P, dS the same way per query row, dQ += dS·K.
// Each gradient row is produced by exactly one CTA, so there are no atomics
// and the result does not depend on timing.  dQ and dK carry the scale.
// ===========================================================================
constexpr int kBwdThreads = 192;                       // 6 warps
constexpr uint32_t kBOffF1 = 0;                        // fixed tiles (K, V) or (Q, dO)
constexpr uint32_t kBOffF2 = kTile;
constexpr uint32_t kBOffG1 = 2 * kTile;                // streamed tiles, 2 stages each
constexpr uint32_t kBOffG2 = kBOffG1 + 2 * kTile;
constexpr uint32_t kBOffP = kBOffG2 + 2 * kTile;       // P (or Pᵀ) bf16: 2 chunks of 64
constexpr uint32_t kBOffDS = kBOffP + 2 * kTile;       // dS (or dSᵀ) bf16
constexpr uint32_t kBOffVec = kBOffDS + 2 * kTile;     // per-column lse·log2e and D, 2 stages
constexpr uint32_t kBOffBar = kBOffVec + 2 * 2 * kBQ * 4;
constexpr int kBNumBars = 10;
constexpr uint32_t kBOffMisc = kBOffBar + kBNumBars * 8;
constexpr uint32_t kBAlloc = kBOffMisc + 16 + 1024;
constexpr uint32_t kTX = 0, kTY = 128, kTA1 = 256, kTA2 = 320;   // tensor memory columns

struct AttnBwdArgs {
  int b, s, heads, nqb;
  int causal;
  float scale, scale_log2;
  const float* lse;          // [b, heads, s] natural log
  const float* D;            // [b, heads, s]
  __nv_bfloat16* dqkv;       // [b·s, 3h], the QKV layout
  int64_t ldq;               // 3h
  int32_t* dev_status;
  uint64_t wait_ns;
  int2 head_cols[kMaxHeads];
};

struct __align__(64) AttnBwdParams {
  CUtensorMap tm_qkv;        // QKV [b·s, 3h], boxes of 64 columns x 128 rows
  CUtensorMap tm_do;         // dO  [b·s, h],  boxes of 64 columns x 128 rows
  AttnBwdArgs a;
};

__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const uint4* __restrict__ O,
                                                            const uint4* __restrict__ dO,
                                                            int64_t rows, int heads, int s,
                                                            float* __restrict__ D) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;   // (row, head)
  if (i >= rows * heads) return;
  const int64_t row = i / heads;
  const int head = static_cast<int>(i - row * heads);
  const uint4* o = O + (row * heads + head) * 8;     // 64 bf16 of this head
  const uint4* g = dO + (row * heads + head) * 8;
  float acc = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 a = __ldg(o + k), c = __ldg(g + k);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc = fmaf(__uint_as_float(aw[q] << 16), __uint_as_float(cw[q] << 16), acc);
      acc = fmaf(__uint_as_float(aw[q] & 0xffff0000u), __uint_as_float(cw[q] & 0xffff0000u), acc);
    }
  }
  const int64_t bb = row / s, pos = row - bb * s;
  D[(bb * heads + head) * s + pos] = acc;
}

__device__ __forceinline__ void bwd_timeout(const AttnBwdArgs& a, volatile int* abort_flag) {
  if (!*abort_flag) {
    *abort_flag = 1;
    if (a.dev_status) atomicOr(a.dev_status, TP_DEVERR_TIMEOUT);
  }
}

template <bool kKV>
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
  float* vecL = reinterpret_cast<float*>(smem + kBOffVec);   // [2][128]
  float* vecD = vecL + 2 * kBQ;                               // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBOffBar);
  uint64_t* f_full = bars;
  uint64_t* g_full = bars + 1;       // [stage]
  uint64_t* g_empty = bars + 3;      // [stage]
  uint64_t* xy_full = bars + 5;
  uint64_t* xy_empty = bars + 6;
  uint64_t* pd_full = bars + 7;
  uint64_t* pd_empty = bars + 8;
  uint64_t* acc_done = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = a.b * a.heads;
  // fixed tile, longest first: under the causal mask key tile t streams the
  // query tiles t.., query tile t the key tiles ..t
  const int ft = kKV ? static_cast<int>(blockIdx.x) / bh
                     : a.nqb - 1 - static_cast<int>(blockIdx.x) / bh;
  const int rem = static_cast<int>(blockIdx.x) % bh;
  const int head = rem / a.b;
  const int batch = rem % a.b;
  const int row0 = batch * a.s;
  // streamed tiles: queries t >= ft (kKV) or keys t <= ft (dQ) under the causal mask
  const int t_begin = (kKV && a.causal) ? ft : 0;
  const int t_end = (!kKV && a.causal) ? ft + 1 : a.nqb;
  const int nt = t_end - t_begin;
  const int qcol = a.head_cols[head].x;
  const int kcol = qcol + a.head_cols[head].y;
  const int vcol = kcol + a.head_cols[head].y;
  const int ocol = head * kHD;                         // this head's columns of dO
  // fixed pair: (K, V) or (Q, dO); streamed pair: (Q, dO) or (K, V)
  const int f1col = kKV ? kcol : qcol, f2col = kKV ? vcol : ocol;
  const int g1col = kKV ? qcol : kcol, g2col = kKV ? ocol : vcol;
  const CUtensorMap* f2map = kKV ? &P.tm_qkv : &P.tm_do;
  const CUtensorMap* g2map = kKV ? &P.tm_do : &P.tm_qkv;

  if (threadIdx.x == 0) {
    mbar_init(f_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&g_full[i], 1);
      mbar_init(&g_empty[i], 1);
    }
    mbar_init(xy_full, 1);
    mbar_init(xy_empty, kSoftmaxThreads);
    mbar_init(pd_full, kSoftmaxThreads);
    mbar_init(pd_empty, 1);
    mbar_init(acc_done, 1);
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
      tma_prefetch_desc(&P.tm_do);
      mbar_arrive_expect_tx(f_full, 2 * kTile);
      tma_load_2d(sF1, &P.tm_qkv, f_full, f1col, row0 + ft * kBQ);
      tma_load_2d(sF2, f2map, f_full, f2col, row0 + ft * kBQ);
      int issued = 0;
      for (int it = 0; it < nt; ++it) {
        const int st = it & 1;
        if (!mbar_wait_bounded(&g_empty[st], (static_cast<uint32_t>(it >> 1) & 1u) ^ 1u, a.wait_ns,
                               abort_flag)) {
          bwd_timeout(a, abort_flag);
          break;
        }
        const int r = row0 + (t_begin + it) * kBQ;
        mbar_arrive_expect_tx(&g_full[st], 2 * kTile);
        tma_load_2d(sG1 + st * kTile, &P.tm_qkv, &g_full[st], g1col, r);
        tma_load_2d(sG2 + st * kTile, g2map, &g_full[st], g2col, r);
        ++issued;
      }
      volatile int keep_waiting = 0;   // every copy lands before the CTA can exit
      mbar_wait_bounded(f_full, 0, a.wait_ns, &keep_waiting);
      for (int it = issued > 2 ? issued - 2 : 0; it < issued; ++it)
        mbar_wait_bounded(&g_full[it & 1], static_cast<uint32_t>(it >> 1) & 1u, a.wait_ns,
                          &keep_waiting);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one_sync()) {
      constexpr uint32_t idS = idesc_bf16_f32(kBQ, kBQ, false, false);   // both K-major
      constexpr uint32_t idA = idesc_bf16_f32(kBQ, kHD, false, true);    // P K-major, G MN-major
      bool ok = mbar_wait_bounded(f_full, 0, a.wait_ns, abort_flag);
      bool any = false;
      const uint32_t f1 = smem_u32(sF1), f2 = smem_u32(sF2);
      const uint32_t pa = smem_u32(sP), da = smem_u32(sDS);
      for (int it = 0; ok && it < nt; ++it) {
        const int st = it & 1;
        const uint32_t ph = static_cast<uint32_t>(it & 1);
        if (!mbar_wait_bounded(&g_full[st], static_cast<uint32_t>(it >> 1) & 1u, a.wait_ns, abort_flag) ||
            !mbar_wait_bounded(xy_empty, ph ^ 1u, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t g1 = smem_u32(sG1 + st * kTile), g2 = smem_u32(sG2 + st * kTile);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k) {
          tc_mma_bf16(tmem + kTX, smem_desc_sw128(f1 + k * 32, 16, 1024),
                      smem_desc_sw128(g1 + k * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          tc_mma_bf16(tmem + kTY, smem_desc_sw128(f2 + k * 32, 16, 1024),
                      smem_desc_sw128(g2 + k * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
        }
        any = true;
        tc_commit(xy_full);
        if (!mbar_wait_bounded(pd_full, ph, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
#pragma unroll
        for (int k = 0; k < kBQ / 16; ++k) {   // K = the streamed tile's 128 rows
          const uint32_t acc = (it > 0 || k > 0) ? 1u : 0u;
          const uint32_t off = (k >> 2) * kTile + (k & 3) * 32;
          if constexpr (kKV)   // dV += Pᵀ·dO
            tc_mma_bf16(tmem + kTA1, smem_desc_sw128(pa + off, 16, 1024),
                        smem_desc_sw128(g2 + k * 2048, 8192, 1024), idA, acc);
          // dK += dSᵀ·Q  or  dQ += dS·K
          tc_mma_bf16(tmem + kTA2, smem_desc_sw128(da + off, 16, 1024),
                      smem_desc_sw128(g1 + k * 2048, 8192, 1024), idA, acc);
        }
        tc_commit(pd_empty);
        tc_commit(&g_empty[st]);
      }
      if (!ok) bwd_timeout(a, abort_flag);
      if (any) tc_commit(acc_done);   // completes once every MMA above has
      if (!any) mbar_arrive(acc_done);
    }
  } else {
    // ------------------------------------------------------------ element-wise
    const int qd = warp & 3;
    const int r = qd * 32 + lane;                  // fixed row = TMEM lane
    const int fpos = ft * kBQ + r;                 // its position in the sequence
    const int sbase = (batch * a.heads + head) * a.s;
    const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
    const float sl = a.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    // the fixed row's own lse and D (dQ kernel)
    const float own_l = (!kKV && fpos < a.s) ? a.lse[sbase + fpos] * kLog2e : 0.0f;
    const float own_d = (!kKV && fpos < a.s) ? a.D[sbase + fpos] : 0.0f;
    uint8_t* prow = sP + r * 128;
    uint8_t* drow = sDS + r * 128;
    const int et = threadIdx.x - 64;               // 0..127
    bool ok = true;
    for (int it = 0; it < nt; ++it) {
      const int st = it & 1;
      const uint32_t ph = static_cast<uint32_t>(it & 1);
      const int t0 = (t_begin + it) * kBQ;         // first position of the streamed tile
      if constexpr (kKV) {   // lse·log2e and D of the streamed queries, one per thread
        const int q = t0 + et;
        vecL[st * kBQ + et] = q < a.s ? a.lse[sbase + q] * kLog2e : 0.0f;
        vecD[st * kBQ + et] = q < a.s ? a.D[sbase + q] : 0.0f;
        // one barrier per tile that also carries every thread's state, so all
        // 128 threads leave together and none is left waiting in it
        ok = __all_sync(0xffffffffu, ok);          // the warp converged for the aligned barrier
        if (!named_barrier_and(1, kSoftmaxThreads, ok)) {
          ok = false;
          break;
        }
      }
      // the warp's lanes agree before the warp-collective tensor-memory loads
      const bool got = __all_sync(0xffffffffu,
                                  mbar_wait_bounded(xy_full, ph, a.wait_ns, abort_flag) &&
                                      mbar_wait_bounded(pd_empty, ph ^ 1u, a.wait_ns, abort_flag));
      if (!got) {
        ok = false;
        if constexpr (kKV) continue;   // leave at the next tile's barrier, with the others
        break;
      }
      tc_fence_after_sync();
      // the mask can only cut the diagonal tile and the tile past the end
      const bool need_mask = (a.causal && t_begin + it == ft) || t0 + kBQ > a.s;
#pragma unroll 1
      for (int c = 0; c < kBQ / 32; ++c) {
        uint32_t xr[32], yr[32];
        tmem_ld_32x32b_x32(tmem + lane_off + kTX + c * 32, xr);
        tmem_ld_32x32b_x32(tmem + lane_off + kTY + c * 32, yr);
        float lv[32], dv[32];   // per-column lse·log2e and D (the streamed queries)
        if constexpr (kKV) {
          const float4* l4 = reinterpret_cast<const float4*>(vecL + st * kBQ + c * 32);
          const float4* d4 = reinterpret_cast<const float4*>(vecD + st * kBQ + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 u = l4[q], w = d4[q];
            lv[4 * q] = u.x; lv[4 * q + 1] = u.y; lv[4 * q + 2] = u.z; lv[4 * q + 3] = u.w;
            dv[4 * q] = w.x; dv[4 * q + 1] = w.y; dv[4 * q + 2] = w.z; dv[4 * q + 3] = w.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            lv[j] = own_l;
            dv[j] = own_d;
          }
        }
        tc_wait_ld();
        float p[32], ds[32];
        if (need_mask) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tpos = t0 + c * 32 + j;      // streamed position of this column
            // rows are keys and columns queries (kKV), or the other way round
            const bool masked = tpos >= a.s || (a.causal && (kKV ? tpos < fpos : tpos > fpos));
            p[j] = masked ? 0.0f : ex2f(fmaf(__uint_as_float(xr[j]), sl, -lv[j]));
            ds[j] = p[j] * (__uint_as_float(yr[j]) - dv[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            p[j] = ex2f(fmaf(__uint_as_float(xr[j]), sl, -lv[j]));
            ds[j] = p[j] * (__uint_as_float(yr[j]) - dv[j]);
          }
        }
        uint8_t* pch = prow + (c >> 1) * kTile;
        uint8_t* dch = drow + (c >> 1) * kTile;
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          const int gr = (c & 1) * 4 + g4;
          uint4 w;
          w.x = pack_bf16x2(p[8 * g4 + 0], p[8 * g4 + 1]);
          w.y = pack_bf16x2(p[8 * g4 + 2], p[8 * g4 + 3]);
          w.z = pack_bf16x2(p[8 * g4 + 4], p[8 * g4 + 5]);
          w.w = pack_bf16x2(p[8 * g4 + 6], p[8 * g4 + 7]);
          *reinterpret_cast<uint4*>(pch + ((gr ^ (r & 7)) << 4)) = w;
          w.x = pack_bf16x2(ds[8 * g4 + 0], ds[8 * g4 + 1]);
          w.y = pack_bf16x2(ds[8 * g4 + 2], ds[8 * g4 + 3]);
          w.z = pack_bf16x2(ds[8 * g4 + 4], ds[8 * g4 + 5]);
          w.w = pack_bf16x2(ds[8 * g4 + 6], ds[8 * g4 + 7]);
          *reinterpret_cast<uint4*>(dch + ((gr ^ (r & 7)) << 4)) = w;
        }
      }
      tc_fence_before_sync();
      mbar_arrive(xy_empty);
      fence_proxy_async_smem();
      mbar_arrive(pd_full);
    }
    // the accumulated gradients of the fixed rows: every lane takes part in
    // the warp-collective tensor-memory loads, only rows inside the sequence
    // are stored
    const bool done =
        __all_sync(0xffffffffu, ok && mbar_wait_bounded<true>(acc_done, 0, a.wait_ns, abort_flag));
    if (!done) {
      if (lane == 0) bwd_timeout(a, abort_flag);
    } else {
      tc_fence_after_sync();
      __nv_bfloat16* dst_row = a.dqkv + static_cast<int64_t>(row0 + fpos) * a.ldq;
#pragma unroll
      for (int which = 0; which < (kKV ? 2 : 1); ++which) {
        // kKV: which 0 -> dK (scaled, acc2), which 1 -> dV (acc1); else dQ (scaled, acc2)
        const uint32_t col = which == 0 ? kTA2 : kTA1;
        const float f = which == 0 ? a.scale : 1.0f;
        __nv_bfloat16* dst = dst_row + (kKV ? (which == 0 ? kcol : vcol) : qcol);
#pragma unroll
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
            if (fpos < a.s) reinterpret_cast<uint4*>(dst + c * 32)[g] = w;
          }
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

template <bool kKV>
tp_status attn_bwd_launch_t(const AttnBwdParams& prm, int64_t grid, cudaStream_t stream) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!configured[dev & 63]) {
    if (cudaFuncSetAttribute(attn_bwd_kernel<kKV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kBAlloc)) != cudaSuccess)
      return TP_ERR_CUDA;
    configured[dev & 63] = true;
  }
  attn_bwd_kernel<kKV><<<static_cast<unsigned>(grid), kBwdThreads, kBAlloc, stream>>>(prm);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
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
  a.npairs = (a.nqb + 1) / 2;
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
  if (!make_tmap_bf16_sw128(&prm.tm, QKV, ncols, static_cast<uint64_t>(b * s), ncols, kHD, kBQ))
    return TP_ERR_CUDA;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!configured[dev & 63]) {
    if (cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kAttnAlloc)) != cudaSuccess)
      return TP_ERR_CUDA;
    configured[dev & 63] = true;
  }
  const int64_t grid = b * heads * a.npairs;
  attn_fwd_kernel<<<static_cast<unsigned>(grid), kAttnThreads, kAttnAlloc, stream>>>(prm);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

size_t attention_bwd_ws_bytes(int64_t b, int64_t s, int heads) {
  return (static_cast<size_t>(b * s) * heads * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

tp_status attention_bwd_launch(const void* QKV, const void* O, const void* dO, const float* lse,
                               int64_t b, int64_t s, int heads, const int64_t* head_offsets, int N,
                               bool causal, float scale, void* dQKV, void* ws, int32_t* dev_status,
                               cudaStream_t stream) {
  if (heads > kMaxHeads) return TP_ERR_UNSUPPORTED;
  float* D = static_cast<float*>(ws);
  {
    const int64_t n = b * s * heads;
    attn_bwd_prep_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
        static_cast<const uint4*>(O), static_cast<const uint4*>(dO), b * s, heads,
        static_cast<int>(s), D);
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
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.lse = lse;
  a.D = D;
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
  if (!make_tmap_bf16_sw128(&prm.tm_qkv, QKV, ncols, rows, ncols, kHD, kBQ)) return TP_ERR_CUDA;
  const uint64_t hcols = static_cast<uint64_t>(heads) * kHD;
  if (!make_tmap_bf16_sw128(&prm.tm_do, dO, hcols, rows, hcols, kHD, kBQ)) return TP_ERR_CUDA;
  const int64_t grid = b * heads * a.nqb;
  if (tp_status st = attn_bwd_launch_t<true>(prm, grid, stream)) return st;
  return attn_bwd_launch_t<false>(prm, grid, stream);
}

}  // namespace tpl
