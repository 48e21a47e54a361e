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
      if (!mbar_wait_bounded(&o_full[g], static_cast<uint32_t>(jb & 1), a.wait_ns,
                                   abort_flag))
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
      if (!mbar_wait_bounded(&s_full[g], static_cast<uint32_t>(j & 1), a.wait_ns,
                                   abort_flag)) {
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

}  // namespace tpl
