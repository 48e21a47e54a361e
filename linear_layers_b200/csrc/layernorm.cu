// layernorm.cu — sequence-parallel dropout-add-LayerNorm for sm_100a.
//
// The residual step of the transformer layer, computed by each sequence
// shard on its own token rows (LayerNorm and Dropout split along the
// sequence; the parameter gradients are summed over shards):
//
//   hs = residual + keep · (x + bias) / (1 − p)        (bf16, the residual stream)
//   y  = (hs − mean) · rstd · gamma + beta              (bf16)
//
// with the mean and the biased variance of each row over the hidden size.
// keep comes from Philox4x32-10 (Salmon et al., SC 2011), written here from
// its definition: element e = row·h + col uses word e mod 4 of the block at
// counter (e div 4, offset) under key seed, and is kept when the word is at
// least floor(p · 2^32).  The backward regenerates the same words instead of
// storing the mask.
//
// HBM-bound: one 16-byte chunk of 8 elements per access, rows held in
// registers between the reductions.  The LayerNorm statistics are taken
// from hs as stored (bf16), so forward and backward see the same values.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstdlib>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace tpl {

namespace {

constexpr int kLnThreads = 128;            // threads per row (forward) / per block (backward)
constexpr int kLnBwdRows = 8;              // rows per backward block

struct DropoutRng {
  uint32_t rk[10][2];                      // the key of each of the 10 rounds
  uint32_t off_lo, off_hi;
  uint32_t threshold;                      // keep when the word >= threshold
  float inv_keep;                          // 1 / (1 − p)
};

// Philox4x32-10 with the round keys (key + r·(0x9E3779B9, 0xBB67AE85))
// precomputed on the host: per round two 32 x 32 -> 64-bit products and two
// three-way XORs.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const DropoutRng& g) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ g.rk[r][0], static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ g.rk[r][1], static_cast<uint32_t>(p0));
  }
  return c;
}

// Keep bits of the 8 elements starting at element e (e a multiple of 8).
__device__ __forceinline__ uint32_t keep_bits8(const DropoutRng& g, uint64_t e) {
  if (g.threshold == 0) return 0xffu;
  const uint64_t q = e >> 2;
  const uint4 w0 = philox4x32_10(make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32),
                                            g.off_lo, g.off_hi), g);
  const uint4 w1 = philox4x32_10(make_uint4(static_cast<uint32_t>(q + 1),
                                            static_cast<uint32_t>((q + 1) >> 32), g.off_lo, g.off_hi),
                                 g);
  const uint32_t t = g.threshold;
  return (w0.x >= t ? 1u : 0u) | (w0.y >= t ? 2u : 0u) | (w0.z >= t ? 4u : 0u) |
         (w0.w >= t ? 8u : 0u) | (w1.x >= t ? 16u : 0u) | (w1.y >= t ? 32u : 0u) |
         (w1.z >= t ? 64u : 0u) | (w1.w >= t ? 128u : 0u);
}

__device__ __forceinline__ void unpack8(const uint4& w, float (&v)[8]) {
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[2 * q] = __uint_as_float(ww[q] << 16);
    v[2 * q + 1] = __uint_as_float(ww[q] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  return make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
}

// Sum over the block's threads in a fixed order (warp tree, then warps in order).
template <int NV>
__device__ __forceinline__ void block_sum(float (&v)[NV], float (*red)[kLnThreads / 32]) {
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  const int w = threadIdx.x >> 5;
  __syncthreads();   // the previous use of red is finished
  if ((threadIdx.x & 31) == 0)
#pragma unroll
    for (int i = 0; i < NV; ++i) red[i][w] = v[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < kLnThreads / 32; ++q) s += red[i][q];
    v[i] = s;
  }
}

template <int CH>
__global__ void __launch_bounds__(kLnThreads, CH <= 2 ? 8 : 4) sp_ln_fwd_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ bias, const uint4* __restrict__ residual,
    const uint4* __restrict__ gamma, const uint4* __restrict__ beta, int h8, float inv_h, float eps,
    DropoutRng rng, uint4* __restrict__ hs_out, uint4* __restrict__ y_out, float* __restrict__ mean_out,
    float* __restrict__ rstd_out, uint8_t* __restrict__ keep_out) {
  __shared__ float red[2][kLnThreads / 32];
  const int64_t row = blockIdx.x;
  float hv[CH][8];
  float s[1] = {0.0f};
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = threadIdx.x + k * kLnThreads;
    if (c < h8) {
      const int64_t o = row * h8 + c;
      float xv[8], rv[8], bv[8];
      unpack8(__ldcs(x + o), xv);
      unpack8(__ldcs(residual + o), rv);
      if (bias) {
        unpack8(__ldg(bias + c), bv);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) bv[i] = 0.0f;
      }
      const uint32_t kb = keep_bits8(rng, static_cast<uint64_t>(o) * 8);
      float t[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        t[i] = rv[i] + (((kb >> i) & 1u) ? (xv[i] + bv[i]) * rng.inv_keep : 0.0f);
      const uint4 packed = pack8(t);
      __stcs(hs_out + o, packed);
      if (keep_out)
        *reinterpret_cast<uint2*>(keep_out + o * 8) = make_uint2(
            ((kb >> 0) & 1u) | (((kb >> 1) & 1u) << 8) | (((kb >> 2) & 1u) << 16) | (((kb >> 3) & 1u) << 24),
            ((kb >> 4) & 1u) | (((kb >> 5) & 1u) << 8) | (((kb >> 6) & 1u) << 16) | (((kb >> 7) & 1u) << 24));
      unpack8(packed, hv[k]);   // the statistics of hs as stored
#pragma unroll
      for (int i = 0; i < 8; ++i) s[0] += hv[k][i];
    }
  }
  block_sum<1>(s, red);
  const float mean = s[0] * inv_h;
  float q[1] = {0.0f};
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = threadIdx.x + k * kLnThreads;
    if (c < h8)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float d = hv[k][i] - mean;
        q[0] = fmaf(d, d, q[0]);
      }
  }
  block_sum<1>(q, red);
  const float rstd = 1.0f / sqrtf(q[0] * inv_h + eps);
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = threadIdx.x + k * kLnThreads;
    if (c < h8) {
      float gv[8], bv[8], yv[8];
      unpack8(__ldg(gamma + c), gv);
      unpack8(__ldg(beta + c), bv);
#pragma unroll
      for (int i = 0; i < 8; ++i) yv[i] = fmaf((hv[k][i] - mean) * rstd, gv[i], bv[i]);
      __stcs(y_out + row * h8 + c, pack8(yv));
    }
  }
  if (threadIdx.x == 0) {
    mean_out[row] = mean;
    rstd_out[row] = rstd;
  }
}

// Warp-wide sum in a fixed order (xor butterfly: every lane ends with the
// same value).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Forward for rows of up to 32·CH chunks (h <= 2048): one warp per row, four
// rows per block, the row in registers (hs kept packed as bf16 between the
// passes, which is what the statistics are taken of, and unpacked again in
// each) and both reductions by shuffles, so no block barrier stands between
// a row's loads and its stores.
template <int CH>
__global__ void __launch_bounds__(kLnThreads, 5) sp_ln_fwd_warp_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ bias, const uint4* __restrict__ residual,
    const uint4* __restrict__ gamma, const uint4* __restrict__ beta, int64_t M, int h8,
    float inv_h, float eps, DropoutRng rng, uint4* __restrict__ hs_out, uint4* __restrict__ y_out,
    float* __restrict__ mean_out, float* __restrict__ rstd_out, uint8_t* __restrict__ keep_out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (kLnThreads / 32) + (threadIdx.x >> 5);
  if (row >= M) return;   // whole warps only
  uint4 hp[CH];   // hs of the row, packed
  float s = 0.0f;
  // every load of the row first, so that all of them are in flight together
  uint4 xw[CH], rw[CH];
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = lane + 32 * k;
    if (c < h8) {
      xw[k] = __ldcs(x + row * h8 + c);
      rw[k] = __ldcs(residual + row * h8 + c);
    }
  }
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = lane + 32 * k;
    if (c < h8) {
      const int64_t o = row * h8 + c;
      float xv[8], rv[8], bv[8];
      unpack8(xw[k], xv);
      unpack8(rw[k], rv);
      if (bias) {
        unpack8(__ldg(bias + c), bv);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) bv[i] = 0.0f;
      }
      const uint32_t kb = keep_bits8(rng, static_cast<uint64_t>(o) * 8);
      float t[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        t[i] = rv[i] + (((kb >> i) & 1u) ? (xv[i] + bv[i]) * rng.inv_keep : 0.0f);
      const uint4 packed = pack8(t);
      hp[k] = packed;
      __stcs(hs_out + o, packed);
      if (keep_out)
        *reinterpret_cast<uint2*>(keep_out + o * 8) = make_uint2(
            ((kb >> 0) & 1u) | (((kb >> 1) & 1u) << 8) | (((kb >> 2) & 1u) << 16) | (((kb >> 3) & 1u) << 24),
            ((kb >> 4) & 1u) | (((kb >> 5) & 1u) << 8) | (((kb >> 6) & 1u) << 16) | (((kb >> 7) & 1u) << 24));
      float hv[8];
      unpack8(packed, hv);   // the statistics of hs as stored
#pragma unroll
      for (int i = 0; i < 8; ++i) s += hv[i];
    }
  }
  const float mean = warp_sum(s) * inv_h;
  float q = 0.0f;
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    if (lane + 32 * k < h8) {
      float hv[8];
      unpack8(hp[k], hv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float d = hv[i] - mean;
        q = fmaf(d, d, q);
      }
    }
  }
  const float rstd = 1.0f / sqrtf(warp_sum(q) * inv_h + eps);
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = lane + 32 * k;
    if (c < h8) {
      float gv[8], bv[8], yv[8], hv[8];
      unpack8(hp[k], hv);
      unpack8(__ldg(gamma + c), gv);
      unpack8(__ldg(beta + c), bv);
#pragma unroll
      for (int i = 0; i < 8; ++i) yv[i] = fmaf((hv[i] - mean) * rstd, gv[i], bv[i]);
      __stcs(y_out + row * h8 + c, pack8(yv));
    }
  }
  if (lane == 0) {
    mean_out[row] = mean;
    rstd_out[row] = rstd;
  }
}

// Staged forward (rows of up to 2048 elements): persistent CTAs, one per SM,
// each owning a contiguous range of rows.  A row's x and residual reach
// shared memory by bulk copy into one of `slots` row slots; the copies of
// all the slots are issued at the start (at M=4096, h=1600 every row of the
// range), so that every read of the kernel is in flight from its first
// microsecond instead of one wave of warps' worth.  Warp w owns slots
// w, w+W, ...: it waits for a slot's row, computes hs and y from shared
// memory into registers and global memory, and refills the slot with the
// row `slots` further on.  gamma, beta and the bias are copied once per CTA.
// No block barrier after the start; every wait is bounded.
constexpr int kLnMaxSlots = 64;

__device__ __forceinline__ void ln_bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int CH, int W>
__global__ void __launch_bounds__(W * 32, 1) sp_ln_fwd_staged_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ bias, const uint4* __restrict__ residual,
    const uint4* __restrict__ gamma, const uint4* __restrict__ beta, int64_t M, int h8,
    int rows_per_cta, int slots, float inv_h, float eps, DropoutRng rng, uint4* __restrict__ hs_out,
    uint4* __restrict__ y_out, float* __restrict__ mean_out, float* __restrict__ rstd_out,
    uint8_t* __restrict__ keep_out, int32_t* dev_status, uint64_t wait_ns) {
  extern __shared__ __align__(128) unsigned char lsm[];
  __shared__ __align__(8) uint64_t full[kLnMaxSlots];
  __shared__ __align__(8) uint64_t par_bar;
  __shared__ int abort_flag;
  // [gamma | beta | bias] then slots × [x row | residual row], h8 uint4 each
  uint4* sg = reinterpret_cast<uint4*>(lsm);
  uint4* sb = sg + h8;
  uint4* sbias = sb + h8;
  uint4* slot0 = sbias + h8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
  const int64_t left = M - row0;
  const int nrows = left < rows_per_cta ? static_cast<int>(left) : rows_per_cta;
  const uint32_t row_bytes = static_cast<uint32_t>(h8) * 16u;
  if (nrows <= 0) return;   // whole CTA
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&par_bar, 1);
    for (int sl = 0; sl < slots; ++sl) mbar_init(&full[sl], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&par_bar, (bias ? 3u : 2u) * row_bytes);
    ln_bulk_load(sg, gamma, row_bytes, &par_bar);
    ln_bulk_load(sb, beta, row_bytes, &par_bar);
    if (bias) ln_bulk_load(sbias, bias, row_bytes, &par_bar);
  }
  auto fill = [&](int sl, int t) {   // one lane: the CTA's row t into slot sl
    uint4* dst = slot0 + static_cast<size_t>(sl) * 2 * h8;
    const int64_t g = row0 + t;
    mbar_arrive_expect_tx(&full[sl], 2u * row_bytes);
    ln_bulk_load(dst, x + g * h8, row_bytes, &full[sl]);
    ln_bulk_load(dst + h8, residual + g * h8, row_bytes, &full[sl]);
  };
  if (lane == 0)
    for (int sl = warp; sl < slots && sl < nrows; sl += W) fill(sl, sl);
  // wait outcomes are made warp-uniform before the warp's shuffles
  bool ok = __all_sync(0xffffffffu, mbar_wait_bounded<true>(&par_bar, 0u, wait_ns, &abort_flag));
  for (int k = 0; ok; ++k) {
    bool any = false;
    for (int sl = warp; sl < slots; sl += W) {
      const int t = sl + k * slots;
      if (t >= nrows) break;
      any = true;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded<true>(&full[sl], static_cast<uint32_t>(k) & 1u,
                                                           wait_ns, &abort_flag))) {
        ok = false;
        break;
      }
      const uint4* xs = slot0 + static_cast<size_t>(sl) * 2 * h8;
      const uint4* rs = xs + h8;
      const int64_t row = row0 + t;
      // hs of the row as stored (bf16-rounded), kept in fp32 for the two
      // statistics passes and the normalisation; the element arithmetic
      // runs on f32x2 pairs
      float hf[CH][8];
      float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int kk = 0; kk < CH; ++kk) {
        const int c = lane + 32 * kk;
        if (c < h8) {
          const int64_t o = row * h8 + c;
          float xv[8], rv[8], bv[8];
          unpack8(xs[c], xv);
          unpack8(rs[c], rv);
          if (bias) {
            unpack8(sbias[c], bv);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) bv[i] = 0.0f;
          }
          const uint32_t kb = keep_bits8(rng, static_cast<uint64_t>(o) * 8);
          // hs = residual + keep·(x + bias)/(1 − p), one rounding after the product
          float tv[8];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float2 xb = __fadd2_rn(make_float2(xv[i], xv[i + 1]), make_float2(bv[i], bv[i + 1]));
            const float2 sc = make_float2(((kb >> i) & 1u) ? rng.inv_keep : 0.0f,
                                          ((kb >> (i + 1)) & 1u) ? rng.inv_keep : 0.0f);
            const float2 tt = __ffma2_rn(xb, sc, make_float2(rv[i], rv[i + 1]));
            tv[i] = tt.x;
            tv[i + 1] = tt.y;
          }
          const uint4 packed = pack8(tv);
          __stcs(hs_out + o, packed);
          if (keep_out)
            *reinterpret_cast<uint2*>(keep_out + o * 8) = make_uint2(
                ((kb >> 0) & 1u) | (((kb >> 1) & 1u) << 8) | (((kb >> 2) & 1u) << 16) | (((kb >> 3) & 1u) << 24),
                ((kb >> 4) & 1u) | (((kb >> 5) & 1u) << 8) | (((kb >> 6) & 1u) << 16) | (((kb >> 7) & 1u) << 24));
          unpack8(packed, hf[kk]);   // the statistics of hs as stored
#pragma unroll
          for (int i = 0; i < 8; i += 2) s2 = __fadd2_rn(s2, make_float2(hf[kk][i], hf[kk][i + 1]));
        }
      }
      // the slot's row is in registers: refill it with the row `slots` on
      __syncwarp();
      if (lane == 0 && t + slots < nrows) {
        fence_proxy_async_smem();
        fill(sl, t + slots);
      }
      const float mean = warp_sum(s2.x + s2.y) * inv_h;
      const float2 nm2 = make_float2(-mean, -mean);
      float2 q2 = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int kk = 0; kk < CH; ++kk) {
        if (lane + 32 * kk < h8) {
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float2 d = __fadd2_rn(make_float2(hf[kk][i], hf[kk][i + 1]), nm2);
            q2 = __ffma2_rn(d, d, q2);
          }
        }
      }
      const float rstd = 1.0f / sqrtf(warp_sum(q2.x + q2.y) * inv_h + eps);
      const float2 rs2 = make_float2(rstd, rstd);
#pragma unroll
      for (int kk = 0; kk < CH; ++kk) {
        const int c = lane + 32 * kk;
        if (c < h8) {
          float gv[8], bv[8], yv[8];
          unpack8(sg[c], gv);
          unpack8(sb[c], bv);
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float2 xh = __fmul2_rn(__fadd2_rn(make_float2(hf[kk][i], hf[kk][i + 1]), nm2), rs2);
            const float2 yy = __ffma2_rn(xh, make_float2(gv[i], gv[i + 1]), make_float2(bv[i], bv[i + 1]));
            yv[i] = yy.x;
            yv[i + 1] = yy.y;
          }
          __stcs(y_out + row * h8 + c, pack8(yv));
        }
      }
      if (lane == 0) {
        mean_out[row] = mean;
        rstd_out[row] = rstd;
      }
    }
    if (!any) break;
  }
  if (!ok && lane == 0 && dev_status) atomicOr(dev_status, TP_DEVERR_TIMEOUT);
}

// Backward, kLnBwdRows rows per block.  Pass A of a row forms Σ g and
// Σ g·xhat (g = dy·gamma); pass B reads the row again (from L1) and writes
// dresidual = rstd·(g − mean(g) − xhat·mean(g·xhat)) + dhs_in and
// dx = keep·dresidual/(1 − p).  Only the block's column sums of dy·xhat, dy
// and dx stay in registers across rows; they are written as this block's
// partial and summed over blocks in block order afterwards.
template <int CH>
__global__ void __launch_bounds__(kLnThreads, CH == 1 ? 6 : CH == 2 ? 4 : CH == 4 ? 2 : 1) sp_ln_bwd_kernel(
    const uint4* __restrict__ dy, const uint4* __restrict__ dhs_in, const uint4* __restrict__ hs,
    const uint4* __restrict__ gamma, const float* __restrict__ mean, const float* __restrict__ rstd,
    int64_t M, int h8, float inv_h, DropoutRng rng, uint4* __restrict__ dx,
    uint4* __restrict__ dresidual, float* __restrict__ part_gamma, float* __restrict__ part_beta,
    float* __restrict__ part_bias) {
  __shared__ float red[4][kLnThreads / 32];
  float ag[CH][8], ab[CH][8], ax[CH][8];   // this block's column sums
#pragma unroll
  for (int k = 0; k < CH; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) ag[k][i] = ab[k][i] = ax[k][i] = 0.0f;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kLnBwdRows;
  // up to two rows per iteration (RPI): their loads are in flight together
  // and their reductions share one pair of block barriers; the widest rows
  // take one at a time to stay within the registers
  constexpr int RPI = CH <= 4 ? 2 : 1;
  for (int rr = 0; rr < kLnBwdRows; rr += RPI) {
    const int64_t rowA = r0 + rr;
    if (rowA >= M) break;   // uniform across the block
    const int nrows = RPI == 2 && rowA + 1 < M ? 2 : 1;
    float mu[RPI], rs[RPI];
    float sums[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // per row: Σ g, Σ g·xhat
#pragma unroll
    for (int q = 0; q < RPI; ++q) {
      mu[q] = q < nrows ? mean[rowA + q] : 0.0f;
      rs[q] = q < nrows ? rstd[rowA + q] : 0.0f;
    }
    uint4 hw[RPI][CH], dw[RPI][CH];
#pragma unroll
    for (int q = 0; q < RPI; ++q)
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int c = threadIdx.x + k * kLnThreads;
        if (q < nrows && c < h8) {
          hw[q][k] = __ldg(hs + (rowA + q) * h8 + c);
          dw[q][k] = __ldg(dy + (rowA + q) * h8 + c);
        }
      }
#pragma unroll
    for (int q = 0; q < RPI; ++q)
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int c = threadIdx.x + k * kLnThreads;
        if (q < nrows && c < h8) {
          float hv[8], dv[8], gv[8];
          unpack8(hw[q][k], hv);
          unpack8(dw[q][k], dv);
          unpack8(__ldg(gamma + c), gv);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float g = dv[i] * gv[i];
            sums[2 * q] += g;
            sums[2 * q + 1] = fmaf(g, (hv[i] - mu[q]) * rs[q], sums[2 * q + 1]);
          }
        }
      }
    block_sum<2 * RPI>(*reinterpret_cast<float(*)[2 * RPI]>(sums), red);
#pragma unroll
    for (int q = 0; q < RPI; ++q) {
      if (q >= nrows) break;   // uniform
      const int64_t row = rowA + q;
      const float mg = sums[2 * q] * inv_h, mgx = sums[2 * q + 1] * inv_h;
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int c = threadIdx.x + k * kLnThreads;
        if (c < h8) {
          const int64_t o = row * h8 + c;
          float hv[8], dv[8], gv[8], din[8], d[8], dxv[8];
          unpack8(hw[q][k], hv);
          unpack8(dw[q][k], dv);
          unpack8(__ldg(gamma + c), gv);
          if (dhs_in) {
            unpack8(__ldcs(dhs_in + o), din);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) din[i] = 0.0f;
          }
          const uint32_t kb = keep_bits8(rng, static_cast<uint64_t>(o) * 8);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float xh = (hv[i] - mu[q]) * rs[q];
            d[i] = fmaf(rs[q], dv[i] * gv[i] - mg - xh * mgx, din[i]);
            dxv[i] = ((kb >> i) & 1u) ? d[i] * rng.inv_keep : 0.0f;
            ag[k][i] = fmaf(dv[i], xh, ag[k][i]);
            ab[k][i] += dv[i];
            ax[k][i] += dxv[i];
          }
          __stcs(dresidual + o, pack8(d));
          __stcs(dx + o, pack8(dxv));
        }
      }
    }
  }
  const int64_t h = static_cast<int64_t>(h8) * 8;
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = threadIdx.x + k * kLnThreads;
    if (c < h8) {
      float* pg = part_gamma + blockIdx.x * h + c * 8;
      float* pb = part_beta + blockIdx.x * h + c * 8;
      *reinterpret_cast<float4*>(pg) = make_float4(ag[k][0], ag[k][1], ag[k][2], ag[k][3]);
      *reinterpret_cast<float4*>(pg + 4) = make_float4(ag[k][4], ag[k][5], ag[k][6], ag[k][7]);
      *reinterpret_cast<float4*>(pb) = make_float4(ab[k][0], ab[k][1], ab[k][2], ab[k][3]);
      *reinterpret_cast<float4*>(pb + 4) = make_float4(ab[k][4], ab[k][5], ab[k][6], ab[k][7]);
      if (part_bias) {
        float* px = part_bias + blockIdx.x * h + c * 8;
        *reinterpret_cast<float4*>(px) = make_float4(ax[k][0], ax[k][1], ax[k][2], ax[k][3]);
        *reinterpret_cast<float4*>(px + 4) = make_float4(ax[k][4], ax[k][5], ax[k][6], ax[k][7]);
      }
    }
  }
}

// out_p[n] = Σ_t part_p[t, n] for the planes p = blockIdx.y, in a fixed
// order: 32 columns per block, 32 row groups of 32 threads; group q sums
// rows q, q+32, … (four loads in flight), then the 32 group sums are added
// in group order.
struct ColumnSums {
  const float* part[3];
  float* out[3];
};

__global__ void __launch_bounds__(1024) column_sums_kernel(ColumnSums cs, int rows, int n) {
  __shared__ float red[32][33];
  const float* part = cs.part[blockIdx.y];
  const int col = blockIdx.x * 32 + (threadIdx.x & 31);
  const int q = threadIdx.x >> 5;
  float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
  if (col < n) {
    int t = q;
    for (; t + 96 < rows; t += 128) {
      s0 += part[static_cast<int64_t>(t) * n + col];
      s1 += part[static_cast<int64_t>(t + 32) * n + col];
      s2 += part[static_cast<int64_t>(t + 64) * n + col];
      s3 += part[static_cast<int64_t>(t + 96) * n + col];
    }
    for (; t < rows; t += 32) s0 += part[static_cast<int64_t>(t) * n + col];
  }
  red[q][threadIdx.x & 31] = (s0 + s1) + (s2 + s3);
  __syncthreads();
  if (q == 0 && col < n) {
    float s = 0.0f;
#pragma unroll
    for (int g = 0; g < 32; ++g) s += red[g][threadIdx.x];
    cs.out[blockIdx.y][col] = s;
  }
}

DropoutRng make_rng(float p, uint64_t seed, uint64_t offset) {
  DropoutRng g;
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    g.rk[r][0] = k0;
    g.rk[r][1] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  g.off_lo = static_cast<uint32_t>(offset);
  g.off_hi = static_cast<uint32_t>(offset >> 32);
  const double t = std::floor(static_cast<double>(p) * 4294967296.0);
  g.threshold = t >= 4294967295.0 ? 0xffffffffu : static_cast<uint32_t>(t);
  g.inv_keep = static_cast<float>(1.0 / (1.0 - static_cast<double>(p)));
  return g;
}

template <int CH>
tp_status ln_fwd_t(const void* x, const void* bias, const void* residual, const void* gamma,
                   const void* beta, int64_t M, int64_t h, const DropoutRng& g, float eps, void* hs,
                   void* y, float* mean, float* rstd, uint8_t* keep, cudaStream_t stream) {
  sp_ln_fwd_kernel<CH><<<static_cast<unsigned>(M), kLnThreads, 0, stream>>>(
      static_cast<const uint4*>(x), static_cast<const uint4*>(bias),
      static_cast<const uint4*>(residual), static_cast<const uint4*>(gamma),
      static_cast<const uint4*>(beta), static_cast<int>(h / 8), 1.0f / static_cast<float>(h), eps, g,
      static_cast<uint4*>(hs), static_cast<uint4*>(y), mean, rstd, keep);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

template <int CH>
tp_status ln_bwd_t(const void* dy, const void* dhs_in, const void* hs, const void* gamma,
                   const float* mean, const float* rstd, int64_t M, int64_t h, const DropoutRng& g,
                   void* dx, void* dres, float* pg, float* pb, float* px, cudaStream_t stream) {
  const int64_t blocks = (M + kLnBwdRows - 1) / kLnBwdRows;
  sp_ln_bwd_kernel<CH><<<static_cast<unsigned>(blocks), kLnThreads, 0, stream>>>(
      static_cast<const uint4*>(dy), static_cast<const uint4*>(dhs_in),
      static_cast<const uint4*>(hs), static_cast<const uint4*>(gamma), mean, rstd, M,
      static_cast<int>(h / 8), 1.0f / static_cast<float>(h), g, static_cast<uint4*>(dx),
      static_cast<uint4*>(dres), pg, pb, px);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

int chunks_per_thread(int64_t h) {
  const int64_t c = (h / 8 + kLnThreads - 1) / kLnThreads;
  return c <= 1 ? 1 : c <= 2 ? 2 : c <= 4 ? 4 : c <= 8 ? 8 : 0;
}

}  // namespace

size_t sp_ln_bwd_ws_bytes(int64_t M, int64_t h) {
  const size_t blocks = static_cast<size_t>((M + kLnBwdRows - 1) / kLnBwdRows);
  const size_t plane = (blocks * static_cast<size_t>(h) * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return 3 * plane;
}

template <int CH>
tp_status ln_fwd_warp_t(const void* x, const void* bias, const void* residual, const void* gamma,
                        const void* beta, int64_t M, int64_t h, const DropoutRng& g, float eps,
                        void* hs, void* y, float* mean, float* rstd, uint8_t* keep,
                        cudaStream_t stream) {
  constexpr int rows = kLnThreads / 32;
  sp_ln_fwd_warp_kernel<CH><<<static_cast<unsigned>((M + rows - 1) / rows), kLnThreads, 0, stream>>>(
      static_cast<const uint4*>(x), static_cast<const uint4*>(bias),
      static_cast<const uint4*>(residual), static_cast<const uint4*>(gamma),
      static_cast<const uint4*>(beta), M, static_cast<int>(h / 8), 1.0f / static_cast<float>(h), eps,
      g, static_cast<uint4*>(hs), static_cast<uint4*>(y), mean, rstd, keep);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

template <int CH, int W>
tp_status ln_fwd_staged_t(const void* x, const void* bias, const void* residual, const void* gamma,
                          const void* beta, int64_t M, int64_t h, const DropoutRng& g, float eps,
                          void* hs, void* y, float* mean, float* rstd, uint8_t* keep,
                          int32_t* dev_status, cudaStream_t stream) {
  static int max_optin[64] = {0};
  static size_t attr_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (max_optin[dev & 63] == 0 &&
      cudaDeviceGetAttribute(&max_optin[dev & 63], cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
          cudaSuccess)
    return TP_ERR_CUDA;
  const size_t row_bytes = static_cast<size_t>(h / 8) * 16;
  const int sms = num_sms();
  const int64_t rows_per_cta = (M + sms - 1) / sms;
  const int64_t grid = (M + rows_per_cta - 1) / rows_per_cta;
  // shared memory: gamma, beta, bias and the row slots, 1 KB left for the
  // static part (barriers)
  const int64_t budget = static_cast<int64_t>(max_optin[dev & 63]) - 1024 - 3 * static_cast<int64_t>(row_bytes);
  int64_t slots = budget / static_cast<int64_t>(2 * row_bytes);
  if (slots > rows_per_cta) slots = rows_per_cta;
  if (slots > kLnMaxSlots) slots = kLnMaxSlots;
  if (slots < 1) return TP_ERR_UNSUPPORTED;
  const size_t smem = (3 + 2 * static_cast<size_t>(slots)) * row_bytes;
  if (smem > attr_set[dev & 63]) {
    if (cudaFuncSetAttribute(sp_ln_fwd_staged_kernel<CH, W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return TP_ERR_CUDA;
    attr_set[dev & 63] = smem;
  }
  sp_ln_fwd_staged_kernel<CH, W><<<static_cast<unsigned>(grid), W * 32, smem, stream>>>(
      static_cast<const uint4*>(x), static_cast<const uint4*>(bias),
      static_cast<const uint4*>(residual), static_cast<const uint4*>(gamma),
      static_cast<const uint4*>(beta), M, static_cast<int>(h / 8), static_cast<int>(rows_per_cta),
      static_cast<int>(slots), 1.0f / static_cast<float>(h), eps, g, static_cast<uint4*>(hs),
      static_cast<uint4*>(y), mean, rstd, keep, dev_status, wait_limit_ns());
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// TP_LN_FWD_WARP=1 takes the register-only warp-per-row forward instead of
// the staged one (sweeps).
bool ln_fwd_warp_forced() {
  const char* e = std::getenv("TP_LN_FWD_WARP");
  return e && e[0] == '1';
}


tp_status sp_ln_fwd_launch(const void* x, const void* bias, const void* residual, const void* gamma,
                           const void* beta, int64_t M, int64_t h, float p, uint64_t seed,
                           uint64_t offset, float eps, void* hs, void* y, float* mean, float* rstd,
                           uint8_t* keep, int32_t* dev_status, cudaStream_t stream) {
  const DropoutRng g = make_rng(p, seed, offset);
  const int64_t h8 = h / 8;
  if (h8 <= 32 * 8 && !ln_fwd_warp_forced()) {
// 16 warps per CTA: 32 measured slower (and spill at 7 or more chunks)
#define TP_LN_STAGED(C) \
  return ln_fwd_staged_t<C, 16>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, dev_status, stream)
    switch ((h8 + 31) / 32) {
      case 1: TP_LN_STAGED(1);
      case 2: TP_LN_STAGED(2);
      case 3: TP_LN_STAGED(3);
      case 4: TP_LN_STAGED(4);
      case 5: TP_LN_STAGED(5);
      case 6: TP_LN_STAGED(6);
      case 7: TP_LN_STAGED(7);
      default: TP_LN_STAGED(8);
    }
#undef TP_LN_STAGED
  }
  if (h8 <= 32 * 2)
    return ln_fwd_warp_t<2>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, stream);
  if (h8 <= 32 * 4)
    return ln_fwd_warp_t<4>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, stream);
  if (h8 <= 32 * 8)
    return ln_fwd_warp_t<8>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, stream);
  switch (chunks_per_thread(h)) {
    case 1: return ln_fwd_t<1>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, stream);
    case 2: return ln_fwd_t<2>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, stream);
    case 4: return ln_fwd_t<4>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, stream);
    case 8: return ln_fwd_t<8>(x, bias, residual, gamma, beta, M, h, g, eps, hs, y, mean, rstd, keep, stream);
  }
  return TP_ERR_UNSUPPORTED;
}

tp_status sp_ln_bwd_launch(const void* dy, const void* dhs_in, const void* hs, const void* gamma,
                           const float* mean, const float* rstd, int64_t M, int64_t h, float p,
                           uint64_t seed, uint64_t offset, void* dx, void* dres, float* dgamma,
                           float* dbeta, float* dbias, void* ws, cudaStream_t stream) {
  const DropoutRng g = make_rng(p, seed, offset);
  const int blocks = static_cast<int>((M + kLnBwdRows - 1) / kLnBwdRows);
  const size_t plane = sp_ln_bwd_ws_bytes(M, h) / 3;
  float* pg = static_cast<float*>(ws);
  float* pb = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + plane);
  float* px = dbias ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 2 * plane) : nullptr;
  tp_status s;
  switch (chunks_per_thread(h)) {
    case 1: s = ln_bwd_t<1>(dy, dhs_in, hs, gamma, mean, rstd, M, h, g, dx, dres, pg, pb, px, stream); break;
    case 2: s = ln_bwd_t<2>(dy, dhs_in, hs, gamma, mean, rstd, M, h, g, dx, dres, pg, pb, px, stream); break;
    case 4: s = ln_bwd_t<4>(dy, dhs_in, hs, gamma, mean, rstd, M, h, g, dx, dres, pg, pb, px, stream); break;
    case 8: s = ln_bwd_t<8>(dy, dhs_in, hs, gamma, mean, rstd, M, h, g, dx, dres, pg, pb, px, stream); break;
    default: return TP_ERR_UNSUPPORTED;
  }
  if (s) return s;
  // the shards' (blocks') partial parameter gradients summed in block order
  const int hi = static_cast<int>(h);
  ColumnSums cs;
  cs.part[0] = pg; cs.part[1] = pb; cs.part[2] = px;
  cs.out[0] = dgamma; cs.out[1] = dbeta; cs.out[2] = dbias;
  column_sums_kernel<<<dim3(static_cast<unsigned>((hi + 31) / 32), dbias ? 3u : 2u), 1024, 0,
                       stream>>>(cs, blocks, hi);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

}  // namespace tpl
