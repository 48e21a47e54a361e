// vocab.cu — vocabulary-parallel embedding and softmax cross-entropy.
//
// Embedding (tensor-model-parallel illustrated, m.youleyou.com, §4.1
// 输入层Embedding): the table is split into N contiguous vocabulary ranges;
// each shard returns its rows for the ids it owns and zeros elsewhere, then
// the shards' outputs are summed.  Exactly one shard owns an in-range id, so
// the kernel forms the sum by routing every token to its owner shard and
// copying that shard's row with 16-byte vector loads and stores, one warp per
// token row.  Out-of-range ids give zero rows and raise TP_DEVERR_RANGE.
//
// Cross-entropy (same page, §5 Cross-Entropy层): instead of gathering the
// [T, v] logits, every shard reduces its own vocabulary range and only
// per-row scalars cross shards.  Here the N shards of one token are the N
// CTAs of a thread-block cluster: each CTA stages its slice of the row in
// shared memory (one HBM read), reduces max / sum-exp / arg-max with warp
// shuffles, publishes (m_i, s_i, target logit, arg-max) in shared memory,
// and after a cluster barrier reads the other shards' scalars through
// distributed shared memory — the on-chip form of the all-reduce.  Each CTA
// then writes its block of dlogits (one HBM write).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace tpl {
namespace {

// ---------------------------------------------------------------------------
// embedding
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(uint4* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

constexpr int kEmbedWarps = 8;
constexpr int kEmbedUnroll = 8;

// out[t] = E_i[id_t - lo_i] for the owner shard i of id_t; zero row if none.
__global__ void __launch_bounds__(kEmbedWarps * 32)
    vp_embed_kernel(const int64_t* __restrict__ ids, int64_t T, const uint4* __restrict__ E,
                    int64_t v, int64_t vec_per_row, int64_t shard_rows, uint4* __restrict__ out,
                    int32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kEmbedWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int64_t id = __ldg(ids + t);
  uint4* dst = out + t * vec_per_row;
  if (id < 0 || id >= v) {
    if (lane == 0 && dev_status) atomicOr(dev_status, TP_DEVERR_RANGE);
    for (int64_t j = lane; j < vec_per_row; j += 32) st_stream(dst + j, make_uint4(0, 0, 0, 0));
    return;
  }
  const int64_t shard = id / shard_rows;           // owner of this id
  const int64_t local = id - shard * shard_rows;   // row inside the owner's range
  const uint4* src = E + (shard * shard_rows + local) * vec_per_row;
  int64_t j = lane;
  for (; j + 32 * (kEmbedUnroll - 1) < vec_per_row; j += 32 * kEmbedUnroll) {
    uint4 r[kEmbedUnroll];
#pragma unroll
    for (int u = 0; u < kEmbedUnroll; ++u) r[u] = ld_stream(src + j + 32 * u);
#pragma unroll
    for (int u = 0; u < kEmbedUnroll; ++u) st_stream(dst + j + 32 * u, r[u]);
  }
  for (; j < vec_per_row; j += 32) st_stream(dst + j, ld_stream(src + j));
}

// ---------------------------------------------------------------------------
// cross-entropy
// ---------------------------------------------------------------------------
constexpr int kXentThreads = 256;          // row-wise fallback
constexpr int kXentClusterThreads = 128;   // per CTA of the cluster kernel




// 1-D bulk copy global -> this CTA's shared memory, completion counted in
// bytes on `bar` (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// (value, index) max with ties to the lower index
__device__ __forceinline__ void argmax_merge(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

__device__ __forceinline__ void block_argmax(float& v, int& i, float* sv, int* si) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, v, off);
    const int i2 = __shfl_xor_sync(0xffffffffu, i, off);
    argmax_merge(v, i, v2, i2);
  }
  if (lane == 0) {
    sv[warp] = v;
    si[warp] = i;
  }
  __syncthreads();
  v = sv[0];
  i = si[0];
  for (int w = 1; w < kXentThreads / 32; ++w) argmax_merge(v, i, sv[w], si[w]);
  __syncthreads();
}

__device__ __forceinline__ float block_sum(float x, float* sv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  if (lane == 0) sv[warp] = x;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < kXentThreads / 32; ++w) s += sv[w];   // fixed order
  __syncthreads();
  return s;
}

// Persistent form: grid = (clusters) x N CTAs, cluster = N CTAs, CTA rank =
// vocabulary shard.  Cluster c handles tokens c, c + C, c + 2C, ...
// Each CTA's slice of a row arrives in shared memory by bulk copy, two
// tokens ahead (double buffered); every thread copies its R float4 into
// registers and the buffer is refilled at once, so HBM reads never wait on
// the reductions.  One HBM read and one HBM write per logit, one exp per
// logit (kept in registers for the gradient).  The shards exchange their
// (max, sum-exp, target logit, arg-max) point to point: lane r of warp 0
// writes the CTA's 16-byte record into shard r's shared memory with an
// asynchronous store that counts its bytes on shard r's barrier; each CTA
// expects N records on its own barrier and combines them in shard order.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {   // three-input max
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Maximum over the full warp in one instruction (sm_100a `redux.sync` on
// f32; NaN inputs are dropped, as by fmaxf).
__device__ __forceinline__ float warp_max_f32(float x) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
  return r;
}

// Gradient stores: fp32 float4, or four bf16 (round to nearest even) in 8 bytes.
__device__ __forceinline__ void store_grad4(float* dst, int j, float4 e) {
  __stcs(reinterpret_cast<float4*>(dst) + j, e);
}
__device__ __forceinline__ void store_grad4(__nv_bfloat16* dst, int j, float4 e) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(e.x, e.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(e.z, e.w);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t*>(&lo);
  w.y = *reinterpret_cast<uint32_t*>(&hi);
  __stcs(reinterpret_cast<uint2*>(dst) + j, w);
}
__device__ __forceinline__ void store_grad1(float* dst, float e) { *dst = e; }
__device__ __forceinline__ void store_grad1(__nv_bfloat16* dst, float e) {
  *dst = __float2bfloat16_rn(e);
}

template <int R, int NT, typename GT>
__global__ void __launch_bounds__(NT, R * NT <= 2048 ? 4 : 2)
    vp_xent_cluster_kernel(const float* logits, const int64_t* __restrict__ targets, int64_t T,
                           int64_t v, int vs, float grad_scale, float* __restrict__ loss,
                           GT* dlogits, int32_t* __restrict__ argmax, int32_t* dev_status,
                           uint64_t wait_ns) {
  extern __shared__ __align__(128) unsigned char xsm[];   // two slices of the row
  __shared__ __align__(16) float rec[2][8][4];   // [token parity][shard] (m, s, tgt, amax)
  __shared__ __align__(8) uint64_t xbar[2];
  __shared__ __align__(8) uint64_t load_bar[2];
  // block-reduction scratch, double buffered by token parity: a warp that
  // runs ahead writes the other half while slow warps still read this one
  __shared__ float red_m2[2][NT / 32];
  __shared__ float red_s2[2][NT / 32];
  __shared__ int red_i2[2][NT / 32];

  constexpr float kLog2e = 1.4426950408889634f;
  const uint32_t shard = cluster_ctarank();
  const int N = static_cast<int>(v / vs);
  const int64_t cluster_id = blockIdx.x / N;
  const int64_t nclusters = gridDim.x / N;
  const int64_t lo = static_cast<int64_t>(shard) * vs;
  const int nvec = vs >> 2;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool need_grad = dlogits != nullptr;
  const uint32_t slice_bytes = static_cast<uint32_t>(vs) * 4u;
  const uint32_t buf_stride = (slice_bytes + 127u) & ~127u;

  if (threadIdx.x == 0) {
    mbar_init(&xbar[0], 1);
    mbar_init(&xbar[1], 1);
    mbar_init(&load_bar[0], 1);
    mbar_init(&load_bar[1], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  cluster_sync_all();   // every CTA's barriers exist before any peer signals them

  auto issue = [&](int b, int64_t tok) {   // one thread
    mbar_arrive_expect_tx(&load_bar[b], slice_bytes);
    const char* src = reinterpret_cast<const char*>(logits + tok * v + lo);
    char* dst = reinterpret_cast<char*>(xsm + b * buf_stride);
    for (uint32_t off = 0; off < slice_bytes; off += 16384u) {
      const uint32_t n = slice_bytes - off < 16384u ? slice_bytes - off : 16384u;
      bulk_load(dst + off, src + off, n, &load_bar[b]);
    }
  };
  if (threadIdx.x == 0) {
    if (cluster_id < T) issue(0, cluster_id);
    if (cluster_id + nclusters < T) issue(1, cluster_id + nclusters);
  }

  int k = 0;
  for (int64_t tok = cluster_id; tok < T; tok += nclusters, ++k) {
    const int p = k & 1;
    const int64_t y = __ldg(targets + tok);
    const bool y_ok = y >= 0 && y < v;
    const bool mine = y_ok && y >= lo && y < lo + vs;
    // this token's N incoming records: 16 bytes each on xbar[p]
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&xbar[p], static_cast<uint32_t>(N) * 16u);
    if (!mbar_wait_cluster_bounded(&load_bar[p], static_cast<uint32_t>(k >> 1) & 1u, wait_ns)) {
      if (threadIdx.x == 0 && dev_status) atomicOr(dev_status, TP_DEVERR_TIMEOUT);
    }
    const float4* buf4 = reinterpret_cast<const float4*>(xsm + p * buf_stride);
    float4 x[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = threadIdx.x + r * NT;
      x[r] = j < nvec ? buf4[j]
                      : make_float4(-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F);
    }
    const float tgt_i =
        (mine && threadIdx.x == 0) ? reinterpret_cast<const float*>(buf4)[y - lo] : 0.0f;

    // 1) each warp's maximum, the first position of it, e = exp(l − m_w) kept
    //    in registers and the warp's sum: one warp-level pass, no barrier
    float mt = -CUDART_INF_F;
#pragma unroll
    for (int r = 0; r < R; ++r) mt = max3f(max3f(mt, x[r].x, x[r].y), x[r].z, x[r].w);
    const float m_w = warp_max_f32(mt);
    int it = 0x7fffffff;
    if (mt == m_w) {   // only lanes holding the warp maximum search
#pragma unroll
      for (int r = R - 1; r >= 0; --r) {   // elements ascend with r: keep the lowest
        const int j = threadIdx.x + r * NT;
        if (x[r].w == m_w) it = 4 * j + 3;
        if (x[r].z == m_w) it = 4 * j + 2;
        if (x[r].y == m_w) it = 4 * j + 1;
        if (x[r].x == m_w) it = 4 * j;
      }
    }
    // a warp whose elements are all padding (−inf) contributes nothing
    const float mL = m_w == -CUDART_INF_F ? 0.0f : m_w * kLog2e;
    // the exponent arguments, the sums and (below) the gradient scaling run
    // on f32x2 pairs
    const float2 l2e2 = make_float2(kLog2e, kLog2e), nml2 = make_float2(-mL, -mL);
    float2 st2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float2 a = __ffma2_rn(make_float2(x[r].x, x[r].y), l2e2, nml2);
      const float2 b = __ffma2_rn(make_float2(x[r].z, x[r].w), l2e2, nml2);
      x[r].x = ex2_approx(a.x);
      x[r].y = ex2_approx(a.y);
      x[r].z = ex2_approx(b.x);
      x[r].w = ex2_approx(b.y);
      st2 = __fadd2_rn(st2, make_float2(x[r].x, x[r].y));
      st2 = __fadd2_rn(st2, make_float2(x[r].z, x[r].w));
    }
    float st = st2.x + st2.y;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) st += __shfl_xor_sync(0xffffffffu, st, off);
    it = __reduce_min_sync(0xffffffffu, it);
    if (lane == 0) {
      red_m2[p][warp] = m_w;
      red_s2[p][warp] = st;
      red_i2[p][warp] = it;
    }
    __syncthreads();   // also: every thread has its slice in registers
    // refill two tokens ahead: warp 1 issues it, so that warp 0, which
    // sends the shard's record, does not wait for the copy to be issued
    if (threadIdx.x == 32 && tok + 2 * nclusters < T) {
      fence_proxy_async_smem();
      issue(p, tok + 2 * nclusters);
    }
    // 2) the shard's record from the warps' in a fixed order:
    //    m_i = max m_w, s_i = Σ s_w·exp(m_w − m_i), first position of m_i
    float m_i = red_m2[p][0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) m_i = fmaxf(m_i, red_m2[p][w]);
    float s_i = 0.f;
    int a_i = 0x7fffffff;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
      const float mw = red_m2[p][w];
      if (mw != -CUDART_INF_F) s_i += red_s2[p][w] * ex2_approx((mw - m_i) * kLog2e);
      if (mw == m_i) a_i = min(a_i, red_i2[p][w]);
    }

    // 4) send this shard's record to every shard of the cluster (itself included)
    if (warp == 0) {
      const float tg = __shfl_sync(0xffffffffu, tgt_i, 0);   // held by thread 0
      if (lane < N)
        st_async_v4(mapa_shared(&rec[p][shard][0], static_cast<uint32_t>(lane)),
                    mapa_shared(&xbar[p], static_cast<uint32_t>(lane)), m_i, s_i, tg,
                    __int_as_float(static_cast<int>(lo) + a_i));
    }
    if (!mbar_wait_cluster_bounded(&xbar[p], static_cast<uint32_t>(k >> 1) & 1u, wait_ns)) {
      if (threadIdx.x == 0 && dev_status) atomicOr(dev_status, TP_DEVERR_TIMEOUT);
    }

    // 5) combine the N records inside each warp: lane r holds shard r's
    float rm = -CUDART_INF_F, rs = 0.f, rt = 0.f;
    int ri = 0x7fffffff;
    if (lane < N) {
      const float4 q = *reinterpret_cast<const float4*>(&rec[p][lane][0]);
      rm = q.x;
      rs = q.y;
      rt = q.z;
      ri = __float_as_int(q.w);
    }
    const float M = warp_max_f32(rm);   // lanes past N hold -inf
    float term = lane < N ? rs * ex2_approx((rm - M) * kLog2e) : 0.f;
    // lowest index among the shards holding M
    const int bi = __reduce_min_sync(0xffffffffu, rm == M ? ri : 0x7fffffff);
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) {
      term += __shfl_xor_sync(0xffffffffu, term, off);
      rt += __shfl_xor_sync(0xffffffffu, rt, off);
    }
    const float S = __shfl_sync(0xffffffffu, term, 0);
    const float tgt = __shfl_sync(0xffffffffu, rt, 0);
    const float lse = M + logf(S);
    if (shard == 0 && threadIdx.x == 0) {
      loss[tok] = y_ok ? lse - tgt : CUDART_NAN_F;
      if (argmax) argmax[tok] = bi;
      if (!y_ok && dev_status) atomicOr(dev_status, TP_DEVERR_RANGE);
    }

    // 6) dlogits block = grad_scale · (e · exp(m_i − lse) − onehot)
    if (need_grad) {
      const float scale = y_ok ? grad_scale * ex2_approx((m_w - lse) * kLog2e) : CUDART_NAN_F;
      GT* dst = dlogits + tok * v + lo;
      const int yl = mine ? static_cast<int>(y - lo) : -1;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int j = threadIdx.x + r * NT;
        if (j < nvec) {
          float4 e;
          const float2 lo2 = __fmul2_rn(make_float2(x[r].x, x[r].y), make_float2(scale, scale));
          const float2 hi2 = __fmul2_rn(make_float2(x[r].z, x[r].w), make_float2(scale, scale));
          e.x = lo2.x;
          e.y = lo2.y;
          e.z = hi2.x;
          e.w = hi2.y;
          if ((yl >> 2) == j) {
            const int q = yl & 3;
            if (q == 0) e.x -= grad_scale;
            if (q == 1) e.y -= grad_scale;
            if (q == 2) e.z -= grad_scale;
            if (q == 3) e.w -= grad_scale;
          }
          store_grad4(dst, j, e);
        }
      }
    }
  }
  cluster_sync_all();   // every peer's writes into this CTA have landed
}

// General path (any N, any alignment): one CTA per token walks the shards'
// ranges in order, reading the row from global memory twice.
template <typename GT>
__global__ void __launch_bounds__(kXentThreads)
    vp_xent_rowwise_kernel(const float* logits, const int64_t* __restrict__ targets, int64_t v,
                           int N, float grad_scale, float* __restrict__ loss, GT* dlogits,
                           int32_t* __restrict__ argmax, int32_t* dev_status) {
  __shared__ float red_v[kXentThreads / 32];
  __shared__ int red_i[kXentThreads / 32];
  const int64_t tok = blockIdx.x;
  const float* row = logits + tok * v;
  const int64_t vs = v / N;
  const int64_t y = __ldg(targets + tok);
  const bool y_ok = y >= 0 && y < v;
  float m = -CUDART_INF_F, S = 0.f, tgt = 0.f;
  float best_v = -CUDART_INF_F;
  int best_i = 0x7fffffff;
  for (int sh = 0; sh < N; ++sh) {
    const int64_t lo = sh * vs;
    float mv = -CUDART_INF_F;
    int mi = 0x7fffffff;
    for (int64_t j = threadIdx.x; j < vs; j += kXentThreads)
      argmax_merge(mv, mi, row[lo + j], static_cast<int>(lo + j));
    block_argmax(mv, mi, red_v, red_i);
    float sacc = 0.f;
    for (int64_t j = threadIdx.x; j < vs; j += kXentThreads) sacc += __expf(row[lo + j] - mv);
    const float s_i = block_sum(sacc, red_v);
    const float m_new = fmaxf(m, mv);
    S = S * __expf(m - m_new) + s_i * __expf(mv - m_new);
    m = m_new;
    argmax_merge(best_v, best_i, mv, mi);
    if (y_ok && y >= lo && y < lo + vs) tgt = row[y];
  }
  const float lse = m + logf(S);
  if (threadIdx.x == 0) {
    loss[tok] = y_ok ? lse - tgt : CUDART_NAN_F;
    if (argmax) argmax[tok] = best_i;
    if (!y_ok && dev_status) atomicOr(dev_status, TP_DEVERR_RANGE);
  }
  if (!dlogits) return;
  __syncthreads();   // every thread has read the row before an in-place write
  for (int64_t j = threadIdx.x; j < v; j += kXentThreads) {
    float d = y_ok ? grad_scale * __expf(row[j] - lse) : CUDART_NAN_F;
    if (j == y) d -= grad_scale;
    store_grad1(dlogits + tok * v + j, d);
  }
}

// loss_sum = Σ_t loss[t], one block, fixed order (deterministic).
__global__ void __launch_bounds__(1024) loss_sum_kernel(const float* loss, int64_t T, float* out) {
  __shared__ float part[1024];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < T; i += 1024) s += loss[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w >= 1; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = part[0];
}

// Combine of the per-slice softmax statistics the logits GEMM records
// (slice k of row t at [k·T + t]): 32 tokens per block, one per lane; warp w
// reads slices w, w + 8, … so that each load is 32 consecutive tokens.  First
// the maximum with its first column, then the sum of s_k·exp(m_k − m); both
// fold the eight warps in warp order, so the result does not depend on timing.
constexpr int kCombWarps = 8;

__global__ void __launch_bounds__(kCombWarps * 32) linear_xent_combine_kernel(
    const float* __restrict__ stat_m, const float* __restrict__ stat_s,
    const int32_t* __restrict__ stat_i, const float* __restrict__ tgt_logit,
    const int64_t* __restrict__ targets, int64_t T, int64_t v, int nslices, float* __restrict__ loss,
    float* __restrict__ lse_out, int32_t* __restrict__ argmax, int32_t* dev_status) {
  __shared__ float part_m[kCombWarps][32];
  __shared__ int part_i[kCombWarps][32];
  __shared__ float part_s[kCombWarps][32];
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  const bool ok = t < T;
  float m = -INFINITY;
  int arg = 0x7fffffff;
  if (ok) {
#pragma unroll 4
    for (int k = w; k < nslices; k += kCombWarps) {
      const float mk = __ldcs(stat_m + k * T + t);
      if (mk > m) {   // slices in increasing column order: ties keep the first
        m = mk;
        arg = stat_i[k * T + t];
      }
    }
  }
  part_m[w][lane] = m;
  part_i[w][lane] = arg;
  __syncthreads();
  float M = part_m[0][lane];
  int A = part_i[0][lane];
#pragma unroll
  for (int q = 1; q < kCombWarps; ++q) {
    const float mq = part_m[q][lane];
    const int aq = part_i[q][lane];
    if (mq > M || (mq == M && aq < A)) {
      M = mq;
      A = aq;
    }
  }
  float S = 0.0f;
  if (ok) {
#pragma unroll 4
    for (int k = w; k < nslices; k += kCombWarps)
      S += __ldcs(stat_s + k * T + t) * expf(stat_m[k * T + t] - M);
  }
  part_s[w][lane] = S;
  __syncthreads();
  if (w == 0 && ok) {
    float tot = 0.0f;
#pragma unroll
    for (int q = 0; q < kCombWarps; ++q) tot += part_s[q][lane];
    const float lse = M + logf(tot);
    const int64_t y = targets[t];
    const bool y_ok = y >= 0 && y < v;
    if (!y_ok && dev_status) atomicOr(dev_status, TP_DEVERR_RANGE);
    loss[t] = y_ok ? lse - tgt_logit[t] : CUDART_NAN_F;
    if (lse_out) lse_out[t] = lse;
    if (argmax) argmax[t] = A;
  }
}

tp_status loss_sum_launch(const float* loss, int64_t T, float* loss_sum, cudaStream_t stream) {
  loss_sum_kernel<<<1, 1024, 0, stream>>>(loss, T, loss_sum);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

template <int R, int NT, typename GT>
tp_status xent_cluster_launch(const float* logits, const int64_t* targets, int64_t T, int64_t v,
                              int N, float grad_scale, float* loss, float* loss_sum, GT* dlogits,
                              int32_t* argmax, int32_t* dev_status, cudaStream_t stream) {
  static int cap[64][9] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t slice = static_cast<size_t>(v / N) * sizeof(float);
  const size_t smem = 2 * ((slice + 127) & ~static_cast<size_t>(127));
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = N;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static size_t cap_smem[64][9] = {{0}};
  // The shared-memory opt-in belongs to the kernel, not to (device, N): it
  // only ever grows, so that a call with a smaller slice cannot lower the
  // limit under a larger one whose occupancy is already cached.
  static size_t attr_smem[64] = {0};
  if (smem > attr_smem[dev & 63]) {
    if (cudaFuncSetAttribute(vp_xent_cluster_kernel<R, NT, GT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return TP_ERR_CUDA;
    attr_smem[dev & 63] = smem;
  }
  int& c = cap[dev & 63][N];
  if (c == 0 || cap_smem[dev & 63][N] != smem) {
    cap_smem[dev & 63][N] = smem;
    int clusters = 0;
    cfg.gridDim = dim3(static_cast<unsigned>(N * num_sms()));
    if (cudaOccupancyMaxActiveClusters(&clusters, vp_xent_cluster_kernel<R, NT, GT>, &cfg) != cudaSuccess ||
        clusters <= 0) {
      cudaGetLastError();
      clusters = num_sms() / N > 0 ? num_sms() / N : 1;
    }
    c = clusters;
  }
  const int64_t clusters = T < c ? T : c;
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * N));
  if (cudaLaunchKernelEx(&cfg, vp_xent_cluster_kernel<R, NT, GT>, logits, targets, T, v,
                         static_cast<int>(v / N), grad_scale, loss, dlogits, argmax, dev_status,
                         wait_limit_ns()) != cudaSuccess)
    return TP_ERR_CUDA;
  note_launches(1);
  return loss_sum ? loss_sum_launch(loss, T, loss_sum, stream) : TP_OK;
}

// ---------------------------------------------------------------------------
// embedding backward: deterministic scatter-add of dOut rows into dE
// ---------------------------------------------------------------------------
// Sort keys (id << 32 | token) ascending: tokens with the same id become a
// contiguous run in token order.  Ids outside [0, v) get the largest key and
// are skipped.
constexpr int64_t kSortSmemKeys = 16384;   // keys sorted inside one CTA (128 KB)
constexpr uint64_t kNoKey = ~0ull;

__device__ __forceinline__ uint64_t embed_key(const int64_t* ids, int64_t T, int64_t v, int64_t i,
                                              int32_t* dev_status) {
  if (i >= T) return kNoKey;
  const int64_t id = ids[i];
  if (id < 0 || id >= v) {
    if (dev_status) atomicOr(dev_status, TP_DEVERR_RANGE);
    return kNoKey;
  }
  return (static_cast<uint64_t>(id) << 32) | static_cast<uint32_t>(i);
}

// Bucketed sort (T <= kSortSmemKeys): CTA b owns ids [b·span, (b+1)·span).
// It scans every token once, gathers its own tokens in token order (warp
// ballots + a block scan), counts the in-range tokens with smaller ids (its
// output offset), sorts its keys in shared memory and writes them in place,
// so keys_out ends up sorted by (id, token); the last CTA fills the tail
// (out-of-range tokens) with the no-key marker.
constexpr int kBucketThreads = 1024;

__global__ void __launch_bounds__(kBucketThreads)
    embed_bucket_sort_kernel(const int64_t* __restrict__ ids, int64_t T, int64_t v, int64_t span,
                             uint64_t* __restrict__ keys_out, int32_t* dev_status) {
  extern __shared__ uint64_t sk[];
  __shared__ int warp_cnt[kBucketThreads / 32];
  __shared__ int warp_below[kBucketThreads / 32];
  __shared__ int scan_tot[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t lo = blockIdx.x * span;
  const int64_t hi = lo + span < v ? lo + span : v;
  int count = 0;       // this bucket's tokens so far (uniform over the block)
  int64_t below = 0;   // in-range tokens with id < lo
  int64_t inrange = 0; // all in-range tokens (for the tail fill)
  for (int64_t base = 0; base < T; base += kBucketThreads) {
    const int64_t t = base + threadIdx.x;
    const int64_t id = t < T ? ids[t] : -1;
    const bool ok = t < T && id >= 0 && id < v;
    if (t < T && !ok && blockIdx.x == 0 && dev_status) atomicOr(dev_status, TP_DEVERR_RANGE);
    const bool mine = ok && id >= lo && id < hi;
    const unsigned bm = __ballot_sync(0xffffffffu, mine);
    const unsigned bb = __ballot_sync(0xffffffffu, ok && id < lo);
    const unsigned bo = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) {
      warp_cnt[warp] = __popc(bm);
      warp_below[warp] = __popc(bb) + (__popc(bo) << 16);
    }
    __syncthreads();
    if (warp == 0) {   // exclusive scan of the warp counts in warp order
      const int c = warp_cnt[lane];
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      int wb = warp_below[lane];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) wb += __shfl_xor_sync(0xffffffffu, wb, off);
      warp_cnt[lane] = incl - c;
      if (lane == 31) scan_tot[0] = incl;
      if (lane == 0) scan_tot[1] = wb;
    }
    __syncthreads();
    const int pos = count + warp_cnt[warp] + __popc(bm & ((1u << lane) - 1u));
    if (mine && pos < kSortSmemKeys)
      sk[pos] = (static_cast<uint64_t>(id) << 32) | static_cast<uint32_t>(t);
    count += scan_tot[0];
    below += scan_tot[1] & 0xffff;
    inrange += scan_tot[1] >> 16;
    __syncthreads();
  }
  int P = 1;
  while (P < count) P <<= 1;
  for (int i = count + threadIdx.x; i < P; i += kBucketThreads) sk[i] = kNoKey;
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {          // bitonic sort, ascending
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P; i += kBucketThreads) {
        const int l = i ^ j;
        if (l > i) {
          const uint64_t a = sk[i], b = sk[l];
          if ((a > b) == ((i & k) == 0)) {
            sk[i] = b;
            sk[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < count; i += kBucketThreads) keys_out[below + i] = sk[i];
  if (blockIdx.x == gridDim.x - 1)
    for (int64_t i = inrange + threadIdx.x; i < T; i += kBucketThreads) keys_out[i] = kNoKey;
}

__global__ void embed_keys_kernel(const int64_t* __restrict__ ids, int64_t T, int64_t v, int64_t P,
                                  uint64_t* __restrict__ keys, int32_t* dev_status) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i < P) keys[i] = embed_key(ids, T, v, i, dev_status);
}

// one compare-exchange stage of a global-memory bitonic sort (large T)
__global__ void bitonic_stage_kernel(uint64_t* keys, int64_t P, int64_t j, int64_t k) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= P) return;
  const int64_t l = i ^ j;
  if (l > i) {
    const uint64_t a = keys[i], b = keys[l];
    if ((a > b) == ((i & k) == 0)) {
      keys[i] = b;
      keys[l] = a;
    }
  }
}

// One warp per (sorted position, 256-column chunk).  A warp whose position
// starts a run of equal ids sums the run's dOut rows in token order (fp32)
// and adds the sum into dE[id] — the only writer of that chunk of that row.
constexpr int kSegWarps = 8;

__global__ void __launch_bounds__(kSegWarps * 32)
    embed_segsum_kernel(const uint64_t* __restrict__ keys, int64_t T,
                        const __nv_bfloat16* __restrict__ dout, int64_t h, int64_t nchunks,
                        float* __restrict__ dE) {
  const int lane = threadIdx.x & 31;
  const int64_t w = blockIdx.x * static_cast<int64_t>(kSegWarps) + (threadIdx.x >> 5);
  const int64_t i = w / nchunks;
  const int64_t chunk = w - i * nchunks;
  if (i >= T) return;
  const uint64_t key = keys[i];
  if (key == kNoKey) return;
  const uint32_t id = static_cast<uint32_t>(key >> 32);
  if (i > 0 && keys[i - 1] != kNoKey && static_cast<uint32_t>(keys[i - 1] >> 32) == id) return;
  const int64_t col = chunk * 256 + lane * 8;
  if (col >= h) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int64_t j = i; j < T; ++j) {
    const uint64_t kj = keys[j];
    if (kj == kNoKey || static_cast<uint32_t>(kj >> 32) != id) break;
    const int64_t t = static_cast<int64_t>(static_cast<uint32_t>(kj));
    const uint4 wv = __ldg(reinterpret_cast<const uint4*>(dout + t * h + col));
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ww[q]));
      acc[2 * q] += f.x;
      acc[2 * q + 1] += f.y;
    }
  }
  float4* dst = reinterpret_cast<float4*>(dE + static_cast<int64_t>(id) * h + col);
  float4 a = dst[0], b = dst[1];
  a.x += acc[0]; a.y += acc[1]; a.z += acc[2]; a.w += acc[3];
  b.x += acc[4]; b.y += acc[5]; b.z += acc[6]; b.w += acc[7];
  dst[0] = a;
  dst[1] = b;
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers (argument validation is done by the entry points)
// ---------------------------------------------------------------------------
tp_status vp_embed_launch(const int64_t* ids, int64_t T, const void* E, int64_t v, int64_t h,
                          int N, int elem_bytes, void* out, int32_t* dev_status,
                          cudaStream_t stream) {
  const int64_t vec_per_row = h * elem_bytes / 16;
  const int64_t blocks = (T + kEmbedWarps - 1) / kEmbedWarps;
  vp_embed_kernel<<<static_cast<unsigned>(blocks), kEmbedWarps * 32, 0, stream>>>(
      ids, T, static_cast<const uint4*>(E), v, vec_per_row, v / N, static_cast<uint4*>(out),
      dev_status);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

template <typename GT>
tp_status vp_xent_launch_t(const float* logits, const int64_t* targets, int64_t T, int64_t v,
                           int N, float grad_scale, float* loss, float* loss_sum, GT* dlogits,
                           int32_t* argmax, int32_t* dev_status, cudaStream_t stream) {
  const int64_t vs = v / N;
  const bool cluster_ok = N >= 1 && N <= 8 && (vs % 4) == 0 && vs <= 16 * 4 * kXentClusterThreads &&
                          (v % 4) == 0 &&
                          (reinterpret_cast<uintptr_t>(logits) % 16) == 0 &&
                          (dlogits == nullptr || (reinterpret_cast<uintptr_t>(dlogits) % 16) == 0);
  if (cluster_ok) {
    // threads per CTA and float4 per thread (the smallest supported R with
    // R * NT * 4 >= vs): fewer, fuller threads amortise the per-token reductions
    constexpr int NT = kXentClusterThreads;
    const int need = static_cast<int>((vs / 4 + NT - 1) / NT);
    if (need <= 2) return xent_cluster_launch<2, NT, GT>(logits, targets, T, v, N, grad_scale, loss,
                                                         loss_sum, dlogits, argmax, dev_status, stream);
    if (need <= 4) return xent_cluster_launch<4, NT, GT>(logits, targets, T, v, N, grad_scale, loss,
                                                         loss_sum, dlogits, argmax, dev_status, stream);
    if (need <= 8) return xent_cluster_launch<8, NT, GT>(logits, targets, T, v, N, grad_scale, loss,
                                                         loss_sum, dlogits, argmax, dev_status, stream);
    if (need <= 13) return xent_cluster_launch<13, NT, GT>(logits, targets, T, v, N, grad_scale,
                                                           loss, loss_sum, dlogits, argmax,
                                                           dev_status, stream);
    return xent_cluster_launch<16, NT, GT>(logits, targets, T, v, N, grad_scale, loss, loss_sum,
                                           dlogits, argmax, dev_status, stream);
  }
  vp_xent_rowwise_kernel<GT><<<static_cast<unsigned>(T), kXentThreads, 0, stream>>>(
      logits, targets, v, N, grad_scale, loss, dlogits, argmax, dev_status);
  note_launches(1);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  return loss_sum ? loss_sum_launch(loss, T, loss_sum, stream) : TP_OK;
}

tp_status vp_xent_launch(const float* logits, const int64_t* targets, int64_t T, int64_t v, int N,
                         float grad_scale, float* loss, float* loss_sum, void* dlogits,
                         bool bf16_grad, int32_t* argmax, int32_t* dev_status,
                         cudaStream_t stream) {
  if (bf16_grad)
    return vp_xent_launch_t<__nv_bfloat16>(logits, targets, T, v, N, grad_scale, loss, loss_sum,
                                           static_cast<__nv_bfloat16*>(dlogits), argmax,
                                           dev_status, stream);
  return vp_xent_launch_t<float>(logits, targets, T, v, N, grad_scale, loss, loss_sum,
                                 static_cast<float*>(dlogits), argmax, dev_status, stream);
}

tp_status linear_xent_combine_launch(const float* stat_m, const float* stat_s,
                                     const int32_t* stat_i, const float* tgt_logit,
                                     const int64_t* targets, int64_t T, int64_t v, float* loss,
                                     float* loss_sum, float* lse, int32_t* argmax,
                                     int32_t* dev_status, cudaStream_t stream) {
  const int nslices = static_cast<int>((v + kXentSlice - 1) / kXentSlice);
  const unsigned blocks = static_cast<unsigned>((T + 31) / 32);
  linear_xent_combine_kernel<<<blocks, kCombWarps * 32, 0, stream>>>(
      stat_m, stat_s, stat_i, tgt_logit, targets, T, v, nslices, loss, lse, argmax, dev_status);
  note_launches(1);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  return loss_sum ? loss_sum_launch(loss, T, loss_sum, stream) : TP_OK;
}

size_t embed_bwd_ws_bytes(int64_t T) {
  int64_t P = 1;
  while (P < T) P <<= 1;
  return static_cast<size_t>(P) * sizeof(uint64_t);
}

tp_status vp_embed_bwd_launch(const int64_t* ids, const void* dout, int64_t T, int64_t v, int64_t h,
                              float* dE, void* ws, int32_t* dev_status, cudaStream_t stream) {
  int64_t P = 1;
  while (P < T) P <<= 1;
  uint64_t* keys = static_cast<uint64_t*>(ws);
  if (P <= kSortSmemKeys) {
    // a bucket may hold every token: room for min(P, kSortSmemKeys) keys
    const int smem = static_cast<int>(P * sizeof(uint64_t));
    static int configured[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (smem > 48 * 1024 && configured[dev & 63] < smem) {
      if (cudaFuncSetAttribute(embed_bucket_sort_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSortSmemKeys * sizeof(uint64_t))) != cudaSuccess)
        return TP_ERR_CUDA;
      configured[dev & 63] = static_cast<int>(kSortSmemKeys * sizeof(uint64_t));
    }
    const int64_t buckets = std::min<int64_t>(v, 2 * static_cast<int64_t>(num_sms()));
    const int64_t span = (v + buckets - 1) / buckets;
    embed_bucket_sort_kernel<<<static_cast<unsigned>((v + span - 1) / span), kBucketThreads, smem,
                               stream>>>(ids, T, v, span, keys, dev_status);
    note_launches(1);
  } else {
    const unsigned blocks = static_cast<unsigned>((P + 255) / 256);
    embed_keys_kernel<<<blocks, 256, 0, stream>>>(ids, T, v, P, keys, dev_status);
    note_launches(1);
    for (int64_t k = 2; k <= P; k <<= 1)
      for (int64_t j = k >> 1; j > 0; j >>= 1) {
        bitonic_stage_kernel<<<blocks, 256, 0, stream>>>(keys, P, j, k);
        note_launches(1);
      }
  }
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  const int64_t nchunks = (h + 255) / 256;
  const int64_t warps = T * nchunks;
  embed_segsum_kernel<<<static_cast<unsigned>((warps + kSegWarps - 1) / kSegWarps), kSegWarps * 32,
                        0, stream>>>(keys, T, static_cast<const __nv_bfloat16*>(dout), h, nchunks, dE);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

}  // namespace tpl
