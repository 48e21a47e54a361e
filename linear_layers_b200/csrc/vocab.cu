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
#include <math_constants.h>

#include <cstdint>

#include "internal.h"

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
constexpr int kXentThreads = 256;

struct ShardStat {   // what one shard publishes for its row
  float m;           // max of the shard's logits
  float s;           // Σ exp(l − m) over the shard
  float tgt;         // target logit if the target is in this shard, else 0
  int amax;          // global index of the first maximum in the shard
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ int ld_dsmem_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
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

// grid = T * N CTAs, cluster = N CTAs (one token), CTA rank = shard.
// Dynamic shared memory: the shard's slice of the row (vs floats).
__global__ void __launch_bounds__(kXentThreads)
    vp_xent_cluster_kernel(const float* logits, const int64_t* __restrict__ targets, int64_t v,
                           int vs, float grad_scale, float* __restrict__ loss, float* dlogits,
                           int32_t* __restrict__ argmax, int32_t* dev_status) {
  extern __shared__ float4 slice4[];
  __shared__ ShardStat stat;
  __shared__ float red_v[kXentThreads / 32];
  __shared__ int red_i[kXentThreads / 32];
  __shared__ float comb[3];   // lse, target logit, valid

  const uint32_t shard = cluster_ctarank();
  const int N = static_cast<int>(v / vs);
  const int64_t tok = blockIdx.x / N;
  const int64_t lo = static_cast<int64_t>(shard) * vs;
  const float4* src4 = reinterpret_cast<const float4*>(logits + tok * v + lo);
  const int nvec = vs >> 2;

  // 1) stage the slice, track the first maximum
  float mv = -CUDART_INF_F;
  int mi = 0x7fffffff;
  for (int j = threadIdx.x; j < nvec; j += kXentThreads) {
    const float4 x = __ldcs(src4 + j);
    slice4[j] = x;
    argmax_merge(mv, mi, x.x, 4 * j);
    argmax_merge(mv, mi, x.y, 4 * j + 1);
    argmax_merge(mv, mi, x.z, 4 * j + 2);
    argmax_merge(mv, mi, x.w, 4 * j + 3);
  }
  block_argmax(mv, mi, red_v, red_i);   // includes __syncthreads: slice visible
  const float m_i = mv;

  const int64_t y = __ldg(targets + tok);
  const bool y_ok = y >= 0 && y < v;
  const bool mine = y_ok && y >= lo && y < lo + vs;
  // read from global: the slice is overwritten in place below, and no CTA
  // writes dlogits (which may alias logits) before the first cluster barrier
  const float tgt_i = (mine && threadIdx.x == 0) ? logits[tok * v + y] : 0.0f;

  // 2) e = exp(l − m_i) in place, and its sum
  const bool need_grad = dlogits != nullptr;
  float sacc = 0.f;
  for (int j = threadIdx.x; j < nvec; j += kXentThreads) {
    float4 x = slice4[j];
    x.x = __expf(x.x - m_i);
    x.y = __expf(x.y - m_i);
    x.z = __expf(x.z - m_i);
    x.w = __expf(x.w - m_i);
    sacc += (x.x + x.y) + (x.z + x.w);
    if (need_grad) slice4[j] = x;
  }
  const float s_i = block_sum(sacc, red_v);

  // 3) publish this shard's scalars; combine all shards' through DSMEM
  if (threadIdx.x == 0) {
    stat.m = m_i;
    stat.s = s_i;
    stat.tgt = tgt_i;
    stat.amax = static_cast<int>(lo) + mi;
  }
  cluster_sync_all();
  if (threadIdx.x == 0) {
    float m = -CUDART_INF_F;
    float ms[16];
    float ss[16];
    float best_v = -CUDART_INF_F;
    int best_i = 0x7fffffff;
    float tgt = 0.f;
    for (int r = 0; r < N; ++r) {
      const uint32_t base = map_to_rank(&stat, r);
      ms[r] = ld_dsmem_f32(base + offsetof(ShardStat, m));
      ss[r] = ld_dsmem_f32(base + offsetof(ShardStat, s));
      tgt += ld_dsmem_f32(base + offsetof(ShardStat, tgt));
      argmax_merge(best_v, best_i, ms[r], ld_dsmem_s32(base + offsetof(ShardStat, amax)));
      m = fmaxf(m, ms[r]);
    }
    float S = 0.f;
    for (int r = 0; r < N; ++r) S += ss[r] * __expf(ms[r] - m);   // shard order
    const float lse = m + logf(S);
    comb[0] = lse;
    comb[1] = tgt;
    comb[2] = y_ok ? 1.f : 0.f;
    if (shard == 0) {
      loss[tok] = y_ok ? lse - tgt : CUDART_NAN_F;
      if (argmax) argmax[tok] = best_i;
      if (!y_ok && dev_status) atomicOr(dev_status, TP_DEVERR_RANGE);
    }
  }
  cluster_sync_all();   // no CTA leaves while a peer may still read its `stat`
  if (!need_grad) return;

  // 4) dlogits block = grad_scale · (e · exp(m_i − lse) − onehot)
  const float lse = comb[0];
  const float scale = y_ok ? grad_scale * __expf(m_i - lse) : CUDART_NAN_F;
  float4* dst4 = reinterpret_cast<float4*>(dlogits + tok * v + lo);
  const int yl = mine ? static_cast<int>(y - lo) : -1;
  for (int j = threadIdx.x; j < nvec; j += kXentThreads) {
    float4 e = slice4[j];
    e.x *= scale;
    e.y *= scale;
    e.z *= scale;
    e.w *= scale;
    if ((yl >> 2) == j) {
      const int k = yl & 3;
      if (k == 0) e.x -= grad_scale;
      if (k == 1) e.y -= grad_scale;
      if (k == 2) e.z -= grad_scale;
      if (k == 3) e.w -= grad_scale;
    }
    __stcs(dst4 + j, e);
  }
}

// General path (any N, any alignment): one CTA per token walks the shards'
// ranges in order, reading the row from global memory twice.
__global__ void __launch_bounds__(kXentThreads)
    vp_xent_rowwise_kernel(const float* logits, const int64_t* __restrict__ targets, int64_t v,
                           int N, float grad_scale, float* __restrict__ loss, float* dlogits,
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
    dlogits[tok * v + j] = d;
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

tp_status vp_xent_launch(const float* logits, const int64_t* targets, int64_t T, int64_t v, int N,
                         float grad_scale, float* loss, float* loss_sum, float* dlogits,
                         int32_t* argmax, int32_t* dev_status, cudaStream_t stream) {
  const int64_t vs = v / N;
  const size_t slice_bytes = static_cast<size_t>(vs) * sizeof(float);
  const bool cluster_ok = N >= 1 && N <= 8 && (vs % 4) == 0 && slice_bytes <= 200 * 1024 &&
                          (T * N) < (1ll << 31) &&
                          (reinterpret_cast<uintptr_t>(logits) % 16) == 0 &&
                          (dlogits == nullptr || (reinterpret_cast<uintptr_t>(dlogits) % 16) == 0);
  if (cluster_ok) {
    static int configured_bytes[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (slice_bytes > 48 * 1024 && configured_bytes[dev & 63] < static_cast<int>(slice_bytes)) {
      if (cudaFuncSetAttribute(vp_xent_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(slice_bytes)) != cudaSuccess)
        return TP_ERR_CUDA;
      configured_bytes[dev & 63] = static_cast<int>(slice_bytes);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(T * N));
    cfg.blockDim = dim3(kXentThreads);
    cfg.dynamicSmemBytes = slice_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = N;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, vp_xent_cluster_kernel, logits, targets, v, static_cast<int>(vs),
                           grad_scale, loss, dlogits, argmax, dev_status) != cudaSuccess)
      return TP_ERR_CUDA;
    note_launches(1);
  } else {
    vp_xent_rowwise_kernel<<<static_cast<unsigned>(T), kXentThreads, 0, stream>>>(
        logits, targets, v, N, grad_scale, loss, dlogits, argmax, dev_status);
    note_launches(1);
    if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  }
  if (loss_sum) {
    loss_sum_kernel<<<1, 1024, 0, stream>>>(loss, T, loss_sum);
    note_launches(1);
    if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  }
  return TP_OK;
}

}  // namespace tpl
