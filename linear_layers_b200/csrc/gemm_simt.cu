// gemm_simt.cu — fp32 CUDA-core path and small reduction helpers.
//
// The fp32 configuration of the layers (the tiny b=2, s=8, h=64 MLP) runs on
// plain FFMA kernels: a 32x32-tile shared-memory GEMM with the same operand
// storages and epilogues as the tensor-core engine (bias + activation,
// activation derivative, plain store, per-split partials).  It exists for
// fp32 accuracy, not speed.  The column-sum finisher used by both paths for
// the bias gradient also lives here.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"

namespace tpl {
namespace {

constexpr int TS = 32;   // tile edge
constexpr int TK = 16;   // k step

__device__ __forceinline__ float act_apply32(float u, int act) {
  if (act == TP_ACT_GELU_TANH) {
    const float z = 0.7978845608028654f * (u + 0.044715f * u * u * u);
    return 0.5f * u * (1.0f + tanhf(z));
  }
  if (act == TP_ACT_GELU_ERF) return 0.5f * u * (1.0f + erff(u * 0.7071067811865476f));
  return u;
}

__device__ __forceinline__ float act_deriv32(float u, int act) {
  if (act == TP_ACT_GELU_TANH) {
    const float t = tanhf(0.7978845608028654f * (u + 0.044715f * u * u * u));
    const float dz = 0.7978845608028654f * (1.0f + 3.0f * 0.044715f * u * u);
    return 0.5f * (1.0f + t) + 0.5f * u * (1.0f - t * t) * dz;
  }
  if (act == TP_ACT_GELU_ERF) {
    return 0.5f * (1.0f + erff(u * 0.7071067811865476f)) +
           u * 0.3989422804014327f * expf(-0.5f * u * u);
  }
  return 1.0f;
}

struct SimtArgs {
  const float* A;
  const float* B;
  int64_t lda, ldb;
  int a_mn, b_mn;
  int M, N, k0, k1;
  int epi, act;
  float* out0;
  float* out1;
  int64_t ldo;
  const float* bias;
  const float* aux;
  int64_t ld_aux;
  float* dbias_part;   // [ceil(M/TS), N]
};

// 32x32 output tile per block of 32x8 threads; each thread owns 4 rows.
__global__ void __launch_bounds__(256) gemm_simt_kernel(SimtArgs a) {
  __shared__ float sA[TK][TS + 1];
  __shared__ float sB[TK][TS + 1];
  __shared__ float sred[8][TS];
  const int tx = threadIdx.x;   // column in tile
  const int ty = threadIdx.y;   // 0..7
  const int row0 = blockIdx.y * TS;
  const int col0 = blockIdx.x * TS;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int kk = a.k0; kk < a.k1; kk += TK) {
    for (int idx = ty * TS + tx; idx < TK * TS; idx += 256) {
      const int k = idx / TS, m = idx % TS;
      const int gk = kk + k, gm = row0 + m, gn = col0 + m;
      float va = 0.f, vb = 0.f;
      if (gk < a.k1 && gm < a.M)
        va = a.a_mn ? a.A[static_cast<int64_t>(gk) * a.lda + gm] : a.A[static_cast<int64_t>(gm) * a.lda + gk];
      if (gk < a.k1 && gn < a.N)
        vb = a.b_mn ? a.B[static_cast<int64_t>(gk) * a.ldb + gn] : a.B[static_cast<int64_t>(gn) * a.ldb + gk];
      sA[k][m] = va;
      sB[k][m] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      const float b = sB[k][tx];
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] = fmaf(sA[k][ty * 4 + r], b, acc[r]);
    }
    __syncthreads();
  }
  const int col = col0 + tx;
  float colsum = 0.f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = row0 + ty * 4 + r;
    if (row >= a.M || col >= a.N) continue;
    float v = acc[r];
    const int64_t o = static_cast<int64_t>(row) * a.ldo + col;
    if (a.epi == EPI_BIAS_ACT) {
      if (a.bias) v += a.bias[col];
      if (a.out0) a.out0[o] = v;
      a.out1[o] = act_apply32(v, a.act);
    } else if (a.epi == EPI_DACT || a.epi == EPI_DACT_Y) {
      const float u = a.aux[static_cast<int64_t>(row) * a.ld_aux + col];
      v *= act_deriv32(u, a.act);
      a.out0[o] = v;
      colsum += v;
      if (a.epi == EPI_DACT_Y) a.out1[o] = act_apply32(u, a.act);   // activation recompute
    } else {
      a.out0[o] = v;
    }
  }
  if ((a.epi == EPI_DACT || a.epi == EPI_DACT_Y) && a.dbias_part) {
    sred[ty][tx] = colsum;
    __syncthreads();
    if (ty == 0 && col < a.N) {
      float s = 0.f;
      for (int i = 0; i < 8; ++i) s += sred[i][tx];
      a.dbias_part[static_cast<int64_t>(blockIdx.y) * a.N + col] = s;
    }
  }
}

// Z = Σ_s part[s] in split order (fp32 Zpart mode of the fp32 path).
__global__ void sum_splits_kernel(const float* part, int splits, int64_t count, float* out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = part[i];
    for (int k = 1; k < splits; ++k) s += part[k * count + i];
    out[i] = s;
  }
}

// dU = dY ⊙ act'(U) (when dU != nullptr) and per-128-row-tile column sums
// of dU into part[tile, n].  One thread per column, 128 rows per block row.
template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T>
__global__ void dact_colsum_kernel(const T* dY, const T* U, int64_t M, int64_t N, int act, T* dU,
                                   float* part) {
  const int64_t n = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (n >= N) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int64_t r1 = r0 + 128 < M ? r0 + 128 : M;
  float s = 0.f;
  for (int64_t r = r0; r < r1; ++r) {
    float g = to_f(dY[r * N + n]);
    if (act != TP_ACT_NONE) g *= act_deriv32(to_f(U[r * N + n]), act);
    if (dU) dU[r * N + n] = from_f<T>(g);
    s += g;
  }
  if (part) part[static_cast<int64_t>(blockIdx.y) * N + n] = s;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// bf16, 8 columns per thread (16-byte loads and stores) over 32 rows per
// block; the activation is a template argument.
template <int ACT>
__global__ void __launch_bounds__(128) dact_colsum_v8_kernel(const uint4* __restrict__ dY,
                                                             const uint4* __restrict__ U,
                                                             int64_t M, int64_t N,
                                                             uint4* __restrict__ dU,
                                                             float* __restrict__ part) {
  const int64_t c8 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n8 = N / 8;
  if (c8 >= n8) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int64_t r1 = r0 + 32 < M ? r0 + 32 : M;
  float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int64_t r = r0; r < r1; ++r) {
    const uint4 g = __ldg(dY + r * n8 + c8);
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
    float v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __uint_as_float(gw[k] << 16);
      v[2 * k + 1] = __uint_as_float(gw[k] & 0xffff0000u);
    }
    if constexpr (ACT != TP_ACT_NONE) {
      const uint4 u = __ldg(U + r * n8 + c8);
      const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[2 * k] *= act_deriv32(__uint_as_float(uw[k] << 16), ACT);
        v[2 * k + 1] *= act_deriv32(__uint_as_float(uw[k] & 0xffff0000u), ACT);
      }
      uint4 o;
      o.x = pack2_bf16(v[0], v[1]);
      o.y = pack2_bf16(v[2], v[3]);
      o.z = pack2_bf16(v[4], v[5]);
      o.w = pack2_bf16(v[6], v[7]);
      if (dU) dU[r * n8 + c8] = o;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) s[k] += v[k];
  }
  if (part) {
    float4* dst = reinterpret_cast<float4*>(part + static_cast<int64_t>(blockIdx.y) * N + c8 * 8);
    dst[0] = make_float4(s[0], s[1], s[2], s[3]);
    dst[1] = make_float4(s[4], s[5], s[6], s[7]);
  }
}

// dbias[n] = Σ_t part[t, n] in a fixed order: 32 columns per block, 8 row
// groups of 32 threads; group q sums tiles q, q+8, q+16, … (four loads in
// flight), then the 8 group sums are added in group order.
__global__ void __launch_bounds__(256) dbias_finish_kernel(const float* part, int tiles, int N,
                                                           float* dbias) {
  __shared__ float red[8][33];
  const int lane = threadIdx.x & 31, q = threadIdx.x >> 5;
  const int n = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (n < N) {
    int t = q;
    for (; t + 24 < tiles; t += 32) {
      const float a = part[static_cast<int64_t>(t) * N + n];
      const float b = part[static_cast<int64_t>(t + 8) * N + n];
      const float c = part[static_cast<int64_t>(t + 16) * N + n];
      const float d = part[static_cast<int64_t>(t + 24) * N + n];
      s += a;
      s += b;
      s += c;
      s += d;
    }
    for (; t < tiles; t += 8) s += part[static_cast<int64_t>(t) * N + n];
  }
  red[q][lane] = s;
  __syncthreads();
  if (q == 0 && n < N) {
    float tot = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) tot += red[g][lane];
    dbias[n] = tot;
  }
}

}  // namespace

tp_status gemm_simt_launch(const GemmProblem& p, cudaStream_t stream) {
  if (p.M <= 0 || p.N <= 0 || p.K <= 0) return TP_ERR_SHAPE;
  SimtArgs a;
  a.A = static_cast<const float*>(p.A);
  a.B = static_cast<const float*>(p.B);
  a.lda = p.lda;
  a.ldb = p.ldb;
  a.a_mn = p.a_mn;
  a.b_mn = p.b_mn;
  a.M = p.M;
  a.N = p.N;
  a.act = p.act;
  a.out1 = static_cast<float*>(p.out1);
  a.ldo = p.ldo;
  a.bias = static_cast<const float*>(p.bias);
  a.aux = static_cast<const float*>(p.aux);
  a.ld_aux = p.ld_aux;
  a.dbias_part = p.dbias_part;
  dim3 block(TS, 8);
  dim3 grid((p.N + TS - 1) / TS, (p.M + TS - 1) / TS);
  if (p.splits <= 1 && !p.zpart) {
    a.epi = p.epi;
    a.out0 = static_cast<float*>(p.out0);
    a.k0 = 0;
    a.k1 = p.K;
    gemm_simt_kernel<<<grid, block, 0, stream>>>(a);
    note_launches(1);
    return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
  }
  // per-split partials into zpart (required here), then an ordered sum
  if (!p.zpart) return TP_ERR_UNSUPPORTED;
  if (p.ldo != p.N) return TP_ERR_UNSUPPORTED;
  const int64_t count = static_cast<int64_t>(p.M) * p.N;
  for (int s = 0; s < p.splits; ++s) {
    a.epi = EPI_STORE_F32;
    a.out0 = p.zpart + s * count;
    a.ldo = p.N;
    a.k0 = p.split_k[s];
    a.k1 = p.split_k[s + 1];
    gemm_simt_kernel<<<grid, block, 0, stream>>>(a);
    note_launches(1);
  }
  const int blocks = static_cast<int>((count + 255) / 256 < 4096 ? (count + 255) / 256 : 4096);
  sum_splits_kernel<<<blocks, 256, 0, stream>>>(p.zpart, p.splits, count,
                                                 static_cast<float*>(p.out0));
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

tp_status dact_colsum_launch(const void* dY, const void* U, int64_t M, int64_t Nout, int act,
                             bool bf16, void* dU, float* dbias_part, cudaStream_t stream,
                             int* tiles) {
  const auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (bf16 && Nout % 8 == 0 && al16(dY) && al16(U) && al16(dU) && al16(dbias_part)) {
    // 32-row partial sums (the workspace holds ceil(M / 32) rows)
    dim3 g(static_cast<unsigned>((Nout / 8 + 127) / 128), static_cast<unsigned>((M + 31) / 32));
    const auto* y = static_cast<const uint4*>(dY);
    const auto* u = static_cast<const uint4*>(U);
    auto* d = static_cast<uint4*>(dU);
    if (act == TP_ACT_GELU_TANH)
      dact_colsum_v8_kernel<TP_ACT_GELU_TANH><<<g, 128, 0, stream>>>(y, u, M, Nout, d, dbias_part);
    else if (act == TP_ACT_GELU_ERF)
      dact_colsum_v8_kernel<TP_ACT_GELU_ERF><<<g, 128, 0, stream>>>(y, u, M, Nout, d, dbias_part);
    else
      dact_colsum_v8_kernel<TP_ACT_NONE><<<g, 128, 0, stream>>>(y, u, M, Nout, d, dbias_part);
    *tiles = static_cast<int>(g.y);
    note_launches(1);
    return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
  }
  dim3 grid(static_cast<unsigned>((Nout + 255) / 256), static_cast<unsigned>((M + 127) / 128));
  *tiles = static_cast<int>(grid.y);
  if (bf16)
    dact_colsum_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(dY), static_cast<const __nv_bfloat16*>(U), M, Nout, act,
        static_cast<__nv_bfloat16*>(dU), dbias_part);
  else
    dact_colsum_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(dY),
                                                        static_cast<const float*>(U), M, Nout, act,
                                                        static_cast<float*>(dU), dbias_part);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

tp_status dbias_finish_launch(const float* part, int tiles, int N, float* dbias,
                              cudaStream_t stream) {
  dbias_finish_kernel<<<(N + 31) / 32, 256, 0, stream>>>(part, tiles, N, dbias);
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

}  // namespace tpl
