// internal.h — declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>
#include <cstddef>

#include "../../include/tplayers.h"

namespace tpl {

constexpr int kMaxSplits = 16;   // K splits of one row-parallel GEMM (and shards with Zpart)

enum EpiKind : int {
  EPI_STORE_BF16 = 0,   // out0 = bf16(acc)
  EPI_BIAS_ACT = 1,     // U = acc + bias; Y = act(U); out0 = U (nullable), out1 = Y
  EPI_DACT = 2,         // dU = acc ⊙ act'(aux); out0 = dU; per-tile column sums of dU
  EPI_STORE_F32 = 3,    // out0 = acc (fp32)
  EPI_SPLIT_SUM = 4,    // fp32 partial per split; the last split of a tile sums them
                        // in split order and stores bf16 to out0
  EPI_XENT_STATS = 5,   // softmax statistics of each 128-column slice of every row:
                        // maximum, Σ exp(acc − maximum), first arg-max; the target
                        // column's accumulator; no output matrix
  EPI_XENT_GRAD = 6,    // out0 = bf16(grad_scale·(exp(acc − lse_row) − [col = target]))
  EPI_DACT_Y = 7        // EPI_DACT, and out1 = act(aux): the activation rebuilt from the
                        // saved pre-activation (recompute), from the same tanh as act'
};

constexpr int kXentSlice = 128;   // columns per softmax-statistics slice

// C[M,N] = A[M,K] · B[K,N] with the operands in one of two storages each:
//   A: a_mn == 0  ->  A stored [M,K] row-major (lda >= K)      (K-major)
//      a_mn == 1  ->  A stored [K,M] row-major (lda >= M)      (MN-major)
//   B: b_mn == 0  ->  B stored [N,K] row-major (ldb >= K)      (K-major)
//      b_mn == 1  ->  B stored [K,N] row-major (ldb >= N)      (MN-major)
struct GemmProblem {
  const void* A = nullptr;
  const void* B = nullptr;
  int64_t lda = 0, ldb = 0;
  int a_mn = 0, b_mn = 0;
  int M = 0, N = 0, K = 0;
  int epi = EPI_STORE_BF16;
  void* out0 = nullptr;
  void* out1 = nullptr;
  int64_t ldo = 0;
  const void* bias = nullptr;      // EPI_BIAS_ACT (bf16 [N]) nullable
  const void* aux = nullptr;       // EPI_DACT: U (bf16, row stride ld_aux)
  int64_t ld_aux = 0;
  float* dbias_part = nullptr;     // EPI_DACT: [ceil(M/128), N] fp32, nullable
  int act = TP_ACT_NONE;
  // EPI_SPLIT_SUM
  int splits = 1;
  int split_k[kMaxSplits + 1] = {0};   // K offsets of the splits (multiples of 64)
  float* zpart = nullptr;          // nullable [splits, M, N] fp32: partials land here
  void* ws = nullptr;              // partial buffer + tile counters (see gemm_ws_bytes)
  size_t ws_bytes = 0;
  int32_t* dev_status = nullptr;
  // EPI_XENT_STATS / EPI_XENT_GRAD (row = token, column = vocabulary entry)
  const int64_t* targets = nullptr;  // [M]
  float* stat_m = nullptr;           // [ceil(N/128), M] slice maxima
  float* stat_s = nullptr;           // [ceil(N/128), M] slice sums of exp(acc − max)
  int32_t* stat_i = nullptr;         // [ceil(N/128), M] slice arg-max (column index)
  float* tgt_logit = nullptr;        // [M] accumulator at the target column
  const float* row_lse = nullptr;    // [M] log-sum-exp of each row (EPI_XENT_GRAD)
  float grad_scale = 1.0f;
};

// Workspace a split GEMM needs: fp32 partial tiles (unless zpart carries
// them) plus one int counter per output tile.
size_t gemm_split_ws_bytes(int M, int N, int splits, bool with_zpart);

tp_status gemm_tc_launch(const GemmProblem& p, cudaStream_t stream);

// Two independent problems with the same epilogue (no split, no partials, no
// dbias) in one launch: the second's tiles fill the first's last wave.
// Returns TP_ERR_UNSUPPORTED for problems it cannot pair.
tp_status gemm_tc_launch_pair(const GemmProblem& p0, const GemmProblem& p1, cudaStream_t stream);

// Arm the one-shot debug injection of the next gemm_tc_launch.
void arm_gemm_injection(int unit, int kb, uint64_t wait_ns);

// Estimated run time (seconds) of a tensor-core GEMM with `splits` K ranges,
// with the tile shape gemm_tc_launch would choose (whole waves of tiles).
double gemm_tc_estimate_s(int M, int N, int K, int splits, int epi);

// fp32 SIMT path (same problem description; operands fp32).
tp_status gemm_simt_launch(const GemmProblem& p, cudaStream_t stream);

// Column sums of the per-tile dbias partials: dbias[n] = Σ_t part[t, n].
tp_status dbias_finish_launch(const float* part, int tiles, int N, float* dbias,
                              cudaStream_t stream);

// Tensor map (a CUtensorMap, 128 bytes) of a row-major bf16 matrix
// [outer, inner] with row stride ld elements: boxes of box_inner x box_outer
// elements, 128-byte swizzle, zero fill outside the matrix.
bool make_tmap_bf16_sw128(void* tmap, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                          uint32_t box_inner, uint32_t box_outer);
// The same for an fp32 matrix (box_inner <= 32: one 128-byte swizzle row).
bool make_tmap_f32_sw128(void* tmap, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                         uint32_t box_inner, uint32_t box_outer);

// Attention core (attn.cu): see tp_attention_fwd.
tp_status attention_fwd_launch(const void* QKV, int64_t b, int64_t s, int heads,
                               const int64_t* head_offsets, int N, bool causal, float scale,
                               void* ctx, float* lse, int32_t* dev_status, cudaStream_t stream);

size_t attention_bwd_ws_bytes(int64_t b, int64_t s, int heads);
tp_status attention_bwd_launch(const void* QKV, const void* O, const void* dO, const float* lse,
                               int64_t b, int64_t s, int heads, const int64_t* head_offsets, int N,
                               bool causal, float scale, void* dQKV, void* ws, int32_t* dev_status,
                               cudaStream_t stream);

// Sequence-parallel dropout-add-LayerNorm (layernorm.cu): see
// tp_sp_dropout_add_ln_fwd / _bwd.  h % 8 == 0, h <= 8192.
size_t sp_ln_bwd_ws_bytes(int64_t M, int64_t h);
tp_status sp_ln_fwd_launch(const void* x, const void* bias, const void* residual, const void* gamma,
                           const void* beta, int64_t M, int64_t h, float p, uint64_t seed,
                           uint64_t offset, float eps, void* hs, void* y, float* mean, float* rstd,
                           uint8_t* keep, int32_t* dev_status, cudaStream_t stream);
tp_status sp_ln_bwd_launch(const void* dy, const void* dhs_in, const void* hs, const void* gamma,
                           const float* mean, const float* rstd, int64_t M, int64_t h, float p,
                           uint64_t seed, uint64_t offset, void* dx, void* dres, float* dgamma,
                           float* dbeta, float* dbias, void* ws, cudaStream_t stream);

// Counts every kernel the library enqueues (tp_launch_count).
void note_launches(int n);

// Device checks shared by the entry points.
tp_status require_sm100();
int num_sms();
uint64_t wait_limit_ns();

}  // namespace tpl
