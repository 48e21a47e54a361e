// tp_api.cu — the extern "C" entry points declared in include/tplayers.h.
//
// Each entry point validates its arguments on the host (returning before
// anything is enqueued), builds the GEMM problem descriptions for the
// tensor-core engine (bf16) or the CUDA-core path (fp32), and enqueues the
// kernels on the caller's stream.  Nothing here allocates, frees or
// synchronises.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace tpl {

tp_status vp_embed_launch(const int64_t* ids, int64_t T, const void* E, int64_t v, int64_t h,
                          int N, int elem_bytes, void* out, int32_t* dev_status,
                          cudaStream_t stream);
tp_status vp_xent_launch(const float* logits, const int64_t* targets, int64_t T, int64_t v, int N,
                         float grad_scale, float* loss, float* loss_sum, void* dlogits,
                         bool bf16_grad, int32_t* argmax, int32_t* dev_status,
                         cudaStream_t stream);

size_t embed_bwd_ws_bytes(int64_t T);
tp_status linear_xent_combine_launch(const float* stat_m, const float* stat_s,
                                     const int32_t* stat_i, const float* tgt_logit,
                                     const int64_t* targets, int64_t T, int64_t v, float* loss,
                                     float* loss_sum, float* lse, int32_t* argmax,
                                     int32_t* dev_status, cudaStream_t stream);
tp_status vp_embed_bwd_launch(const int64_t* ids, const void* dout, int64_t T, int64_t v, int64_t h,
                              float* dE, void* ws, int32_t* dev_status, cudaStream_t stream);

namespace {

constexpr int kDefaultSms = 148;

struct DeviceInfo {
  int checked = 0;
  int ok = 0;
  int sms = kDefaultSms;
};
DeviceInfo g_dev[64];
std::mutex g_dev_mu;

DeviceInfo* device_info() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
      d.ok = (major == 10 && minor == 0);
      d.sms = sms > 0 ? sms : kDefaultSms;
    } else {
      cudaGetLastError();
    }
    d.checked = 1;
  }
  return &d;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Shard offsets: the caller's, or the even split.  Returns TP_OK and fills
// `offs` (N+1 entries) or an error.
tp_status shard_offsets(const int64_t* user, int64_t total, int32_t N, std::vector<int64_t>& offs) {
  if (N < 1) return TP_ERR_SHAPE;
  offs.assign(N + 1, 0);
  if (user == nullptr) {
    if (total % N) return TP_ERR_SHAPE;
    for (int i = 0; i <= N; ++i) offs[i] = total / N * i;
    return TP_OK;
  }
  for (int i = 0; i <= N; ++i) offs[i] = user[i];
  if (offs[0] != 0 || offs[N] != total) return TP_ERR_SHAPE;
  for (int i = 0; i < N; ++i)
    if (offs[i + 1] <= offs[i]) return TP_ERR_SHAPE;
  return TP_OK;
}

bool dims_ok(std::initializer_list<int64_t> d) {
  for (int64_t x : d)
    if (x <= 0 || x > (1ll << 30)) return false;
  return true;
}

inline int64_t elem_bytes(tp_dtype dt) { return dt == TP_DTYPE_BF16 ? 2 : 4; }

// Row lengths must keep TMA / vector rows 16-byte aligned.
bool rows_aligned(tp_dtype dt, std::initializer_list<int64_t> lens) {
  const int64_t q = dt == TP_DTYPE_BF16 ? 8 : 4;
  for (int64_t x : lens)
    if (x % q) return false;
  return true;
}

bool ptrs_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p != nullptr && !aligned16(p)) return false;
  return true;
}

// ---------------------------------------------------------------------------
// split choice for the row-parallel (shard-summing) GEMMs
// ---------------------------------------------------------------------------
// Units of work = output tiles x splits; a split is a contiguous group of
// shards.  More splits fill the last wave of SMs better but write fp32
// partials.  Cost model (relative): compute / wave efficiency + partial
// traffic at HBM speed.  Splits must be a divisor of N with every group
// boundary on a 64-element k-block.
int choose_splits(int64_t M, int64_t Nout, int64_t K, const std::vector<int64_t>& offs, int sms) {
  (void)sms;
  const int N = static_cast<int>(offs.size()) - 1;
  const double hbm = 6.5e12;
  double best_cost = 0;
  int best = 1;
  for (int S = 1; S <= N && S <= kMaxSplits; ++S) {
    if (N % S) continue;
    bool aligned = true;
    for (int g = 1; g < S; ++g)
      if (offs[g * (N / S)] % 64) aligned = false;
    if (!aligned) continue;
    if (S > 1 && K / S < 512) continue;   // keep main loops long enough
    // whole waves of the chosen tile shape, plus the fp32 partials written
    // and read back by the splits but the last
    double cost = gemm_tc_estimate_s(static_cast<int>(M), static_cast<int>(Nout),
                                     static_cast<int>(K), S, S > 1 ? EPI_SPLIT_SUM : EPI_STORE_BF16);
    if (S > 1) cost += static_cast<double>(S - 1) * M * Nout * 4.0 * 2.0 / hbm;
    if (S == 1 || cost < best_cost * 0.98) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

void fill_splits(GemmProblem& g, const std::vector<int64_t>& offs, int S) {
  const int N = static_cast<int>(offs.size()) - 1;
  g.splits = S;
  for (int s = 0; s <= S; ++s) g.split_k[s] = static_cast<int>(offs[s * (N / S)]);
}

int sms_or_default() {
  DeviceInfo* d = device_info();
  return d ? d->sms : kDefaultSms;
}

// Workspace layout of the MLP / linear ops (bf16 path):
//   [split partials + counters of the row-parallel GEMM]   (aligned 256)
//   [dbias per-tile partials, ceil(M/128) x F fp32]         (aligned 256)
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t row_split_ws(int64_t M, int64_t Nout, int64_t K, int32_t N, bool zpart) {
  std::vector<int64_t> offs;
  if (shard_offsets(nullptr, K, N, offs) != TP_OK) return 0;
  const int S = choose_splits(M, Nout, K, offs, sms_or_default());
  // the chosen split's partials + counters, or the counters alone that a
  // call with Zpart (one split per shard, partials in Zpart) needs
  const size_t a = gemm_split_ws_bytes(static_cast<int>(M), static_cast<int>(Nout), S, false);
  const size_t b = gemm_split_ws_bytes(static_cast<int>(M), static_cast<int>(Nout), 2, true);
  (void)zpart;
  return align256(a > b ? a : b);
}

// dbias partials: one fp32 row per 32-row tile (the finest tiling any path uses)
// slice maxima, slice sums, slice arg-max ([ceil(v/128), T] each), target logits [T]
size_t linear_xent_ws_bytes(int64_t T, int64_t v) {
  const size_t plane = align256(static_cast<size_t>((v + kXentSlice - 1) / kXentSlice) * T * 4);
  return 3 * plane + align256(static_cast<size_t>(T) * 4);
}

size_t dbias_ws(int64_t M, int64_t F) { return align256(((M + 31) / 32) * F * sizeof(float)); }

// Run a row-parallel GEMM C[M,Nout] = Σ_i A[:, off_i:off_{i+1}]·B[off_i:off_{i+1}, :]
// (K = sum of the shards).  Zpart forces one split per shard.
tp_status run_row_parallel(GemmProblem g, const std::vector<int64_t>& offs, float* zpart,
                           void* ws, size_t ws_bytes, bool bf16, cudaStream_t stream) {
  const int N = static_cast<int>(offs.size()) - 1;
  int S;
  if (zpart) {
    if (N > kMaxSplits) return TP_ERR_UNSUPPORTED;
    S = N;
    if (bf16)
      for (int i = 1; i < N; ++i)
        if (offs[i] % 64) return TP_ERR_UNSUPPORTED;
  } else {
    S = bf16 ? choose_splits(g.M, g.N, g.K, offs, sms_or_default()) : 1;
    // a workspace sized for other shard offsets only costs the split: the
    // unsplit form (all shards summed in one accumulator) needs none
    if (S > 1 && (ws == nullptr || ws_bytes < gemm_split_ws_bytes(g.M, g.N, S, false))) S = 1;
  }
  fill_splits(g, offs, S);
  g.zpart = zpart;
  g.ws = ws;
  g.ws_bytes = ws_bytes;
  return bf16 ? gemm_tc_launch(g, stream) : gemm_simt_launch(g, stream);
}

uint64_t g_wait_ns = 0;
std::once_flag g_wait_once;

}  // namespace

std::atomic<uint64_t> g_launches{0};

void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int num_sms() { return sms_or_default(); }

uint64_t wait_limit_ns() {
  std::call_once(g_wait_once, [] {
    g_wait_ns = 2000000000ull;   // 2 s: far above any legitimate stage wait
    if (const char* e = std::getenv("TP_WAIT_LIMIT_MS")) {
      const long long ms = std::atoll(e);
      if (ms > 0) g_wait_ns = static_cast<uint64_t>(ms) * 1000000ull;
    }
  });
  return g_wait_ns;
}

tp_status require_sm100() {
  DeviceInfo* d = device_info();
  if (!d || !d->ok) return TP_ERR_DEVICE;
  return TP_OK;
}

}  // namespace tpl

using namespace tpl;

extern "C" {

const char* tp_status_string(tp_status s) {
  switch (s) {
    case TP_OK: return "ok";
    case TP_ERR_NULL: return "a required pointer is NULL";
    case TP_ERR_SHAPE: return "invalid or inconsistent sizes";
    case TP_ERR_ALIGN: return "pointer or row length breaks the 16-byte alignment rule";
    case TP_ERR_DTYPE: return "unknown dtype or activation";
    case TP_ERR_UNSUPPORTED: return "request not supported by the library";
    case TP_ERR_CUDA: return "CUDA call failed while enqueueing";
    case TP_ERR_WORKSPACE: return "workspace missing or too small";
    case TP_ERR_DEVICE: return "no sm_100 device is current";
    default: return "unknown status";
  }
}

int32_t tp_version(void) { return 100; }

uint64_t tp_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t tp_workspace_bytes(tp_op op, int64_t M, int64_t h, int64_t F, int32_t N) {
  if (M <= 0 || h <= 0 || F <= 0 || N < 1) return 0;
  switch (op) {
    case TP_OP_MLP_FWD:   // row GEMM Z = Y·B over K = F
      return row_split_ws(M, h, F, N, false);
    case TP_OP_MLP_BWD:   // dX = dU·Aᵀ over K = F, plus dbias partials
      return row_split_ws(M, h, F, N, false) + dbias_ws(M, F);
    case TP_OP_ROW_LINEAR_FWD:   // (M, Nout=h, Kin=F)
      return row_split_ws(M, h, F, N, false);
    case TP_OP_COL_LINEAR_BWD:   // (M, K=h, Nout=F): dX over K=Nout, dbias partials
      return row_split_ws(M, h, F, N, false) + dbias_ws(M, F);
    case TP_OP_ROW_LINEAR_BWD:
      return 0;
    case TP_OP_EMBED_BWD:   // (T, h, v, N): sort keys of the T tokens
      return align256(embed_bwd_ws_bytes(M));
    case TP_OP_LINEAR_XENT:   // (T, h, v, N): slice statistics + target logits
      return linear_xent_ws_bytes(M, F);
    case TP_OP_SP_LN_BWD:     // (M, h, h, N): per-block partial parameter gradients
      return sp_ln_bwd_ws_bytes(M, h);
    case TP_OP_ATTENTION_BWD: // (b·s, n_heads, 64, N): rowsum(dO ⊙ O), fp32 dQ accumulator
      return attention_bwd_ws_bytes(M, 1, static_cast<int>(h));
  }
  return 0;
}

tp_status tp_mlp_fwd(const void* X, const void* A, const void* bias, const void* B, int64_t M,
                     int64_t h, int64_t F, int32_t N, const int64_t* shard_offsets_,
                     tp_dtype dt, tp_act act, void* U, void* Y, void* Z, float* Zpart, void* ws,
                     size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!X || !A || !B || !U || !Y || !Z) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16 && dt != TP_DTYPE_F32) return TP_ERR_DTYPE;
  if (act < TP_ACT_NONE || act > TP_ACT_GELU_ERF) return TP_ERR_DTYPE;
  if (!dims_ok({M, h, F})) return TP_ERR_SHAPE;
  std::vector<int64_t> offs;
  if (tp_status s = shard_offsets(shard_offsets_, F, N, offs)) return s;
  if (!rows_aligned(dt, {h, F}) || !ptrs_aligned({X, A, bias, B, U, Y, Z, Zpart, ws}))
    return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  const bool bf16 = dt == TP_DTYPE_BF16;
  cudaStream_t st = as_stream(stream);

  // column-parallel GEMM over all shards: U = X·A + bias, Y = act(U)
  GemmProblem g1;
  g1.A = X; g1.lda = h; g1.a_mn = 0;
  g1.B = A; g1.ldb = F; g1.b_mn = 1;
  g1.M = static_cast<int>(M); g1.N = static_cast<int>(F); g1.K = static_cast<int>(h);
  g1.epi = EPI_BIAS_ACT; g1.act = act; g1.bias = bias;
  g1.out0 = U; g1.out1 = Y; g1.ldo = F;
  g1.dev_status = dev_status;
  tp_status s = bf16 ? gemm_tc_launch(g1, st) : gemm_simt_launch(g1, st);
  if (s) return s;

  // row-parallel GEMM with the g all-reduce fused: Z = Σ_i Y_i·B_i
  GemmProblem g2;
  g2.A = Y; g2.lda = F; g2.a_mn = 0;
  g2.B = B; g2.ldb = h; g2.b_mn = 1;
  g2.M = static_cast<int>(M); g2.N = static_cast<int>(h); g2.K = static_cast<int>(F);
  g2.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  g2.out0 = Z; g2.ldo = h;
  g2.dev_status = dev_status;
  return run_row_parallel(g2, offs, Zpart, ws, ws_bytes, bf16, st);
}

}  // extern "C"

namespace tpl {
namespace {

// The MLP backward; with recompute the dGeLU GEMM's epilogue also writes
// Y = act(U) into Y (which the dB GEMM then reads), otherwise Y is the saved
// activation.
tp_status mlp_bwd_impl(const void* X, const void* A, const void* B, const void* U, void* Y,
                       bool recompute, const void* dZ, int64_t M, int64_t h, int64_t F, int32_t N,
                       const int64_t* shard_offsets_, tp_dtype dt, tp_act act, void* dU, void* dX,
                       void* dA, float* dbias, void* dB, void* ws, size_t ws_bytes,
                       int32_t* dev_status, void* stream) {
  if (!X || !A || !B || !U || !Y || !dZ || !dU || !dX || !dA || !dB) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16 && dt != TP_DTYPE_F32) return TP_ERR_DTYPE;
  if (act < TP_ACT_NONE || act > TP_ACT_GELU_ERF) return TP_ERR_DTYPE;
  if (!dims_ok({M, h, F})) return TP_ERR_SHAPE;
  std::vector<int64_t> offs;
  if (tp_status s = shard_offsets(shard_offsets_, F, N, offs)) return s;
  if (!rows_aligned(dt, {h, F}) ||
      !ptrs_aligned({X, A, B, U, Y, dZ, dU, dX, dA, dbias, dB, ws}))
    return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  const bool bf16 = dt == TP_DTYPE_BF16;
  cudaStream_t st = as_stream(stream);

  // dbias partial rows: one per 128-row piece (tensor cores) or per 32-row tile (fp32 path)
  const int64_t mtiles = bf16 ? (M + 127) / 128 : (M + 31) / 32;
  const size_t split_bytes = bf16 ? row_split_ws(M, h, F, N, false) : 0;
  const size_t dbias_bytes = dbias ? dbias_ws(M, F) : 0;
  if (split_bytes + dbias_bytes > 0 && (ws == nullptr || ws_bytes < split_bytes + dbias_bytes))
    return TP_ERR_WORKSPACE;
  float* dbias_part =
      dbias ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + split_bytes) : nullptr;

  // g backward = identity; dU = (dZ·Bᵀ) ⊙ act'(U), per-tile column sums for dbias
  GemmProblem g3;
  g3.A = dZ; g3.lda = h; g3.a_mn = 0;
  g3.B = B; g3.ldb = h; g3.b_mn = 0;            // B [F,h] read as Bᵀ: K-major
  g3.M = static_cast<int>(M); g3.N = static_cast<int>(F); g3.K = static_cast<int>(h);
  g3.epi = recompute ? EPI_DACT_Y : EPI_DACT; g3.act = act; g3.aux = U; g3.ld_aux = F;
  g3.out0 = dU; g3.ldo = F; g3.dbias_part = dbias_part;
  if (recompute) g3.out1 = Y;
  g3.dev_status = dev_status;
  tp_status s = bf16 ? gemm_tc_launch(g3, st) : gemm_simt_launch(g3, st);
  if (s) return s;

  // dB_i = Y_iᵀ·dZ and dA_i = Xᵀ·dU_i (independent: one launch in bf16)
  GemmProblem g4;
  g4.A = Y; g4.lda = F; g4.a_mn = 1;
  g4.B = dZ; g4.ldb = h; g4.b_mn = 1;
  g4.M = static_cast<int>(F); g4.N = static_cast<int>(h); g4.K = static_cast<int>(M);
  g4.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  g4.out0 = dB; g4.ldo = h;
  g4.dev_status = dev_status;
  GemmProblem g5;
  g5.A = X; g5.lda = h; g5.a_mn = 1;
  g5.B = dU; g5.ldb = F; g5.b_mn = 1;
  g5.M = static_cast<int>(h); g5.N = static_cast<int>(F); g5.K = static_cast<int>(M);
  g5.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  g5.out0 = dA; g5.ldo = F;
  g5.dev_status = dev_status;
  if (bf16) {
    if ((s = gemm_tc_launch_pair(g4, g5, st))) return s;
  } else {
    if ((s = gemm_simt_launch(g4, st))) return s;
    if ((s = gemm_simt_launch(g5, st))) return s;
  }

  // f backward: dX = Σ_i dU_i·A_iᵀ
  GemmProblem g6;
  g6.A = dU; g6.lda = F; g6.a_mn = 0;
  g6.B = A; g6.ldb = F; g6.b_mn = 0;            // A [h,F] read as Aᵀ: K-major
  g6.M = static_cast<int>(M); g6.N = static_cast<int>(h); g6.K = static_cast<int>(F);
  g6.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  g6.out0 = dX; g6.ldo = h;
  g6.dev_status = dev_status;
  if ((s = run_row_parallel(g6, offs, nullptr, ws, split_bytes, bf16, st))) return s;

  if (dbias) return dbias_finish_launch(dbias_part, static_cast<int>(mtiles), static_cast<int>(F),
                                        dbias, st);
  return TP_OK;
}

}  // namespace
}  // namespace tpl

extern "C" {

tp_status tp_mlp_bwd(const void* X, const void* A, const void* B, const void* U, const void* Y,
                     const void* dZ, int64_t M, int64_t h, int64_t F, int32_t N,
                     const int64_t* shard_offsets_, tp_dtype dt, tp_act act, void* dU, void* dX,
                     void* dA, float* dbias, void* dB, void* ws, size_t ws_bytes,
                     int32_t* dev_status, void* stream) {
  return tpl::mlp_bwd_impl(X, A, B, U, const_cast<void*>(Y), false, dZ, M, h, F, N,
                           shard_offsets_, dt, act, dU, dX, dA, dbias, dB, ws, ws_bytes,
                           dev_status, stream);
}

tp_status tp_mlp_bwd_recompute(const void* X, const void* A, const void* B, const void* U,
                               void* Y, const void* dZ, int64_t M, int64_t h, int64_t F,
                               int32_t N, const int64_t* shard_offsets_, tp_dtype dt, tp_act act,
                               void* dU, void* dX, void* dA, float* dbias, void* dB, void* ws,
                               size_t ws_bytes, int32_t* dev_status, void* stream) {
  return tpl::mlp_bwd_impl(X, A, B, U, Y, true, dZ, M, h, F, N, shard_offsets_, dt, act, dU, dX,
                           dA, dbias, dB, ws, ws_bytes, dev_status, stream);
}

}  // extern "C"

extern "C" {

tp_status tp_col_linear_fwd(const void* X, const void* W, const void* bias, int64_t M, int64_t K,
                            int64_t Nout, int32_t N, const int64_t* shard_offsets_, tp_dtype dt,
                            tp_act act, void* U, void* Y, int32_t* dev_status, void* stream) {
  if (!X || !W || !Y || (act != TP_ACT_NONE && !U)) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16 && dt != TP_DTYPE_F32) return TP_ERR_DTYPE;
  if (act < TP_ACT_NONE || act > TP_ACT_GELU_ERF) return TP_ERR_DTYPE;
  if (!dims_ok({M, K, Nout})) return TP_ERR_SHAPE;
  std::vector<int64_t> offs;
  if (tp_status s = shard_offsets(shard_offsets_, Nout, N, offs)) return s;
  if (!rows_aligned(dt, {K, Nout}) || !ptrs_aligned({X, W, bias, U, Y})) return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  const bool bf16 = dt == TP_DTYPE_BF16;
  GemmProblem g;
  g.A = X; g.lda = K; g.a_mn = 0;
  g.B = W; g.ldb = Nout; g.b_mn = 1;
  g.M = static_cast<int>(M); g.N = static_cast<int>(Nout); g.K = static_cast<int>(K);
  g.epi = EPI_BIAS_ACT; g.act = act; g.bias = bias;
  g.out0 = U; g.out1 = Y; g.ldo = Nout;
  g.dev_status = dev_status;
  return bf16 ? gemm_tc_launch(g, as_stream(stream)) : gemm_simt_launch(g, as_stream(stream));
}

}  // extern "C"

namespace tpl {
tp_status dact_colsum_launch(const void* dY, const void* U, int64_t M, int64_t Nout, int act,
                             bool bf16, void* dU, float* dbias_part, cudaStream_t stream,
                             int* tiles);
}

extern "C" {

tp_status tp_col_linear_bwd(const void* X, const void* W, const void* U, const void* dY,
                            int64_t M, int64_t K, int64_t Nout, int32_t N,
                            const int64_t* shard_offsets_, tp_dtype dt, tp_act act, void* dU,
                            void* dX, void* dW, float* dbias, void* ws, size_t ws_bytes,
                            int32_t* dev_status, void* stream) {
  if (!X || !W || !dY || !dX || !dW) return TP_ERR_NULL;
  if (act != TP_ACT_NONE && (!U || !dU)) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16 && dt != TP_DTYPE_F32) return TP_ERR_DTYPE;
  if (act < TP_ACT_NONE || act > TP_ACT_GELU_ERF) return TP_ERR_DTYPE;
  if (!dims_ok({M, K, Nout})) return TP_ERR_SHAPE;
  std::vector<int64_t> offs;
  if (tp_status s = shard_offsets(shard_offsets_, Nout, N, offs)) return s;
  if (!rows_aligned(dt, {K, Nout}) || !ptrs_aligned({X, W, U, dY, dU, dX, dW, dbias, ws}))
    return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  const bool bf16 = dt == TP_DTYPE_BF16;
  cudaStream_t st = as_stream(stream);
  const size_t split_bytes = bf16 ? row_split_ws(M, K, Nout, N, false) : 0;
  int64_t mtiles = (M + 127) / 128;   // partial rows of the column sums (set by their kernel)
  const size_t dbias_bytes = dbias ? dbias_ws(M, Nout) : 0;
  if (split_bytes + dbias_bytes > 0 && (ws == nullptr || ws_bytes < split_bytes + dbias_bytes))
    return TP_ERR_WORKSPACE;
  float* dbias_part =
      dbias ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + split_bytes) : nullptr;

  // dU = dY ⊙ act'(U) and its per-tile column sums (one element-wise pass)
  const void* grad = dY;
  if (act != TP_ACT_NONE || dbias) {
    void* dst = act != TP_ACT_NONE ? dU : nullptr;
    int tiles = static_cast<int>(mtiles);
    if (tp_status s = dact_colsum_launch(dY, U, M, Nout, act, bf16, dst, dbias_part, st, &tiles))
      return s;
    mtiles = tiles;
    if (act != TP_ACT_NONE) grad = dU;
  }
  // dW = Xᵀ·dU
  GemmProblem gw;
  gw.A = X; gw.lda = K; gw.a_mn = 1;
  gw.B = grad; gw.ldb = Nout; gw.b_mn = 1;
  gw.M = static_cast<int>(K); gw.N = static_cast<int>(Nout); gw.K = static_cast<int>(M);
  gw.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  gw.out0 = dW; gw.ldo = Nout;
  gw.dev_status = dev_status;
  // f backward: dX = Σ_i dU_i·W_iᵀ
  GemmProblem gx;
  gx.A = grad; gx.lda = Nout; gx.a_mn = 0;
  gx.B = W; gx.ldb = Nout; gx.b_mn = 0;
  gx.M = static_cast<int>(M); gx.N = static_cast<int>(K); gx.K = static_cast<int>(Nout);
  gx.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  gx.out0 = dX; gx.ldo = K;
  gx.dev_status = dev_status;
  tp_status s;
  if (bf16 && choose_splits(M, K, Nout, offs, sms_or_default()) == 1) {
    // the shard sum stays in the accumulator: dW and dX in one launch
    fill_splits(gx, offs, 1);
    if ((s = gemm_tc_launch_pair(gw, gx, st))) return s;
  } else {
    if ((s = bf16 ? gemm_tc_launch(gw, st) : gemm_simt_launch(gw, st))) return s;
    if ((s = run_row_parallel(gx, offs, nullptr, ws, split_bytes, bf16, st))) return s;
  }
  if (dbias) return dbias_finish_launch(dbias_part, static_cast<int>(mtiles),
                                        static_cast<int>(Nout), dbias, st);
  return TP_OK;
}

tp_status tp_row_linear_fwd(const void* Xin, const void* W, int64_t M, int64_t Kin, int64_t Nout,
                            int32_t N, const int64_t* shard_offsets_, tp_dtype dt, void* Z,
                            float* Zpart, void* ws, size_t ws_bytes, int32_t* dev_status,
                            void* stream) {
  if (!Xin || !W || !Z) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16 && dt != TP_DTYPE_F32) return TP_ERR_DTYPE;
  if (!dims_ok({M, Kin, Nout})) return TP_ERR_SHAPE;
  std::vector<int64_t> offs;
  if (tp_status s = shard_offsets(shard_offsets_, Kin, N, offs)) return s;
  if (!rows_aligned(dt, {Kin, Nout}) || !ptrs_aligned({Xin, W, Z, Zpart, ws})) return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  const bool bf16 = dt == TP_DTYPE_BF16;
  GemmProblem g;
  g.A = Xin; g.lda = Kin; g.a_mn = 0;
  g.B = W; g.ldb = Nout; g.b_mn = 1;
  g.M = static_cast<int>(M); g.N = static_cast<int>(Nout); g.K = static_cast<int>(Kin);
  g.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  g.out0 = Z; g.ldo = Nout;
  g.dev_status = dev_status;
  return run_row_parallel(g, offs, Zpart, ws, ws_bytes, bf16, as_stream(stream));
}

tp_status tp_row_linear_bwd(const void* Xin, const void* W, const void* dZ, int64_t M,
                            int64_t Kin, int64_t Nout, int32_t N, const int64_t* shard_offsets_,
                            tp_dtype dt, void* dXin, void* dW, int32_t* dev_status,
                            void* stream) {
  if (!Xin || !W || !dZ || !dXin || !dW) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16 && dt != TP_DTYPE_F32) return TP_ERR_DTYPE;
  if (!dims_ok({M, Kin, Nout})) return TP_ERR_SHAPE;
  std::vector<int64_t> offs;
  if (tp_status s = shard_offsets(shard_offsets_, Kin, N, offs)) return s;
  if (!rows_aligned(dt, {Kin, Nout}) || !ptrs_aligned({Xin, W, dZ, dXin, dW})) return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  const bool bf16 = dt == TP_DTYPE_BF16;
  cudaStream_t st = as_stream(stream);
  // g backward = identity: dXin = dZ·Wᵀ
  GemmProblem gx;
  gx.A = dZ; gx.lda = Nout; gx.a_mn = 0;
  gx.B = W; gx.ldb = Nout; gx.b_mn = 0;
  gx.M = static_cast<int>(M); gx.N = static_cast<int>(Kin); gx.K = static_cast<int>(Nout);
  gx.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  gx.out0 = dXin; gx.ldo = Kin;
  gx.dev_status = dev_status;
  // dW = Xinᵀ·dZ (independent of dXin: one launch in bf16)
  GemmProblem gw;
  gw.A = Xin; gw.lda = Kin; gw.a_mn = 1;
  gw.B = dZ; gw.ldb = Nout; gw.b_mn = 1;
  gw.M = static_cast<int>(Kin); gw.N = static_cast<int>(Nout); gw.K = static_cast<int>(M);
  gw.epi = bf16 ? EPI_STORE_BF16 : EPI_STORE_F32;
  gw.out0 = dW; gw.ldo = Nout;
  gw.dev_status = dev_status;
  if (bf16) return gemm_tc_launch_pair(gx, gw, st);
  tp_status s = gemm_simt_launch(gx, st);
  if (s) return s;
  return gemm_simt_launch(gw, st);
}

tp_status vp_embed(const int64_t* ids, int64_t T, const void* E, int64_t v, int64_t h, int32_t N,
                   tp_dtype dt, void* out, int32_t* dev_status, void* stream) {
  if (!ids || !E || !out) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16 && dt != TP_DTYPE_F32) return TP_ERR_DTYPE;
  if (!dims_ok({T, v, h}) || N < 1 || v % N) return TP_ERR_SHAPE;
  if (!rows_aligned(dt, {h}) || !ptrs_aligned({E, out}) || (reinterpret_cast<uintptr_t>(ids) & 7))
    return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  return vp_embed_launch(ids, T, E, v, h, N, static_cast<int>(elem_bytes(dt)), out, dev_status,
                         as_stream(stream));
}

tp_status tp_logits_fwd(const void* H, const void* E, int64_t T, int64_t h, int64_t v, int32_t N,
                        float* logits, int32_t* dev_status, void* stream) {
  if (!H || !E || !logits) return TP_ERR_NULL;
  if (!dims_ok({T, h, v}) || N < 1 || v % N) return TP_ERR_SHAPE;
  if (h % 8 || v % 4 || !ptrs_aligned({H, E, logits})) return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  // one launch over every vocabulary shard: logits[:, lo_i:hi_i] = H·E_iᵀ
  GemmProblem g;
  g.A = H; g.lda = h; g.a_mn = 0;
  g.B = E; g.ldb = h; g.b_mn = 0;               // E [v,h] read as Eᵀ: K-major
  g.M = static_cast<int>(T); g.N = static_cast<int>(v); g.K = static_cast<int>(h);
  g.epi = EPI_STORE_F32;
  g.out0 = logits; g.ldo = v;
  g.dev_status = dev_status;
  return gemm_tc_launch(g, as_stream(stream));
}

tp_status vp_xent(const float* logits, const int64_t* targets, int64_t T, int64_t v, int32_t N,
                  float grad_scale, float* loss, float* loss_sum, float* dlogits,
                  int32_t* argmax, int32_t* dev_status, void* stream) {
  if (!logits || !targets || !loss) return TP_ERR_NULL;
  if (!dims_ok({T, v}) || N < 1 || v % N) return TP_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(logits) & 3) || (reinterpret_cast<uintptr_t>(targets) & 7))
    return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  return vp_xent_launch(logits, targets, T, v, N, grad_scale, loss, loss_sum, dlogits, false,
                        argmax, dev_status, as_stream(stream));
}

}  // extern "C"

extern "C" {

tp_status vp_xent_bf16_grad(const float* logits, const int64_t* targets, int64_t T, int64_t v,
                            int32_t N, float grad_scale, float* loss, float* loss_sum,
                            void* dlogits, int32_t* argmax, int32_t* dev_status, void* stream) {
  if (!logits || !targets || !loss || !dlogits) return TP_ERR_NULL;
  if (!dims_ok({T, v}) || N < 1 || v % N) return TP_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(logits) & 3) || (reinterpret_cast<uintptr_t>(targets) & 7) ||
      (reinterpret_cast<uintptr_t>(dlogits) & 1))
    return TP_ERR_ALIGN;
  if (static_cast<const void*>(logits) == dlogits) return TP_ERR_UNSUPPORTED;
  if (tp_status s = require_sm100()) return s;
  return vp_xent_launch(logits, targets, T, v, N, grad_scale, loss, loss_sum, dlogits, true, argmax,
                        dev_status, as_stream(stream));
}

tp_status tp_sp_dropout_add_ln_fwd(const void* x, const void* bias, const void* residual,
                                   const void* gamma, const void* beta, int64_t M, int64_t h,
                                   int32_t N, float p, uint64_t seed, uint64_t offset, float eps,
                                   void* hs, void* y, float* mean, float* rstd, uint8_t* keep_out,
                                   int32_t* dev_status, void* stream) {
  if (!x || !residual || !gamma || !beta || !hs || !y || !mean || !rstd) return TP_ERR_NULL;
  if (!dims_ok({M, h}) || N < 1 || M % N) return TP_ERR_SHAPE;
  if (!(p >= 0.0f && p < 1.0f) || !(eps > 0.0f)) return TP_ERR_SHAPE;
  if (h % 8 || h > 8192) return h % 8 ? TP_ERR_ALIGN : TP_ERR_UNSUPPORTED;
  if (!ptrs_aligned({x, bias, residual, gamma, beta, hs, y}) ||
      (reinterpret_cast<uintptr_t>(keep_out) & 7))
    return TP_ERR_ALIGN;
  if (tp_status st = require_sm100()) return st;
  return sp_ln_fwd_launch(x, bias, residual, gamma, beta, M, h, p, seed, offset, eps, hs, y, mean,
                          rstd, keep_out, dev_status, as_stream(stream));
}

tp_status tp_sp_dropout_add_ln_bwd(const void* dy, const void* dhs_in, const void* hs,
                                   const void* gamma, const float* mean, const float* rstd,
                                   int64_t M, int64_t h, int32_t N, float p, uint64_t seed,
                                   uint64_t offset, void* dx, void* dresidual, float* dgamma,
                                   float* dbeta, float* dbias, void* ws, size_t ws_bytes,
                                   int32_t* dev_status, void* stream) {
  (void)dev_status;
  if (!dy || !hs || !gamma || !mean || !rstd || !dx || !dresidual || !dgamma || !dbeta)
    return TP_ERR_NULL;
  if (!dims_ok({M, h}) || N < 1 || M % N) return TP_ERR_SHAPE;
  if (!(p >= 0.0f && p < 1.0f)) return TP_ERR_SHAPE;
  if (h % 8 || h > 8192) return h % 8 ? TP_ERR_ALIGN : TP_ERR_UNSUPPORTED;
  if (!ptrs_aligned({dy, dhs_in, hs, gamma, dx, dresidual, dgamma, dbeta, dbias, ws}))
    return TP_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < sp_ln_bwd_ws_bytes(M, h)) return TP_ERR_WORKSPACE;
  if (tp_status st = require_sm100()) return st;
  return sp_ln_bwd_launch(dy, dhs_in, hs, gamma, mean, rstd, M, h, p, seed, offset, dx, dresidual,
                          dgamma, dbeta, dbias, ws, as_stream(stream));
}

tp_status tp_attention_fwd(const void* QKV, int64_t b, int64_t s, int32_t n_heads,
                           int32_t head_dim, int32_t N, const int64_t* head_offsets,
                           int32_t causal, float scale, void* ctx, float* lse,
                           int32_t* dev_status, void* stream) {
  if (!QKV || !ctx) return TP_ERR_NULL;
  if (b <= 0 || s <= 0 || n_heads <= 0 || N < 1 || N > n_heads || b * s > (1ll << 30))
    return TP_ERR_SHAPE;
  if (head_dim != 64 || n_heads > 256) return TP_ERR_UNSUPPORTED;
  if (!ptrs_aligned({QKV, ctx}) || (reinterpret_cast<uintptr_t>(lse) & 3)) return TP_ERR_ALIGN;
  std::vector<int64_t> offs(N + 1);
  if (head_offsets == nullptr) {   // contiguous split, the first n_heads mod N shards one larger
    offs[0] = 0;
    for (int i = 0; i < N; ++i) offs[i + 1] = offs[i] + n_heads / N + (i < n_heads % N ? 1 : 0);
  } else {
    for (int i = 0; i <= N; ++i) offs[i] = head_offsets[i];
    if (offs[0] != 0 || offs[N] != n_heads) return TP_ERR_SHAPE;
    for (int i = 0; i < N; ++i)
      if (offs[i + 1] <= offs[i]) return TP_ERR_SHAPE;
  }
  if (!(scale > 0.0f) || !std::isfinite(scale)) scale = 1.0f / std::sqrt(static_cast<float>(head_dim));
  if (tp_status st = require_sm100()) return st;
  return attention_fwd_launch(QKV, b, s, n_heads, offs.data(), N, causal != 0, scale, ctx, lse,
                              dev_status, as_stream(stream));
}

tp_status tp_attention_bwd(const void* QKV, const void* ctx, const void* dctx, const float* lse,
                           int64_t b, int64_t s, int32_t n_heads, int32_t head_dim, int32_t N,
                           const int64_t* head_offsets, int32_t causal, float scale, void* dQKV,
                           void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!QKV || !ctx || !dctx || !lse || !dQKV) return TP_ERR_NULL;
  if (b <= 0 || s <= 0 || n_heads <= 0 || N < 1 || N > n_heads || b * s > (1ll << 30))
    return TP_ERR_SHAPE;
  if (head_dim != 64 || n_heads > 256) return TP_ERR_UNSUPPORTED;
  if (!ptrs_aligned({QKV, ctx, dctx, dQKV, ws}) || (reinterpret_cast<uintptr_t>(lse) & 3))
    return TP_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < attention_bwd_ws_bytes(b, s, n_heads)) return TP_ERR_WORKSPACE;
  std::vector<int64_t> offs(N + 1);
  if (head_offsets == nullptr) {
    offs[0] = 0;
    for (int i = 0; i < N; ++i) offs[i + 1] = offs[i] + n_heads / N + (i < n_heads % N ? 1 : 0);
  } else {
    for (int i = 0; i <= N; ++i) offs[i] = head_offsets[i];
    if (offs[0] != 0 || offs[N] != n_heads) return TP_ERR_SHAPE;
    for (int i = 0; i < N; ++i)
      if (offs[i + 1] <= offs[i]) return TP_ERR_SHAPE;
  }
  if (!(scale > 0.0f) || !std::isfinite(scale)) scale = 1.0f / std::sqrt(static_cast<float>(head_dim));
  if (tp_status st = require_sm100()) return st;
  return attention_bwd_launch(QKV, ctx, dctx, lse, b, s, n_heads, offs.data(), N, causal != 0,
                              scale, dQKV, ws, dev_status, as_stream(stream));
}

tp_status tp_linear_xent_fwd(const void* H, const void* E, const int64_t* targets, int64_t T,
                             int64_t h, int64_t v, int32_t N, float* loss, float* loss_sum,
                             float* lse, int32_t* argmax, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream) {
  if (!H || !E || !targets || !loss) return TP_ERR_NULL;
  if (!dims_ok({T, h, v}) || N < 1 || v % N) return TP_ERR_SHAPE;
  if (h % 8 || !ptrs_aligned({H, E}) || (reinterpret_cast<uintptr_t>(targets) & 7)) return TP_ERR_ALIGN;
  const size_t need = linear_xent_ws_bytes(T, v);
  if (ws == nullptr || ws_bytes < need) return TP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255) return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  const size_t plane = align256(static_cast<size_t>((v + kXentSlice - 1) / kXentSlice) * T * 4);
  uint8_t* w = static_cast<uint8_t*>(ws);
  GemmProblem g;
  g.A = H; g.lda = h; g.a_mn = 0;
  g.B = E; g.ldb = h; g.b_mn = 0;               // E [v,h] read as Eᵀ: K-major
  g.M = static_cast<int>(T); g.N = static_cast<int>(v); g.K = static_cast<int>(h);
  g.epi = EPI_XENT_STATS;
  g.targets = targets;
  g.stat_m = reinterpret_cast<float*>(w);
  g.stat_s = reinterpret_cast<float*>(w + plane);
  g.stat_i = reinterpret_cast<int32_t*>(w + 2 * plane);
  g.tgt_logit = reinterpret_cast<float*>(w + 3 * plane);
  g.dev_status = dev_status;
  cudaStream_t st = as_stream(stream);
  if (tp_status s = gemm_tc_launch(g, st)) return s;
  return linear_xent_combine_launch(g.stat_m, g.stat_s, g.stat_i, g.tgt_logit, targets, T, v, loss,
                                    loss_sum, lse, argmax, dev_status, st);
}

tp_status tp_linear_xent_dlogits(const void* H, const void* E, const int64_t* targets,
                                 const float* lse, int64_t T, int64_t h, int64_t v, int32_t N,
                                 float grad_scale, void* dlogits, int32_t* dev_status,
                                 void* stream) {
  if (!H || !E || !targets || !lse || !dlogits) return TP_ERR_NULL;
  if (!dims_ok({T, h, v}) || N < 1 || v % N) return TP_ERR_SHAPE;
  if (h % 8 || v % 8 || !ptrs_aligned({H, E, dlogits}) ||
      (reinterpret_cast<uintptr_t>(targets) & 7) || (reinterpret_cast<uintptr_t>(lse) & 3))
    return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  GemmProblem g;
  g.A = H; g.lda = h; g.a_mn = 0;
  g.B = E; g.ldb = h; g.b_mn = 0;
  g.M = static_cast<int>(T); g.N = static_cast<int>(v); g.K = static_cast<int>(h);
  g.epi = EPI_XENT_GRAD;
  g.out0 = dlogits; g.ldo = v;
  g.targets = targets;
  g.row_lse = lse;
  g.grad_scale = grad_scale;
  g.dev_status = dev_status;
  return gemm_tc_launch(g, as_stream(stream));
}

tp_status tp_logits_bwd(const void* dlogits, const void* H, const void* E, int64_t T, int64_t h,
                        int64_t v, int32_t N, void* dH, float* dE, int32_t* dev_status,
                        void* stream) {
  if (!dlogits || !H || !E || !dH || !dE) return TP_ERR_NULL;
  if (!dims_ok({T, h, v}) || N < 1 || v % N) return TP_ERR_SHAPE;
  if (h % 8 || v % 8 || !ptrs_aligned({dlogits, H, E, dH, dE})) return TP_ERR_ALIGN;
  if (tp_status s = require_sm100()) return s;
  cudaStream_t st = as_stream(stream);
  std::vector<int64_t> offs;
  if (tp_status s = shard_offsets(nullptr, v, N, offs)) return s;
  // dH = Σ_i dlogits_i·E_i: the vocabulary shards are the K ranges of one accumulator
  GemmProblem gh;
  gh.A = dlogits; gh.lda = v; gh.a_mn = 0;
  gh.B = E; gh.ldb = h; gh.b_mn = 1;            // E [v,h] = [K, N]
  gh.M = static_cast<int>(T); gh.N = static_cast<int>(h); gh.K = static_cast<int>(v);
  gh.epi = EPI_STORE_BF16;
  gh.out0 = dH; gh.ldo = h;
  gh.dev_status = dev_status;
  if (tp_status s = run_row_parallel(gh, offs, nullptr, nullptr, 0, true, st)) return s;
  // dE = dlogitsᵀ·H, one block of rows per shard
  GemmProblem ge;
  ge.A = dlogits; ge.lda = v; ge.a_mn = 1;      // dlogits [T,v] read as [K, M]
  ge.B = H; ge.ldb = h; ge.b_mn = 1;            // H [T,h] = [K, N]
  ge.M = static_cast<int>(v); ge.N = static_cast<int>(h); ge.K = static_cast<int>(T);
  ge.epi = EPI_STORE_F32;
  ge.out0 = dE; ge.ldo = h;
  ge.dev_status = dev_status;
  return gemm_tc_launch(ge, st);
}

tp_status vp_embed_bwd(const int64_t* ids, const void* dout, int64_t T, int64_t v, int64_t h,
                       int32_t N, float* dE, void* ws, size_t ws_bytes, int32_t* dev_status,
                       void* stream) {
  if (!ids || !dout || !dE) return TP_ERR_NULL;
  if (!dims_ok({T, v, h}) || N < 1 || v % N || T > (1ll << 31) || v > (1ll << 31))
    return TP_ERR_SHAPE;
  if (h % 8 || !ptrs_aligned({dout, dE, ws}) || (reinterpret_cast<uintptr_t>(ids) & 7))
    return TP_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < embed_bwd_ws_bytes(T)) return TP_ERR_WORKSPACE;
  if (tp_status s = require_sm100()) return s;
  return vp_embed_bwd_launch(ids, dout, T, v, h, dE, ws, dev_status, as_stream(stream));
}

}  // extern "C"
