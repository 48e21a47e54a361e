// noalloc.cu — tp_row_linear_fwd_noalloc: the row-parallel linear forward
// for callers that cannot allocate device memory or pass a workspace.
//
// The shards' fp32 partial tiles and the per-tile arrival counters of the
// split shard-sum GEMM live in g_noalloc_scratch, a file-scope static device
// array.  In host code that name is only a host-side stand-in for the
// symbol, never a device address: the address is looked up once per device
// with cudaGetSymbolAddress (with that device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace tpl {
namespace {

constexpr size_t kScratchBytes = TP_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.
tp_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return TP_ERR_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return TP_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace tpl

using namespace tpl;

extern "C" tp_status tp_row_linear_fwd_noalloc(const void* Xin, const void* W, int64_t M,
                                               int64_t Kin, int64_t Nout, int32_t N,
                                               const int64_t* shard_offsets, tp_dtype dt, void* Z,
                                               int32_t* dev_status, void* stream) {
  if (!Xin || !W || !Z) return TP_ERR_NULL;
  if (dt != TP_DTYPE_BF16) return TP_ERR_DTYPE;
  if (M <= 0 || Kin <= 0 || Nout <= 0 || M > (1 << 30) || Kin > (1 << 30) || Nout > (1 << 30))
    return TP_ERR_SHAPE;
  if (N < 1) return TP_ERR_SHAPE;
  if (N > kMaxSplits) return TP_ERR_UNSUPPORTED;
  int64_t offs[kMaxSplits + 1];
  for (int i = 0; i <= N; ++i) {
    if (shard_offsets) {
      offs[i] = shard_offsets[i];
    } else {
      if (Kin % N) return TP_ERR_SHAPE;
      offs[i] = Kin / N * i;
    }
  }
  if (offs[0] != 0 || offs[N] != Kin) return TP_ERR_SHAPE;
  for (int i = 0; i < N; ++i)
    if (offs[i + 1] <= offs[i]) return TP_ERR_SHAPE;
  for (int i = 1; i < N; ++i)
    if (offs[i] % 64) return TP_ERR_UNSUPPORTED;
  if (Kin % 8 || Nout % 8 || !aligned16(Xin) || !aligned16(W) || !aligned16(Z))
    return TP_ERR_ALIGN;
  // one partial per shard (a single shard needs no partials and no scratch)
  const size_t need =
      gemm_split_ws_bytes(static_cast<int>(M), static_cast<int>(Nout), N, false);
  if (need > kScratchBytes) return TP_ERR_WORKSPACE;
  if (tp_status s = require_sm100()) return s;
  void* scratch = nullptr;
  if (tp_status s = scratch_address(&scratch)) return s;

  GemmProblem g;
  g.A = Xin; g.lda = Kin; g.a_mn = 0;
  g.B = W; g.ldb = Nout; g.b_mn = 1;
  g.M = static_cast<int>(M); g.N = static_cast<int>(Nout); g.K = static_cast<int>(Kin);
  g.epi = EPI_STORE_BF16;
  g.out0 = Z; g.ldo = Nout;
  g.dev_status = dev_status;
  g.splits = N;
  for (int s = 0; s <= N; ++s) g.split_k[s] = static_cast<int>(offs[s]);
  g.zpart = nullptr;
  g.ws = scratch;
  g.ws_bytes = kScratchBytes;
  return gemm_tc_launch(g, static_cast<cudaStream_t>(stream));
}
