// noalloc.cu — tp_row_linear_fwd_noalloc: the row-parallel linear forward
// for callers that cannot allocate device memory or pass a workspace.
//
// The shards' fp32 partial tiles and the per-tile arrival counters of the
// split shard-sum GEMM live in g_noalloc_scratch, a file-scope static device
// array.  In host code that name is only a host-side stand-in for the
// symbol, never a device address: the address is looked up with
// cudaGetSymbolAddress while the caller's device (and context) is current,
// and cached per CUDA context, so a caller on a context of its own (or on a
// primary context created again after cudaDeviceReset) gets the address that
// is valid in that context.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace tpl {
namespace {

constexpr size_t kScratchBytes = TP_NOALLOC_SCRATCH_BYTES;
constexpr int kCacheSlots = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct ScratchSlot {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
ScratchSlot g_scratch_cache[kCacheSlots];
int g_scratch_next = 0;
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch array in the current context.  The first
// call in a context makes the runtime load the library's module there (and
// may create the device's primary context), so it belongs before any stream
// capture.
tp_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return TP_ERR_DEVICE;
  }
  CtxGetCurrentFn get = ctx_get_current_fn();
  if (get == nullptr) return TP_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return TP_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (ctx != nullptr)
    for (const ScratchSlot& s : g_scratch_cache)
      if (s.ctx == ctx && s.addr != nullptr) {
        *out = s.addr;
        return TP_OK;
      }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return TP_ERR_CUDA;
  }
  // with no context current before, the lookup made the device's primary
  // context current
  if (ctx == nullptr && (get(&ctx) != CUDA_SUCCESS || ctx == nullptr)) return TP_ERR_CUDA;
  // A context handle can be reused after its context is destroyed; the new
  // context then simply replaces the old entry's address on its first call.
  ScratchSlot& slot = g_scratch_cache[g_scratch_next];
  g_scratch_next = (g_scratch_next + 1) % kCacheSlots;
  slot.ctx = ctx;
  slot.addr = p;
  *out = p;
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
