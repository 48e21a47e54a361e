/*
 * tplayers.h — C ABI of the B200 tensor-parallel layers library (libtplayers.so).
 *
 * Megatron-style tensor parallelism on ONE GPU: the N shards of a layer are
 * partitions of device memory, and the sums the pages perform with
 * all-reduces (the g operator after the row-parallel GEMM, the f operator in
 * backward, the embedding and the cross-entropy reductions) are on-device
 * reductions fused into the kernels that produce the partials.
 *
 * Sources, cited by page title and section:
 *   [MLP-TP] "Megatron-LM：张量并行与大规模训练" (astro-blog-cod.pages.dev),
 *            §2.1 MLP 层的张量并行, §2.2 Self-Attention 的张量并行.
 *   [TP-ILL] tensor-model-parallel illustrated (m.youleyou.com/wenzhang/3143730),
 *            §1.1 按行切分权重, §1.2 按列切分权重, §2.1 MLP层的张量模型并行计算方法,
 *            §3.1 Multihead-Attention的计算方法, §4.1 输入层Embedding,
 *            §4.2 输出层Embedding, §5 Cross-Entropy层.
 *   [APX]    "Megatron-LM 介绍" (apxml.com), §核心贡献 (column-parallel Y_i = X·A_i).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All matrices are dense ROW-MAJOR with no padding: X [M,h], A [h,F],
 *    bias [F], B [F,h], Z [M,h] (the pages' math orientation, not the
 *    [out,in] weight layout).  Shard i of A owns columns [off_i, off_{i+1});
 *    shard i of B owns the same range of rows.
 *  - shard_offsets: nullable int64 HOST array of N+1 increasing offsets with
 *    off_0 = 0 and off_N = F.  NULL means the even split off_i = i*F/N, which
 *    requires F % N == 0 (else TP_ERR_SHAPE).
 *  - The CALLER OWNS EVERY BUFFER.  The library never allocates or frees
 *    memory and never synchronises; all work is enqueued on `stream`
 *    (a cudaStream_t, passed as void*; NULL = legacy default stream) and the
 *    call returns before it completes.
 *  - Every size (M, h, F, K, Nout, T, v, b·s, ...) lies in [1, 2^30]; a size
 *    outside that range returns TP_ERR_SHAPE.  An empty batch is therefore
 *    not a call: skip it on the host.
 *  - Argument errors are returned synchronously, before anything is
 *    enqueued.  Errors found on the device (an id or target out of range, a
 *    bounded wait that ran out) are OR-ed as TP_DEVERR_* bits into
 *    *dev_status, an int32 in device memory (nullable); read it after the
 *    stream has completed.
 *  - bf16 tensors: base pointers 16-byte aligned and every row length a
 *    multiple of 8 elements (the tensor-memory-accelerator copy rule);
 *    fp32 tensors: 16-byte aligned, row lengths a multiple of 4.  Violations
 *    return TP_ERR_ALIGN.
 *  - bf16 storage, fp32 accumulation; every bf16 store rounds to nearest even.
 *  - Thread safety: calls on different streams may overlap as long as they
 *    do not share output or workspace buffers.
 */
#ifndef TPLAYERS_H_
#define TPLAYERS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TP_API __attribute__((visibility("default")))
#else
#define TP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t tp_status;

enum {
  TP_OK = 0,
  TP_ERR_NULL = 1,        /* a required pointer is NULL */
  TP_ERR_SHAPE = 2,       /* a size is <= 0, inconsistent, or not divisible as required */
  TP_ERR_ALIGN = 3,       /* a pointer or row length breaks the alignment rules above */
  TP_ERR_DTYPE = 4,       /* unknown dtype or activation code */
  TP_ERR_UNSUPPORTED = 5, /* valid request the library does not implement */
  TP_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed while enqueueing */
  TP_ERR_WORKSPACE = 7,   /* workspace NULL or smaller than tp_workspace_bytes() */
  TP_ERR_DEVICE = 8       /* no usable sm_100 device is current */
};

/* Bits OR-ed into *dev_status by the kernels. */
enum {
  TP_DEVERR_RANGE = 1,    /* an embedding id or xent target outside [0, v) */
  TP_DEVERR_TIMEOUT = 2   /* a bounded pipeline wait ran out; outputs are garbage */
};

typedef enum { TP_DTYPE_BF16 = 0, TP_DTYPE_F32 = 1 } tp_dtype;

/* Activation of the column-parallel GEMM.  The pages name GeLU without a
 * formula; GELU_TANH = 0.5·x·(1 + tanh(√(2/π)·(x + 0.044715·x³))) is the
 * default, GELU_ERF = x·Φ(x). */
typedef enum { TP_ACT_NONE = 0, TP_ACT_GELU_TANH = 1, TP_ACT_GELU_ERF = 2 } tp_act;

/* Operations whose workspace size tp_workspace_bytes() reports. */
typedef enum {
  TP_OP_MLP_FWD = 0,
  TP_OP_MLP_BWD = 1,
  TP_OP_ROW_LINEAR_FWD = 2,
  TP_OP_COL_LINEAR_BWD = 3,
  TP_OP_ROW_LINEAR_BWD = 4,
  TP_OP_EMBED_BWD = 5,    /* pass (T, h, v, N): T tokens */
  TP_OP_LINEAR_XENT = 6,  /* pass (T, h, v, N) */
  TP_OP_SP_LN_BWD = 7,    /* pass (M, h, h, N): M token rows of width h */
  TP_OP_ATTENTION_BWD = 8 /* pass (b·s, n_heads, 64, N) */
} tp_op;

/*
 * Diagnostics: check the bounded-wait path on the device.  Launches one CTA
 * that waits, with the same bounded mbarrier wait the kernels use, on a
 * barrier that nothing arrives on.  After limit_us microseconds the wait
 * gives up, the kernel ORs TP_DEVERR_TIMEOUT into *dev_status (required) and
 * returns normally: no trap, no fault, the context stays usable.
 */
TP_API tp_status tp_selftest_wait_timeout(int32_t* dev_status, uint32_t limit_us, void* stream);

/*
 * Diagnostics: exercise the real pipeline's failure path.  Arms a one-shot
 * injection for the NEXT tensor-core GEMM launch of this process (any entry
 * point; the TP-MLP forward's first launch is its column GEMM): in that
 * launch the TMA producers of the CTA (pair) that owns work unit `unit`
 * stop, without a word, before loading k-block `kblock` of it, as a
 * producer that died would.  The MMA issuer's wait for that k-block then
 * runs out after wait_limit_us (the launch's every bounded wait uses that
 * limit); the kernel ORs TP_DEVERR_TIMEOUT into *dev_status, lets the copies
 * and MMAs already issued finish, frees its tensor memory and returns.  The
 * outputs of that launch are garbage; later launches are unaffected.  Units
 * are numbered split-major over the output tiles (unit 0 is the first K range
 * of the first tile); an injection naming a unit or k-block the launch does
 * not reach does nothing.  Host-side only: nothing here faults or traps.
 *   Returns TP_ERR_SHAPE for a negative unit or kblock, or a limit of 0 or
 *   above 10 s.
 */
TP_API tp_status tp_debug_stall_next_gemm(int32_t unit, int32_t kblock, uint32_t wait_limit_us);

/* Human-readable text of a status code (static storage, never NULL). */
TP_API const char* tp_status_string(tp_status s);

/* Library version as 10000*major + 100*minor + patch. */
TP_API int32_t tp_version(void);

/* Number of kernels this library has enqueued since it was loaded (all
 * devices, all threads).  Diagnostics only: lets a caller count the
 * library's launches inside a timed region. */
TP_API uint64_t tp_launch_count(void);

/*
 * Workspace bytes an op needs for these sizes (M rows, h model width,
 * F = ffn / output width, N shards).  For TP_OP_ROW_LINEAR_FWD pass
 * (M, Nout, Kin, N).  Returns 0 when the op needs none.  The library
 * clears the parts that must start at zero on every call.
 */
TP_API size_t tp_workspace_bytes(tp_op op, int64_t M, int64_t h, int64_t F, int32_t N);

/*
 * TP-MLP forward   [MLP-TP] §2.1 (formula and pseudocode); [TP-ILL] §2.1.
 *
 *   f forward is the identity: every shard reads the same X.
 *   Shard i:  U_i = X·A_i + bias_i,  Y_i = act(U_i),  Z_i = Y_i·B_i.
 *   g forward: Z = Σ_i Z_i (the all-reduce), fused on the device: the
 *   row-parallel GEMM walks the shards' K ranges and sums them in its
 *   accumulator or, in split mode, in a fixed-order epilogue reduction.
 *
 *   X    [M,h]   dt           in
 *   A    [h,F]   dt           in   (column shards)
 *   bias [F]     dt           in   nullable (= zero)
 *   B    [F,h]   dt           in   (row shards)
 *   U    [M,F]   dt           out  pre-activation, kept for backward
 *   Y    [M,F]   dt           out  activation, kept for backward
 *   Z    [M,h]   dt           out
 *   Zpart [N,M,h] fp32        out  nullable: each shard's partial Z_i before
 *                                  the sum (needs every off_i % 64 == 0 in bf16)
 *   ws, ws_bytes                   workspace, >= tp_workspace_bytes(TP_OP_MLP_FWD, M, h, F, N)
 *                                  (may be NULL when that is 0)
 */
TP_API tp_status tp_mlp_fwd(const void* X, const void* A, const void* bias, const void* B,
                     int64_t M, int64_t h, int64_t F, int32_t N,
                     const int64_t* shard_offsets, tp_dtype dt, tp_act act,
                     void* U, void* Y, void* Z, float* Zpart,
                     void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * TP-MLP backward   [TP-ILL] §1.1, §1.2, §2.1 (f and g backward).
 *
 *   g backward is the identity: dZ reaches every shard.
 *   Shard i:  dU_i = (dZ·B_iᵀ) ⊙ act'(U_i)     (dGeLU fused in the epilogue)
 *             dB_i = Y_iᵀ·dZ,  dA_i = Xᵀ·dU_i,  dbias_i = Σ_rows dU_i
 *   f backward: dX = Σ_i dU_i·A_iᵀ (the all-reduce), fused like Z above.
 *
 *   X, A, B, U, Y, dZ   as in/out of the forward (U, Y from tp_mlp_fwd)
 *   dU    [M,F] dt      out  (also the intermediate that dA and dX read)
 *   dX    [M,h] dt      out
 *   dA    [h,F] dt      out
 *   dbias [F]   fp32    out  nullable
 *   dB    [F,h] dt      out
 *   ws, ws_bytes        >= tp_workspace_bytes(TP_OP_MLP_BWD, M, h, F, N)
 */
TP_API tp_status tp_mlp_bwd(const void* X, const void* A, const void* B, const void* U,
                     const void* Y, const void* dZ,
                     int64_t M, int64_t h, int64_t F, int32_t N,
                     const int64_t* shard_offsets, tp_dtype dt, tp_act act,
                     void* dU, void* dX, void* dA, float* dbias, void* dB,
                     void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * TP-MLP backward with activation recompute   [FW] "Megatron-LM框架概览"
 * §3.2 (the recompute row of the feature table: activations are dropped
 * after the forward and rebuilt in the backward); [EVO] Megatron history page
 * §2.3 "序列并行与激活重计算" (selective recompute of the MLP's costliest part).
 *
 *   Exactly tp_mlp_bwd, except that the forward's activation Y is not an
 *   input: only the pre-activation U [M,F] was kept.  The dGeLU GEMM, which
 *   reads U for act'(U) anyway, also writes Y = act(U) into Y [M,F] (an
 *   output here, bf16 or fp32 like U), and the dB GEMM reads it from there.
 *   Y may be a scratch buffer shared between layers, or U itself: every
 *   element of U is read by the thread that then overwrites it, so Y == U
 *   recomputes in place (U is then lost).  Same workspace as
 *   TP_OP_MLP_BWD; same errors.
 */
TP_API tp_status tp_mlp_bwd_recompute(const void* X, const void* A, const void* B, const void* U,
                                      void* Y, const void* dZ,
                                      int64_t M, int64_t h, int64_t F, int32_t N,
                                      const int64_t* shard_offsets, tp_dtype dt, tp_act act,
                                      void* dU, void* dX, void* dA, float* dbias, void* dB,
                                      void* ws, size_t ws_bytes, int32_t* dev_status,
                                      void* stream);

/*
 * Column-parallel linear, forward   [TP-ILL] §1.2; [APX] §核心贡献; the QKV
 * projection of [MLP-TP] §2.2 / [TP-ILL] §3.1 with per-shard heads.
 *
 *   U = X·W + bias, Y = act(U) over all N column shards of W in one launch.
 *   X [M,K] in; W [K,Nout] in; bias [Nout] nullable; Y [M,Nout] out;
 *   U [M,Nout] out, required unless act == TP_ACT_NONE (then may be NULL).
 *   shard_offsets partition Nout (e.g. 3·64·heads_i for per-shard heads).
 *   The shard boundaries do not change any value: a column split is exact.
 */
TP_API tp_status tp_col_linear_fwd(const void* X, const void* W, const void* bias,
                            int64_t M, int64_t K, int64_t Nout, int32_t N,
                            const int64_t* shard_offsets, tp_dtype dt, tp_act act,
                            void* U, void* Y, int32_t* dev_status, void* stream);

/*
 * Column-parallel linear, backward   [TP-ILL] §1.2 (f backward sums the
 * shards' dX partials).
 *
 *   dU = dY ⊙ act'(U) (dU may alias dY when act == NONE: then it is not
 *   written); dW = Xᵀ·dU [K,Nout]; dbias = Σ_rows dU [Nout] fp32 (nullable);
 *   dX = Σ_i dU_i·W_iᵀ [M,K].
 */
TP_API tp_status tp_col_linear_bwd(const void* X, const void* W, const void* U, const void* dY,
                            int64_t M, int64_t K, int64_t Nout, int32_t N,
                            const int64_t* shard_offsets, tp_dtype dt, tp_act act,
                            void* dU, void* dX, void* dW, float* dbias,
                            void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * Row-parallel linear, forward   [TP-ILL] §1.1; the output projection of
 * [MLP-TP] §2.2 followed by its all-reduce.
 *
 *   Z = Σ_i Xin[:, off_i:off_{i+1}]·W[off_i:off_{i+1}, :]   Xin [M,Kin],
 *   W [Kin,Nout], Z [M,Nout] dt; Zpart [N,M,Nout] fp32 nullable as above.
 */
TP_API tp_status tp_row_linear_fwd(const void* Xin, const void* W,
                            int64_t M, int64_t Kin, int64_t Nout, int32_t N,
                            const int64_t* shard_offsets, tp_dtype dt,
                            void* Z, float* Zpart,
                            void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * Row-parallel linear, backward   [TP-ILL] §1.1 (g backward is the identity).
 *
 *   dXin = dZ·Wᵀ [M,Kin] (each shard's columns are its own dX_i);
 *   dW = Xinᵀ·dZ [Kin,Nout].
 */
TP_API tp_status tp_row_linear_bwd(const void* Xin, const void* W, const void* dZ,
                            int64_t M, int64_t Kin, int64_t Nout, int32_t N,
                            const int64_t* shard_offsets, tp_dtype dt,
                            void* dXin, void* dW, int32_t* dev_status, void* stream);

/*
 * Row-parallel linear forward that allocates nothing.  (No counterpart on
 * the pages: this is a deployment variant of tp_row_linear_fwd.)
 *
 * Some callers cannot call cudaMalloc or pass in a workspace: code that runs
 * inside a host framework which owns every device allocation, or a plugin
 * whose interface only hands over input and output pointers.  This entry
 * point computes the same Z = Σ_i Xin_i·W_i as tp_row_linear_fwd, always
 * with one partial product per shard and the fused fixed-order sum, but keeps
 * the shards' fp32 partials and the per-tile counters in a scratch array
 * that is a static __device__ variable of the library.
 *
 *   - Scratch: TP_NOALLOC_SCRATCH_BYTES per GPU, reserved on every GPU that
 *     loads the library and held until the process exits.  Calls whose
 *     partials do not fit (ceil(M/128)·ceil(Nout/256)·N tiles of 128 KB plus
 *     a counter each) return TP_ERR_WORKSPACE without enqueueing anything.
 *   - bf16 only (TP_ERR_DTYPE otherwise); N <= 16; every shard offset a
 *     multiple of 64 (TP_ERR_UNSUPPORTED otherwise).
 *   - The first call in a CUDA context looks up the scratch address there
 *     (cudaGetSymbolAddress, with the caller's device and context current)
 *     and caches it for that context, so callers on their own contexts, or
 *     on a primary context created again after cudaDeviceReset, get an
 *     address valid where they run; make that first call before any stream
 *     capture.  No call allocates or frees memory.
 *   - Every call on a device shares the one scratch array, and it keeps the
 *     previous call's contents (the counters are cleared by each call).
 *     Calls that overlap on the GPU — on two streams, or from two threads —
 *     race on it and give wrong results: serialise them.
 *   Arguments as for tp_row_linear_fwd (no Zpart, no workspace).
 */
#define TP_NOALLOC_SCRATCH_BYTES (32u << 20)
TP_API tp_status tp_row_linear_fwd_noalloc(const void* Xin, const void* W,
                                           int64_t M, int64_t Kin, int64_t Nout, int32_t N,
                                           const int64_t* shard_offsets, tp_dtype dt,
                                           void* Z, int32_t* dev_status, void* stream);

/*
 * Vocabulary-parallel input embedding   [TP-ILL] §4.1.
 *
 *   The table E [v,h] is split into N contiguous row ranges
 *   [i·v/N, (i+1)·v/N) (needs v % N == 0).  Shard i returns E[id] for the ids
 *   in its range and a zero row otherwise; the N results are summed.  The
 *   kernel forms that sum as an owner select: exactly one shard owns each
 *   in-range id, so the sum is that shard's row (bit for bit, for every
 *   value except -0.0, which the literal sum with +0.0 would turn into +0.0).
 *   Ids outside [0, v) give a zero row and set TP_DEVERR_RANGE.
 *
 *   ids [T] int64 in (device); E [v,h] dt in; out [T,h] dt out.
 */
TP_API tp_status vp_embed(const int64_t* ids, int64_t T, const void* E, int64_t v, int64_t h,
                   int32_t N, tp_dtype dt, void* out, int32_t* dev_status, void* stream);

/*
 * Output-embedding logits   [TP-ILL] §4.2 (the output layer shares the word
 * embedding table): logits[:, lo_i:hi_i] = H·E_iᵀ for every vocabulary
 * shard i, one launch, no gather (the blocks are written side by side).
 *
 *   H [T,h] bf16 in; E [v,h] bf16 in; logits [T,v] fp32 out.  v % N == 0.
 */
TP_API tp_status tp_logits_fwd(const void* H, const void* E, int64_t T, int64_t h, int64_t v,
                        int32_t N, float* logits, int32_t* dev_status, void* stream);

/*
 * Vocabulary-parallel softmax cross-entropy   [TP-ILL] §5.
 *
 *   Row t of logits [T,v] fp32 is split into N contiguous vocabulary ranges
 *   (v % N == 0).  Each shard computes its maximum m_i, its sum
 *   s_i = Σ exp(l − m_i), its share of the target logit and its arg-max; the
 *   shards combine m = max m_i, S = Σ s_i·exp(m_i − m) (the all-reduce of the
 *   softmax denominators, with the maxima added for range safety) and
 *
 *     loss[t]    = log S + m − l[t, y_t]
 *     dlogits    = grad_scale · (exp(l − m)/S − onehot(y_t))   (nullable)
 *     argmax[t]  = lowest index of the row maximum (int32, nullable)
 *     loss_sum   = Σ_t loss[t] in a fixed order (fp32 [1], nullable)
 *
 *   targets [T] int64 (device).  A target outside [0, v) sets
 *   TP_DEVERR_RANGE, its loss is NaN and its dlogits row is NaN.
 *   dlogits may alias logits (in-place gradient).
 */
TP_API tp_status vp_xent(const float* logits, const int64_t* targets, int64_t T, int64_t v,
                  int32_t N, float grad_scale, float* loss, float* loss_sum,
                  float* dlogits, int32_t* argmax, int32_t* dev_status, void* stream);

/*
 * Vocabulary-parallel cross-entropy with a bf16 gradient   [TP-ILL] §5.
 *
 *   Exactly vp_xent, except that dlogits [T,v] is written in bf16 (round to
 *   nearest even), the storage the output-layer backward GEMMs read; it is
 *   required here and may not alias the fp32 logits.
 */
TP_API tp_status vp_xent_bf16_grad(const float* logits, const int64_t* targets, int64_t T,
                                   int64_t v, int32_t N, float grad_scale, float* loss,
                                   float* loss_sum, void* dlogits, int32_t* argmax,
                                   int32_t* dev_status, void* stream);

/*
 * Output-embedding backward   [TP-ILL] §4.2 (the output layer shares the word
 * embedding table).
 *
 *   dH = Σ_i dlogits_i·E_i   [T,h] bf16 — vocabulary shard i holds columns
 *        [i·v/N, (i+1)·v/N) of dlogits and rows of E; the shards' partials are
 *        summed in one accumulator (the all-reduce of the pages' layout);
 *   dE = dlogitsᵀ·H          [v,h] fp32 — each shard's block of rows is its own.
 *
 *   dlogits [T,v] bf16, H [T,h] bf16, E [v,h] bf16 in; v % N == 0,
 *   v % 8 == 0, h % 8 == 0.  dE is overwritten (see vp_embed_bwd to add the
 *   input-side gradient of a tied table).
 */
TP_API tp_status tp_logits_bwd(const void* dlogits, const void* H, const void* E, int64_t T,
                               int64_t h, int64_t v, int32_t N, void* dH, float* dE,
                               int32_t* dev_status, void* stream);

/*
 * Vocabulary-parallel input-embedding backward   [TP-ILL] §4.1, §4.2.
 *
 *   dE[x] += Σ_{t: ids[t] = x} dout[t]   for every x in [0, v): shard i adds
 *   the gradient rows of the ids in its own range [i·v/N, (i+1)·v/N).  The
 *   sum over repeated ids runs in token order (tokens sorted by (id, token)),
 *   so the result is bitwise reproducible; each touched row is written once.
 *   Adding onto the dE of tp_logits_bwd gives the gradient of a table shared
 *   by the input and output layers (the sum the pages prescribe).
 *
 *   ids [T] int64 (device), dout [T,h] bf16, dE [v,h] fp32 (read and
 *   written); ids outside [0, v) are skipped and set TP_DEVERR_RANGE.
 *   ws, ws_bytes >= tp_workspace_bytes(TP_OP_EMBED_BWD, T, h, v, N).
 */
TP_API tp_status vp_embed_bwd(const int64_t* ids, const void* dout, int64_t T, int64_t v,
                              int64_t h, int32_t N, float* dE, void* ws, size_t ws_bytes,
                              int32_t* dev_status, void* stream);

/*
 * Attention core between the projections, per-shard heads   [MLP-TP] §2.2;
 * [TP-ILL] §3.1 (heads are independent, so each GPU computes attention for
 * its own heads with no communication; only the output projection's sum
 * follows).
 *
 *   For every sequence and head:  O = softmax(Q·Kᵀ·scale + mask)·V, with the
 *   causal mask (key j hidden from query i for j > i) when causal != 0.
 *
 *   QKV [b·s, 3·n_heads·64] bf16: the column-parallel projection's output in
 *   the shard-major layout — shard i (heads [head_offsets[i],
 *   head_offsets[i+1])) holds its Q heads, then its K heads, then its V
 *   heads, each head 64 columns; row = batch·s + position.
 *   ctx [b·s, n_heads·64] bf16 out: heads in order, so shard i's context is
 *   the column block [64·head_offsets[i], 64·head_offsets[i+1]) — the input of
 *   its rows of tp_row_linear_fwd.  lse [b, n_heads, s] fp32 (nullable): the
 *   natural-log sum of exp of each query's scaled, masked scores.
 *   head_offsets: N+1 increasing head indices from 0 to n_heads, or NULL for
 *   the contiguous split that gives the first n_heads mod N shards one head
 *   more (25 heads over 4: 7, 6, 6, 6).  scale <= 0 selects 1/sqrt(64).
 *   head_dim must be 64 and n_heads <= 256 (else TP_ERR_UNSUPPORTED); any
 *   s >= 1.  QKV and ctx 16-byte aligned.
 *   The formula is an image lost from the pages; this is the standard
 *   scaled dot-product attention of the GPT-2 layer, without dropout.
 */
TP_API tp_status tp_attention_fwd(const void* QKV, int64_t b, int64_t s, int32_t n_heads,
                                  int32_t head_dim, int32_t N, const int64_t* head_offsets,
                                  int32_t causal, float scale, void* ctx, float* lse,
                                  int32_t* dev_status, void* stream);

/*
 * Backward of the attention core, per-shard heads   [MLP-TP] §2.2;
 * [TP-ILL] §3.1 (each shard differentiates its own heads; no communication).
 *
 *   For every sequence and head, with P = softmax(Q·Kᵀ·scale + mask) and
 *   dO the gradient at the context:
 *     dV = Pᵀ·dO,  dS = P ⊙ (dO·Vᵀ − rowsum(dO ⊙ O)),
 *     dQ = scale·dS·K,  dK = scale·dSᵀ·Q,
 *   written into dQKV [b·s, 3·n_heads·64] bf16 in the same shard-major layout
 *   as QKV (the upstream gradient of the column-parallel projection).
 *
 *   QKV as in tp_attention_fwd; ctx [b·s, n_heads·64] bf16 its output O;
 *   dctx the same shape, the gradient dO; lse [b, n_heads, s] fp32 from
 *   tp_attention_fwd.  causal, scale and head_offsets must be the forward's.
 *   One CTA per 128-key tile of a head computes that tile's dK and dV rows
 *   (reproducible bit for bit) and adds its share of dQ into an fp32
 *   accumulator in the workspace; the adds of different key tiles land in
 *   any order, so dQ may differ between runs by the rounding of that sum.
 *   ws, ws_bytes >= tp_workspace_bytes(TP_OP_ATTENTION_BWD, b·s, n_heads,
 *   64, N) (rowsum(dO ⊙ O) per query and head, then the fp32 dQ
 *   accumulator, b·s·n_heads·64 floats).  head_dim 64, n_heads <= 256.
 */
TP_API tp_status tp_attention_bwd(const void* QKV, const void* ctx, const void* dctx,
                                  const float* lse, int64_t b, int64_t s, int32_t n_heads,
                                  int32_t head_dim, int32_t N, const int64_t* head_offsets,
                                  int32_t causal, float scale, void* dQKV, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * Sequence-parallel dropout-add-LayerNorm   [EVO] Megatron history page §2.3
 * "序列并行与激活重计算" (LayerNorm and Dropout split along the sequence:
 * each shard handles its own token rows, so their activations are split too).
 *
 *   hs = residual + keep · (x + bias) / (1 − p)            [M,h] bf16 out
 *   y  = (hs − mean)·rstd·gamma + beta                      [M,h] bf16 out
 *   mean, rstd [M] fp32 out: mean and 1/sqrt(biased variance + eps) of hs
 *   as stored (bf16).
 *
 *   Shard i owns rows [i·M/N, (i+1)·M/N) (M % N == 0); on one device all
 *   shards run in one launch.  keep: element e = row·h + col uses word e mod 4
 *   of Philox4x32-10 (Salmon et al., SC 2011) at counter (e div 4 as two
 *   32-bit words, offset as two 32-bit words) under key seed (two 32-bit
 *   words), and is kept when the word is >= floor(p·2^32); 0 <= p < 1, p = 0
 *   disables dropout.  keep_out [M,h] uint8 (nullable) receives the mask.
 *   x, residual, gamma, beta bf16; bias [h] bf16 nullable; h % 8 == 0,
 *   h <= 8192, pointers 16-byte aligned.  The formulas are not printed on
 *   the pages: this is the transformer's residual step as Megatron writes it.
 *   For h <= 2048 the rows reach shared memory by bulk copy and every wait
 *   for a copy is bounded: if one runs out, TP_DEVERR_TIMEOUT is ORed into
 *   *dev_status (nullable) and the rows not yet computed are left as they
 *   were.
 */
TP_API tp_status tp_sp_dropout_add_ln_fwd(const void* x, const void* bias, const void* residual,
                                          const void* gamma, const void* beta, int64_t M,
                                          int64_t h, int32_t N, float p, uint64_t seed,
                                          uint64_t offset, float eps, void* hs, void* y,
                                          float* mean, float* rstd, uint8_t* keep_out,
                                          int32_t* dev_status, void* stream);

/*
 * Its backward, same passage.  dy [M,h]: gradient at y; dhs_in [M,h]
 * (nullable): gradient reaching the residual stream hs from later layers.
 *
 *   dresidual = rstd·(g − mean(g) − xhat·mean(g·xhat)) + dhs_in,
 *               g = dy·gamma, xhat = (hs − mean)·rstd      [M,h] bf16 out
 *   dx        = keep · dresidual / (1 − p)                   [M,h] bf16 out
 *   dgamma = Σ_rows dy·xhat, dbeta = Σ_rows dy, dbias = Σ_rows dx   [h] fp32
 *
 *   The row sums are each shard's partial gradients summed over the shards
 *   (the sequence-parallel all-reduce), in a fixed order.  keep is
 *   regenerated from (p, seed, offset), which must be the forward's.
 *   dbias nullable.  ws, ws_bytes >= tp_workspace_bytes(TP_OP_SP_LN_BWD, M,
 *   h, h, N).
 */
TP_API tp_status tp_sp_dropout_add_ln_bwd(const void* dy, const void* dhs_in, const void* hs,
                                          const void* gamma, const float* mean, const float* rstd,
                                          int64_t M, int64_t h, int32_t N, float p, uint64_t seed,
                                          uint64_t offset, void* dx, void* dresidual,
                                          float* dgamma, float* dbeta, float* dbias, void* ws,
                                          size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * Output layer and cross-entropy in one pass, without the logits matrix
 *   [TP-ILL] §4.2 (logits = H·Eᵀ against the shared table) and §5 (the loss
 *   from per-part maxima and rescaled sums, so that no part of the [T,v]
 *   logits has to be gathered).
 *
 *   The logits GEMM keeps its accumulators on chip: for every 128-column
 *   slice of every row it records the maximum m_k, s_k = Σ exp(l − m_k), the
 *   first column holding m_k and, in the slice that holds the target, the
 *   target logit.  A second kernel combines the slices by §5's rule,
 *   m = max m_k, S = Σ s_k·exp(m_k − m), and writes
 *
 *     loss[t]    = m + log S − l[t, y_t]            fp32 [T]
 *     lse[t]     = m + log S                        fp32 [T]   (nullable)
 *     argmax[t]  = lowest index of the row maximum  int32 [T]  (nullable)
 *     loss_sum   = Σ_t loss[t], fixed order         fp32 [1]   (nullable)
 *
 *   The vocabulary shards i (rows [i·v/N, (i+1)·v/N) of E, v % N == 0) are
 *   memory partitions of E; the slices are a finer partition of the same
 *   columns, combined by the same rule.  H [T,h] bf16, E [v,h] bf16,
 *   targets [T] int64; h % 8 == 0, H and E 16-byte aligned.  A target outside
 *   [0, v) sets TP_DEVERR_RANGE and gives loss NaN.
 *   ws, ws_bytes >= tp_workspace_bytes(TP_OP_LINEAR_XENT, T, h, v, N)
 *   (the slice statistics: 12·ceil(v/128)·T bytes plus 4·T).
 *   No counterpart of the fused form is printed on the pages: it is their
 *   output-layer GEMM and §5 loss evaluated without storing the logits.
 */
TP_API tp_status tp_linear_xent_fwd(const void* H, const void* E, const int64_t* targets,
                                    int64_t T, int64_t h, int64_t v, int32_t N, float* loss,
                                    float* loss_sum, float* lse, int32_t* argmax, void* ws,
                                    size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * Gradient of that loss with respect to the logits, recomputed   [TP-ILL] §5.
 *
 *   dlogits[t, j] = grad_scale · (exp(l[t, j] − lse[t]) − [j = y_t])   bf16 [T,v]
 *
 *   with l = H·Eᵀ recomputed by the GEMM in fp32 and lse from
 *   tp_linear_xent_fwd, so that the fp32 logits are never stored; the result
 *   is the input of tp_logits_bwd.  v % 8 == 0, h % 8 == 0, H, E and dlogits
 *   16-byte aligned.  A row whose target lies outside [0, v) is NaN and sets
 *   TP_DEVERR_RANGE.
 */
TP_API tp_status tp_linear_xent_dlogits(const void* H, const void* E, const int64_t* targets,
                                        const float* lse, int64_t T, int64_t h, int64_t v,
                                        int32_t N, float grad_scale, void* dlogits,
                                        int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TPLAYERS_H_ */
