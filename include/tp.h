/*
 * tp.h -- C ABI of the single-GPU tensor-parallel (TP) block library, libtp.so.
 *
 * The library computes the Megatron tensor-parallel MLP and attention block
 * with all p shards held as separate buffers on ONE GPU, so each "collective"
 * of the method (all-reduce, reduce-scatter, all-gather) is a local kernel
 * over HBM. Sources, cited by page title and section:
 *   [TP-blog]    "企业官网建设流程全解析" (2kiu.com), a TP walkthrough: §2.1 column
 *                parallel, §2.2 row parallel, §2.3 pairing, §3.1 attention split
 *                by heads, §3.2 MLP with gate/up in one column shard, §3.3
 *                normalisation, §4.1 collectives, §4.3 sequence parallelism,
 *                §6.1 divisibility checks before model init.
 *   [TP-wiki]    "张量并行" (ai-infra-wiki): 两种切法 (Y = GELU(XA)B,
 *                XA = [XA_1, XA_2], XB = X_1B_1 + X_2B_2), 序列维度的补充：Megatron-SP.
 *   [TP-scratch] "大模型分布式训练篇——从零实现 Tensor Parallel" (makesence), §四:
 *                column forward identity / backward all-reduce, and the mirror.
 *   [TP-basics]  "Tensor Parallelism基础：模型切分原理" (bjdmk), 实现细节: the
 *                F.linear [out, in] weight layout, row bias added once after the sum.
 *
 * Conventions for every call
 *   - Pointers named in the argument lists are DEVICE pointers unless stated.
 *     Arrays of per-shard pointers (`const void* const* X`) are HOST arrays of
 *     n (= p unless stated) device pointers; the array itself is read during
 *     the call only.
 *   - Tensors are dense row-major. Weights use the [out, in] layout of
 *     F.linear; activations are [T, features] with T = batch * seq tokens in
 *     sequence-major order (row = s * batch + b), so a sequence shard is a
 *     contiguous block of rows.
 *   - Element types follow the plan dtype (TP_BF16: bf16 storage, fp32
 *     accumulation; TP_F32: fp32 throughout) except where a parameter is
 *     typed `float*`: statistics and bias / LayerNorm-parameter gradients
 *     are always fp32.
 *   - Every device pointer must be 16-byte aligned and every row (the
 *     innermost extent times the element size) a multiple of 16 bytes.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it; they take no locks and never synchronise.
 *   - Ownership: the caller owns every tensor. The plan owns host metadata and
 *     a device workspace that the library allocates (cudaMalloc) the first
 *     time a call needs scratch space and frees in tp_plan_destroy.
 *   - Errors: argument, shape, divisibility and alignment errors are detected
 *     on the host and returned BEFORE any launch, with detail text available
 *     from tp_last_error() (thread-local). A failed launch returns TP_ERR_CUDA.
 *     Kernels never trap: a device wait that runs past its time limit sets a
 *     device status word and the kernel returns; read it with
 *     tp_get_device_status().
 *   - A plan may be used from one host thread at a time.
 */
#ifndef TP_H_
#define TP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TP_MAX_SHARDS 16

#if defined(__GNUC__)
#define TP_API __attribute__((visibility("default")))
#else
#define TP_API
#endif

typedef struct tp_plan tp_plan; /* opaque, host side */

typedef enum {
  TP_OK = 0,
  TP_ERR_ARG = 1,          /* NULL / out-of-range argument */
  TP_ERR_DIVISIBILITY = 2, /* a dimension is not divisible by p ([TP-blog] §6.1) */
  TP_ERR_ALIGN = 3,        /* pointer or row not 16-byte aligned */
  TP_ERR_DTYPE = 4,        /* combination not available for this dtype */
  TP_ERR_UNSUPPORTED = 5,  /* shape beyond what the kernels support */
  TP_ERR_CUDA = 6,         /* CUDA runtime / driver error (detail in tp_last_error) */
  TP_ERR_TIMEOUT = 7,      /* a device-side wait gave up (from tp_get_device_status) */
  TP_ERR_NO_DEVICE = 8     /* no usable sm_100 device */
} tp_status;

typedef enum { TP_F32 = 0, TP_BF16 = 1 } tp_dtype;

/* Activation between the column and the row GEMM of the MLP.
 * GELU is the exact erf form; SWIGLU is H = SiLU(gate) * up with the column
 * shard holding [G_i; U_i] (gate rows first) ([TP-blog] §3.2). */
typedef enum { TP_ACT_NONE = 0, TP_ACT_GELU = 1, TP_ACT_SWIGLU = 2 } tp_act;

/* Which projection a GEMM call is for; fixes the shard shapes.
 *   TP_MLP:     column W1 [n1, hidden] (n1 = ffn, or 2*ffn for SwiGLU),
 *               row W2 [hidden, ffn].
 *   TP_QKV:     column Wqkv [3*hidden, hidden], rows [Wq; Wk; Wv], split by
 *               whole heads ([TP-blog] §3.1). No activation.
 *   TP_OUTPROJ: row Wo [hidden, hidden], input = local heads' outputs.
 *   TP_VOCAB:   column output head W [Vp, hidden] split by vocab rows (Vp the
 *               padded vocab, see tp_plan_set_vocab); no activation. */
typedef enum { TP_MLP = 0, TP_QKV = 1, TP_OUTPROJ = 2, TP_VOCAB = 3 } tp_which;

/* Norm of a hidden-sharded activation (tp_norm_sharded_*). */
typedef enum { TP_NORM_LAYER = 0, TP_NORM_RMS = 1 } tp_norm_kind;

/* ---------------------------------------------------------------- plan */

/* Create a plan for one block. Checks, before anything else ([TP-blog] §6.1):
 * p in [1, TP_MAX_SHARDS]; hidden % p, heads % p, hidden % heads, ffn % p
 * (and the doubled gate+up column count 2*ffn % p for SwiGLU) all zero.
 * ffn may be 0 (attention-only plan); heads may be 0 (MLP-only plan).
 *   partial_dtype: element type of the full-shape partial sums that
 *     tp_row_fwd_partial and tp_column_bwd write and tp_reduce_partials,
 *     tp_reduce_scatter_seq and tp_all_gather_seq_bwd read. Either `dtype`
 *     (the partials travel in the activation type, as an all-reduce of the
 *     layer output would carry them) or TP_F32 (twice the bytes, but each
 *     partial reaches the fp32 sum unrounded: [TP-wiki] notes that the
 *     all-reduce changes the floating-point summation, and this bounds the
 *     change to the one final rounding). TP_F32 plans take TP_F32 only;
 *     anything else returns TP_ERR_DTYPE.
 * Allocates no device memory. Returns TP_ERR_DIVISIBILITY naming the failing
 * dimension (tp_last_error), TP_ERR_ARG for non-positive sizes. */
TP_API tp_status tp_plan_create(int hidden, int ffn, int heads, int p, tp_dtype dtype,
                         tp_act act, tp_dtype partial_dtype, tp_plan** out);
TP_API void tp_plan_destroy(tp_plan* plan);

/* Vocab of the embedding / output head ([TP-blog] §6.2: the vocab is padded
 * up to a size the split divides). Sets the plan's padded vocab Vp, the
 * smallest multiple of 8*p >= vocab (each shard then holds Vp/p rows, a
 * multiple of 8, i.e. 16-byte rows in bf16), and writes it to *vocab_padded
 * (NULL ok). */
TP_API tp_status tp_plan_set_vocab(tp_plan* plan, int vocab, int* vocab_padded);

/* Write a text description of every shard shape into buf (host, n bytes,
 * always NUL-terminated) -- the shape print [TP-blog] §6.1/§6.4 asks for. */
TP_API tp_status tp_plan_describe(const tp_plan* plan, char* buf, size_t n);

TP_API const char* tp_status_string(tp_status s);
TP_API const char* tp_last_error(void);

/* Device-side error report ([TP-blog] §6: fail fast and say why). Synchronises
 * `stream`, reads the device status word of the current device, clears it and
 * returns what it held: TP_OK (nothing happened), TP_ERR_TIMEOUT (a kernel's
 * bounded wait gave up; the kernel returned early and its outputs are
 * undefined) or TP_ERR_ARG (a kernel met an out-of-range token id or label).
 * The word is per device and shared by every plan, so `plan` may be NULL; a
 * non-NULL plan is only validated. If the read itself fails the call returns
 * TP_ERR_CUDA or TP_ERR_NO_DEVICE and leaves the word unchanged. */
TP_API tp_status tp_get_device_status(const tp_plan* plan, void* stream);

/* Self-test of the device-side failure path ([TP-blog] §6: fail fast, never
 * hang). Launches one CTA whose single thread waits, through the same bounded
 * wait every pipelined kernel of the library uses, on an mbarrier that no one
 * will arrive at. After limit_ns nanoseconds (0 < limit_ns <= 1e9, else
 * TP_ERR_ARG) the wait gives up, sets TP_ERR_TIMEOUT in the device status
 * word (read it with tp_get_device_status) and the kernel returns; the
 * context stays usable. gave_up (device int*, NULL ok) receives 1. Faults,
 * traps and hangs nothing. */
TP_API tp_status tp_selftest_wait_timeout(int64_t limit_ns, int* gave_up, void* stream);

/* Number of kernel launches this thread has issued through the library
 * since the last reset (host counter; used to report launch counts). */
TP_API uint64_t tp_launch_count(int reset);

/* ------------------------------------------------------------ sharding
 * Bit-exact copies between a full weight and its p shards.
 * [TP-blog] §2.1 (column: blocks of the output dim), §2.2 (row: blocks of the
 * input dim), §3.1 (QKV: whole heads from each of Wq, Wk, Wv), §3.2 (SwiGLU:
 * shard i = [G rows i*f/p.., U rows i*f/p..]).
 *   column, TP_MLP:  W_full [n1, hidden] -> W_shards[i] [n1/p, hidden]
 *   column, TP_QKV:  W_full [3h, h]      -> W_shards[i] [3h/p, h] = [Q_i; K_i; V_i]
 *   row,    TP_MLP:  W_full [h, ffn]     -> W_shards[i] [h, ffn/p]
 *   row,    TP_OUTPROJ: W_full [h, h]    -> W_shards[i] [h, h/p]
 * The bias variants shard a column bias the same way (vectors). */
TP_API tp_status tp_shard_column(const tp_plan* plan, tp_which which, const void* W_full,
                          void* const* W_shards, void* stream);
TP_API tp_status tp_unshard_column(const tp_plan* plan, tp_which which, const void* const* W_shards,
                            void* W_full, void* stream);
TP_API tp_status tp_shard_row(const tp_plan* plan, tp_which which, const void* W_full,
                       void* const* W_shards, void* stream);
TP_API tp_status tp_unshard_row(const tp_plan* plan, tp_which which, const void* const* W_shards,
                         void* W_full, void* stream);
TP_API tp_status tp_shard_column_bias(const tp_plan* plan, tp_which which, const void* b_full,
                               void* const* b_shards, void* stream);

/* ------------------------------------------------------------- forward */

/* Column-parallel GEMM of every shard in one launch, with its epilogue.
 * [TP-blog] §2.1, [TP-wiki] 两种切法 (XA = [XA_1, ..., XA_p], no communication),
 * [TP-basics] (column bias sharded with its columns).
 *   X:    [T, hidden], replicated input.
 *   W[i]: column shard i (see the sharding calls).
 *   bias: NULL, or bias[i] = shard i of the column bias (length of W[i]'s rows).
 *         Not allowed with SwiGLU.
 *   TP_MLP, GELU:   Z[i] [T, ffn/p] = X W[i]^T + bias[i] (pre-activation, may be
 *                   NULL when no backward follows); H[i] [T, ffn/p] = GELU(Z[i]).
 *   TP_MLP, SWIGLU: Z[i] [T, 2*ffn/p] = [Zg | Zu] (may be NULL);
 *                   H[i] [T, ffn/p] = SiLU(Zg) * Zu.
 *   TP_MLP, NONE:   H[i] = X W[i]^T + bias[i]; Z must be NULL.
 *   TP_QKV:         H[i] [T, 3h/p] = [Q_i | K_i | V_i] = X W[i]^T + bias[i];
 *                   Z must be NULL.
 * bf16 plans run the tcgen05 tensor-core kernel; fp32 plans an fp32 FMA kernel. */
TP_API tp_status tp_column_fwd(tp_plan* plan, tp_which which, int64_t T, const void* X,
                        const void* const* W, const void* const* bias, void* const* Z,
                        void* const* H, void* stream);

/* Row-parallel GEMM of every shard: P[i] [T, hidden] = H[i] W[i]^T, the
 * full-shape partial sums, with NO bias ([TP-blog] §2.2, [TP-wiki] XB = X_1B_1 +
 * X_2B_2). H[i] is [T, ffn/p] (TP_MLP) or [T, h/p] (TP_OUTPROJ); W[i] the row
 * shard; P[i] is stored in the plan's partial dtype. */
TP_API tp_status tp_row_fwd_partial(tp_plan* plan, tp_which which, int64_t T, const void* const* H,
                             const void* const* W, void* const* P, void* stream);

/* Row-parallel GEMM with the sum over shards fused into it: one launch in
 * which every output tile accumulates all p shards' K-slices in the same TMEM
 * accumulator, Y = sum_i H[i] W[i]^T (fp32) + bias once (NULL ok) + residual
 * (NULL ok), rounded once. Same result as tp_row_fwd_partial followed by
 * tp_reduce_partials (TP-blog §2.2, TP-basics: bias once after the sum)
 * without writing or re-reading the p partials. Y [T, hidden]; Y must not
 * alias an input. bf16 plans only. */
TP_API tp_status tp_row_fwd_reduce(tp_plan* plan, tp_which which, int64_t T, const void* const* H,
                                   const void* const* W, const void* bias, const void* residual,
                                   void* Y, void* stream);

/* The same with the sequence-parallel reduce-scatter fused in (TP-blog §4.3):
 * rows [j*T/p, (j+1)*T/p) of the sum (+ bias, + residual_seq[j]) go to
 * Y_seq[j] [T/p, hidden]. residual_seq may be NULL. */
TP_API tp_status tp_row_fwd_reduce_scatter_seq(tp_plan* plan, tp_which which, int64_t T,
                                               const void* const* H, const void* const* W,
                                               const void* bias, const void* const* residual_seq,
                                               void* const* Y_seq, void* stream);

/* The all-reduce of the row layer, done locally: Y = sum_{i<n} P[i] (fp32, in
 * order 0..n-1), then + bias once (NULL ok), then + residual (NULL ok).
 * [TP-blog] §2.2, [TP-basics] (bias once, after the sum). P[i] [T, hidden] in
 * the plan's partial dtype; residual, Y [T, hidden] and bias [hidden] in the
 * plan dtype. Y may alias residual. */
TP_API tp_status tp_reduce_partials(tp_plan* plan, int64_t T, int n, const void* const* P,
                             const void* bias, const void* residual, void* Y, void* stream);

/* Sequence-parallel form of the reduction ([TP-blog] §4.3, [TP-wiki] Megatron-SP):
 * Y_seq[j] [T/n, hidden] = rows [j*T/n, (j+1)*T/n) of (sum_i P[i] + bias),
 * plus residual_seq[j] (NULL array ok). T % n must be 0. Types as
 * tp_reduce_partials (P[i] in the partial dtype). */
TP_API tp_status tp_reduce_scatter_seq(tp_plan* plan, int64_t T, int n, const void* const* P,
                                const void* bias, const void* const* residual_seq,
                                void* const* Y_seq, void* stream);

/* All-gather along the sequence: X_full [T, hidden] = rows of X_seq[0..n-1]
 * ([T/n, hidden] each) in order. Bit-exact copy. */
TP_API tp_status tp_all_gather_seq(tp_plan* plan, int64_t T, int n, const void* const* X_seq,
                            void* X_full, void* stream);

/* LayerNorm over the full hidden dim ([TP-blog] §3.3): y = (x - mean) * rstd *
 * gamma + beta, biased variance, eps = 1e-5. x, y [rows, hidden]; gamma, beta
 * [hidden]; mean, rstd [rows] fp32 outputs (either may be NULL). The mean and
 * then the variance about it are two exact passes over the row (fp32).
 * hidden a multiple of 8 and <= 16384 (bf16) or 8192 (fp32), else
 * TP_ERR_UNSUPPORTED. */
TP_API tp_status tp_layernorm_fwd(tp_plan* plan, int64_t rows, const void* x, const void* gamma,
                           const void* beta, void* y, float* mean, float* rstd, void* stream);

/* LayerNorm on each sequence shard fused with the all-gather that follows it
 * in Megatron-SP ([TP-blog] §4.3): Y_full row j*T/n + r = LN(X_seq[j] row r)
 * (each row is read from its shard once and written to Y_full once).
 * mean, rstd: [T] fp32 in full-sequence order (NULL ok). Limits and numerics
 * as tp_layernorm_fwd. */
TP_API tp_status tp_layernorm_all_gather_seq(tp_plan* plan, int64_t T, int n, const void* const* X_seq,
                                      const void* gamma, const void* beta, void* Y_full,
                                      float* mean, float* rstd, void* stream);

/* Vocab-parallel embedding lookup ([TP-blog] §6.2, [TP-wiki] 工程实践): E[i]
 * [Vp/p, hidden] is shard i of the padded embedding (vocab ids [i*Vp/p,
 * (i+1)*Vp/p)); ids [T] int32 (device). Y [T, hidden] = the row of the owning
 * shard, i.e. the sum over shards of the partial lookups (each shard
 * contributes zeros outside its range). Ids outside [0, vocab) give a zero
 * row and set the device status word (tp_get_device_status -> TP_ERR_ARG). */
TP_API tp_status tp_embedding_fwd(tp_plan* plan, int64_t T, const int32_t* ids,
                                  const void* const* E, void* Y, void* stream);

/* Backward of the lookup: dE[i] [Vp/p, hidden] (plan dtype, overwritten) =
 * for each vocab row v of shard i, the sum over tokens with id == v of dY[t]
 * (fp32, in token order, deterministic); rows no token uses are zero; ids
 * outside [0, vocab) are skipped. Uses the plan's device workspace (a stable
 * bucket sort of the token indices, about Vp/16 * (ceil(T/1024) + 1) + 2 T ints).
 * TP_ERR_UNSUPPORTED for Vp > 196608 or T > 2^31 - 1. */
TP_API tp_status tp_embedding_bwd(tp_plan* plan, int64_t T, const int32_t* ids, const void* dY,
                                  void* const* dE, void* stream);

/* Vocab-parallel cross-entropy on sharded logits ([TP-blog] §6.2: each shard
 * computes only its vocab slice's logits and partial loss; the per-row
 * scalars -- local max, local sum of exponentials, target logit -- are
 * reduced over shards). logits[i] [T, Vp/p] (e.g. from tp_column_fwd with
 * TP_VOCAB); labels [T] int32 (device; < 0 = ignored token). loss [T] fp32 =
 * logsumexp over the real vocab columns (padding excluded) minus the target
 * logit (0 for ignored tokens); lse [T] fp32 (NULL ok). dlogits[i] (NULL array
 * skips; may alias logits[i]) = (softmax - onehot) * grad_scale, zero on
 * padding columns and ignored tokens. Labels >= vocab set the device status. */
TP_API tp_status tp_vocab_cross_entropy(tp_plan* plan, int64_t T, const void* const* logits,
                                        const int32_t* labels, float grad_scale, float* loss,
                                        float* lse, void* const* dlogits, void* stream);

/* LayerNorm / RMSNorm of rows whose hidden dim is split over the p shards,
 * with the statistics formed the way [TP-blog] §3.3 describes: every shard's
 * local sums (sum x and sum x^2; RMSNorm only sum x^2) are summed over shards
 * into one scalar per row, and every shard normalises its slice with them.
 *   X[i], Y[i]: [rows, hidden/p] (columns [i*h/p, (i+1)*h/p) of the row);
 *   gamma[i], beta[i]: [hidden/p] (beta ignored, may be NULL, for RMSNorm);
 *   mean (LayerNorm only), rstd: [rows] fp32 outputs (NULL ok).
 * LayerNorm uses var = E[x^2] - mean^2 (the local-sums form), eps = 1e-5.
 * hidden/p must be a multiple of 8; hidden <= 16384 (bf16) or 8192 (fp32),
 * else TP_ERR_UNSUPPORTED. */
TP_API tp_status tp_norm_sharded_fwd(tp_plan* plan, tp_norm_kind kind, int64_t rows,
                                     const void* const* X, const void* const* gamma,
                                     const void* const* beta, void* const* Y, float* mean,
                                     float* rstd, void* stream);

/* Causal attention of each shard's local heads ([TP-blog] §3.1: full sequence,
 * whole heads, no cross-shard step). QKV[i] [seq*batch, 3*h/p] = [Q_i|K_i|V_i]
 * (the TP_QKV column output); O[i] [seq*batch, h/p] with head j of the shard
 * in columns [j*d, (j+1)*d); LSE[i] [batch, heads/p, seq] fp32 log-sum-exp of
 * each row's scaled, masked scores (NULL ok when no backward follows).
 * softmax(Q K^T / sqrt(d), causal j <= i) V. */
TP_API tp_status tp_attention_fwd(tp_plan* plan, int batch, int seq, const void* const* QKV,
                           void* const* O, float* const* LSE, void* stream);

/* ------------------------------------------------------------ backward */

/* Streams of the backward calls (scheduling only: the pages' backward
 * ([TP-scratch] §四) fixes what is computed, not the launch order, and has no
 * counterpart of these switches): tp_row_bwd (dZ and dW) and the column
 * backward calls (dX and dW) issue two GEMMs that read the same inputs. When
 * either leaves SMs idle (few output tiles), the activation-gradient GEMM runs
 * on a side stream the library creates per device, forked from `stream` by an
 * event, and `stream` waits for it before the call returns: the results are
 * ordered on `stream` as with one stream, also inside a stream capture (the
 * fork and join become graph edges). Environment TP_BWD_CONCURRENT=0 keeps
 * every launch on `stream`. Calls on one plan must not overlap in time (they
 * share the plan's workspace). */

/* Deferred backward (a scheduling option; the results are the same): with
 * on != 0, the plan's bf16 tp_row_bwd and column backward calls run the
 * activation gradient (dZ / dX) on `stream` and put the weight gradient (no K
 * split) and the bias sums on the device's side stream, forked from `stream`
 * at the call, and do NOT join them: dW and dbias are valid on a stream only
 * after tp_backward_join on it. They read the call's inputs (dY, H, X, dZ)
 * when they run, so those buffers must stay unchanged until the join, and the
 * call's dW / dbias must not be read before it. Deferred bias sums use scratch
 * of their own, so later calls of the same plan may run meanwhile. TP_ERR_ARG
 * if plan is NULL. */
TP_API tp_status tp_set_backward_defer(tp_plan* plan, int on);

/* Make `stream` wait for all work issued so far on the current device's side
 * stream (the deferred weight gradients and bias sums of every plan). An
 * event wait: it returns at once on the host, and works inside a capture. */
TP_API tp_status tp_backward_join(void* stream);

/* Grouped weight gradients (on != 0): tp_row_bwd leaves its weight-gradient
 * GEMM (dW_i = dY^T H_i) waiting in the plan, and the next tp_column_bwd*
 * call on the same plan and stream launches it together with its own
 * (dW_i = dZ_i^T X) as one grouped GEMM over both shard sets: the same tiles
 * and results, one partly empty last wave instead of two. Until then dW of
 * the row backward is not written, and its inputs dY and H must stay
 * unchanged. tp_flush_wgrad launches a waiting one alone (on the stream it was
 * issued on); so does any backward call that cannot take it along (another
 * stream, the deferred mode, a GEMM on the side stream, no dW), and switching
 * grouping off. bf16 plans; fp32 plans run every GEMM at once. */
TP_API tp_status tp_set_wgrad_grouping(tp_plan* plan, int on);
TP_API tp_status tp_flush_wgrad(tp_plan* plan);

/* Row layer backward for every shard ([TP-scratch] §四: the input gradient of
 * the row layer needs no reduction; dY is replicated).
 *   dY [T, hidden]; H[i] the row input of shard i; W[i] the row shard.
 *   TP_MLP: dZ[i] = act'(dH_i) with dH_i = dY W[i]: GELU: dZ[i] [T, ffn/p] =
 *     dH_i * GELU'(Z[i]); SWIGLU: Z[i] = [Zg|Zu], dZ[i] [T, 2ffn/p] =
 *     [dH_i * Zu * SiLU'(Zg) | dH_i * SiLU(Zg)]; NONE: dZ[i] = dH_i.
 *   TP_OUTPROJ: dZ[i] [T, h/p] = dY W[i] (Z ignored).
 *   dW[i] = dY^T H[i] (shape of W[i]; NULL array skips);
 *   dbias [hidden] fp32 = sum over tokens of dY, computed once (NULL skips). */
TP_API tp_status tp_row_bwd(tp_plan* plan, tp_which which, int64_t T, const void* dY,
                     const void* const* H, const void* const* W, const void* const* Z,
                     void* const* dZ, void* const* dW, float* dbias, void* stream);

/* Column layer backward for every shard ([TP-scratch] §四: forward identity,
 * backward sum of the input gradient).
 *   X [T, hidden]; dZ[i] the gradient of shard i's pre-activation output;
 *   W[i] the column shard. dW[i] = dZ[i]^T X (NULL array skips); dbias[i] fp32
 *   = sum over tokens of dZ[i] (NULL array skips); dX_partials[i] [T, hidden] =
 *   dZ[i] W[i] in the plan's partial dtype, to be summed by tp_reduce_partials
 *   (or tp_all_gather_seq_bwd). */
TP_API tp_status tp_column_bwd(tp_plan* plan, tp_which which, int64_t T, const void* X,
                        const void* const* dZ, const void* const* W, void* const* dW,
                        float* const* dbias, void* const* dX_partials, void* stream);

/* Column layer backward with the sum of the input gradient fused into its
 * GEMM ([TP-scratch] §四: the column layer's backward all-reduces dX): dW[i],
 * dbias[i] as in tp_column_bwd; dX [T, hidden] = sum_i dZ[i] W[i] accumulated
 * over all shards in one TMEM accumulator and rounded once. bf16 plans only. */
TP_API tp_status tp_column_bwd_reduce(tp_plan* plan, tp_which which, int64_t T, const void* X,
                                      const void* const* dZ, const void* const* W, void* const* dW,
                                      float* const* dbias, void* dX, void* stream);

/* The same with the sequence-parallel reduce-scatter fused in: rows
 * [j*T/p, (j+1)*T/p) of dX go to dX_seq[j] [T/p, hidden]. */
TP_API tp_status tp_column_bwd_reduce_scatter_seq(tp_plan* plan, tp_which which, int64_t T,
                                                  const void* X, const void* const* dZ,
                                                  const void* const* W, void* const* dW,
                                                  float* const* dbias, void* const* dX_seq,
                                                  void* stream);

/* Backward of tp_reduce_scatter_seq: the all-gather of the dY sequence shards
 * into dY_full [T, hidden] (the conjugate of the reduce-scatter, [TP-wiki]
 * Megatron-SP). */
TP_API tp_status tp_reduce_scatter_seq_bwd(tp_plan* plan, int64_t T, int n, const void* const* dY_seq,
                                    void* dY_full, void* stream);

/* Backward of tp_all_gather_seq: the reduce-scatter of the n full-shape dX
 * partials (partial dtype) into sequence shards dX_seq[j] [T/n, hidden]
 * (plan dtype). */
TP_API tp_status tp_all_gather_seq_bwd(tp_plan* plan, int64_t T, int n, const void* const* dX_partials,
                                void* const* dX_seq, void* stream);

/* LayerNorm backward ([TP-blog] §3.3: the statistics span the whole hidden
 * dim, so dx of a row needs the row's two reductions; §4.3 / [TP-wiki]
 * Megatron-SP: LayerNorm runs on sequence shards with replicated gamma and
 * beta, so their gradients are sums over every shard's rows).
 * dx [rows, hidden] (plan dtype) = rstd * (g - mean_h(g) - xhat * mean_h(g *
 * xhat)) with g = dy * gamma and xhat = (x - mean) * rstd; dgamma = sum_rows
 * dy * xhat, dbeta = sum_rows dy, [hidden] fp32 (deterministic; when
 * accumulate != 0 they are added to the existing contents, so the sequence
 * shards' sums can be chained). mean/rstd from the forward. dres (NULL ok,
 * [rows, hidden], may alias dx) is added to dx: the gradient of the residual
 * branch around a pre-LN sublayer (x1 = x + f(LN(x)) gives dx = dres +
 * LN'(x)^T df), so the sum needs no launch of its own. Uses the plan's
 * device workspace for per-CTA partials. */
TP_API tp_status tp_layernorm_bwd(tp_plan* plan, int64_t rows, const void* x, const void* gamma,
                           const void* dy, const float* mean, const float* rstd, const void* dres,
                           void* dx, float* dgamma, float* dbeta, int accumulate, void* stream);

/* Backward of tp_norm_sharded_fwd: dX[i] [rows, hidden/p]; dgamma[i] (and
 * dbeta[i] for LayerNorm; NULL array ok) [hidden/p] fp32 sums over rows
 * (deterministic: fixed per-CTA partials in the plan's workspace, summed in a
 * fixed order). The per-row means of the backward are again local sums
 * reduced over shards. One pass over X and dY. */
TP_API tp_status tp_norm_sharded_bwd(tp_plan* plan, tp_norm_kind kind, int64_t rows,
                                     const void* const* X, const void* const* gamma,
                                     const void* const* dY, const float* mean, const float* rstd,
                                     void* const* dX, float* const* dgamma, float* const* dbeta,
                                     void* stream);

/* Attention backward of each shard's local heads ([TP-blog] §3.1: a shard's
 * attention touches only its own whole heads over the full sequence, so the
 * backward, like the forward, has no cross-shard step; the shard sum follows
 * in the QKV column backward). From QKV[i], O[i], dO[i] and LSE[i] of the
 * forward, writes dQKV[i] [seq*batch, 3h/p] = [dQ|dK|dV], the chain rule of
 * softmax(Q K^T / sqrt(d), causal) V with P recomputed from LSE:
 * dV = P^T dO; dS = P * (dO V^T - rowsum(dO * O)); dQ = dS K / sqrt(d);
 * dK = dS^T Q / sqrt(d). bf16 plans, head_dim 64 or 128. */
TP_API tp_status tp_attention_bwd(tp_plan* plan, int batch, int seq, const void* const* QKV,
                           const void* const* O, const void* const* dO,
                           const float* const* LSE, void* const* dQKV, void* stream);

/* Column sums over rows: out[c] = sum_r x[r, c] in fp32 (fixed order;
 * accumulate != 0 adds to out) -- the bias gradient of a layer, db = the sum
 * over tokens of its output gradient ([TP-basics] 实现细节: the row bias is
 * one full vector, so its gradient is the column sum of dY once; the column
 * bias shard i gets the column sums of dZ_i). x [rows, cols] in the plan
 * dtype. One launch:
 * blocks sum row splits into the plan's workspace and the last block of each
 * column slab adds the splits in order. The plan's first reduction on a
 * device allocates its workspace and arrival counters, so it must not be the
 * first call inside a stream capture (TP_ERR_ARG). */
TP_API tp_status tp_column_sum(tp_plan* plan, int64_t rows, int64_t cols, const void* x, float* out,
                        int accumulate, void* stream);

/* Column sums that allocate nothing: same result as tp_column_sum (out[c] =
 * sum_r x[r, c] in fp32, x [rows, cols] of `dtype`, accumulate != 0 adds to
 * out), for callers that cannot call cudaMalloc -- for example a framework
 * whose caching allocator already owns the device memory (a cudaMalloc from
 * the side can fail or fragment its pool), or a latency-sensitive loop that
 * must not pay cudaMalloc's implicit device synchronisation. It takes no plan.
 * The pages have no counterpart of this call; it exists for such callers only.
 *   - Scratch: a fixed device array inside libtp.so of 512 Ki floats (2 MiB);
 *     every GPU that loads the library holds it until the process exits.
 *     cols > 524288 returns TP_ERR_UNSUPPORTED; larger column counts lower the
 *     number of row splits (each split needs cols floats).
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture. Under CUDA's lazy module loading that first call is
 *     also where the library's module, and with it the array, is loaded onto
 *     the device: the driver reserves the 2 MiB then, and the call may
 *     synchronise. A caller that needs no allocation at all inside some
 *     section makes one call first (rows = 0 is enough: it writes zeros, or
 *     nothing in accumulate mode, to out) before entering it.
 *   - x must be dense: row r starts at x + r * cols (no leading dimension).
 *   - The cached address belongs to the device's current context: calls
 *     after cudaDeviceReset in the same process are not supported.
 *   - Every call shares the one array, so calls that overlap on the GPU (two
 *     streams, or two host threads) race and corrupt each other's sums:
 *     serialise them. Each call overwrites every scratch entry it reads, so
 *     nothing from an earlier call leaks into a later one.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call
 *     (beyond the module load of the first call, above). */
TP_API tp_status tp_column_sum_static(int64_t rows, int64_t cols, tp_dtype dtype, const void* x,
                                      float* out, int accumulate, void* stream);

/* ------------------------------------------------------------------------
 * Across GPUs over peer memory: the p shards split over `world` ranks (one
 * process per GPU), every rank's buffers mapped into every other rank's
 * address space with CUDA IPC. The row layer's all-reduce ([TP-blog] §4.1:
 * each GPU holds a partial sum and every GPU needs the full result) is split
 * into a reduce-scatter and an all-gather ([TP-wiki] 序列维度的补充：
 * Megatron-SP: all-reduce = reduce-scatter + all-gather at the same traffic),
 * and the reduce-scatter's transfer is fused into the GEMM that produces the
 * partial sum. Three asynchronous calls on the caller's stream, each taken by
 * every rank with the same `epoch` (a counter that starts at 1 and grows by
 * one per all-reduce; the group's flag words start at zero):
 *   1. push    tp_row_fwd_push_peer / tp_column_bwd_push_peer: the GEMM sums
 *              this rank's shards in its accumulator and its epilogue stores
 *              row block j (rows [j*T/world, (j+1)*T/world)) straight into
 *              rank j's receive buffer, slot <rank>, with plain stores through
 *              the peer mapping; then this rank's "arrived" flag is raised on
 *              every rank.
 *   2. reduce  tp_peer_reduce: waits until every rank's block has arrived,
 *              sums the world slots in rank order in fp32, adds bias and
 *              residual once, rounds once, stores the block to each of the
 *              n_out destinations (every rank's output at this rank's rows:
 *              the all-gather; or this rank's sequence shard only: the
 *              Megatron-SP reduce-scatter), then raises this rank's "done"
 *              flag on every rank.
 *   3. wait    tp_peer_wait: waits until every rank's "done" flag is up: all
 *              of this rank's output blocks have been written, and every rank
 *              has finished reading its receive buffer, so the next push may
 *              begin.
 * Waits are bounded (tp_peer_set_wait_limit, default 5 s): a rank that never
 * arrives makes the waiting kernel set TP_ERR_TIMEOUT in the device status
 * word and return. bf16 plans only. No call here issues a TMA load, and no
 * library kernel is given a peer's memory. */
#define TP_PEER_HANDLE_BYTES 64
#define TP_PEER_FLAG_WORDS (2 * TP_MAX_SHARDS) /* [0, MAX): arrived from rank s; [MAX, 2 MAX): done */
#define TP_PEER_FLAG_BYTES 256                  /* flag words padded to keep what follows aligned */

typedef struct tp_peer_group {
  int world;                      /* ranks, 1..TP_MAX_SHARDS */
  int rank;                       /* this rank, 0..world-1 */
  int64_t recv_elems;             /* capacity of each receive buffer, in elements */
  uint32_t* flags[TP_MAX_SHARDS]; /* rank d's TP_PEER_FLAG_WORDS flag words (device, zeroed) */
  void* recv[TP_MAX_SHARDS];      /* rank d's receive buffer (device): world slots of [T/world, hidden] */
} tp_peer_group;

/* Buffers of the exchange above ([TP-blog] §4.1: every GPU holds a partial
 * sum that the others need; here each rank's receive buffer and flag words,
 * mapped into the other ranks' processes).
 * Device memory that other processes can map: `bytes` (> 0) from cudaMalloc
 * on the current device, zero-filled, its IPC handle written to `handle`
 * (TP_PEER_HANDLE_BYTES host bytes). Free with tp_peer_free. */
TP_API tp_status tp_peer_alloc(size_t bytes, void** ptr, void* handle);
TP_API tp_status tp_peer_free(void* ptr);
/* Map another process's tp_peer_alloc memory (its handle bytes) into this
 * process; unmap with tp_peer_close. A handle from this same process is
 * refused by CUDA (TP_ERR_CUDA): a rank uses its own pointer directly. */
TP_API tp_status tp_peer_open(const void* handle, void** ptr);
TP_API tp_status tp_peer_close(void* ptr);
/* Wait limit of the peer waits in nanoseconds, (0, 60e9]; 0 restores the
 * default. Applies to launches made after the call, from any thread. */
TP_API tp_status tp_peer_set_wait_limit(int64_t ns);

/* Step 1 for the row layer: Y_r = sum over this rank's p shards of H[i]
 * W[i]^T (fp32 accumulator, rounded once to bf16), row block j pushed into
 * g->recv[j] slot g->rank ([T/world, hidden] at element offset
 * rank*(T/world)*hidden). No bias or residual here (step 2 adds them once).
 * T % world == 0 and T*hidden <= g->recv_elems. */
TP_API tp_status tp_row_fwd_push_peer(tp_plan* plan, tp_which which, int64_t T, const void* const* H,
                                      const void* const* W, const tp_peer_group* g, uint32_t epoch,
                                      void* stream);
/* Step 1 for the column layer's backward ([TP-scratch] §四: the input
 * gradient is all-reduced): dW[i], dbias[i] as in tp_column_bwd, and dX_r =
 * sum over this rank's shards of dZ[i] W[i] pushed by row block as above. */
TP_API tp_status tp_column_bwd_push_peer(tp_plan* plan, tp_which which, int64_t T, const void* X,
                                         const void* const* dZ, const void* const* W, void* const* dW,
                                         float* const* dbias, const tp_peer_group* g, uint32_t epoch,
                                         void* stream);
/* Step 2: out[k] [T/world, hidden] = sum_{s<world} slot s of this rank's
 * receive buffer (fp32, in order 0..world-1) + bias [hidden] (NULL ok) +
 * residual [T/world, hidden] (this rank's rows; NULL ok), rounded to bf16,
 * for k < n_out (1 <= n_out <= TP_MAX_SHARDS; out is a host array of device
 * pointers, local or peer). hidden % 8 == 0. */
TP_API tp_status tp_peer_reduce(const tp_peer_group* g, int64_t T, int hidden, const void* bias,
                                const void* residual, int n_out, void* const* out, uint32_t epoch,
                                void* stream);
/* Step 3: the stream waits (on the device) for every rank's step 2. */
TP_API tp_status tp_peer_wait(const tp_peer_group* g, uint32_t epoch, void* stream);

/* The Megatron-SP all-gather along the sequence ([TP-wiki] Megatron-SP: the
 * next layer's column GEMM needs the whole sequence) over peer memory, in two
 * of the steps above: this rank's shard is stored into out[d] (rank d's
 * gathered buffer at this rank's rows, [rows, cols]) for every d < world with
 * plain stores, then this rank's "done" word is raised on every rank; then
 * tp_peer_wait (step 3, same epoch) waits until every rank's shard has
 * arrived. A gathered buffer is written by the next all-gather's pushes, so
 * its readers must have finished by then: in a layer they do, because the
 * exchange that follows them (the reduce-scatter and its wait) cannot finish
 * on any rank before every rank has passed them. x and out[d] bf16, dense,
 * cols % 8 == 0. */
TP_API tp_status tp_all_gather_push_peer(const tp_peer_group* g, int64_t rows, int cols, const void* x,
                                         void* const* out, uint32_t epoch, void* stream);
/* The same with the LayerNorm of the shard fused in ([TP-blog] §3.3, as
 * tp_layernorm_fwd: x [rows, hidden] of this rank, gamma, beta [hidden], mean
 * and rstd [rows] fp32 (NULL ok)): each normalised row is pushed to every
 * rank's gathered buffer. bf16 plans only. */
TP_API tp_status tp_layernorm_all_gather_push_peer(tp_plan* plan, const tp_peer_group* g, int64_t rows,
                                                   const void* x, const void* gamma, const void* beta,
                                                   void* const* out, float* mean, float* rstd,
                                                   uint32_t epoch, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TP_H_ */
