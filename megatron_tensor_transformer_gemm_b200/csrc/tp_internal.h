// Internal host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "tp.h"

namespace tpi {
struct GemmBatch;
}

struct tp_plan {
  int hidden;
  int ffn;
  int heads;
  int p;
  int head_dim;
  int vocab;         // 0 until tp_plan_set_vocab
  int vocab_padded;  // multiple of 8 * p
  tp_dtype dtype;
  tp_dtype partial_dtype;  // element type of the full-shape partial sums
  tp_act act;
  // Device scratch, allocated on first need (cudaMalloc), grown on demand.
  void* ws;
  size_t ws_bytes;
  int ws_device;
  // Arrival counters of single-launch reductions (zero at rest: the last
  // block of each reduction sets its counter back), allocated on first need;
  // the upper half serves work deferred to the side stream.
  unsigned* cnt;
  int cnt_device;
  // Deferred backward (tp_set_backward_defer): weight gradients and bias sums
  // run on the device's side stream, with scratch of their own (ws2).
  int defer_bwd;
  void* ws2;
  size_t ws2_bytes;
  int ws2_device;
  // Grouped weight gradients (tp_set_wgrad_grouping): the row backward's
  // weight-gradient batch waits here (launched by the next column backward
  // together with its own, or by tp_flush_wgrad) on stream wg_st.
  int group_wgrad;
  tpi::GemmBatch* wg_pend;  // NULL when nothing waits
  cudaStream_t wg_st;
};

namespace tpi {

// Programmatic dependent launch: every kernel of the library begins with
// pdl_entry() (tp_device.cuh) before it touches global memory, so a launch
// may start while the kernel before it on the stream finishes, and its
// wait resolves when that kernel has completed and its writes are visible.
// On unless the environment variable TP_PDL is "0".
bool pdl_enabled();

// Launch `kernel` on `st` with the programmatic-serialization attribute (when
// enabled). Launch errors surface through cudaGetLastError as with <<<>>>.
template <typename... Exp, typename... Act>
inline cudaError_t launch(void (*kernel)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Act&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Act&&>(args)...);
}

// Record `fmt` as this thread's last error and return `s`.
tp_status fail(tp_status s, const char* fmt, ...);
// TP_OK if e == cudaSuccess, else TP_ERR_CUDA with the CUDA error text.
tp_status cuda_status(cudaError_t e, const char* what);
// Check for a launch error right after a kernel launch; counts the launch.
tp_status after_launch(const char* what, int launches = 1);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dsize(tp_dtype t) { return t == TP_BF16 ? 2 : 4; }

// Grid of a persistent kernel: min(units, SMs x resident CTAs of `kernel` at
// `threads` and `smem` bytes of dynamic shared memory), at least 1. Raises the
// kernel's dynamic shared-memory limit to `smem` when needed. Both the limit
// and the occupancy are cached per device, kernel and size, so a repeated call
// makes no driver query.
tp_status persistent_grid(const void* kernel, int threads, int smem, int64_t units, int64_t* grid);

// Device address of this device's status word (set by kernels on a timeout).
tp_status device_status_word(unsigned** out);
// Scratch of at least `bytes` on the current device, owned by the plan.
tp_status workspace(tp_plan* plan, size_t bytes, void** out);
// The plan's kPlanCounters arrival counters on the current device (zero at
// rest). The first call on a device allocates and zeroes them (not allowed
// while `st` is being captured).
constexpr int kPlanCounters = 4096;
tp_status plan_counters(tp_plan* plan, cudaStream_t st, unsigned** out);
// Scratch for the work a deferred backward puts on the side stream (never
// shared with the caller's stream).
tp_status workspace2(tp_plan* plan, size_t bytes, void** out);

// Validation helpers: each returns TP_OK or records an error.
tp_status check_ptr(const void* p, const char* name);
tp_status check_ptrs(const void* const* arr, int n, const char* name, bool allow_null_array);
tp_status check_row_bytes(int64_t cols, tp_dtype t, const char* name);

// Pointer arrays passed to kernels by value.
struct PtrArray {
  const void* p[TP_MAX_SHARDS];
};
struct MutPtrArray {
  void* p[TP_MAX_SHARDS];
};

// ---------------------------------------------------------------- launchers
// Element-wise / copy / reduction kernels (tp_reduce.cu).
tp_status launch_copy_2d(const void* src, int64_t src_ld, void* dst, int64_t dst_ld, int64_t rows,
                         int64_t cols, size_t esize, cudaStream_t st);
// P[i] are of type `pt`; bias, residual and the outputs of type `dt`.
tp_status launch_reduce(const PtrArray& P, int n, const void* bias, const void* residual,
                        const PtrArray& residual_seq, bool res_seq, const MutPtrArray& out,
                        bool out_is_seq, int nout, int64_t T, int64_t cols, tp_dtype pt,
                        tp_dtype dt, cudaStream_t st);
tp_status launch_gather(const PtrArray& src, int n, void* dst, int64_t T, int64_t cols,
                        tp_dtype dt, cudaStream_t st);
// ws_offset: the partials start this many bytes into the plan's workspace
// (a multiple of 256), leaving the bytes before it to concurrent work.
tp_status launch_column_sum(tp_plan* plan, const void* x, int64_t rows, int64_t cols, int64_t ld,
                            float* out, int accumulate, tp_dtype dt, cudaStream_t st,
                            size_t ws_offset = 0);
// The same for n inputs of one shape at once (one launch).
tp_status launch_column_sum_grouped(tp_plan* plan, const PtrArray& x, int n, int64_t rows,
                                    int64_t cols, int64_t ld, const MutPtrArray& out, int accumulate,
                                    tp_dtype dt, cudaStream_t st, size_t ws_offset = 0);
// Column sums deferred to the side stream: partials in workspace2, counters in
// the upper half of the plan's counters.
tp_status launch_column_sum_deferred(tp_plan* plan, const PtrArray& x, int n, int64_t rows,
                                     int64_t cols, int64_t ld, const MutPtrArray& out, tp_dtype dt,
                                     cudaStream_t st);

// LayerNorm (tp_layernorm.cu).
tp_status launch_layernorm_fwd(const PtrArray& x_seq, int n, int64_t rows_per_src, int64_t cols,
                               const void* gamma, const void* beta, void* y, float* mean,
                               float* rstd, tp_dtype dt, cudaStream_t st,
                               const MutPtrArray* ydst = nullptr, int n_dst = 0);
tp_status launch_layernorm_bwd(tp_plan* plan, const void* x, const void* gamma, const void* dy,
                               const float* mean, const float* rstd, const void* dres, void* dx,
                               float* dgamma, float* dbeta, int accumulate, int64_t rows,
                               int64_t cols, tp_dtype dt, cudaStream_t st);

// Vocab-parallel embedding and cross-entropy (tp_vocab.cu).
tp_status launch_embedding_fwd(const int32_t* ids, const PtrArray& E, int vocab, int64_t Vs,
                               int64_t T, int64_t h, tp_dtype dt, void* Y, cudaStream_t st);
tp_status embedding_bwd_workspace(int64_t T, int64_t Vp, size_t* bytes);
tp_status launch_embedding_bwd(const int32_t* ids, int64_t T, const void* dY, int64_t h, int vocab,
                               int64_t Vp, int64_t Vs, const MutPtrArray& dE, tp_dtype dt,
                               void* ws, cudaStream_t st);
tp_status launch_vocab_ce(const PtrArray& L, const MutPtrArray& G, int p, int64_t Vs, int vocab,
                          const int32_t* labels, float scale, float* loss, float* lse, int64_t T,
                          tp_dtype dt, cudaStream_t st);

// Norms of hidden-sharded rows (tp_layernorm.cu).
tp_status launch_norm_sharded_fwd(bool rms, const PtrArray& X, const PtrArray& G,
                                  const PtrArray& B, const MutPtrArray& Y, int p, int64_t rows,
                                  int64_t h, float* mean, float* rstd, tp_dtype dt,
                                  cudaStream_t st);
tp_status launch_norm_sharded_bwd(tp_plan* plan, bool rms, const PtrArray& X, const PtrArray& G,
                                  const PtrArray& DY, const MutPtrArray& DX, const MutPtrArray& dg,
                                  const MutPtrArray& db, int p, int64_t rows, int64_t h,
                                  const float* mean, const float* rstd, tp_dtype dt,
                                  cudaStream_t st, int accumulate = 0,
                                  const PtrArray& DRES = PtrArray{});

// ------------------------------------------------------------------- GEMM
// One GEMM problem of a grouped launch: D[M, N] = A[M, K] . B[N, K]^T.
// A element (m, k) lives at A + m*lda + k when !a_mn (K-major) and at
// A + k*lda + m when a_mn (MN-major); likewise B with (n, k).
enum Epi : int {
  EPI_STORE = 0,       // D = acc (+ bias[n])
  EPI_BIAS_GELU = 1,   // Z = acc + bias; D2 (H) = GELU(Z); D (Z) optional
  EPI_SWIGLU = 2,      // gate/up pair: D (Z = [Zg|Zu]) optional, D2 (H) = SiLU(g) * u
  EPI_DGELU = 3,       // dH = acc; D (dZ) = dH * GELU'(aux Z)
  EPI_DSWIGLU = 4,     // dH = acc; aux = [Zg|Zu]; D (dZ) = [dH*u*SiLU'(g) | dH*SiLU(g)]
};

struct GemmProblem {
  int M, N, K;
  const void* A;
  int64_t lda;
  const void* B;
  int64_t ldb;
  void* D;
  int64_t ldd;
  void* D2;
  int64_t ldd2;
  const void* bias;  // [N] (plan dtype), EPI_STORE / EPI_BIAS_GELU only
  const void* aux;   // Z for EPI_DGELU / EPI_DSWIGLU
  int64_t ldaux;
  int nh;            // SwiGLU: columns of each half ([Zg|Zu] offset of Zu)
};

struct GemmBatch {
  int n;
  GemmProblem g[TP_MAX_SHARDS];
  bool a_mn;
  bool b_mn;
  int epi;
  bool out_f32;  // D written as fp32 (bf16 otherwise)
  // K-concatenated: the n problems are K segments of ONE output, D = sum_i
  // A_i B_i^T (the shards' sum happens in the accumulator). M, N, D, ldd,
  // bias and aux (a residual added in the epilogue) come from g[0]; each
  // g[i] gives A, lda, B, ldb, K of its segment. EPI_STORE only.
  bool kcat;
  // Row scatter of that single output: row r goes to out_seq[r / rows_per_out]
  // (row r % rows_per_out, stride g[0].ldd), plus res_seq[j] rows if given.
  int scatter_n;  // 0 = off, else number of output blocks
  int64_t rows_per_out;
  void* out_seq[TP_MAX_SHARDS];
  const void* res_seq[TP_MAX_SHARDS];
  // Outputs that may be another GPU's memory (a peer group's receive
  // buffers): the epilogue writes them with plain stores, never TMA.
  bool plain_stores;
  // Split K (bf16 path, EPI_STORE, fp32 outputs, every problem with the same
  // K): ksplit > 1 runs each output tile ksplit times over consecutive K
  // ranges, split s writing its fp32 partial at g[i].D + s * split_stride.
  int ksplit;
  int64_t split_stride;
};

// bf16 tcgen05 tensor-core path (tp_gemm_sm100.cu).
tp_status launch_gemm_bf16(const GemmBatch& b, cudaStream_t st);
// Whether a bf16 launch of b has at least as many tiles as CTA units (pairs or
// CTAs) on this device, i.e. leaves no SM idle in its first wave.
bool gemm_fills_gpu(const GemmBatch& b);
// The K split that minimises the estimated time of a batch of plain bf16-output
// GEMMs of equal shape, counting the fp32 partials' reduce (1 = no split, <= 16).
int gemm_split_k(const GemmBatch& b);
// fp32 FMA path (tp_gemm_simt.cu): the same epilogues, grouping and K concatenation.
tp_status launch_gemm_f32(const GemmBatch& b, cudaStream_t st);

// Peer-memory steps (tp_peer.cu): validation of a peer group, and the flag
// raise that follows a grid which wrote into other ranks' memory.
tp_status check_peer_group(const tp_peer_group* g);
tp_status launch_peer_signal(const tp_peer_group* g, int word, uint32_t epoch, cudaStream_t st);

// Attention core (tp_attention.cu).
tp_status launch_attention_fwd(const tp_plan* plan, int batch, int seq, const PtrArray& qkv,
                               const MutPtrArray& o, float* const* lse, cudaStream_t st);
tp_status launch_attention_bwd(tp_plan* plan, int batch, int seq, const PtrArray& qkv,
                               const PtrArray& o, const PtrArray& dO, const float* const* lse,
                               const MutPtrArray& dqkv, cudaStream_t st);

}  // namespace tpi

// Return the status of `expr` from the enclosing function unless it is TP_OK.
#define TP_TRY(expr)            \
  do {                          \
    tp_status _s = (expr);      \
    if (_s != TP_OK) return _s; \
  } while (0)
