// extern "C" entry points of libtp.so: plan management, host-side validation
// and dispatch to the kernels. Every check happens before any launch.
#include <cuda.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <tuple>
#include <new>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {
thread_local char g_last_error[1024] = "";
thread_local uint64_t g_launches = 0;

__device__ unsigned g_device_status;  // per device: bit 0 = a wait timed out

constexpr int kMaxDevices = 64;
unsigned* g_status_addr[kMaxDevices] = {};
std::mutex g_status_mu;

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
}  // namespace

namespace tp_selftest {
// One thread waits, through the same bounded wait the pipelined kernels use,
// on an mbarrier that expects one arrival which never comes: the wait gives
// up after limit_ns, sets the status word and the kernel returns.
__global__ void selftest_wait_kernel(unsigned* status, uint64_t limit_ns, int* gave_up) {
  tpd::pdl_entry();
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  tpd::mbar_init(&bar, 1);
  abort_flag = 0;
  tpd::fence_barrier_init();
  const bool ok = tpd::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
  if (gave_up) *gave_up = ok ? 0 : 1;
}
}  // namespace tp_selftest

namespace tpi {

tp_status fail(tp_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

tp_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return TP_OK;
  return fail(TP_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("TP_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

tp_status after_launch(const char* what, int launches) {
  g_launches += static_cast<uint64_t>(launches);
  return cuda_status(cudaGetLastError(), what);
}

namespace {
std::mutex g_occ_mu;
std::map<std::tuple<int, const void*, int, int>, int> g_occ;  // (dev, kernel, threads, smem) -> CTAs per SM
std::map<std::pair<int, const void*>, int> g_smem_limit;        // (dev, kernel) -> dynamic smem limit set
int g_sms[kMaxDevices] = {};
}  // namespace

tp_status persistent_grid(const void* kernel, int threads, int smem, int64_t units, int64_t* grid) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return fail(TP_ERR_NO_DEVICE, "no current CUDA device");
  }
  std::lock_guard<std::mutex> lk(g_occ_mu);
  if (!g_sms[dev]) {
    int n = 0;
    tp_status s = cuda_status(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev),
                              "cudaDeviceGetAttribute(SM count)");
    if (s != TP_OK) return s;
    g_sms[dev] = n > 0 ? n : 1;
  }
  const auto key = std::make_tuple(dev, kernel, threads, smem);
  auto it = g_occ.find(key);
  if (it == g_occ.end()) {
    int& lim = g_smem_limit[std::make_pair(dev, kernel)];
    if (smem > lim) {
      tp_status s = cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                                "cudaFuncSetAttribute(dynamic shared memory)");
      if (s != TP_OK) return s;
      lim = smem;
    }
    int per_sm = 0;
    tp_status s = cuda_status(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem),
                              "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (s != TP_OK) return s;
    it = g_occ.emplace(key, per_sm > 0 ? per_sm : 1).first;
  }
  *grid = std::max<int64_t>(1, std::min<int64_t>(units, static_cast<int64_t>(g_sms[dev]) * it->second));
  return TP_OK;
}

tp_status device_status_word(unsigned** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return fail(TP_ERR_NO_DEVICE, "no current CUDA device");
  }
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_addr[dev]) {
    void* p = nullptr;
    tp_status s = cuda_status(cudaGetSymbolAddress(&p, g_device_status), "cudaGetSymbolAddress");
    if (s != TP_OK) return s;
    g_status_addr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_status_addr[dev];
  return TP_OK;
}

tp_status workspace(tp_plan* plan, size_t bytes, void** out) {
  int dev = 0;
  tp_status s = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (s != TP_OK) return s;
  if (plan->ws && (plan->ws_bytes < bytes || plan->ws_device != dev)) {
    // Grow (or move to another device): release the old block first. The
    // caller's stream may still use it, so wait for the device.
    cudaDeviceSynchronize();
    int cur = dev;
    if (plan->ws_device != dev) cudaSetDevice(plan->ws_device);
    cudaFree(plan->ws);
    if (plan->ws_device != dev) cudaSetDevice(cur);
    plan->ws = nullptr;
    plan->ws_bytes = 0;
  }
  if (!plan->ws) {
    size_t want = bytes < (1u << 20) ? (1u << 20) : bytes;
    s = cuda_status(cudaMalloc(&plan->ws, want), "cudaMalloc(workspace)");
    if (s != TP_OK) {
      plan->ws = nullptr;
      return s;
    }
    plan->ws_bytes = want;
    plan->ws_device = dev;
  }
  *out = plan->ws;
  return TP_OK;
}

tp_status plan_counters(tp_plan* plan, cudaStream_t st, unsigned** out) {
  int dev = 0;
  tp_status s = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (s != TP_OK) return s;
  if (plan->cnt && plan->cnt_device == dev) {
    *out = plan->cnt;
    return TP_OK;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return fail(TP_ERR_ARG, "the plan's first reduction on a device must run before a stream capture");
  }
  if (plan->cnt) {  // moved to another device
    cudaDeviceSynchronize();
    cudaSetDevice(plan->cnt_device);
    cudaFree(plan->cnt);
    cudaSetDevice(dev);
    plan->cnt = nullptr;
  }
  void* p = nullptr;
  s = cuda_status(cudaMalloc(&p, 2 * kPlanCounters * sizeof(unsigned)), "cudaMalloc(counters)");
  if (s != TP_OK) return s;
  // zero, and finished, before any kernel on any stream can use them
  s = cuda_status(cudaMemsetAsync(p, 0, 2 * kPlanCounters * sizeof(unsigned), st), "cudaMemsetAsync(counters)");
  if (s == TP_OK) s = cuda_status(cudaStreamSynchronize(st), "cudaStreamSynchronize(counters)");
  if (s != TP_OK) {
    cudaFree(p);
    return s;
  }
  plan->cnt = static_cast<unsigned*>(p);
  plan->cnt_device = dev;
  *out = plan->cnt;
  return TP_OK;
}

tp_status workspace2(tp_plan* plan, size_t bytes, void** out) {
  int dev = 0;
  tp_status s = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (s != TP_OK) return s;
  if (plan->ws2 && (plan->ws2_bytes < bytes || plan->ws2_device != dev)) {
    cudaDeviceSynchronize();  // side-stream work may still use the old block
    int cur = dev;
    if (plan->ws2_device != dev) cudaSetDevice(plan->ws2_device);
    cudaFree(plan->ws2);
    if (plan->ws2_device != dev) cudaSetDevice(cur);
    plan->ws2 = nullptr;
    plan->ws2_bytes = 0;
  }
  if (!plan->ws2) {
    size_t want = bytes < (1u << 20) ? (1u << 20) : bytes;
    s = cuda_status(cudaMalloc(&plan->ws2, want), "cudaMalloc(side workspace)");
    if (s != TP_OK) {
      plan->ws2 = nullptr;
      return s;
    }
    plan->ws2_bytes = want;
    plan->ws2_device = dev;
  }
  *out = plan->ws2;
  return TP_OK;
}

tp_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(TP_ERR_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(TP_ERR_ALIGN, "%s (%p) is not 16-byte aligned", name, p);
  return TP_OK;
}

tp_status check_ptrs(const void* const* arr, int n, const char* name, bool allow_null_array) {
  if (!arr) {
    if (allow_null_array) return TP_OK;
    return fail(TP_ERR_ARG, "%s (pointer array) is NULL", name);
  }
  for (int i = 0; i < n; ++i) {
    if (!arr[i]) return fail(TP_ERR_ARG, "%s[%d] is NULL", name, i);
    if (!aligned16(arr[i]))
      return fail(TP_ERR_ALIGN, "%s[%d] (%p) is not 16-byte aligned", name, i, arr[i]);
  }
  return TP_OK;
}

tp_status check_row_bytes(int64_t cols, tp_dtype t, const char* name) {
  if ((cols * static_cast<int64_t>(dsize(t))) % 16 != 0)
    return fail(TP_ERR_ALIGN, "%s: a row of %lld elements is not a multiple of 16 bytes", name,
                static_cast<long long>(cols));
  return TP_OK;
}

}  // namespace tpi

using namespace tpi;

namespace {

tp_status check_plan(const tp_plan* plan) {
  if (!plan) return fail(TP_ERR_ARG, "plan is NULL");
  return TP_OK;
}

// Rows of W_i for the column layer and the matching width of Z_i / H_i.
struct ColShape {
  int n_w;   // rows of the column shard W_i (= columns of Z_i)
  int n_h;   // columns of H_i
  int k;     // hidden
};

tp_status col_shape(const tp_plan* plan, tp_which which, ColShape* cs) {
  const int p = plan->p;
  if (which == TP_MLP) {
    if (plan->ffn <= 0) return fail(TP_ERR_ARG, "plan has no MLP (ffn = 0)");
    int f = plan->ffn / p;
    cs->n_h = f;
    cs->n_w = plan->act == TP_ACT_SWIGLU ? 2 * f : f;
  } else if (which == TP_QKV) {
    if (plan->heads <= 0) return fail(TP_ERR_ARG, "plan has no attention (heads = 0)");
    cs->n_w = cs->n_h = 3 * plan->hidden / p;
  } else if (which == TP_VOCAB) {
    if (plan->vocab_padded <= 0) return fail(TP_ERR_ARG, "plan has no vocab (tp_plan_set_vocab)");
    cs->n_w = cs->n_h = plan->vocab_padded / p;
  } else {
    return fail(TP_ERR_ARG, "projection %d is not column-parallel", static_cast<int>(which));
  }
  cs->k = plan->hidden;
  return TP_OK;
}

// Input width K_i of the row shard.
tp_status row_k(const tp_plan* plan, tp_which which, int* k) {
  if (which == TP_MLP) {
    if (plan->ffn <= 0) return fail(TP_ERR_ARG, "plan has no MLP (ffn = 0)");
    *k = plan->ffn / plan->p;
  } else if (which == TP_OUTPROJ) {
    if (plan->heads <= 0) return fail(TP_ERR_ARG, "plan has no attention (heads = 0)");
    *k = plan->hidden / plan->p;
  } else {
    return fail(TP_ERR_ARG, "projection %d is not row-parallel", static_cast<int>(which));
  }
  return TP_OK;
}

tp_status check_T(int64_t T) {
  if (T < 0) return fail(TP_ERR_ARG, "T = %lld is negative", static_cast<long long>(T));
  if (T > 0x7fffffffLL) return fail(TP_ERR_UNSUPPORTED, "T = %lld exceeds 2^31 - 1", (long long)T);
  return TP_OK;
}

PtrArray to_arr(const void* const* a, int n) {
  PtrArray r{};
  for (int i = 0; i < n && a; ++i) r.p[i] = a[i];
  return r;
}
MutPtrArray to_marr(void* const* a, int n) {
  MutPtrArray r{};
  for (int i = 0; i < n && a; ++i) r.p[i] = a[i];
  return r;
}

// A backward call's activation-gradient GEMM (dX or dH) and its weight
// gradient read the same inputs and write different outputs. When either
// leaves SMs idle (small problems: a few tiles per launch), the activation
// gradient runs on a side stream of the device beside the weight gradient:
// fork (the side stream waits for the caller's stream), the GEMM on the side
// stream, then the caller's stream waits for it before the call returns. The
// side GEMM uses no workspace (the weight gradient's split-K partials and the
// bias sums do, on the caller's stream). Works inside stream capture (the
// fork and join become graph edges). TP_BWD_CONCURRENT=0 keeps one stream.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

tp_status side_stream(SideStream** out) {
  constexpr int kMaxDev = 64;
  static SideStream side[kMaxDev];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return fail(TP_ERR_NO_DEVICE, "no current CUDA device");
  }
  std::lock_guard<std::mutex> lk(mu);
  SideStream& sd = side[dev];
  if (!sd.s) {
    SideStream n;
    tp_status r = cuda_status(cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking), "cudaStreamCreate(side)");
    if (r == TP_OK) r = cuda_status(cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming), "cudaEventCreate(fork)");
    if (r == TP_OK) r = cuda_status(cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming), "cudaEventCreate(join)");
    if (r != TP_OK) {
      if (n.join) cudaEventDestroy(n.join);
      if (n.fork) cudaEventDestroy(n.fork);
      if (n.s) cudaStreamDestroy(n.s);
      return r;
    }
    sd = n;
  }
  *out = &sd;
  return TP_OK;
}

bool concurrent_bwd(const tp_plan* plan, const GemmBatch& act_grad, const GemmBatch& wgrad) {
  if (plan->dtype != TP_BF16) return false;
  const char* e = getenv("TP_BWD_CONCURRENT");
  if (e && e[0] == '0') return false;
  return !gemm_fills_gpu(act_grad) || !gemm_fills_gpu(wgrad);
}

// Runs `act_grad` on the side stream (forked from st); more work may follow
// it there (stream()). When it goes out of scope, st waits for everything
// issued on the side stream: every return path of the call joins.
class SideGemm {
 public:
  SideGemm(const tp_plan* plan, const GemmBatch& act_grad, cudaStream_t st) : st_(st) {
    status_ = side_stream(&sd_);
    if (status_ != TP_OK) return;
    status_ = cuda_status(cudaEventRecord(sd_->fork, st), "cudaEventRecord(fork)");
    if (status_ == TP_OK) status_ = cuda_status(cudaStreamWaitEvent(sd_->s, sd_->fork, 0), "cudaStreamWaitEvent(fork)");
    if (status_ != TP_OK) {
      sd_ = nullptr;
      return;
    }
    status_ = plan->dtype == TP_BF16 ? launch_gemm_bf16(act_grad, sd_->s) : launch_gemm_f32(act_grad, sd_->s);
  }
  ~SideGemm() {
    if (!sd_) return;
    if (cudaEventRecord(sd_->join, sd_->s) == cudaSuccess) cudaStreamWaitEvent(st_, sd_->join, 0);
    else cudaStreamSynchronize(sd_->s);  // cannot join by event: finish the side work now
    cudaGetLastError();
  }
  tp_status status() const { return status_; }
  cudaStream_t stream() const { return sd_ ? sd_->s : st_; }

 private:
  SideStream* sd_ = nullptr;
  cudaStream_t st_;
  tp_status status_ = TP_OK;
};

// Launch grouped GEMMs in the plan dtype; fp32 takes EPI_STORE only.
tp_status run_gemm(const tp_plan* plan, const GemmBatch& b, cudaStream_t st) {
  if (plan->dtype == TP_BF16) return launch_gemm_bf16(b, st);
  return launch_gemm_f32(b, st);
}

// A weight-gradient batch (every problem the same shape, outputs D[i] dense
// [M, N] in the plan dtype). Problems with few output tiles and a long K (the
// token dim) leave most SMs idle, so for bf16 plans, when the estimate says so,
// the GEMM splits K: split s writes fp32 partials of every D[i] into the plan's
// workspace and one reduce sums the splits in order into D[i].
// allow_split = false when another GEMM shares the GPU with this one (the
// split's estimate assumes every SM; measured on the 12-layer stack beside
// the side stream's GEMM: no split 240.1 TFLOP/s, split 237.8, and 48 fewer
// launches a step).
// The K split run_wgrad takes for w (1: none).
int wgrad_split(const tp_plan* plan, const GemmBatch& w, bool allow_split) {
  if (plan->dtype != TP_BF16) return 1;
  // a split forced through TP_GEMM_SPLITK (tests) applies in either case
  const int s = allow_split || getenv("TP_GEMM_SPLITK") ? gemm_split_k(w) : 1;
  if (s <= 1 || s > TP_MAX_SHARDS) return 1;
  for (int i = 0; i < w.n; ++i)
    if (w.g[i].ldd != w.g[0].N) return 1;
  return s;
}
// Workspace bytes run_wgrad uses for w (its split's fp32 partials), rounded up to 256.
size_t wgrad_workspace(const tp_plan* plan, const GemmBatch& w, bool allow_split) {
  const int s = wgrad_split(plan, w, allow_split);
  if (s <= 1) return 0;
  const size_t b = static_cast<size_t>(s) * w.n * w.g[0].M * w.g[0].N * sizeof(float);
  return (b + 255) / 256 * 256;
}

tp_status run_wgrad(tp_plan* plan, GemmBatch w, cudaStream_t st, bool allow_split = true) {
  if (plan->dtype != TP_BF16) return run_gemm(plan, w, st);
  const int s = wgrad_split(plan, w, allow_split);
  if (s <= 1) return launch_gemm_bf16(w, st);
  const int n = w.n;
  const int64_t M = w.g[0].M, N = w.g[0].N, mn = M * N, elems = n * mn;
  void* ws = nullptr;
  TP_TRY(workspace(plan, static_cast<size_t>(s) * elems * sizeof(float), &ws));
  float* part = static_cast<float*>(ws);
  MutPtrArray outs{};
  for (int i = 0; i < n; ++i) {
    outs.p[i] = w.g[i].D;
    w.g[i].D = part + i * mn;
  }
  w.ksplit = s;
  w.split_stride = elems;
  w.out_f32 = true;
  TP_TRY(launch_gemm_bf16(w, st));
  PtrArray P{};
  for (int j = 0; j < s; ++j) P.p[j] = part + j * elems;
  return launch_reduce(P, s, nullptr, nullptr, PtrArray{}, false, outs, true, n, n * M, N, TP_F32,
                       TP_BF16, st);
}

// Launch the weight gradients a row backward left waiting, alone, on the
// stream it was issued on.
tp_status flush_wgrad(tp_plan* plan) {
  if (!plan->wg_pend) return TP_OK;
  std::unique_ptr<GemmBatch> w(plan->wg_pend);
  plan->wg_pend = nullptr;
  return run_wgrad(plan, *w, plan->wg_st);
}

// Whether two weight-gradient batches can run as one launch: the same
// operand layouts, epilogue and output type, the same K (tokens), room for
// both in one batch, and the same stream.
bool wgrad_mergeable(const GemmBatch& a, const GemmBatch& b, cudaStream_t sa, cudaStream_t sb) {
  return sa == sb && a.n + b.n <= TP_MAX_SHARDS && a.a_mn == b.a_mn && a.b_mn == b.b_mn &&
         a.epi == b.epi && a.out_f32 == b.out_f32 && !a.kcat && !b.kcat && a.scatter_n == 0 &&
         b.scatter_n == 0 && a.g[0].K == b.g[0].K;
}

// The weight-gradient step of a backward call: with grouping on, a row
// backward's batch waits for the next column backward, which launches both
// in one grouped GEMM (one partly empty last wave instead of two).
tp_status issue_wgrad(tp_plan* plan, const GemmBatch& w, cudaStream_t st, bool allow_split, bool row) {
  if (plan->group_wgrad && plan->dtype == TP_BF16 && allow_split) {
    if (row) {
      TP_TRY(flush_wgrad(plan));
      plan->wg_pend = new (std::nothrow) GemmBatch(w);
      if (!plan->wg_pend) return fail(TP_ERR_ARG, "out of host memory for a pending weight gradient");
      plan->wg_st = st;
      return TP_OK;
    }
    if (plan->wg_pend && wgrad_mergeable(*plan->wg_pend, w, plan->wg_st, st)) {
      std::unique_ptr<GemmBatch> pend(plan->wg_pend);
      plan->wg_pend = nullptr;
      GemmBatch m = *pend;
      for (int i = 0; i < w.n; ++i) m.g[m.n + i] = w.g[i];
      m.n += w.n;
      return run_wgrad(plan, m, st);
    }
  }
  TP_TRY(flush_wgrad(plan));
  return run_wgrad(plan, w, st, allow_split);
}

}  // namespace

extern "C" {

const char* tp_status_string(tp_status s) {
  switch (s) {
    case TP_OK: return "TP_OK";
    case TP_ERR_ARG: return "TP_ERR_ARG";
    case TP_ERR_DIVISIBILITY: return "TP_ERR_DIVISIBILITY";
    case TP_ERR_ALIGN: return "TP_ERR_ALIGN";
    case TP_ERR_DTYPE: return "TP_ERR_DTYPE";
    case TP_ERR_UNSUPPORTED: return "TP_ERR_UNSUPPORTED";
    case TP_ERR_CUDA: return "TP_ERR_CUDA";
    case TP_ERR_TIMEOUT: return "TP_ERR_TIMEOUT";
    case TP_ERR_NO_DEVICE: return "TP_ERR_NO_DEVICE";
  }
  return "TP_ERR_UNKNOWN";
}

const char* tp_last_error(void) { return g_last_error; }

uint64_t tp_launch_count(int reset) {
  uint64_t n = g_launches;
  if (reset) g_launches = 0;
  return n;
}

tp_status tp_plan_create(int hidden, int ffn, int heads, int p, tp_dtype dtype, tp_act act,
                         tp_dtype partial_dtype, tp_plan** out) {
  if (!out) return fail(TP_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (p < 1 || p > TP_MAX_SHARDS)
    return fail(TP_ERR_ARG, "p = %d outside [1, %d]", p, TP_MAX_SHARDS);
  if (hidden <= 0) return fail(TP_ERR_ARG, "hidden = %d must be positive", hidden);
  if (ffn < 0 || heads < 0) return fail(TP_ERR_ARG, "ffn and heads must be >= 0");
  if (dtype != TP_F32 && dtype != TP_BF16) return fail(TP_ERR_DTYPE, "unknown dtype %d", dtype);
  if (partial_dtype != dtype && partial_dtype != TP_F32)
    return fail(TP_ERR_DTYPE, "partial dtype %d: the partials are stored in the plan dtype or in fp32",
                partial_dtype);
  if (act != TP_ACT_NONE && act != TP_ACT_GELU && act != TP_ACT_SWIGLU)
    return fail(TP_ERR_ARG, "unknown activation %d", act);
  if (hidden % p) return fail(TP_ERR_DIVISIBILITY, "hidden = %d is not divisible by p = %d", hidden, p);
  if (heads > 0) {
    if (heads % p)
      return fail(TP_ERR_DIVISIBILITY, "heads = %d is not divisible by p = %d", heads, p);
    if (hidden % heads)
      return fail(TP_ERR_DIVISIBILITY, "hidden = %d is not divisible by heads = %d", hidden, heads);
  }
  if (ffn > 0) {
    if (ffn % p) return fail(TP_ERR_DIVISIBILITY, "ffn = %d is not divisible by p = %d", ffn, p);
    if (act == TP_ACT_SWIGLU && (2 * ffn) % (2 * p))
      return fail(TP_ERR_DIVISIBILITY, "gate+up columns 2*ffn = %d do not split into p = %d pairs",
                  2 * ffn, p);
  }
  tp_plan* plan = new (std::nothrow) tp_plan();
  if (!plan) return fail(TP_ERR_ARG, "out of host memory");
  plan->hidden = hidden;
  plan->ffn = ffn;
  plan->heads = heads;
  plan->p = p;
  plan->head_dim = heads > 0 ? hidden / heads : 0;
  plan->vocab = 0;
  plan->vocab_padded = 0;
  plan->dtype = dtype;
  plan->partial_dtype = partial_dtype;
  plan->act = act;
  plan->ws = nullptr;
  plan->ws_bytes = 0;
  plan->ws_device = -1;
  plan->cnt = nullptr;
  plan->cnt_device = -1;
  plan->defer_bwd = 0;
  plan->ws2 = nullptr;
  plan->ws2_bytes = 0;
  plan->ws2_device = -1;
  plan->group_wgrad = 0;
  plan->wg_pend = nullptr;
  plan->wg_st = nullptr;
  *out = plan;
  return TP_OK;
}

void tp_plan_destroy(tp_plan* plan) {
  if (!plan) return;
  delete plan->wg_pend;  // a weight gradient still waiting is dropped, not launched
  plan->wg_pend = nullptr;
  int cur = 0;
  cudaGetDevice(&cur);
  if (plan->ws) {
    cudaSetDevice(plan->ws_device);
    cudaDeviceSynchronize();
    cudaFree(plan->ws);
  }
  if (plan->cnt) {
    cudaSetDevice(plan->cnt_device);
    cudaDeviceSynchronize();
    cudaFree(plan->cnt);
  }
  if (plan->ws2) {
    cudaSetDevice(plan->ws2_device);
    cudaDeviceSynchronize();
    cudaFree(plan->ws2);
  }
  cudaSetDevice(cur);
  cudaGetLastError();
  delete plan;
}

tp_status tp_set_backward_defer(tp_plan* plan, int on) {
  TP_TRY(check_plan(plan));
  plan->defer_bwd = on ? 1 : 0;
  return TP_OK;
}

tp_status tp_flush_wgrad(tp_plan* plan) {
  TP_TRY(check_plan(plan));
  return flush_wgrad(plan);
}

tp_status tp_set_wgrad_grouping(tp_plan* plan, int on) {
  TP_TRY(check_plan(plan));
  if (!on) TP_TRY(flush_wgrad(plan));
  plan->group_wgrad = on ? 1 : 0;
  return TP_OK;
}

tp_status tp_backward_join(void* stream) {
  SideStream* sd = nullptr;
  TP_TRY(side_stream(&sd));
  cudaStream_t st = as_stream(stream);
  TP_TRY(cuda_status(cudaEventRecord(sd->join, sd->s), "cudaEventRecord(join)"));
  return cuda_status(cudaStreamWaitEvent(st, sd->join, 0), "cudaStreamWaitEvent(join)");
}

tp_status tp_plan_describe(const tp_plan* plan, char* buf, size_t n) {
  TP_TRY(check_plan(plan));
  if (!buf || n == 0) return fail(TP_ERR_ARG, "buf is NULL or empty");
  const int p = plan->p, h = plan->hidden, f = plan->ffn;
  const char* act = plan->act == TP_ACT_GELU ? "gelu" : plan->act == TP_ACT_SWIGLU ? "swiglu" : "none";
  int w = snprintf(buf, n,
                   "tp_plan: hidden=%d ffn=%d heads=%d head_dim=%d p=%d dtype=%s partials=%s act=%s\n",
                   h, f, plan->heads, plan->head_dim, p, plan->dtype == TP_BF16 ? "bf16" : "f32",
                   plan->partial_dtype == TP_BF16 ? "bf16" : "f32", act);
  auto add = [&](const char* fmt, auto... args) {
    if (w >= 0 && static_cast<size_t>(w) < n) w += snprintf(buf + w, n - w, fmt, args...);
  };
  if (f > 0) {
    int n1 = plan->act == TP_ACT_SWIGLU ? 2 * f / p : f / p;
    add("  MLP column shard W1_i: [%d, %d]%s; Z_i: [T, %d]; H_i: [T, %d]\n", n1, h,
        plan->act == TP_ACT_SWIGLU ? " = [G_i; U_i]" : "", n1, f / p);
    add("  MLP row shard W2_i: [%d, %d]; partial P_i: [T, %d]\n", h, f / p, h);
  }
  if (plan->heads > 0) {
    add("  QKV column shard: [%d, %d] = [Q_i; K_i; V_i], %d heads x %d each\n", 3 * h / p, h,
        plan->heads / p, plan->head_dim);
    add("  out-proj row shard Wo_i: [%d, %d]\n", h, h / p);
  }
  if (plan->vocab_padded > 0)
    add("  vocab shard (embedding / output head): [%d, %d] (vocab %d padded to %d)\n",
        plan->vocab_padded / p, h, plan->vocab, plan->vocab_padded);
  add("  sequence shard (SP): [T/%d, %d]\n", p, h);
  return TP_OK;
}

tp_status tp_get_device_status(const tp_plan* plan, void* stream) {
  (void)plan;  // the word is per device, shared by every plan
  unsigned* addr = nullptr;
  TP_TRY(device_status_word(&addr));
  unsigned v = 0;
  TP_TRY(cuda_status(cudaStreamSynchronize(as_stream(stream)), "cudaStreamSynchronize"));
  TP_TRY(cuda_status(cudaMemcpy(&v, addr, sizeof(v), cudaMemcpyDeviceToHost), "read status"));
  unsigned zero = 0;
  TP_TRY(cuda_status(cudaMemcpy(addr, &zero, sizeof(zero), cudaMemcpyHostToDevice), "clear status"));
  if (v & 1u) return fail(TP_ERR_TIMEOUT, "a kernel's bounded wait gave up (status word 0x%x)", v);
  if (v & 2u) return fail(TP_ERR_ARG, "a kernel met an out-of-range token id or label (status word 0x%x)", v);
  return TP_OK;
}

tp_status tp_selftest_wait_timeout(int64_t limit_ns, int* gave_up, void* stream) {
  if (limit_ns <= 0 || limit_ns > 1000000000LL)
    return fail(TP_ERR_ARG, "limit_ns = %lld outside (0, 1e9]", (long long)limit_ns);
  if (gave_up && (reinterpret_cast<uintptr_t>(gave_up) & 3u))
    return fail(TP_ERR_ALIGN, "gave_up is not 4-byte aligned");
  unsigned* addr = nullptr;
  TP_TRY(device_status_word(&addr));
  (void)tpi::launch(tp_selftest::selftest_wait_kernel, dim3(1), dim3(32), 0, as_stream(stream), addr, static_cast<uint64_t>(limit_ns), gave_up);
  return after_launch("selftest_wait_timeout");
}

// ------------------------------------------------------------------ sharding

static tp_status shard_copy(const tp_plan* plan, tp_which which, bool column, const void* full,
                            void* const* shards_out, const void* const* shards_in, bool to_shards,
                            cudaStream_t st) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_ptr(full, to_shards ? "W_full" : "W_full (out)"));
  const int p = plan->p, h = plan->hidden;
  const void* const* shards = to_shards ? reinterpret_cast<const void* const*>(shards_out) : shards_in;
  TP_TRY(check_ptrs(shards, p, "W_shards", false));
  const size_t es = dsize(plan->dtype);
  char* F = static_cast<char*>(const_cast<void*>(full));
  // Each shard is a set of (src block -> dst block) 2-D copies.
  auto copy = [&](const char* src, int64_t sld, char* dst, int64_t dld, int64_t rows, int64_t cols) {
    return launch_copy_2d(src, sld, dst, dld, rows, cols, es, st);
  };
  if (column) {
    if (which == TP_MLP) {
      if (plan->ffn <= 0) return fail(TP_ERR_ARG, "plan has no MLP");
      const int f = plan->ffn, k = f / p;
      TP_TRY(check_row_bytes(h, plan->dtype, "hidden"));
      for (int i = 0; i < p; ++i) {
        char* S = static_cast<char*>(const_cast<void*>(shards[i]));
        if (plan->act == TP_ACT_SWIGLU) {
          // [G_i; U_i]: gate rows then the matching up rows.
          const int64_t rows[2] = {static_cast<int64_t>(i) * k, static_cast<int64_t>(f) + i * k};
          for (int half = 0; half < 2; ++half) {
            char* fb = F + rows[half] * h * es;
            char* sb = S + static_cast<int64_t>(half) * k * h * es;
            TP_TRY(to_shards ? copy(fb, h, sb, h, k, h) : copy(sb, h, fb, h, k, h));
          }
        } else {
          char* fb = F + static_cast<int64_t>(i) * k * h * es;
          TP_TRY(to_shards ? copy(fb, h, S, h, k, h) : copy(S, h, fb, h, k, h));
        }
      }
      return TP_OK;
    }
    if (which == TP_QKV) {
      if (plan->heads <= 0) return fail(TP_ERR_ARG, "plan has no attention");
      const int rows = h / p;  // heads/p * head_dim rows from each of Wq, Wk, Wv
      TP_TRY(check_row_bytes(h, plan->dtype, "hidden"));
      for (int i = 0; i < p; ++i) {
        char* S = static_cast<char*>(const_cast<void*>(shards[i]));
        for (int part = 0; part < 3; ++part) {
          char* fb = F + (static_cast<int64_t>(part) * h + static_cast<int64_t>(i) * rows) * h * es;
          char* sb = S + static_cast<int64_t>(part) * rows * h * es;
          TP_TRY(to_shards ? copy(fb, h, sb, h, rows, h) : copy(sb, h, fb, h, rows, h));
        }
      }
      return TP_OK;
    }
    if (which == TP_VOCAB) {
      if (plan->vocab_padded <= 0) return fail(TP_ERR_ARG, "plan has no vocab (tp_plan_set_vocab)");
      const int rows = plan->vocab_padded / p;
      TP_TRY(check_row_bytes(h, plan->dtype, "hidden"));
      for (int i = 0; i < p; ++i) {
        char* S = static_cast<char*>(const_cast<void*>(shards[i]));
        char* fb = F + static_cast<int64_t>(i) * rows * h * es;
        TP_TRY(to_shards ? copy(fb, h, S, h, rows, h) : copy(S, h, fb, h, rows, h));
      }
      return TP_OK;
    }
    return fail(TP_ERR_ARG, "projection %d is not column-parallel", static_cast<int>(which));
  }
  int k = 0;
  TP_TRY(row_k(plan, which, &k));
  const int kin = k * p;
  TP_TRY(check_row_bytes(k, plan->dtype, "row shard width"));
  for (int i = 0; i < p; ++i) {
    char* S = static_cast<char*>(const_cast<void*>(shards[i]));
    char* fb = F + static_cast<int64_t>(i) * k * es;
    TP_TRY(to_shards ? copy(fb, kin, S, k, h, k) : copy(S, k, fb, kin, h, k));
  }
  return TP_OK;
}

tp_status tp_shard_column(const tp_plan* plan, tp_which which, const void* W_full,
                          void* const* W_shards, void* stream) {
  return shard_copy(plan, which, true, W_full, W_shards, nullptr, true, as_stream(stream));
}
tp_status tp_unshard_column(const tp_plan* plan, tp_which which, const void* const* W_shards,
                            void* W_full, void* stream) {
  return shard_copy(plan, which, true, W_full, nullptr, W_shards, false, as_stream(stream));
}
tp_status tp_shard_row(const tp_plan* plan, tp_which which, const void* W_full,
                       void* const* W_shards, void* stream) {
  return shard_copy(plan, which, false, W_full, W_shards, nullptr, true, as_stream(stream));
}
tp_status tp_unshard_row(const tp_plan* plan, tp_which which, const void* const* W_shards,
                         void* W_full, void* stream) {
  return shard_copy(plan, which, false, W_full, nullptr, W_shards, false, as_stream(stream));
}

tp_status tp_shard_column_bias(const tp_plan* plan, tp_which which, const void* b_full,
                               void* const* b_shards, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_ptr(b_full, "b_full"));
  const int p = plan->p;
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(b_shards), p, "b_shards", false));
  const size_t es = dsize(plan->dtype);
  cudaStream_t st = as_stream(stream);
  const char* B = static_cast<const char*>(b_full);
  auto copy = [&](const char* src, char* dst, int64_t n) {
    return launch_copy_2d(src, n, dst, n, 1, n, es, st);
  };
  for (int i = 0; i < p; ++i) {
    char* S = static_cast<char*>(b_shards[i]);
    if (which == TP_MLP) {
      if (plan->ffn <= 0) return fail(TP_ERR_ARG, "plan has no MLP");
      const int f = plan->ffn, k = f / p;
      if (plan->act == TP_ACT_SWIGLU) {
        TP_TRY(copy(B + static_cast<int64_t>(i) * k * es, S, k));
        TP_TRY(copy(B + (static_cast<int64_t>(f) + i * k) * es, S + k * es, k));
      } else {
        TP_TRY(copy(B + static_cast<int64_t>(i) * k * es, S, k));
      }
    } else if (which == TP_QKV) {
      if (plan->heads <= 0) return fail(TP_ERR_ARG, "plan has no attention");
      const int h = plan->hidden, rows = h / p;
      for (int part = 0; part < 3; ++part)
        TP_TRY(copy(B + (static_cast<int64_t>(part) * h + static_cast<int64_t>(i) * rows) * es,
                    S + static_cast<int64_t>(part) * rows * es, rows));
    } else {
      return fail(TP_ERR_ARG, "projection %d is not column-parallel", static_cast<int>(which));
    }
  }
  return TP_OK;
}

// ------------------------------------------------------------------- forward

tp_status tp_column_fwd(tp_plan* plan, tp_which which, int64_t T, const void* X,
                        const void* const* W, const void* const* bias, void* const* Z,
                        void* const* H, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  ColShape cs{};
  TP_TRY(col_shape(plan, which, &cs));
  const int p = plan->p;
  const tp_act act = which == TP_MLP ? plan->act : TP_ACT_NONE;
  TP_TRY(check_ptr(X, "X"));
  TP_TRY(check_ptrs(W, p, "W", false));
  TP_TRY(check_ptrs(bias, p, "bias", true));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(Z), p, "Z", true));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(H), p, "H", false));
  TP_TRY(check_row_bytes(cs.k, plan->dtype, "hidden"));
  TP_TRY(check_row_bytes(cs.n_h, plan->dtype, "H_i width"));
  if (act == TP_ACT_SWIGLU && bias)
    return fail(TP_ERR_ARG, "a column bias is not supported with SwiGLU");
  if (act == TP_ACT_NONE && Z)
    return fail(TP_ERR_ARG, "Z must be NULL when there is no activation");
  if (T == 0) return TP_OK;
  cudaStream_t st = as_stream(stream);

  GemmBatch b{};
  b.n = p;
  b.a_mn = false;
  b.b_mn = false;
  b.out_f32 = plan->dtype == TP_F32;
  for (int i = 0; i < p; ++i) {
    GemmProblem& g = b.g[i];
    g.M = static_cast<int>(T);
    g.K = cs.k;
    g.A = X;
    g.lda = cs.k;
    g.B = W[i];
    g.ldb = cs.k;
    g.bias = bias ? bias[i] : nullptr;
  }
  if (act == TP_ACT_NONE) {
    b.epi = EPI_STORE;
    for (int i = 0; i < p; ++i) {
      b.g[i].N = cs.n_w;
      b.g[i].D = H[i];
      b.g[i].ldd = cs.n_h;
    }
  } else if (act == TP_ACT_GELU) {
    b.epi = EPI_BIAS_GELU;
    for (int i = 0; i < p; ++i) {
      b.g[i].N = cs.n_w;
      b.g[i].D = Z ? Z[i] : nullptr;
      b.g[i].ldd = cs.n_w;
      b.g[i].D2 = H[i];
      b.g[i].ldd2 = cs.n_h;
    }
  } else {
    b.epi = EPI_SWIGLU;
    for (int i = 0; i < p; ++i) {
      b.g[i].N = cs.n_h;  // gate/up pairs
      b.g[i].nh = cs.n_h;
      b.g[i].D = Z ? Z[i] : nullptr;
      b.g[i].ldd = cs.n_w;
      b.g[i].D2 = H[i];
      b.g[i].ldd2 = cs.n_h;
    }
  }
  return run_gemm(plan, b, st);
}

tp_status tp_row_fwd_partial(tp_plan* plan, tp_which which, int64_t T, const void* const* H,
                             const void* const* W, void* const* P, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  int k = 0;
  TP_TRY(row_k(plan, which, &k));
  const int p = plan->p, h = plan->hidden;
  TP_TRY(check_ptrs(H, p, "H", false));
  TP_TRY(check_ptrs(W, p, "W", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(P), p, "P", false));
  TP_TRY(check_row_bytes(k, plan->dtype, "row shard width"));
  TP_TRY(check_row_bytes(h, plan->partial_dtype, "hidden"));
  if (T == 0) return TP_OK;
  GemmBatch b{};
  b.n = p;
  b.epi = EPI_STORE;
  b.out_f32 = plan->partial_dtype == TP_F32;
  for (int i = 0; i < p; ++i) {
    GemmProblem& g = b.g[i];
    g.M = static_cast<int>(T);
    g.N = h;
    g.K = k;
    g.A = H[i];
    g.lda = k;
    g.B = W[i];
    g.ldb = k;
    g.D = P[i];
    g.ldd = h;
  }
  return run_gemm(plan, b, as_stream(stream));
}

// Row GEMM with the shard sum fused (K-concatenated over shards), writing the
// full output or (scatter) its sequence shards.
// With a peer group (peer != NULL, scatter false, no bias or residual) row
// block j goes to slot <rank> of rank j's receive buffer with plain stores.
static tp_status check_peer_push(const tp_plan* plan, const tp_peer_group* g, int64_t T) {
  TP_TRY(check_peer_group(g));
  if (plan->dtype != TP_BF16) return fail(TP_ERR_DTYPE, "peer pushes need a bf16 plan");
  if (T % g->world)
    return fail(TP_ERR_DIVISIBILITY, "T = %lld is not divisible by world = %d", (long long)T, g->world);
  if (T * plan->hidden > g->recv_elems)
    return fail(TP_ERR_ARG, "T x hidden = %lld exceeds the receive buffers (%lld elements)",
                (long long)(T * plan->hidden), (long long)g->recv_elems);
  return TP_OK;
}

static void peer_push_targets(GemmBatch& b, const tp_peer_group* g, int64_t T, int h) {
  const int64_t t = T / g->world;
  b.scatter_n = g->world;
  b.rows_per_out = t;
  b.plain_stores = true;
  for (int j = 0; j < g->world; ++j) {
    b.out_seq[j] = static_cast<__nv_bfloat16*>(g->recv[j]) + static_cast<int64_t>(g->rank) * t * h;
    b.res_seq[j] = nullptr;
  }
  b.g[0].D = b.out_seq[0];
}

static tp_status row_fwd_reduce_common(tp_plan* plan, tp_which which, int64_t T,
                                       const void* const* H, const void* const* W, const void* bias,
                                       const void* residual, const void* const* residual_seq,
                                       void* Y, void* const* Y_seq, bool scatter, cudaStream_t st,
                                       const tp_peer_group* peer = nullptr) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  int k = 0;
  TP_TRY(row_k(plan, which, &k));
  const int p = plan->p, h = plan->hidden;
  TP_TRY(check_ptrs(H, p, "H", false));
  TP_TRY(check_ptrs(W, p, "W", false));
  if (bias) TP_TRY(check_ptr(bias, "bias"));
  TP_TRY(check_row_bytes(k, plan->dtype, "row shard width"));
  TP_TRY(check_row_bytes(h, plan->dtype, "hidden"));
  if (peer) {
    TP_TRY(check_peer_push(plan, peer, T));
  } else if (scatter) {
    if (T % p) return fail(TP_ERR_DIVISIBILITY, "T = %lld is not divisible by p = %d", (long long)T, p);
    TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(Y_seq), p, "Y_seq", false));
    TP_TRY(check_ptrs(residual_seq, p, "residual_seq", true));
  } else {
    TP_TRY(check_ptr(Y, "Y"));
    if (residual) TP_TRY(check_ptr(residual, "residual"));
  }
  if (T == 0) return TP_OK;
  GemmBatch b{};
  b.n = p;
  b.kcat = true;
  b.epi = EPI_STORE;
  for (int i = 0; i < p; ++i) {
    GemmProblem& g = b.g[i];
    g.M = static_cast<int>(T);
    g.N = h;
    g.K = k;
    g.A = H[i];
    g.lda = k;
    g.B = W[i];
    g.ldb = k;
  }
  b.g[0].D = scatter ? Y_seq[0] : Y;
  b.g[0].ldd = h;
  b.g[0].bias = bias;
  b.g[0].aux = scatter ? nullptr : residual;
  b.g[0].ldaux = h;
  if (peer) {
    peer_push_targets(b, peer, T, h);
  } else if (scatter) {
    b.scatter_n = p;
    b.rows_per_out = T / p;
    for (int j = 0; j < p; ++j) {
      b.out_seq[j] = Y_seq[j];
      b.res_seq[j] = residual_seq ? residual_seq[j] : nullptr;
    }
  }
  return run_gemm(plan, b, st);
}

tp_status tp_row_fwd_reduce(tp_plan* plan, tp_which which, int64_t T, const void* const* H,
                            const void* const* W, const void* bias, const void* residual, void* Y,
                            void* stream) {
  return row_fwd_reduce_common(plan, which, T, H, W, bias, residual, nullptr, Y, nullptr, false,
                               as_stream(stream));
}

tp_status tp_row_fwd_reduce_scatter_seq(tp_plan* plan, tp_which which, int64_t T,
                                        const void* const* H, const void* const* W,
                                        const void* bias, const void* const* residual_seq,
                                        void* const* Y_seq, void* stream) {
  return row_fwd_reduce_common(plan, which, T, H, W, bias, nullptr, residual_seq, nullptr, Y_seq,
                               true, as_stream(stream));
}

tp_status tp_row_fwd_push_peer(tp_plan* plan, tp_which which, int64_t T, const void* const* H,
                               const void* const* W, const tp_peer_group* g, uint32_t epoch,
                               void* stream) {
  const cudaStream_t st = as_stream(stream);
  TP_TRY(row_fwd_reduce_common(plan, which, T, H, W, nullptr, nullptr, nullptr, nullptr, nullptr,
                               false, st, g));
  return launch_peer_signal(g, g->rank, epoch, st);
}

static tp_status reduce_common(tp_plan* plan, int64_t T, int n, const void* const* P,
                               const void* bias, const void* residual,
                               const void* const* residual_seq, void* Y,
                               void* const* Y_seq, bool scatter, cudaStream_t st) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  if (n < 1 || n > TP_MAX_SHARDS) return fail(TP_ERR_ARG, "n = %d outside [1, %d]", n, TP_MAX_SHARDS);
  const int h = plan->hidden;
  TP_TRY(check_ptrs(P, n, "P", false));
  if (bias) TP_TRY(check_ptr(bias, "bias"));
  if (residual) TP_TRY(check_ptr(residual, "residual"));
  TP_TRY(check_row_bytes(h, plan->dtype, "hidden"));
  TP_TRY(check_row_bytes(h, plan->partial_dtype, "hidden (partials)"));
  if (scatter) {
    if (T % n) return fail(TP_ERR_DIVISIBILITY, "T = %lld is not divisible by n = %d", (long long)T, n);
    TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(Y_seq), n, "Y_seq", false));
    TP_TRY(check_ptrs(residual_seq, n, "residual_seq", true));
  } else {
    TP_TRY(check_ptr(Y, "Y"));
  }
  if (T == 0) return TP_OK;
  MutPtrArray out{};
  int nout = 1;
  if (scatter) {
    out = to_marr(Y_seq, n);
    nout = n;
  } else {
    out.p[0] = Y;
  }
  return launch_reduce(to_arr(P, n), n, bias, residual, to_arr(residual_seq, n),
                       scatter && residual_seq != nullptr, out, scatter, nout, T, h,
                       plan->partial_dtype, plan->dtype, st);
}

tp_status tp_reduce_partials(tp_plan* plan, int64_t T, int n, const void* const* P,
                             const void* bias, const void* residual, void* Y, void* stream) {
  return reduce_common(plan, T, n, P, bias, residual, nullptr, Y, nullptr, false,
                       as_stream(stream));
}

tp_status tp_reduce_scatter_seq(tp_plan* plan, int64_t T, int n, const void* const* P,
                                const void* bias, const void* const* residual_seq,
                                void* const* Y_seq, void* stream) {
  return reduce_common(plan, T, n, P, bias, nullptr, residual_seq, nullptr, Y_seq, true,
                       as_stream(stream));
}

tp_status tp_all_gather_seq(tp_plan* plan, int64_t T, int n, const void* const* X_seq,
                            void* X_full, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  if (n < 1 || n > TP_MAX_SHARDS) return fail(TP_ERR_ARG, "n = %d outside [1, %d]", n, TP_MAX_SHARDS);
  if (T % n) return fail(TP_ERR_DIVISIBILITY, "T = %lld is not divisible by n = %d", (long long)T, n);
  TP_TRY(check_ptrs(X_seq, n, "X_seq", false));
  TP_TRY(check_ptr(X_full, "X_full"));
  TP_TRY(check_row_bytes(plan->hidden, plan->dtype, "hidden"));
  if (T == 0) return TP_OK;
  return launch_gather(to_arr(X_seq, n), n, X_full, T, plan->hidden, plan->dtype, as_stream(stream));
}

tp_status tp_reduce_scatter_seq_bwd(tp_plan* plan, int64_t T, int n, const void* const* dY_seq,
                                    void* dY_full, void* stream) {
  return tp_all_gather_seq(plan, T, n, dY_seq, dY_full, stream);
}

tp_status tp_all_gather_seq_bwd(tp_plan* plan, int64_t T, int n, const void* const* dX_partials,
                                void* const* dX_seq, void* stream) {
  return tp_reduce_scatter_seq(plan, T, n, dX_partials, nullptr, nullptr, dX_seq, stream);
}

static tp_status check_ln(const tp_plan* plan) {
  const int h = plan->hidden;
  if (h % 8) return fail(TP_ERR_UNSUPPORTED, "LayerNorm needs hidden %% 8 == 0 (hidden = %d)", h);
  if (h > 16384) return fail(TP_ERR_UNSUPPORTED, "LayerNorm supports hidden <= 16384 (got %d)", h);
  return check_row_bytes(h, plan->dtype, "hidden");
}

tp_status tp_layernorm_fwd(tp_plan* plan, int64_t rows, const void* x, const void* gamma,
                           const void* beta, void* y, float* mean, float* rstd, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(rows));
  TP_TRY(check_ptr(x, "x"));
  TP_TRY(check_ptr(gamma, "gamma"));
  TP_TRY(check_ptr(beta, "beta"));
  TP_TRY(check_ptr(y, "y"));
  TP_TRY(check_ln(plan));
  if (rows == 0) return TP_OK;
  PtrArray xs{};
  xs.p[0] = x;
  return launch_layernorm_fwd(xs, 1, rows, plan->hidden, gamma, beta, y, mean, rstd, plan->dtype,
                              as_stream(stream));
}

tp_status tp_layernorm_all_gather_seq(tp_plan* plan, int64_t T, int n, const void* const* X_seq,
                                      const void* gamma, const void* beta, void* Y_full,
                                      float* mean, float* rstd, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  if (n < 1 || n > TP_MAX_SHARDS) return fail(TP_ERR_ARG, "n = %d outside [1, %d]", n, TP_MAX_SHARDS);
  if (T % n) return fail(TP_ERR_DIVISIBILITY, "T = %lld is not divisible by n = %d", (long long)T, n);
  TP_TRY(check_ptrs(X_seq, n, "X_seq", false));
  TP_TRY(check_ptr(gamma, "gamma"));
  TP_TRY(check_ptr(beta, "beta"));
  TP_TRY(check_ptr(Y_full, "Y_full"));
  TP_TRY(check_ln(plan));
  if (T == 0) return TP_OK;
  return launch_layernorm_fwd(to_arr(X_seq, n), n, T / n, plan->hidden, gamma, beta, Y_full, mean,
                              rstd, plan->dtype, as_stream(stream));
}

tp_status tp_layernorm_all_gather_push_peer(tp_plan* plan, const tp_peer_group* g, int64_t rows,
                                           const void* x, const void* gamma, const void* beta,
                                           void* const* out, float* mean, float* rstd, uint32_t epoch,
                                           void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(rows));
  TP_TRY(check_peer_group(g));
  if (plan->dtype != TP_BF16) return fail(TP_ERR_DTYPE, "peer pushes need a bf16 plan");
  TP_TRY(check_ptr(x, "x"));
  TP_TRY(check_ptr(gamma, "gamma"));
  TP_TRY(check_ptr(beta, "beta"));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(out), g->world, "out", false));
  TP_TRY(check_ln(plan));
  const cudaStream_t st = as_stream(stream);
  if (rows > 0) {
    PtrArray xs{};
    xs.p[0] = x;
    MutPtrArray dst{};
    for (int d = 0; d < g->world; ++d) dst.p[d] = out[d];
    TP_TRY(launch_layernorm_fwd(xs, 1, rows, plan->hidden, gamma, beta, nullptr, mean, rstd, plan->dtype,
                                st, &dst, g->world));
  }
  return launch_peer_signal(g, TP_MAX_SHARDS + g->rank, epoch, st);
}

tp_status tp_layernorm_bwd(tp_plan* plan, int64_t rows, const void* x, const void* gamma,
                           const void* dy, const float* mean, const float* rstd, const void* dres,
                           void* dx, float* dgamma, float* dbeta, int accumulate, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(rows));
  TP_TRY(check_ptr(x, "x"));
  TP_TRY(check_ptr(gamma, "gamma"));
  TP_TRY(check_ptr(dy, "dy"));
  TP_TRY(check_ptr(mean, "mean"));
  TP_TRY(check_ptr(rstd, "rstd"));
  TP_TRY(check_ptr(dx, "dx"));
  TP_TRY(check_ptr(dgamma, "dgamma"));
  TP_TRY(check_ptr(dbeta, "dbeta"));
  if (dres) TP_TRY(check_ptr(dres, "dres"));
  TP_TRY(check_ln(plan));
  return launch_layernorm_bwd(plan, x, gamma, dy, mean, rstd, dres, dx, dgamma, dbeta, accumulate,
                              rows, plan->hidden, plan->dtype, as_stream(stream));
}

tp_status tp_plan_set_vocab(tp_plan* plan, int vocab, int* vocab_padded) {
  TP_TRY(check_plan(plan));
  if (vocab <= 0) return fail(TP_ERR_ARG, "vocab = %d must be positive", vocab);
  const int64_t unit = 8LL * plan->p;
  const int64_t vp = ((vocab + unit - 1) / unit) * unit;
  if (vp > 0x7fffffffLL) return fail(TP_ERR_UNSUPPORTED, "vocab too large");
  plan->vocab = vocab;
  plan->vocab_padded = static_cast<int>(vp);
  if (vocab_padded) *vocab_padded = plan->vocab_padded;
  return TP_OK;
}

static tp_status check_vocab(const tp_plan* plan, int64_t T) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  if (plan->vocab_padded <= 0) return fail(TP_ERR_ARG, "plan has no vocab (tp_plan_set_vocab)");
  return check_row_bytes(plan->hidden, plan->dtype, "hidden");
}

tp_status tp_embedding_fwd(tp_plan* plan, int64_t T, const int32_t* ids, const void* const* E,
                           void* Y, void* stream) {
  TP_TRY(check_vocab(plan, T));
  const int p = plan->p;
  TP_TRY(check_ptr(ids, "ids"));
  TP_TRY(check_ptrs(E, p, "E", false));
  TP_TRY(check_ptr(Y, "Y"));
  if (T == 0) return TP_OK;
  return launch_embedding_fwd(ids, to_arr(E, p), plan->vocab, plan->vocab_padded / p, T,
                              plan->hidden, plan->dtype, Y, as_stream(stream));
}

tp_status tp_embedding_bwd(tp_plan* plan, int64_t T, const int32_t* ids, const void* dY,
                           void* const* dE, void* stream) {
  TP_TRY(check_vocab(plan, T));
  const int p = plan->p;
  if (T > 0) {
    TP_TRY(check_ptr(ids, "ids"));
    TP_TRY(check_ptr(dY, "dY"));
  }
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dE), p, "dE", false));
  size_t bytes = 0;
  TP_TRY(embedding_bwd_workspace(T, plan->vocab_padded, &bytes));
  void* ws = nullptr;
  TP_TRY(workspace(plan, bytes, &ws));
  return launch_embedding_bwd(ids, T, dY, plan->hidden, plan->vocab, plan->vocab_padded,
                              plan->vocab_padded / p, to_marr(dE, p), plan->dtype, ws,
                              as_stream(stream));
}

tp_status tp_vocab_cross_entropy(tp_plan* plan, int64_t T, const void* const* logits,
                                 const int32_t* labels, float grad_scale, float* loss, float* lse,
                                 void* const* dlogits, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  if (plan->vocab_padded <= 0) return fail(TP_ERR_ARG, "plan has no vocab (tp_plan_set_vocab)");
  const int p = plan->p;
  TP_TRY(check_ptrs(logits, p, "logits", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dlogits), p, "dlogits", true));
  TP_TRY(check_ptr(labels, "labels"));
  TP_TRY(check_ptr(loss, "loss"));
  if (T == 0) return TP_OK;
  MutPtrArray g{};
  if (dlogits)
    for (int i = 0; i < p; ++i) g.p[i] = dlogits[i];
  return launch_vocab_ce(to_arr(logits, p), g, p, plan->vocab_padded / p, plan->vocab, labels,
                         grad_scale, loss, lse, T, plan->dtype, as_stream(stream));
}

static tp_status check_norm_sharded(const tp_plan* plan, tp_norm_kind kind, int64_t rows) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(rows));
  if (kind != TP_NORM_LAYER && kind != TP_NORM_RMS) return fail(TP_ERR_ARG, "unknown norm kind %d", kind);
  const int h = plan->hidden, p = plan->p;
  if ((h / p) % 8) return fail(TP_ERR_UNSUPPORTED, "hidden/p = %d must be a multiple of 8", h / p);
  const int hmax = plan->dtype == TP_BF16 ? 16384 : 8192;  // 2048 16-byte vectors a row
  if (h > hmax) return fail(TP_ERR_UNSUPPORTED, "norms support hidden <= %d (got %d)", hmax, h);
  return TP_OK;
}

tp_status tp_norm_sharded_fwd(tp_plan* plan, tp_norm_kind kind, int64_t rows, const void* const* X,
                              const void* const* gamma, const void* const* beta, void* const* Y,
                              float* mean, float* rstd, void* stream) {
  TP_TRY(check_norm_sharded(plan, kind, rows));
  const int p = plan->p;
  TP_TRY(check_ptrs(X, p, "X", false));
  TP_TRY(check_ptrs(gamma, p, "gamma", false));
  if (kind == TP_NORM_LAYER) TP_TRY(check_ptrs(beta, p, "beta", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(Y), p, "Y", false));
  if (rows == 0) return TP_OK;
  return launch_norm_sharded_fwd(kind == TP_NORM_RMS, to_arr(X, p), to_arr(gamma, p),
                                 to_arr(kind == TP_NORM_LAYER ? beta : nullptr, p), to_marr(Y, p), p,
                                 rows, plan->hidden, mean, rstd, plan->dtype, as_stream(stream));
}

tp_status tp_norm_sharded_bwd(tp_plan* plan, tp_norm_kind kind, int64_t rows, const void* const* X,
                              const void* const* gamma, const void* const* dY, const float* mean,
                              const float* rstd, void* const* dX, float* const* dgamma,
                              float* const* dbeta, void* stream) {
  TP_TRY(check_norm_sharded(plan, kind, rows));
  const int p = plan->p;
  TP_TRY(check_ptrs(X, p, "X", false));
  TP_TRY(check_ptrs(gamma, p, "gamma", false));
  TP_TRY(check_ptrs(dY, p, "dY", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dX), p, "dX", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dgamma), p, "dgamma", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dbeta), p, "dbeta", true));
  TP_TRY(check_ptr(rstd, "rstd"));
  if (kind == TP_NORM_LAYER) TP_TRY(check_ptr(mean, "mean"));
  MutPtrArray dg{}, db{};
  for (int i = 0; i < p; ++i) {
    dg.p[i] = dgamma[i];
    db.p[i] = dbeta ? dbeta[i] : nullptr;
  }
  return launch_norm_sharded_bwd(plan, kind == TP_NORM_RMS, to_arr(X, p), to_arr(gamma, p),
                                 to_arr(dY, p), to_marr(dX, p), dg, db, p, rows, plan->hidden, mean,
                                 rstd, plan->dtype, as_stream(stream));
}

tp_status tp_column_sum(tp_plan* plan, int64_t rows, int64_t cols, const void* x, float* out,
                        int accumulate, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(rows));
  if (cols <= 0 || cols > 0x7fffffffLL) return fail(TP_ERR_ARG, "cols = %lld", (long long)cols);
  if (rows > 0) TP_TRY(check_ptr(x, "x"));
  TP_TRY(check_ptr(out, "out"));
  TP_TRY(check_row_bytes(cols, plan->dtype, "cols"));
  return launch_column_sum(plan, x, rows, cols, cols, out, accumulate, plan->dtype,
                           as_stream(stream));
}

tp_status tp_attention_fwd(tp_plan* plan, int batch, int seq, const void* const* QKV,
                           void* const* O, float* const* LSE, void* stream) {
  TP_TRY(check_plan(plan));
  if (plan->heads <= 0) return fail(TP_ERR_ARG, "plan has no attention (heads = 0)");
  if (batch <= 0 || seq <= 0) return fail(TP_ERR_ARG, "batch and seq must be positive");
  if (plan->dtype != TP_BF16) return fail(TP_ERR_DTYPE, "attention runs in bf16 only");
  const int p = plan->p;
  TP_TRY(check_ptrs(QKV, p, "QKV", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(O), p, "O", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(LSE), p, "LSE", true));
  if (plan->head_dim != 64 && plan->head_dim != 128)
    return fail(TP_ERR_UNSUPPORTED, "attention supports head_dim 64 or 128 (got %d)", plan->head_dim);
  return launch_attention_fwd(plan, batch, seq, to_arr(QKV, p), to_marr(O, p), LSE,
                              as_stream(stream));
}

tp_status tp_attention_bwd(tp_plan* plan, int batch, int seq, const void* const* QKV,
                           const void* const* O, const void* const* dO, const float* const* LSE,
                           void* const* dQKV, void* stream) {
  TP_TRY(check_plan(plan));
  if (plan->heads <= 0) return fail(TP_ERR_ARG, "plan has no attention (heads = 0)");
  if (batch <= 0 || seq <= 0) return fail(TP_ERR_ARG, "batch and seq must be positive");
  if (plan->dtype != TP_BF16) return fail(TP_ERR_DTYPE, "attention runs in bf16 only");
  const int p = plan->p;
  TP_TRY(check_ptrs(QKV, p, "QKV", false));
  TP_TRY(check_ptrs(O, p, "O", false));
  TP_TRY(check_ptrs(dO, p, "dO", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(LSE), p, "LSE", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dQKV), p, "dQKV", false));
  if (plan->head_dim != 64 && plan->head_dim != 128)
    return fail(TP_ERR_UNSUPPORTED, "attention supports head_dim 64 or 128 (got %d)", plan->head_dim);
  return launch_attention_bwd(plan, batch, seq, to_arr(QKV, p), to_arr(O, p), to_arr(dO, p), LSE,
                              to_marr(dQKV, p), as_stream(stream));
}

// ------------------------------------------------------------------ backward

tp_status tp_row_bwd(tp_plan* plan, tp_which which, int64_t T, const void* dY,
                     const void* const* H, const void* const* W, const void* const* Z,
                     void* const* dZ, void* const* dW, float* dbias, void* stream) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  int k = 0;
  TP_TRY(row_k(plan, which, &k));
  const int p = plan->p, h = plan->hidden;
  const tp_act act = which == TP_OUTPROJ ? TP_ACT_NONE : plan->act;
  const int nz = act == TP_ACT_SWIGLU ? 2 * k : k;  // width of Z_i / dZ_i
  TP_TRY(check_ptr(dY, "dY"));
  TP_TRY(check_ptrs(W, p, "W", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dZ), p, "dZ", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dW), p, "dW", true));
  TP_TRY(check_ptrs(H, p, "H", dW == nullptr));
  if (act != TP_ACT_NONE) TP_TRY(check_ptrs(Z, p, "Z", false));
  if (dbias) TP_TRY(check_ptr(dbias, "dbias"));
  TP_TRY(check_row_bytes(k, plan->dtype, "row shard width"));
  TP_TRY(check_row_bytes(h, plan->dtype, "hidden"));
  if (T == 0) return TP_OK;
  cudaStream_t st = as_stream(stream);

  // dH_i = dY W_i (W_i is [h, k]: (n = j, k = c) at W_i + c*k + j -> MN-major B),
  // with the activation derivative fused in the epilogue.
  GemmBatch b{};
  b.n = p;
  b.a_mn = false;
  b.b_mn = true;
  b.out_f32 = plan->dtype == TP_F32;
  for (int i = 0; i < p; ++i) {
    GemmProblem& g = b.g[i];
    g.M = static_cast<int>(T);
    g.N = k;
    g.K = h;
    g.A = dY;
    g.lda = h;
    g.B = W[i];
    g.ldb = k;
    g.D = dZ[i];
    g.ldd = nz;
    g.aux = act != TP_ACT_NONE ? Z[i] : nullptr;
    g.ldaux = nz;
    g.nh = k;
  }
  b.epi = act == TP_ACT_GELU ? EPI_DGELU : act == TP_ACT_SWIGLU ? EPI_DSWIGLU : EPI_STORE;
  GemmBatch w{};
  if (dW) {
    // dW_i [h, k] = dY^T H_i: A(m, t) = dY[t, m] (MN-major), B(n, t) = H_i[t, n] (MN-major).
    w.n = p;
    w.a_mn = true;
    w.b_mn = true;
    w.epi = EPI_STORE;
    w.out_f32 = plan->dtype == TP_F32;
    for (int i = 0; i < p; ++i) {
      GemmProblem& g = w.g[i];
      g.M = h;
      g.N = k;
      g.K = static_cast<int>(T);
      g.A = dY;
      g.lda = h;
      g.B = H[i];
      g.ldb = k;
      g.D = dW[i];
      g.ldd = k;
    }
  }
  if (plan->defer_bwd && plan->dtype == TP_BF16 && (dW || dbias)) {
    // Deferred: dH on the caller's stream, dW and db on the side stream,
    // joined by tp_backward_join (dW without a K split: no shared scratch).
    TP_TRY(flush_wgrad(plan));
    SideStream* sd = nullptr;
    TP_TRY(side_stream(&sd));
    TP_TRY(cuda_status(cudaEventRecord(sd->fork, st), "cudaEventRecord(fork)"));
    TP_TRY(cuda_status(cudaStreamWaitEvent(sd->s, sd->fork, 0), "cudaStreamWaitEvent(fork)"));
    TP_TRY(run_gemm(plan, b, st));
    if (dW) TP_TRY(launch_gemm_bf16(w, sd->s));
    if (dbias) {
      PtrArray X{};
      MutPtrArray O{};
      X.p[0] = dY;
      O.p[0] = dbias;
      TP_TRY(launch_column_sum_deferred(plan, X, 1, T, h, h, O, plan->dtype, sd->s));
    }
    return TP_OK;
  }
  // dH beside the weight gradient (joined when this call returns), or before it
  std::unique_ptr<SideGemm> side;
  if (dW && concurrent_bwd(plan, b, w)) {
    side.reset(new SideGemm(plan, b, st));
    TP_TRY(side->status());
  } else {
    TP_TRY(run_gemm(plan, b, st));
  }
  // The bias gradient reads only dY: beside the weight gradient too (after dH on
  // the side stream, its partials past the weight gradient's workspace).
  if (dbias)
    TP_TRY(launch_column_sum(plan, dY, T, h, h, dbias, 0, plan->dtype, side ? side->stream() : st,
                             side ? wgrad_workspace(plan, w, false) : 0));
  if (dW) TP_TRY(issue_wgrad(plan, w, st, !side, true));
  return TP_OK;
}

// dX mode: 0 = partials (dX_out[i] per shard), 1 = summed (dX_out[0] full),
// 2 = summed and scattered by sequence (dX_out[j] = rows of shard j),
// 3 = summed and pushed by row block into the peer group's receive buffers.
static tp_status column_bwd_common(tp_plan* plan, tp_which which, int64_t T, const void* X,
                                   const void* const* dZ, const void* const* W, void* const* dW,
                                   float* const* dbias, void* const* dX_out, int mode,
                                   cudaStream_t st, const tp_peer_group* peer = nullptr) {
  TP_TRY(check_plan(plan));
  TP_TRY(check_T(T));
  ColShape cs{};
  TP_TRY(col_shape(plan, which, &cs));
  const int p = plan->p, h = plan->hidden;
  const int n = cs.n_w;
  TP_TRY(check_ptrs(dZ, p, "dZ", false));
  TP_TRY(check_ptrs(W, p, "W", false));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dW), p, "dW", true));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dbias), p, "dbias", true));
  const int nout = mode == 1 ? 1 : p;
  if (mode == 3) TP_TRY(check_peer_push(plan, peer, T));
  else TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(dX_out), nout, "dX", mode == 0));
  if (mode == 2 && T % p)
    return fail(TP_ERR_DIVISIBILITY, "T = %lld is not divisible by p = %d", (long long)T, p);
  if (dW) TP_TRY(check_ptr(X, "X"));
  TP_TRY(check_row_bytes(n, plan->dtype, "dZ_i width"));
  TP_TRY(check_row_bytes(h, plan->dtype, "hidden"));
  if (mode == 0) TP_TRY(check_row_bytes(h, plan->partial_dtype, "hidden (dX partials)"));
  if (T == 0) return TP_OK;
  GemmBatch w{};
  if (dW) {
    // dW_i [n, h] = dZ_i^T X: A(m, t) = dZ_i[t, m] (MN-major), B(c, t) = X[t, c] (MN-major).
    w.n = p;
    w.a_mn = true;
    w.b_mn = true;
    w.epi = EPI_STORE;
    w.out_f32 = plan->dtype == TP_F32;
    for (int i = 0; i < p; ++i) {
      GemmProblem& g = w.g[i];
      g.M = n;
      g.N = h;
      g.K = static_cast<int>(T);
      g.A = dZ[i];
      g.lda = n;
      g.B = X;
      g.ldb = h;
      g.D = dW[i];
      g.ldd = h;
    }
  }
  GemmBatch d{};
  if (dX_out || mode == 3) {
    // dX_i [T, h] = dZ_i W_i: A = dZ_i (K-major), B(c, j) = W_i[j, c] (MN-major).
    d.n = p;
    d.a_mn = false;
    d.b_mn = true;
    d.epi = EPI_STORE;
    d.out_f32 = (mode == 0 ? plan->partial_dtype : plan->dtype) == TP_F32;
    d.kcat = mode != 0;
    for (int i = 0; i < p; ++i) {
      GemmProblem& g = d.g[i];
      g.M = static_cast<int>(T);
      g.N = h;
      g.K = n;
      g.A = dZ[i];
      g.lda = n;
      g.B = W[i];
      g.ldb = h;
      g.D = mode == 3 ? nullptr : mode == 0 ? dX_out[i] : dX_out[0];
      g.ldd = h;
    }
    if (mode == 2) {
      d.scatter_n = p;
      d.rows_per_out = T / p;
      for (int j = 0; j < p; ++j) d.out_seq[j] = dX_out[j];
    } else if (mode == 3) {
      peer_push_targets(d, peer, T, h);
    }
  }
  const bool has_dx = dX_out || mode == 3;
  if (plan->defer_bwd && plan->dtype == TP_BF16 && (dW || dbias)) {
    // Deferred: dX on the caller's stream, dW and db on the side stream,
    // joined by tp_backward_join (dW without a K split: no shared scratch).
    TP_TRY(flush_wgrad(plan));
    SideStream* sd = nullptr;
    TP_TRY(side_stream(&sd));
    TP_TRY(cuda_status(cudaEventRecord(sd->fork, st), "cudaEventRecord(fork)"));
    TP_TRY(cuda_status(cudaStreamWaitEvent(sd->s, sd->fork, 0), "cudaStreamWaitEvent(fork)"));
    if (has_dx) TP_TRY(run_gemm(plan, d, st));
    if (dW) TP_TRY(launch_gemm_bf16(w, sd->s));
    if (dbias)
      TP_TRY(launch_column_sum_deferred(plan, to_arr(dZ, p), p, T, n, n,
                                        to_marr(reinterpret_cast<void* const*>(dbias), p), plan->dtype, sd->s));
    return TP_OK;
  }
  // dX beside the weight gradient (joined when this call returns), or after it
  std::unique_ptr<SideGemm> side;
  if (dW && has_dx && concurrent_bwd(plan, d, w)) {
    side.reset(new SideGemm(plan, d, st));
    TP_TRY(side->status());
  }
  // The bias gradients read only dZ: beside the weight gradient too (after dX on
  // the side stream, their partials past the weight gradient's workspace).
  if (dbias)
    TP_TRY(launch_column_sum_grouped(plan, to_arr(dZ, p), p, T, n, n,
                                     to_marr(reinterpret_cast<void* const*>(dbias), p), 0, plan->dtype,
                                     side ? side->stream() : st, side ? wgrad_workspace(plan, w, false) : 0));
  if (dW) TP_TRY(issue_wgrad(plan, w, st, !side, false));
  else TP_TRY(flush_wgrad(plan));
  if (has_dx && !side) TP_TRY(run_gemm(plan, d, st));
  return TP_OK;
}

tp_status tp_column_bwd(tp_plan* plan, tp_which which, int64_t T, const void* X,
                        const void* const* dZ, const void* const* W, void* const* dW,
                        float* const* dbias, void* const* dX_partials, void* stream) {
  return column_bwd_common(plan, which, T, X, dZ, W, dW, dbias, dX_partials, 0, as_stream(stream));
}

tp_status tp_column_bwd_reduce(tp_plan* plan, tp_which which, int64_t T, const void* X,
                               const void* const* dZ, const void* const* W, void* const* dW,
                               float* const* dbias, void* dX, void* stream) {
  void* out[1] = {dX};
  return column_bwd_common(plan, which, T, X, dZ, W, dW, dbias, out, 1, as_stream(stream));
}

tp_status tp_column_bwd_reduce_scatter_seq(tp_plan* plan, tp_which which, int64_t T,
                                           const void* X, const void* const* dZ,
                                           const void* const* W, void* const* dW,
                                           float* const* dbias, void* const* dX_seq,
                                           void* stream) {
  return column_bwd_common(plan, which, T, X, dZ, W, dW, dbias, dX_seq, 2, as_stream(stream));
}

tp_status tp_column_bwd_push_peer(tp_plan* plan, tp_which which, int64_t T, const void* X,
                                  const void* const* dZ, const void* const* W, void* const* dW,
                                  float* const* dbias, const tp_peer_group* g, uint32_t epoch,
                                  void* stream) {
  const cudaStream_t st = as_stream(stream);
  TP_TRY(column_bwd_common(plan, which, T, X, dZ, W, dW, dbias, nullptr, 3, st, g));
  return launch_peer_signal(g, g->rank, epoch, st);
}

}  // extern "C"
