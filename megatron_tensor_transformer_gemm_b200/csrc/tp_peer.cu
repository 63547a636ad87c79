// Across GPUs over peer memory: the row layer's all-reduce as a reduce-scatter
// whose transfer the producing GEMM makes from its epilogue (tp_api.cu, the
// push calls), then the reduce of the received slots with an all-gather push
// of the result, then a wait for every rank's push ("张量并行", Megatron-SP:
// all-reduce = reduce-scatter + all-gather at the same traffic; TP walkthrough
// §4.1: the row output's partial sums are all-reduced).
//
// Ordering between GPUs uses flag words in each rank's memory:
//   - a step that has written into other ranks' memory is followed on its
//     stream by peer_signal_kernel, which (after the writer grid completed)
//     fences at system scope and stores the epoch with release semantics into
//     each destination's flag word for this rank;
//   - a step that reads what others wrote first loads those flag words with
//     acquire semantics at system scope until each reached the epoch.
// Every wait is bounded by the peer wait limit; on time-out the kernel sets
// the device status word and returns without touching the data.
#include <algorithm>
#include <atomic>
#include <cstring>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {

using tpi::fail;

constexpr uint64_t kDefaultPeerWaitNs = 5000000000ull;  // 5 s
std::atomic<uint64_t> g_peer_wait_ns{kDefaultPeerWaitNs};

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until *f has reached `epoch` (wrap-safe comparison). On time-out
// it sets the status word and returns false.
__device__ bool wait_flag(const uint32_t* f, uint32_t epoch, uint64_t limit_ns, unsigned* status) {
  if (static_cast<int32_t>(ld_acquire_sys(f) - epoch) >= 0) return true;
  const uint64_t t0 = tpd::globaltimer();
  for (uint32_t it = 1; it < tpd::kWaitLimitPolls; ++it) {
    __nanosleep(128);
    if (static_cast<int32_t>(ld_acquire_sys(f) - epoch) >= 0) return true;
    if ((it & 63u) == 0 && tpd::globaltimer() - t0 > limit_ns) break;
  }
  atomicOr(status, tpd::kStatusTimeout);
  return false;
}

struct SignalParams {
  uint32_t* word[TP_MAX_SHARDS];  // one flag word per destination rank
  int n;
  uint32_t epoch;
};

// Raise the flags after the previous grid on the stream (the writer) has
// completed: griddepcontrol.wait in pdl_entry returns once its memory
// operations are performed; the system-scope fence then orders them before
// the release store that the destination's acquire load observes.
__global__ void peer_signal_kernel(const __grid_constant__ SignalParams p) {
  tpd::pdl_entry();
  const int i = threadIdx.x;
  if (i < p.n) {
    __threadfence_system();
    st_release_sys(p.word[i], p.epoch);
  }
}

__global__ void peer_wait_kernel(const uint32_t* done, int n, uint32_t epoch, uint64_t limit_ns,
                                 unsigned* status) {
  tpd::pdl_entry();
  const int i = threadIdx.x;
  if (i < n) (void)wait_flag(done + i, epoch, limit_ns, status);
}

struct ReduceParams {
  const __nv_bfloat16* recv;  // this rank's receive buffer: world slots of [t, h]
  const uint32_t* arrived;    // this rank's arrived words, one per source rank
  const __nv_bfloat16* bias;  // [h] or null
  const __nv_bfloat16* res;   // [t, h] or null
  __nv_bfloat16* out[TP_MAX_SHARDS];
  int n_out, world, rank;
  int64_t t, vpr;  // rows of a slot; 16-byte vectors per row (h / 8)
  uint32_t epoch;
  uint64_t limit_ns;
  unsigned* status;
};

__device__ __forceinline__ void acc8(float (&a)[8], const uint4& u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = tpd::unpack_bf16x2(w[k]);
    a[2 * k] += f.x;
    a[2 * k + 1] += f.y;
  }
}

// out[k][r, :] = sum_{s<world} slot_s[r, :] (fp32, order 0..world-1) + bias +
// res[r, :], rounded to bf16, for every destination k. A thread owns one
// 16-byte vector (8 columns) of a row and walks the slot's rows and vectors
// with the grid's stride, two vectors per step with all their loads issued
// before the sums. Each CTA first waits for every source's block: thread s
// polls source s's word, so the system-scope acquire loads overlap.
template <int NMAX>
__global__ void __launch_bounds__(256) peer_reduce_kernel(const __grid_constant__ ReduceParams p) {
  tpd::pdl_entry();
  const bool ok = threadIdx.x >= p.world || wait_flag(p.arrived + threadIdx.x, p.epoch, p.limit_ns, p.status);
  if (!__syncthreads_and(ok)) return;
  const int64_t total = p.t * p.vpr;
  const int64_t slot = p.t * p.vpr * 8;  // elements per slot
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float b[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) b[k] = 0.f;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < total; v += 2 * stride) {
    const int64_t v2 = v + stride;
    const bool two = v2 < total;
    uint4 u1[NMAX], u2[NMAX];
#pragma unroll
    for (int s = 0; s < NMAX; ++s) {
      if (s < p.world) {
        const __nv_bfloat16* base = p.recv + s * slot;
        u1[s] = __ldcs(reinterpret_cast<const uint4*>(base + v * 8));
        if (two) u2[s] = __ldcs(reinterpret_cast<const uint4*>(base + v2 * 8));
      }
    }
    float a1[8], a2[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a1[k] = a2[k] = 0.f;
#pragma unroll
    for (int s = 0; s < NMAX; ++s) {
      if (s < p.world) {
        acc8(a1, u1[s]);
        if (two) acc8(a2, u2[s]);
      }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (half == 1 && !two) break;
      const int64_t vv = half ? v2 : v;
      float(&a)[8] = half ? a2 : a1;
      const int64_t cv = vv % p.vpr;
      if (p.bias) {
        for (int k = 0; k < 8; ++k) b[k] = 0.f;
        acc8(b, __ldg(reinterpret_cast<const uint4*>(p.bias) + cv));
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] += b[k];
      }
      if (p.res) acc8(a, __ldcs(reinterpret_cast<const uint4*>(p.res) + vv));
      const uint4 o = make_uint4(tpd::pack_bf16x2(a[0], a[1]), tpd::pack_bf16x2(a[2], a[3]),
                                 tpd::pack_bf16x2(a[4], a[5]), tpd::pack_bf16x2(a[6], a[7]));
      // destinations in rotated order, so the ranks' pushes spread over the peers
      for (int k = 0; k < p.n_out; ++k) {
        int d = p.rank + 1 + k;
        while (d >= p.n_out) d -= p.n_out;
        reinterpret_cast<uint4*>(p.out[d])[vv] = o;
      }
    }
  }
}

struct PushParams {
  const uint4* src;  // [rows, cols] bf16 as 16-byte vectors, dense
  uint4* out[TP_MAX_SHARDS];
  int n_out, rank;
  int64_t total;     // vectors
};

// out[k][v] = src[v] for every destination, in rotated order as in the reduce.
__global__ void __launch_bounds__(256) peer_push_kernel(const __grid_constant__ PushParams p) {
  tpd::pdl_entry();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < p.total; v += stride) {
    const uint4 x = __ldcs(p.src + v);
    for (int k = 0; k < p.n_out; ++k) {
      int d = p.rank + 1 + k;
      while (d >= p.n_out) d -= p.n_out;
      p.out[d][v] = x;
    }
  }
}

}  // namespace

namespace tpi {

tp_status check_peer_group(const tp_peer_group* g) {
  if (!g) return fail(TP_ERR_ARG, "peer group is NULL");
  if (g->world < 1 || g->world > TP_MAX_SHARDS)
    return fail(TP_ERR_ARG, "peer group world = %d outside [1, %d]", g->world, TP_MAX_SHARDS);
  if (g->rank < 0 || g->rank >= g->world)
    return fail(TP_ERR_ARG, "peer group rank = %d outside [0, %d)", g->rank, g->world);
  if (g->recv_elems < 0) return fail(TP_ERR_ARG, "peer group recv_elems = %lld", (long long)g->recv_elems);
  for (int d = 0; d < g->world; ++d) {
    if (!g->flags[d] || !g->recv[d]) return fail(TP_ERR_ARG, "peer group: rank %d's flags or receive buffer is NULL", d);
    if (!aligned16(g->flags[d]) || !aligned16(g->recv[d]))
      return fail(TP_ERR_ALIGN, "peer group: rank %d's flags or receive buffer is not 16-byte aligned", d);
  }
  return TP_OK;
}

// Raise flag word `word` on every rank of the group to `epoch`, after the
// previous grid on `st` has completed.
tp_status launch_peer_signal(const tp_peer_group* g, int word, uint32_t epoch, cudaStream_t st) {
  SignalParams sp{};
  sp.n = g->world;
  sp.epoch = epoch;
  for (int d = 0; d < g->world; ++d) sp.word[d] = g->flags[d] + word;
  (void)launch(peer_signal_kernel, dim3(1), dim3(32), 0, st, sp);
  return after_launch("peer_signal");
}

}  // namespace tpi

using namespace tpi;

extern "C" {

tp_status tp_peer_alloc(size_t bytes, void** ptr, void* handle) {
  if (!ptr || !handle) return fail(TP_ERR_ARG, "tp_peer_alloc: ptr and handle must be non-NULL");
  if (bytes == 0) return fail(TP_ERR_ARG, "tp_peer_alloc: bytes = 0");
  *ptr = nullptr;
  void* p = nullptr;
  TP_TRY(cuda_status(cudaMalloc(&p, bytes), "cudaMalloc (peer memory)"));
  cudaIpcMemHandle_t h;
  tp_status s = cuda_status(cudaMemset(p, 0, bytes), "cudaMemset (peer memory)");
  if (s == TP_OK) s = cuda_status(cudaIpcGetMemHandle(&h, p), "cudaIpcGetMemHandle");
  if (s != TP_OK) {
    cudaFree(p);
    return s;
  }
  static_assert(sizeof(cudaIpcMemHandle_t) == TP_PEER_HANDLE_BYTES, "IPC handle size");
  memcpy(handle, &h, sizeof(h));
  *ptr = p;
  return TP_OK;
}

tp_status tp_peer_free(void* ptr) {
  if (!ptr) return TP_OK;
  return cuda_status(cudaFree(ptr), "cudaFree (peer memory)");
}

tp_status tp_peer_open(const void* handle, void** ptr) {
  if (!ptr || !handle) return fail(TP_ERR_ARG, "tp_peer_open: handle and ptr must be non-NULL");
  *ptr = nullptr;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  return cuda_status(cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess), "cudaIpcOpenMemHandle");
}

tp_status tp_peer_close(void* ptr) {
  if (!ptr) return TP_OK;
  return cuda_status(cudaIpcCloseMemHandle(ptr), "cudaIpcCloseMemHandle");
}

tp_status tp_peer_set_wait_limit(int64_t ns) {
  if (ns < 0 || ns > 60000000000LL) return fail(TP_ERR_ARG, "peer wait limit %lld ns outside [0, 60e9]", (long long)ns);
  g_peer_wait_ns.store(ns == 0 ? kDefaultPeerWaitNs : static_cast<uint64_t>(ns));
  return TP_OK;
}

tp_status tp_peer_reduce(const tp_peer_group* g, int64_t T, int hidden, const void* bias,
                         const void* residual, int n_out, void* const* out, uint32_t epoch,
                         void* stream) {
  TP_TRY(check_peer_group(g));
  if (T < 0) return fail(TP_ERR_ARG, "T = %lld", (long long)T);
  if (hidden <= 0 || hidden % 8)
    return fail(TP_ERR_ALIGN, "hidden = %d is not a positive multiple of 8 (16-byte rows)", hidden);
  if (T % g->world)
    return fail(TP_ERR_DIVISIBILITY, "T = %lld is not divisible by world = %d", (long long)T, g->world);
  if (T * hidden > g->recv_elems)
    return fail(TP_ERR_ARG, "T x hidden = %lld exceeds the receive buffers (%lld elements)",
                (long long)(T * hidden), (long long)g->recv_elems);
  if (n_out < 1 || n_out > TP_MAX_SHARDS) return fail(TP_ERR_ARG, "n_out = %d outside [1, %d]", n_out, TP_MAX_SHARDS);
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(out), n_out, "out", false));
  if (bias) TP_TRY(check_ptr(bias, "bias"));
  if (residual) TP_TRY(check_ptr(residual, "residual"));
  unsigned* status = nullptr;
  TP_TRY(device_status_word(&status));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ReduceParams p{};
  p.recv = static_cast<const __nv_bfloat16*>(g->recv[g->rank]);
  p.arrived = g->flags[g->rank];
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.res = static_cast<const __nv_bfloat16*>(residual);
  for (int k = 0; k < n_out; ++k) p.out[k] = static_cast<__nv_bfloat16*>(out[k]);
  p.n_out = n_out;
  p.world = g->world;
  p.rank = g->rank;
  p.t = T / g->world;
  p.vpr = hidden / 8;
  p.epoch = epoch;
  p.limit_ns = g_peer_wait_ns.load();
  p.status = status;
  // one CTA per 512 vectors (two per thread), at most as many as are resident at once
  // (SM count and occupancy cached per device)
  const int64_t units = std::max<int64_t>(1, (p.t * p.vpr + 511) / 512);
  auto run = [&](auto kernel) -> tp_status {
    int64_t grid = 1;
    TP_TRY(persistent_grid(reinterpret_cast<const void*>(kernel), 256, 0, units, &grid));
    (void)launch(kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, p);
    return TP_OK;
  };
  if (g->world <= 2) TP_TRY(run(peer_reduce_kernel<2>));
  else if (g->world <= 4) TP_TRY(run(peer_reduce_kernel<4>));
  else if (g->world <= 8) TP_TRY(run(peer_reduce_kernel<8>));
  else TP_TRY(run(peer_reduce_kernel<TP_MAX_SHARDS>));
  TP_TRY(after_launch("peer_reduce"));
  return launch_peer_signal(g, TP_MAX_SHARDS + g->rank, epoch, st);
}

tp_status tp_all_gather_push_peer(const tp_peer_group* g, int64_t rows, int cols, const void* x,
                                  void* const* out, uint32_t epoch, void* stream) {
  TP_TRY(check_peer_group(g));
  if (rows < 0) return fail(TP_ERR_ARG, "rows = %lld", (long long)rows);
  if (cols <= 0 || cols % 8)
    return fail(TP_ERR_ALIGN, "cols = %d is not a positive multiple of 8 (16-byte rows)", cols);
  TP_TRY(check_ptr(x, "x"));
  TP_TRY(check_ptrs(reinterpret_cast<const void* const*>(out), g->world, "out", false));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (rows > 0) {
    PushParams p{};
    p.src = static_cast<const uint4*>(x);
    for (int d = 0; d < g->world; ++d) p.out[d] = static_cast<uint4*>(out[d]);
    p.n_out = g->world;
    p.rank = g->rank;
    p.total = rows * (cols / 8);
    int64_t grid = 1;
    TP_TRY(persistent_grid(reinterpret_cast<const void*>(peer_push_kernel), 256, 0,
                           std::max<int64_t>(1, (p.total + 255) / 256), &grid));
    (void)launch(peer_push_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, p);
    TP_TRY(after_launch("peer_push"));
  }
  return launch_peer_signal(g, TP_MAX_SHARDS + g->rank, epoch, st);
}

tp_status tp_peer_wait(const tp_peer_group* g, uint32_t epoch, void* stream) {
  TP_TRY(check_peer_group(g));
  unsigned* status = nullptr;
  TP_TRY(device_status_word(&status));
  (void)launch(peer_wait_kernel, dim3(1), dim3(32), 0, reinterpret_cast<cudaStream_t>(stream),
               static_cast<const uint32_t*>(g->flags[g->rank] + TP_MAX_SHARDS), g->world, epoch,
               g_peer_wait_ns.load(), status);
  return after_launch("peer_wait");
}

}  // extern "C"
