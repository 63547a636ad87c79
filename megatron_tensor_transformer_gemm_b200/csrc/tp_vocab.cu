// Vocab-parallel embedding and cross-entropy (TP walkthrough 2kiu.com §6.2;
// 张量并行 wiki, 工程实践): the padded vocab Vp is split into p shards of
// Vs = Vp / p rows; shard i owns vocab ids [i*Vs, (i+1)*Vs).
//
//  embed_fwd   Y[t] = E_{s}[id - s*Vs] with s the owning shard: the sum over
//              shards of the partial lookups (zero outside a shard's range) has
//              exactly one non-zero term, so the kernel reads it directly.
//  embed_bwd   dE[v] = sum over tokens with id == v of dY[t], deterministic: a
//              CTA owns 32 vocab rows x 512 columns, walks the ids in token
//              order and accumulates the matching dY rows in fp32 in shared
//              memory (no atomics), then writes its rows to the owning shard.
//  ce          per token row: max, sum of exp and the target logit over the
//              real (non-padding) columns of all shards -- the shards' local
//              max / sum / target reduced over shards -- then loss = lse - z_t
//              and the gradient of the scaled loss, (softmax - onehot) * scale,
//              written to dlogits (which may alias the logits).
#include <algorithm>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {

using tpi::MutPtrArray;
using tpi::PtrArray;

constexpr unsigned kStatusBadIndex = 2u;

__global__ void embed_fwd_kernel(const int32_t* ids, const __grid_constant__ PtrArray E, int vocab,
                                 int64_t Vs, int64_t T, int64_t vpr, uint4* Y,
                                 unsigned* status) {
  const int64_t total = T * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vpr, c = i - t * vpr;
    const int id = ids[t];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (id >= 0 && id < vocab) {
      const int s = static_cast<int>(id / Vs);
      v = reinterpret_cast<const uint4*>(E.p[s])[(id - s * Vs) * vpr + c];
    } else if (c == 0) {
      atomicOr(status, kStatusBadIndex);
    }
    Y[t * vpr + c] = v;
  }
}

constexpr int kEmbRows = 32;    // vocab rows per CTA
constexpr int kEmbCols = 512;   // columns per CTA (2 per thread)
constexpr int kEmbThreads = 256;
constexpr int kIdTile = 1024;

// dE rows [v0, v0 + 32) x columns [c0, c0 + 512) of the padded vocab.
template <typename T>
__global__ void __launch_bounds__(kEmbThreads) embed_bwd_kernel(
    const int32_t* ids, int64_t ntok, const T* dY, int64_t h, int vocab, int64_t Vs, int64_t Vp,
    const __grid_constant__ MutPtrArray dE) {
  extern __shared__ float acc[];  // [kEmbRows][kEmbCols]
  __shared__ int match[kIdTile];
  __shared__ int nmatch;
  __shared__ int wcount[kEmbThreads / 32];
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * kEmbRows;
  const int64_t c0 = static_cast<int64_t>(blockIdx.y) * kEmbCols;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kEmbRows * kEmbCols; i += kEmbThreads) acc[i] = 0.f;
  __syncthreads();
  for (int64_t base = 0; base < ntok; base += kIdTile) {
    // Ordered compaction of this tile's matching tokens: thread tid checks
    // tokens base + tid*4 .. +3, warp ballots give each match its rank.
    int mine[4], cnt = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t t = base + tid * 4 + k;
      mine[k] = -1;
      if (t < ntok) {
        const int id = ids[t];
        if (id >= v0 && id < v0 + kEmbRows && id < vocab) {
          mine[k] = static_cast<int>(t - base);
          ++cnt;
        }
      }
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) wcount[warp] = incl;
    __syncthreads();
    int woff = 0, total = 0;
    for (int w = 0; w < kEmbThreads / 32; ++w) {
      if (w < warp) woff += wcount[w];
      total += wcount[w];
    }
    int pos = woff + incl - cnt;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (mine[k] >= 0) match[pos++] = mine[k];
    if (tid == 0) nmatch = total;
    __syncthreads();
    // Accumulate the matches in token order; thread tid owns columns 2 tid, 2 tid + 1.
    const int64_t col = c0 + 2 * tid;
    for (int m = 0; m < nmatch; ++m) {
      const int64_t t = base + match[m];
      const int r = ids[t] - static_cast<int>(v0);
      if (col < h) {
        float a, b;
        if constexpr (sizeof(T) == 2) {
          const float2 f = tpd::unpack_bf16x2(*reinterpret_cast<const uint32_t*>(dY + t * h + col));
          a = f.x;
          b = f.y;
        } else {
          a = dY[t * h + col];
          b = dY[t * h + col + 1];
        }
        acc[r * kEmbCols + 2 * tid] += a;
        acc[r * kEmbCols + 2 * tid + 1] += b;
      }
    }
    __syncthreads();
  }
  // Write the rows to their shards (every padded row gets written: zeros if unused).
  for (int r = 0; r < kEmbRows; ++r) {
    const int64_t v = v0 + r;
    if (v >= Vp) break;
    const int s = static_cast<int>(v / Vs);
    const int64_t col = c0 + 2 * tid;
    if (col < h) {
      T* dst = static_cast<T*>(dE.p[s]) + (v - s * Vs) * h + col;
      if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<uint32_t*>(dst) =
            tpd::pack_bf16x2(acc[r * kEmbCols + 2 * tid], acc[r * kEmbCols + 2 * tid + 1]);
      } else {
        dst[0] = acc[r * kEmbCols + 2 * tid];
        dst[1] = acc[r * kEmbCols + 2 * tid + 1];
      }
    }
  }
}

template <int THREADS>
__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, u) : v + u;
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < THREADS / 32; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

template <typename T>
__device__ __forceinline__ float ld_logit(const void* p, int64_t i) {
  if constexpr (sizeof(T) == 2) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  else return static_cast<const float*>(p)[i];
}

template <typename T>
__device__ __forceinline__ void st_grad(void* p, int64_t i, float v) {
  if constexpr (sizeof(T) == 2) static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else static_cast<float*>(p)[i] = v;
}

// One CTA per token row t.
template <typename T, int THREADS>
__global__ void __launch_bounds__(THREADS) vocab_ce_kernel(
    const __grid_constant__ PtrArray L, const __grid_constant__ MutPtrArray G, int p, int64_t Vs,
    int vocab, const int32_t* labels, float scale, float* loss, float* lse_out,
    unsigned* status) {
  __shared__ float red[THREADS / 32];
  __shared__ float ztarget;
  const int64_t t = blockIdx.x;
  const int label = labels[t];
  const int64_t row_total = static_cast<int64_t>(p) * Vs;
  if (threadIdx.x == 0) {
    ztarget = 0.f;
    if (label >= vocab) atomicOr(status, kStatusBadIndex);
  }
  // pass 1: max over real columns (and the target logit)
  float mx = -INFINITY;
  for (int64_t v = threadIdx.x; v < row_total; v += THREADS) {
    if (v >= vocab) break;
    const int s = static_cast<int>(v / Vs);
    const float z = ld_logit<T>(L.p[s], t * Vs + (v - s * Vs));
    mx = fmaxf(mx, z);
    if (v == label) ztarget = z;
  }
  const float m = block_reduce<THREADS>(mx, red, true);
  // pass 2: sum of exp(z - m)
  float se = 0.f;
  for (int64_t v = threadIdx.x; v < vocab; v += THREADS) {
    const int s = static_cast<int>(v / Vs);
    se += expf(ld_logit<T>(L.p[s], t * Vs + (v - s * Vs)) - m);
  }
  const float S = block_reduce<THREADS>(se, red, false);
  const float lse = m + logf(S);
  const bool ignore = label < 0 || label >= vocab;
  if (threadIdx.x == 0) {
    loss[t] = ignore ? 0.f : lse - ztarget;
    if (lse_out) lse_out[t] = lse;
  }
  // pass 3: gradient of scale * loss (zero for ignored tokens and padding columns)
  if (G.p[0] == nullptr) return;
  for (int64_t v = threadIdx.x; v < row_total; v += THREADS) {
    const int s = static_cast<int>(v / Vs);
    const int64_t off = t * Vs + (v - s * Vs);
    float g = 0.f;
    if (!ignore && v < vocab) g = (expf(ld_logit<T>(L.p[s], off) - lse) - (v == label ? 1.f : 0.f)) * scale;
    st_grad<T>(G.p[s], off, g);
  }
}

int sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  return n;
}

}  // namespace

namespace tpi {

tp_status launch_embedding_fwd(const int32_t* ids, const PtrArray& E, int vocab, int64_t Vs,
                               int64_t T, int64_t h, tp_dtype dt, void* Y, cudaStream_t st) {
  unsigned* status = nullptr;
  tp_status s = device_status_word(&status);
  if (s != TP_OK) return s;
  const int64_t vpr = h * static_cast<int64_t>(dsize(dt)) / 16;
  const int64_t total = T * vpr;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, sms() * 16LL));
  embed_fwd_kernel<<<blocks, 256, 0, st>>>(ids, E, vocab, Vs, T, vpr, static_cast<uint4*>(Y), status);
  return after_launch("embedding_fwd");
}

tp_status launch_embedding_bwd(const int32_t* ids, int64_t T, const void* dY, int64_t h, int vocab,
                               int64_t Vp, int64_t Vs, const MutPtrArray& dE, tp_dtype dt,
                               cudaStream_t st) {
  const int smem = kEmbRows * kEmbCols * 4;
  static bool attr[2] = {false, false};
  const int k = dt == TP_BF16 ? 0 : 1;
  if (!attr[k]) {
    cudaError_t e = dt == TP_BF16
        ? cudaFuncSetAttribute(embed_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
        : cudaFuncSetAttribute(embed_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    tp_status s = cuda_status(e, "cudaFuncSetAttribute(embedding_bwd)");
    if (s != TP_OK) return s;
    attr[k] = true;
  }
  dim3 grid(static_cast<unsigned>((Vp + kEmbRows - 1) / kEmbRows),
            static_cast<unsigned>((h + kEmbCols - 1) / kEmbCols));
  if (dt == TP_BF16)
    embed_bwd_kernel<__nv_bfloat16><<<grid, kEmbThreads, smem, st>>>(
        ids, T, static_cast<const __nv_bfloat16*>(dY), h, vocab, Vs, Vp, dE);
  else
    embed_bwd_kernel<float><<<grid, kEmbThreads, smem, st>>>(ids, T, static_cast<const float*>(dY), h,
                                                            vocab, Vs, Vp, dE);
  return after_launch("embedding_bwd");
}

tp_status launch_vocab_ce(const PtrArray& L, const MutPtrArray& G, int p, int64_t Vs, int vocab,
                          const int32_t* labels, float scale, float* loss, float* lse, int64_t T,
                          tp_dtype dt, cudaStream_t st) {
  unsigned* status = nullptr;
  tp_status s = device_status_word(&status);
  if (s != TP_OK) return s;
  if (dt == TP_BF16)
    vocab_ce_kernel<__nv_bfloat16, 256><<<static_cast<unsigned>(T), 256, 0, st>>>(
        L, G, p, Vs, vocab, labels, scale, loss, lse, status);
  else
    vocab_ce_kernel<float, 256><<<static_cast<unsigned>(T), 256, 0, st>>>(L, G, p, Vs, vocab, labels,
                                                                         scale, loss, lse, status);
  return after_launch("vocab_cross_entropy");
}

}  // namespace tpi
