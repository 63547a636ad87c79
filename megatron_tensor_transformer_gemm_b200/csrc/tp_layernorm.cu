// LayerNorm over the full hidden dim, forward (optionally fused with the
// sequence all-gather of Megatron-SP: each output row comes from the sequence
// shard that owns it) and backward (dx per row; dgamma/dbeta as deterministic
// two-pass column sums).
//
// One CTA normalises one row; a thread owns up to 8 16-byte vectors of it, so
// the row stays in registers between the statistics and the output pass.
// Statistics are fp32: mean, then the biased variance of (x - mean).
#include <algorithm>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {

using tpi::PtrArray;

constexpr float kEps = 1e-5f;
constexpr int kVptMax = 8;  // 16-byte vectors per thread

template <typename T>
struct LnVec;
template <>
struct LnVec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const void* p, float* f) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    float2 a = tpd::unpack_bf16x2(u.x), b = tpd::unpack_bf16x2(u.y);
    float2 c = tpd::unpack_bf16x2(u.z), d = tpd::unpack_bf16x2(u.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
  }
  __device__ static void store(void* p, const float* f) {
    *reinterpret_cast<uint4*>(p) =
        make_uint4(tpd::pack_bf16x2(f[0], f[1]), tpd::pack_bf16x2(f[2], f[3]),
                   tpd::pack_bf16x2(f[4], f[5]), tpd::pack_bf16x2(f[6], f[7]));
  }
};
template <>
struct LnVec<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float* f) {
    float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  __device__ static void store(void* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};

// Sum over the CTA (THREADS <= 1024), same result in every thread.
template <int THREADS>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  constexpr int W = THREADS / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < W; ++w) s += red[w];
  return s;
}

// y row r = LN(x row r); x row r is row (r - j*rows_per_src) of src.p[j].
template <typename T, int THREADS>
__global__ void __launch_bounds__(THREADS) ln_fwd_kernel(const __grid_constant__ PtrArray src, int64_t rows_per_src,
                                                         int64_t cols, const T* gamma,
                                                         const T* beta, T* y, float* mean_out,
                                                         float* rstd_out) {
  constexpr int V = LnVec<T>::N;
  __shared__ float red[THREADS / 32];
  const int64_t r = blockIdx.x;
  const int j = static_cast<int>(r / rows_per_src);
  const T* x = static_cast<const T*>(src.p[j]) + (r - j * rows_per_src) * cols;
  const int vpr = static_cast<int>(cols / V);
  float v[kVptMax][V];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      LnVec<T>::load(x + static_cast<int64_t>(c) * V, v[i]);
#pragma unroll
      for (int k = 0; k < V; ++k) s += v[i][k];
    }
  }
  const float mean = block_sum<THREADS>(s, red) / static_cast<float>(cols);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
#pragma unroll
      for (int k = 0; k < V; ++k) {
        const float d = v[i][k] - mean;
        q += d * d;
      }
    }
  }
  const float var = block_sum<THREADS>(q, red) / static_cast<float>(cols);
  const float rstd = rsqrtf(var + kEps);
  T* yr = y + r * cols;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      float g[V], b[V], o[V];
      LnVec<T>::load(gamma + static_cast<int64_t>(c) * V, g);
      LnVec<T>::load(beta + static_cast<int64_t>(c) * V, b);
#pragma unroll
      for (int k = 0; k < V; ++k) o[k] = (v[i][k] - mean) * rstd * g[k] + b[k];
      LnVec<T>::store(yr + static_cast<int64_t>(c) * V, o);
    }
  }
  if (threadIdx.x == 0) {
    if (mean_out) mean_out[r] = mean;
    if (rstd_out) rstd_out[r] = rstd;
  }
}

// dx row r = rstd * (gy - mean(gy) - xhat * mean(gy * xhat)), gy = dy * gamma.
template <typename T, int THREADS>
__global__ void __launch_bounds__(THREADS) ln_bwd_dx_kernel(const T* x, const T* gamma,
                                                            const T* dy, const float* mean_in,
                                                            const float* rstd_in, T* dx,
                                                            int64_t cols) {
  constexpr int V = LnVec<T>::N;
  __shared__ float red[THREADS / 32];
  const int64_t r = blockIdx.x;
  const int vpr = static_cast<int>(cols / V);
  const float mean = mean_in[r], rstd = rstd_in[r];
  float xh[kVptMax][V], gy[kVptMax][V];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      float g[V], d[V];
      LnVec<T>::load(x + r * cols + static_cast<int64_t>(c) * V, xh[i]);
      LnVec<T>::load(dy + r * cols + static_cast<int64_t>(c) * V, d);
      LnVec<T>::load(gamma + static_cast<int64_t>(c) * V, g);
#pragma unroll
      for (int k = 0; k < V; ++k) {
        xh[i][k] = (xh[i][k] - mean) * rstd;
        gy[i][k] = d[k] * g[k];
        s1 += gy[i][k];
        s2 += gy[i][k] * xh[i][k];
      }
    }
  }
  const float m1 = block_sum<THREADS>(s1, red) / static_cast<float>(cols);
  const float m2 = block_sum<THREADS>(s2, red) / static_cast<float>(cols);
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      float o[V];
#pragma unroll
      for (int k = 0; k < V; ++k) o[k] = rstd * (gy[i][k] - m1 - xh[i][k] * m2);
      LnVec<T>::store(dx + r * cols + static_cast<int64_t>(c) * V, o);
    }
  }
}

// dgamma / dbeta, pass 1: block (32 column vectors x 8 row lanes) over rows
// [split*rps, ...): part[split][0][col] = sum dy * xhat, part[split][1][col] = sum dy.
template <typename T>
__global__ void __launch_bounds__(256) ln_bwd_param_pass1(const T* x, const T* dy,
                                                          const float* mean_in,
                                                          const float* rstd_in, int64_t rows,
                                                          int64_t cols, int64_t rps,
                                                          float* part) {
  constexpr int V = LnVec<T>::N;
  __shared__ float red[2][8][32 * V + 1];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t vpr = cols / V;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rps;
  const int64_t r1 = min(rows, r0 + rps);
  float ag[V], ab[V];
#pragma unroll
  for (int k = 0; k < V; ++k) ag[k] = ab[k] = 0.f;
  if (cv < vpr) {
    for (int64_t r = r0 + ty; r < r1; r += 8) {
      float xv[V], dv[V];
      LnVec<T>::load(x + r * cols + cv * V, xv);
      LnVec<T>::load(dy + r * cols + cv * V, dv);
      const float mean = mean_in[r], rstd = rstd_in[r];
#pragma unroll
      for (int k = 0; k < V; ++k) {
        ag[k] += dv[k] * ((xv[k] - mean) * rstd);
        ab[k] += dv[k];
      }
    }
  }
#pragma unroll
  for (int k = 0; k < V; ++k) {
    red[0][ty][tx * V + k] = ag[k];
    red[1][ty][tx * V + k] = ab[k];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * V; c += 256) {
    float sg = 0.f, sb = 0.f;
#pragma unroll
    for (int yy = 0; yy < 8; ++yy) {
      sg += red[0][yy][c];
      sb += red[1][yy][c];
    }
    const int64_t col = static_cast<int64_t>(blockIdx.x) * 32 * V + c;
    if (col < cols) {
      part[(static_cast<int64_t>(blockIdx.y) * 2 + 0) * cols + col] = sg;
      part[(static_cast<int64_t>(blockIdx.y) * 2 + 1) * cols + col] = sb;
    }
  }
}

__global__ void ln_bwd_param_pass2(const float* part, int splits, int64_t cols, float* dgamma,
                                   float* dbeta, int accumulate) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float sg = 0.f, sb = 0.f;
  for (int k = 0; k < splits; ++k) {
    sg += part[(static_cast<int64_t>(k) * 2 + 0) * cols + c];
    sb += part[(static_cast<int64_t>(k) * 2 + 1) * cols + c];
  }
  dgamma[c] = accumulate ? dgamma[c] + sg : sg;
  dbeta[c] = accumulate ? dbeta[c] + sb : sb;
}

int threads_for(int64_t vpr) {
  if (vpr <= 64 * kVptMax) return 64;
  if (vpr <= 128 * kVptMax) return 128;
  return 256;
}

int num_sms() {
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

tp_status launch_layernorm_fwd(const PtrArray& x_seq, int n, int64_t rows_per_src, int64_t cols,
                               const void* gamma, const void* beta, void* y, float* mean,
                               float* rstd, tp_dtype dt, cudaStream_t st) {
  const int64_t rows = rows_per_src * n;
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = cols / V;
  if (vpr > 256 * kVptMax) return fail(TP_ERR_UNSUPPORTED, "LayerNorm row too long (%lld)", (long long)cols);
  const int th = threads_for(vpr);
#define TP_LN_FWD(T, TH)                                                                        \
  ln_fwd_kernel<T, TH><<<static_cast<unsigned>(rows), TH, 0, st>>>(                            \
      x_seq, rows_per_src, cols, static_cast<const T*>(gamma), static_cast<const T*>(beta),     \
      static_cast<T*>(y), mean, rstd)
  if (dt == TP_BF16) {
    if (th == 64) TP_LN_FWD(__nv_bfloat16, 64);
    else if (th == 128) TP_LN_FWD(__nv_bfloat16, 128);
    else TP_LN_FWD(__nv_bfloat16, 256);
  } else {
    if (th == 64) TP_LN_FWD(float, 64);
    else if (th == 128) TP_LN_FWD(float, 128);
    else TP_LN_FWD(float, 256);
  }
#undef TP_LN_FWD
  return after_launch("layernorm_fwd");
}

tp_status launch_layernorm_bwd(tp_plan* plan, const void* x, const void* gamma, const void* dy,
                               const float* mean, const float* rstd, void* dx, float* dgamma,
                               float* dbeta, int accumulate, int64_t rows, int64_t cols,
                               tp_dtype dt, cudaStream_t st) {
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = cols / V;
  if (vpr > 256 * kVptMax) return fail(TP_ERR_UNSUPPORTED, "LayerNorm row too long (%lld)", (long long)cols);
  const int gx = static_cast<int>((vpr + 31) / 32);
  int64_t splits = std::max<int64_t>(1, (static_cast<int64_t>(num_sms()) * 8) / gx);
  splits = std::min<int64_t>(splits, std::max<int64_t>(1, (rows + 63) / 64));
  splits = std::min<int64_t>(splits, 1024);
  const int64_t rps = rows > 0 ? (rows + splits - 1) / splits : 1;
  splits = rows > 0 ? (rows + rps - 1) / rps : 0;
  void* ws = nullptr;
  tp_status s = workspace(plan, static_cast<size_t>(std::max<int64_t>(splits, 1)) * 2 * cols * sizeof(float), &ws);
  if (s != TP_OK) return s;
  float* part = static_cast<float*>(ws);
  if (rows > 0) {
    const int th = threads_for(vpr);
#define TP_LN_BWD(T, TH)                                                                        \
  ln_bwd_dx_kernel<T, TH><<<static_cast<unsigned>(rows), TH, 0, st>>>(                         \
      static_cast<const T*>(x), static_cast<const T*>(gamma), static_cast<const T*>(dy), mean,  \
      rstd, static_cast<T*>(dx), cols)
    if (dt == TP_BF16) {
      if (th == 64) TP_LN_BWD(__nv_bfloat16, 64);
      else if (th == 128) TP_LN_BWD(__nv_bfloat16, 128);
      else TP_LN_BWD(__nv_bfloat16, 256);
    } else {
      if (th == 64) TP_LN_BWD(float, 64);
      else if (th == 128) TP_LN_BWD(float, 128);
      else TP_LN_BWD(float, 256);
    }
#undef TP_LN_BWD
    s = after_launch("layernorm_bwd/dx");
    if (s != TP_OK) return s;
    dim3 grid(gx, static_cast<unsigned>(splits));
    if (dt == TP_BF16)
      ln_bwd_param_pass1<__nv_bfloat16><<<grid, 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(dy), mean, rstd,
          rows, cols, rps, part);
    else
      ln_bwd_param_pass1<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x),
                                                      static_cast<const float*>(dy), mean, rstd,
                                                      rows, cols, rps, part);
    s = after_launch("layernorm_bwd/param1");
    if (s != TP_OK) return s;
  }
  ln_bwd_param_pass2<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(
      part, static_cast<int>(splits), cols, dgamma, dbeta, accumulate);
  return after_launch("layernorm_bwd/param2");
}

}  // namespace tpi

// ---------------------------------------------------------------------------
// Norms of rows whose hidden dim is split over p shards (each shard holds
// columns [i*h/p, (i+1)*h/p) in its own buffer). The row statistics are sums
// of the shards' local sums -- on one GPU that reduction over shards is part
// of the CTA's row reduction -- and each shard's slice is normalised with them.
// LayerNorm uses the one-pass variance E[x^2] - mean^2 that the local-sums
// method implies; RMSNorm needs only sum x^2.
// ---------------------------------------------------------------------------
namespace {

using tpi::MutPtrArray;

template <typename T, int THREADS, bool RMS>
__global__ void __launch_bounds__(THREADS) norm_hsh_fwd_kernel(
    const __grid_constant__ PtrArray X, const __grid_constant__ PtrArray G,
    const __grid_constant__ PtrArray B, const __grid_constant__ MutPtrArray Y, int vps,
    int64_t hs, int64_t h, float* mean_out, float* rstd_out) {
  constexpr int V = LnVec<T>::N;
  __shared__ float red[THREADS / 32];
  const int64_t r = blockIdx.x;
  const int vpr = static_cast<int>(h / V);
  float v[kVptMax][V];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      const int sh = c / vps, lc = c - sh * vps;
      LnVec<T>::load(static_cast<const T*>(X.p[sh]) + r * hs + static_cast<int64_t>(lc) * V, v[i]);
#pragma unroll
      for (int k = 0; k < V; ++k) {
        s1 += v[i][k];
        s2 += v[i][k] * v[i][k];
      }
    }
  }
  const float S2 = block_sum<THREADS>(s2, red);
  float mean = 0.f;
  if (!RMS) mean = block_sum<THREADS>(s1, red) / static_cast<float>(h);
  const float var = RMS ? S2 / static_cast<float>(h) : fmaxf(S2 / static_cast<float>(h) - mean * mean, 0.f);
  const float rstd = rsqrtf(var + kEps);
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      const int sh = c / vps, lc = c - sh * vps;
      float g[V], b[V], o[V];
      LnVec<T>::load(static_cast<const T*>(G.p[sh]) + static_cast<int64_t>(lc) * V, g);
      if (!RMS) LnVec<T>::load(static_cast<const T*>(B.p[sh]) + static_cast<int64_t>(lc) * V, b);
#pragma unroll
      for (int k = 0; k < V; ++k) o[k] = (v[i][k] - mean) * rstd * g[k] + (RMS ? 0.f : b[k]);
      LnVec<T>::store(static_cast<T*>(Y.p[sh]) + r * hs + static_cast<int64_t>(lc) * V, o);
    }
  }
  if (threadIdx.x == 0) {
    if (mean_out && !RMS) mean_out[r] = mean;
    if (rstd_out) rstd_out[r] = rstd;
  }
}

template <typename T, int THREADS, bool RMS>
__global__ void __launch_bounds__(THREADS) norm_hsh_bwd_dx_kernel(
    const __grid_constant__ PtrArray X, const __grid_constant__ PtrArray G,
    const __grid_constant__ PtrArray DY, const __grid_constant__ MutPtrArray DX, int vps,
    int64_t hs, int64_t h, const float* mean_in, const float* rstd_in) {
  constexpr int V = LnVec<T>::N;
  __shared__ float red[THREADS / 32];
  const int64_t r = blockIdx.x;
  const int vpr = static_cast<int>(h / V);
  const float mean = RMS ? 0.f : mean_in[r], rstd = rstd_in[r];
  float xh[kVptMax][V], gy[kVptMax][V];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      const int sh = c / vps, lc = c - sh * vps;
      float g[V], d[V];
      LnVec<T>::load(static_cast<const T*>(X.p[sh]) + r * hs + static_cast<int64_t>(lc) * V, xh[i]);
      LnVec<T>::load(static_cast<const T*>(DY.p[sh]) + r * hs + static_cast<int64_t>(lc) * V, d);
      LnVec<T>::load(static_cast<const T*>(G.p[sh]) + static_cast<int64_t>(lc) * V, g);
#pragma unroll
      for (int k = 0; k < V; ++k) {
        xh[i][k] = (xh[i][k] - mean) * rstd;
        gy[i][k] = d[k] * g[k];
        s1 += gy[i][k];
        s2 += gy[i][k] * xh[i][k];
      }
    }
  }
  const float m2 = block_sum<THREADS>(s2, red) / static_cast<float>(h);
  const float m1 = RMS ? 0.f : block_sum<THREADS>(s1, red) / static_cast<float>(h);
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      const int sh = c / vps, lc = c - sh * vps;
      float o[V];
#pragma unroll
      for (int k = 0; k < V; ++k) o[k] = rstd * (gy[i][k] - m1 - xh[i][k] * m2);
      LnVec<T>::store(static_cast<T*>(DX.p[sh]) + r * hs + static_cast<int64_t>(lc) * V, o);
    }
  }
}

// dgamma / dbeta of a hidden-sharded norm, pass 1: block (32 column vectors x
// 8 row lanes) of shard blockIdx.z over rows [split*rps, ...):
// part[split][0][col] = sum dy * xhat, part[split][1][col] = sum dy (col in 0..h).
template <typename T, bool RMS>
__global__ void __launch_bounds__(256) norm_hsh_param_pass1(
    const __grid_constant__ PtrArray X, const __grid_constant__ PtrArray DY, const float* mean_in,
    const float* rstd_in, int64_t rows, int64_t hs, int64_t h, int64_t rps, float* part) {
  constexpr int V = LnVec<T>::N;
  __shared__ float red[2][8][32 * V + 1];
  const int sh = blockIdx.z;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t vps = hs / V;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rps;
  const int64_t r1 = min(rows, r0 + rps);
  const T* x = static_cast<const T*>(X.p[sh]);
  const T* dy = static_cast<const T*>(DY.p[sh]);
  float ag[V], ab[V];
#pragma unroll
  for (int k = 0; k < V; ++k) ag[k] = ab[k] = 0.f;
  if (cv < vps) {
    for (int64_t r = r0 + ty; r < r1; r += 8) {
      float xv[V], dv[V];
      LnVec<T>::load(x + r * hs + cv * V, xv);
      LnVec<T>::load(dy + r * hs + cv * V, dv);
      const float mean = RMS ? 0.f : mean_in[r], rstd = rstd_in[r];
#pragma unroll
      for (int k = 0; k < V; ++k) {
        ag[k] += dv[k] * ((xv[k] - mean) * rstd);
        ab[k] += dv[k];
      }
    }
  }
#pragma unroll
  for (int k = 0; k < V; ++k) {
    red[0][ty][tx * V + k] = ag[k];
    red[1][ty][tx * V + k] = ab[k];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * V; c += 256) {
    float sg = 0.f, sb = 0.f;
#pragma unroll
    for (int yy = 0; yy < 8; ++yy) {
      sg += red[0][yy][c];
      sb += red[1][yy][c];
    }
    const int64_t lcol = static_cast<int64_t>(blockIdx.x) * 32 * V + c;
    if (lcol < hs) {
      const int64_t col = static_cast<int64_t>(sh) * hs + lcol;
      part[(static_cast<int64_t>(blockIdx.y) * 2 + 0) * h + col] = sg;
      part[(static_cast<int64_t>(blockIdx.y) * 2 + 1) * h + col] = sb;
    }
  }
}

__global__ void norm_hsh_param_pass2(const float* part, int splits, int64_t hs, int64_t h,
                                     const __grid_constant__ MutPtrArray dg,
                                     const __grid_constant__ MutPtrArray db) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= h) return;
  float sg = 0.f, sb = 0.f;
  for (int k = 0; k < splits; ++k) {
    sg += part[(static_cast<int64_t>(k) * 2 + 0) * h + c];
    sb += part[(static_cast<int64_t>(k) * 2 + 1) * h + c];
  }
  const int sh = static_cast<int>(c / hs);
  const int64_t lc = c - sh * hs;
  static_cast<float*>(dg.p[sh])[lc] = sg;
  if (db.p[sh]) static_cast<float*>(db.p[sh])[lc] = sb;
}

}  // namespace

namespace tpi {

tp_status launch_norm_sharded_fwd(bool rms, const PtrArray& X, const PtrArray& G,
                                  const PtrArray& B, const MutPtrArray& Y, int p, int64_t rows,
                                  int64_t h, float* mean, float* rstd, tp_dtype dt,
                                  cudaStream_t st) {
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = h / V, hs = h / p;
  if (vpr > 256 * kVptMax) return fail(TP_ERR_UNSUPPORTED, "norm row too long (%lld)", (long long)h);
  const int vps = static_cast<int>(hs / V);
  const int th = threads_for(vpr);
#define TP_NH_FWD(T, TH, R)                                                                        \
  norm_hsh_fwd_kernel<T, TH, R><<<static_cast<unsigned>(rows), TH, 0, st>>>(X, G, B, Y, vps, hs, h, \
                                                                          mean, rstd)
#define TP_NH_FWD_T(T, R)              \
  if (th == 64) TP_NH_FWD(T, 64, R);   \
  else if (th == 128) TP_NH_FWD(T, 128, R); \
  else TP_NH_FWD(T, 256, R)
  if (dt == TP_BF16) {
    if (rms) { TP_NH_FWD_T(__nv_bfloat16, true); } else { TP_NH_FWD_T(__nv_bfloat16, false); }
  } else {
    if (rms) { TP_NH_FWD_T(float, true); } else { TP_NH_FWD_T(float, false); }
  }
#undef TP_NH_FWD_T
#undef TP_NH_FWD
  return after_launch("norm_sharded_fwd");
}

tp_status launch_norm_sharded_bwd(tp_plan* plan, bool rms, const PtrArray& X, const PtrArray& G,
                                  const PtrArray& DY, const MutPtrArray& DX, const MutPtrArray& dg,
                                  const MutPtrArray& db, int p, int64_t rows, int64_t h,
                                  const float* mean, const float* rstd, tp_dtype dt,
                                  cudaStream_t st) {
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = h / V, hs = h / p;
  if (vpr > 256 * kVptMax) return fail(TP_ERR_UNSUPPORTED, "norm row too long (%lld)", (long long)h);
  const int vps = static_cast<int>(hs / V);
  const int gx = static_cast<int>((hs / V + 31) / 32);
  int64_t splits = std::max<int64_t>(1, (static_cast<int64_t>(num_sms()) * 8) / (gx * p));
  splits = std::min<int64_t>(splits, std::max<int64_t>(1, (rows + 63) / 64));
  splits = std::min<int64_t>(splits, 1024);
  const int64_t rps = rows > 0 ? (rows + splits - 1) / splits : 1;
  splits = rows > 0 ? (rows + rps - 1) / rps : 0;
  void* ws = nullptr;
  tp_status s = workspace(plan, static_cast<size_t>(std::max<int64_t>(splits, 1)) * 2 * h * sizeof(float), &ws);
  if (s != TP_OK) return s;
  float* part = static_cast<float*>(ws);
  if (rows > 0) {
    const int th = threads_for(vpr);
#define TP_NH_BWD(T, TH, R)                                                                 \
  norm_hsh_bwd_dx_kernel<T, TH, R><<<static_cast<unsigned>(rows), TH, 0, st>>>(X, G, DY, DX, \
                                                                              vps, hs, h, mean, rstd)
#define TP_NH_BWD_T(T, R)              \
  if (th == 64) TP_NH_BWD(T, 64, R);   \
  else if (th == 128) TP_NH_BWD(T, 128, R); \
  else TP_NH_BWD(T, 256, R)
    if (dt == TP_BF16) {
      if (rms) { TP_NH_BWD_T(__nv_bfloat16, true); } else { TP_NH_BWD_T(__nv_bfloat16, false); }
    } else {
      if (rms) { TP_NH_BWD_T(float, true); } else { TP_NH_BWD_T(float, false); }
    }
#undef TP_NH_BWD_T
#undef TP_NH_BWD
    s = after_launch("norm_sharded_bwd/dx");
    if (s != TP_OK) return s;
    dim3 grid(gx, static_cast<unsigned>(splits), p);
    if (dt == TP_BF16) {
      if (rms) norm_hsh_param_pass1<__nv_bfloat16, true><<<grid, 256, 0, st>>>(X, DY, mean, rstd, rows, hs, h, rps, part);
      else norm_hsh_param_pass1<__nv_bfloat16, false><<<grid, 256, 0, st>>>(X, DY, mean, rstd, rows, hs, h, rps, part);
    } else {
      if (rms) norm_hsh_param_pass1<float, true><<<grid, 256, 0, st>>>(X, DY, mean, rstd, rows, hs, h, rps, part);
      else norm_hsh_param_pass1<float, false><<<grid, 256, 0, st>>>(X, DY, mean, rstd, rows, hs, h, rps, part);
    }
    s = after_launch("norm_sharded_bwd/param1");
    if (s != TP_OK) return s;
  }
  norm_hsh_param_pass2<<<static_cast<unsigned>((h + 255) / 256), 256, 0, st>>>(
      part, static_cast<int>(splits), hs, h, dg, db);
  return after_launch("norm_sharded_bwd/param2");
}

}  // namespace tpi
