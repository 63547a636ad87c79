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

using tpi::MutPtrArray;
using tpi::PtrArray;

constexpr float kEps = 1e-5f;
constexpr int kVptMax = 8;  // 16-byte vectors per thread

template <typename T>
struct LnVec;
template <>
struct LnVec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const void* p, float* f) { unpack(*reinterpret_cast<const uint4*>(p), f); }
  __device__ static void unpack(const uint4 u, float* f) {
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
  __device__ static void load(const void* p, float* f) { unpack(*reinterpret_cast<const uint4*>(p), f); }
  __device__ static void unpack(const uint4 u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
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

// y row r = LN(x row r); x row r is row (r - j*rows_per_src) of src.p[j], so a
// sequence all-gather is part of the load. One CTA per row, many resident per
// SM: each row's chain (load, two sums, store) overlaps the other rows' loads.
// The slice stays packed in registers; the mean and the biased variance about
// it are two exact passes over those registers, each summed over the CTA with
// one barrier (each sum has a buffer of its own, and a CTA takes one row).
// Row r of y goes to ydst.p[0] (MULTI = false) or to each of the n_dst outputs
// (MULTI: an all-gather pushed into other GPUs' buffers over peer memory).
template <typename T, int THREADS, bool MULTI>
__global__ void __launch_bounds__(THREADS) ln_fwd_kernel(const __grid_constant__ PtrArray src, int64_t rows_per_src,
                                                         int64_t cols, const T* gamma,
                                                         const T* beta, const __grid_constant__ MutPtrArray ydst,
                                                         int n_dst, float* mean_out, float* rstd_out) {
  tpd::pdl_entry();
  constexpr int V = LnVec<T>::N;
  constexpr int W = THREADS / 32;
  __shared__ float red1[W], red2[W];
  const int64_t r = blockIdx.x;
  const int64_t j = r / rows_per_src;
  const uint4* x = reinterpret_cast<const uint4*>(static_cast<const T*>(src.p[j]) + (r - j * rows_per_src) * cols);
  const int vpr = static_cast<int>(cols / V);
  const float inv_h = 1.f / static_cast<float>(cols);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4 xr[kVptMax];
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    xr[i] = c < vpr ? __ldcs(x + c) : make_uint4(0, 0, 0, 0);  // read once: streaming
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    if (threadIdx.x + i * THREADS < vpr) {
      float v[V];
      LnVec<T>::unpack(xr[i], v);
#pragma unroll
      for (int e = 0; e < V; ++e) s += v[e];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red1[warp] = s;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < W; ++w) t += red1[w];
  const float mean = t * inv_h;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    if (threadIdx.x + i * THREADS < vpr) {
      float v[V];
      LnVec<T>::unpack(xr[i], v);
#pragma unroll
      for (int e = 0; e < V; ++e) q += (v[e] - mean) * (v[e] - mean);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  if (lane == 0) red2[warp] = q;
  __syncthreads();
  float u = 0.f;
#pragma unroll
  for (int w = 0; w < W; ++w) u += red2[w];
  const float rstd = rsqrtf(u * inv_h + kEps);
  uint4* y1 = reinterpret_cast<uint4*>(static_cast<T*>(ydst.p[0]) + r * cols);
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
      float v[V], g[V], b[V], o[V];
      LnVec<T>::unpack(xr[i], v);
      LnVec<T>::load(gamma + static_cast<int64_t>(c) * V, g);
      LnVec<T>::load(beta + static_cast<int64_t>(c) * V, b);
#pragma unroll
      for (int e = 0; e < V; ++e) o[e] = (v[e] - mean) * rstd * g[e] + b[e];
      if (MULTI) {
        for (int d = 0; d < n_dst; ++d)
          LnVec<T>::store(reinterpret_cast<uint4*>(static_cast<T*>(ydst.p[d]) + r * cols) + c, o);
      } else {
        LnVec<T>::store(y1 + c, o);
      }
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
                                                            const float* rstd_in, const T* dres,
                                                            T* dx, int64_t cols) {
  tpd::pdl_entry();
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
      if (dres) {
        float rr[V];
        LnVec<T>::load(dres + r * cols + static_cast<int64_t>(c) * V, rr);
#pragma unroll
        for (int k = 0; k < V; ++k) o[k] += rr[k];
      }
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
  tpd::pdl_entry();
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

// Sums of the per-CTA partials part[k][0|1][c] over k in [k0, k1) for
// kPass2Cols columns c0 + lane: warp w takes k = k0 + w, k0 + w + 8, ... in
// increasing order, then the eight warps' sums are added in warp order (fixed
// order: deterministic). Lane 0..31 of warp 0 returns true with the column's
// two sums.
constexpr int kPass2Cols = 32;
template <bool CG = false>  // CG: load through L2 only (partials other blocks of this launch wrote)
__device__ __forceinline__ bool param_colsum_range(const float* part, int k0, int k1, int64_t cols,
                                                   int64_t c, float* sg_out, float* sb_out) {
  __shared__ float rg[8][32], rb[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float sg = 0.f, sb = 0.f;
  if (c < cols) {
#pragma unroll 4
    for (int k = k0 + warp; k < k1; k += 8) {
      const float* pg = part + (static_cast<int64_t>(k) * 2 + 0) * cols + c;
      sg += CG ? __ldcg(pg) : *pg;
      sb += CG ? __ldcg(pg + cols) : pg[cols];
    }
  }
  rg[warp][lane] = sg;
  rb[warp][lane] = sb;
  __syncthreads();
  if (warp != 0 || c >= cols) return false;
  sg = rg[0][lane];
  sb = rb[0][lane];
#pragma unroll
  for (int w = 1; w < 8; ++w) {
    sg += rg[w][lane];
    sb += rb[w][lane];
  }
  *sg_out = sg;
  *sb_out = sb;
  return true;
}
__device__ __forceinline__ bool param_colsum(const float* part, int splits, int64_t cols, int64_t c,
                                             float* sg_out, float* sb_out) {
  return param_colsum_range(part, 0, splits, cols, c, sg_out, sb_out);
}

// Many partials (one per CTA of a wide persistent grid): first sum them in
// groups of kParamGroup consecutive k, each group by its own CTAs in the fixed
// order above, into inter[g][0|1][c]; pass 2 then sums the groups in order.
constexpr int kParamGroup = 64;
__global__ void __launch_bounds__(256) param_group_sum(const float* part, int splits, int64_t cols,
                                                       float* inter) {
  tpd::pdl_entry();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kPass2Cols + (threadIdx.x & 31);
  const int g = static_cast<int>(blockIdx.y);
  const int k1 = min(splits, (g + 1) * kParamGroup);
  float sg, sb;
  if (!param_colsum_range(part, g * kParamGroup, k1, cols, c, &sg, &sb)) return;
  inter[(static_cast<int64_t>(g) * 2 + 0) * cols + c] = sg;
  inter[(static_cast<int64_t>(g) * 2 + 1) * cols + c] = sb;
}

// 256 threads per CTA, kPass2Cols columns per CTA.
__global__ void __launch_bounds__(256) ln_bwd_param_pass2(const float* part, int splits, int64_t cols,
                                                          float* dgamma, float* dbeta, int accumulate) {
  tpd::pdl_entry();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kPass2Cols + (threadIdx.x & 31);
  float sg, sb;
  if (!param_colsum(part, splits, cols, c, &sg, &sb)) return;
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
                               float* rstd, tp_dtype dt, cudaStream_t st, const MutPtrArray* ydst,
                               int n_dst) {
  const int64_t rows = rows_per_src * n;
  if (rows == 0) return TP_OK;
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = cols / V;
  if (vpr > 256 * kVptMax) return fail(TP_ERR_UNSUPPORTED, "LayerNorm row too long (%lld)", (long long)cols);
  const int th = threads_for(vpr);
  MutPtrArray dst{};
  if (ydst && n_dst > 0) {
    dst = *ydst;
  } else {
    dst.p[0] = y;
    n_dst = 1;
  }
#define TP_LN_FWD(T, TH)                                                                        \
  (void)(n_dst > 1 ? tpi::launch(ln_fwd_kernel<T, TH, true>, dim3(static_cast<unsigned>(rows)), dim3(TH), 0, st, \
                                 x_seq, rows_per_src, cols, static_cast<const T*>(gamma),       \
                                 static_cast<const T*>(beta), dst, n_dst, mean, rstd)           \
                   : tpi::launch(ln_fwd_kernel<T, TH, false>, dim3(static_cast<unsigned>(rows)), dim3(TH), 0, st, \
                                 x_seq, rows_per_src, cols, static_cast<const T*>(gamma),       \
                                 static_cast<const T*>(beta), dst, n_dst, mean, rstd))
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
                               const float* mean, const float* rstd, const void* dres, void* dx,
                               float* dgamma, float* dbeta, int accumulate, int64_t rows,
                               int64_t cols, tp_dtype dt, cudaStream_t st) {
  // The backward formula takes the saved mean and rstd, so a LayerNorm over the
  // whole row is the hidden-sharded one with a single shard: its one-pass,
  // staged kernel serves whenever the row fits it.
  if (cols % 8 == 0 && cols <= (dt == TP_BF16 ? 16384 : 8192)) {
    PtrArray X{}, G{}, DY{};
    MutPtrArray DX{}, dg{}, db{};
    X.p[0] = x;
    G.p[0] = gamma;
    DY.p[0] = dy;
    DX.p[0] = dx;
    dg.p[0] = dgamma;
    db.p[0] = dbeta;
    PtrArray R{};
    R.p[0] = dres;
    return launch_norm_sharded_bwd(plan, false, X, G, DY, DX, dg, db, 1, rows, cols, mean, rstd, dt, st,
                                   accumulate, R);
  }
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
  (void)tpi::launch(ln_bwd_dx_kernel<T, TH>, dim3(static_cast<unsigned>(rows)), dim3(TH), 0, st,                          \
      static_cast<const T*>(x), static_cast<const T*>(gamma), static_cast<const T*>(dy), mean,  \
      rstd, static_cast<const T*>(dres), static_cast<T*>(dx), cols)
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
      (void)tpi::launch(ln_bwd_param_pass1<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, 
          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(dy), mean, rstd,
          rows, cols, rps, part);
    else
      (void)tpi::launch(ln_bwd_param_pass1<float>, dim3(grid), dim3(256), 0, st, static_cast<const float*>(x),
                                                      static_cast<const float*>(dy), mean, rstd,
                                                      rows, cols, rps, part);
    s = after_launch("layernorm_bwd/param1");
    if (s != TP_OK) return s;
  }
  (void)tpi::launch(ln_bwd_param_pass2, dim3(static_cast<unsigned>((cols + kPass2Cols - 1) / kPass2Cols)), dim3(256), 0, st, 
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

// Rows staged in shared memory (the backward): CTA b takes rows b, b + G, ... and
// keeps STAGES of them in flight; a row's p shard slices arrive by bulk copy
// (one per shard, completing on the stage's mbarrier) while the CTA works on
// the rows before it. Thread tid owns the row's 16-byte vectors
// tid + i * THREADS (vector c lies in shard c / vps), the same for every row.
// thread 0: start the copies of row r of `a` (and, if given, of `b`: placed
// after a's row) into `dst`, one bulk copy per shard slice, completing on `bar`.
__device__ __forceinline__ void issue_row(const PtrArray& a, const PtrArray* b, int p, int64_t r,
                                          uint32_t shard_bytes, uint8_t* dst, uint64_t* bar) {
  const int nbuf = b ? 2 : 1;
  tpd::mbar_arrive_expect_tx(bar, shard_bytes * static_cast<uint32_t>(p * nbuf));
  for (int s = 0; s < p; ++s)
    tpd::bulk_load(dst + static_cast<size_t>(s) * shard_bytes,
                   static_cast<const uint8_t*>(a.p[s]) + r * shard_bytes, shard_bytes, bar);
  if (b)
    for (int s = 0; s < p; ++s)
      tpd::bulk_load(dst + static_cast<size_t>(p + s) * shard_bytes,
                     static_cast<const uint8_t*>(b->p[s]) + r * shard_bytes, shard_bytes, bar);
}

// thread 0: store row r of the p shard buffers of `y` from `src` (its shard
// slices back to back), one bulk copy per shard, as one bulk group.
__device__ __forceinline__ void store_row(const MutPtrArray& y, int p, int64_t r, uint32_t shard_bytes,
                                          const uint8_t* src) {
  for (int s = 0; s < p; ++s)
    tpd::bulk_store(static_cast<uint8_t*>(y.p[s]) + r * shard_bytes, src + static_cast<size_t>(s) * shard_bytes,
                    shard_bytes);
  tpd::bulk_commit();
}

// Sum of a float pair over the CTA with one barrier, which also carries every
// thread's wait result (false for all if any thread's ok is false). The
// caller's previous barrier (end of the previous row) keeps red from being
// overwritten while still read.
template <int THREADS>
__device__ __forceinline__ bool block_sum2_ok(float2& v, bool ok, float2* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
  }
  constexpr int W = THREADS / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  if (!__syncthreads_and(ok)) return false;
  float2 s = make_float2(0.f, 0.f);
#pragma unroll
  for (int w = 0; w < W; ++w) {
    s.x += red[w].x;
    s.y += red[w].y;
  }
  v = s;
  return true;
}

// Forward of a hidden-sharded norm, one CTA per row: vector c of the row is
// vector c - j*vps of shard j = c / vps. The slice stays packed in registers;
// one barrier sums (sum x, sum x^2) over the CTA, the local sums of every shard
// reduced in one step.
template <typename T, int THREADS, bool RMS>
__global__ void __launch_bounds__(THREADS) norm_hsh_row_fwd_kernel(
    const __grid_constant__ PtrArray X, const __grid_constant__ PtrArray G,
    const __grid_constant__ PtrArray B, const __grid_constant__ MutPtrArray Y, int vps, int64_t h,
    float* mean_out, float* rstd_out) {
  tpd::pdl_entry();
  constexpr int V = LnVec<T>::N;
  constexpr int W = THREADS / 32;
  __shared__ float2 red[W];
  const int64_t r = blockIdx.x;
  const int vpr = static_cast<int>(h / V);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // shard and offset of vector c = tid + i*THREADS, stepped from i to i + 1
  // (one division per thread instead of one per vector)
  const int step_sh = THREADS / vps, step_lc = THREADS - step_sh * vps;
  int sh[kVptMax], lc[kVptMax];
  sh[0] = static_cast<int>(threadIdx.x) / vps;
  lc[0] = static_cast<int>(threadIdx.x) - sh[0] * vps;
#pragma unroll
  for (int i = 1; i < kVptMax; ++i) {
    sh[i] = sh[i - 1] + step_sh;
    lc[i] = lc[i - 1] + step_lc;
    if (lc[i] >= vps) {
      lc[i] -= vps;
      ++sh[i];
    }
  }
  uint4 xr[kVptMax];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    xr[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x + i * THREADS < vpr)
      xr[i] = __ldcs(reinterpret_cast<const uint4*>(X.p[sh[i]]) + r * vps + lc[i]);
  }
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    if (threadIdx.x + i * THREADS < vpr) {
      float x[V];
      LnVec<T>::unpack(xr[i], x);
#pragma unroll
      for (int e = 0; e < V; ++e) {
        s1 += x[e];
        s2 += x[e] * x[e];
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  }
  if (lane == 0) red[warp] = make_float2(s1, s2);
  __syncthreads();
  float2 tot = make_float2(0.f, 0.f);
#pragma unroll
  for (int w = 0; w < W; ++w) {
    tot.x += red[w].x;
    tot.y += red[w].y;
  }
  const float mean = RMS ? 0.f : tot.x / static_cast<float>(h);
  const float var = RMS ? tot.y / static_cast<float>(h) : fmaxf(tot.y / static_cast<float>(h) - mean * mean, 0.f);
  const float rstd = rsqrtf(var + kEps);
#pragma unroll
  for (int i = 0; i < kVptMax; ++i) {
    if (threadIdx.x + i * THREADS < vpr) {
      float x[V], g[V], bb[V], o[V];
      LnVec<T>::unpack(xr[i], x);
      LnVec<T>::load(static_cast<const T*>(G.p[sh[i]]) + static_cast<int64_t>(lc[i]) * V, g);
      if (!RMS) LnVec<T>::load(static_cast<const T*>(B.p[sh[i]]) + static_cast<int64_t>(lc[i]) * V, bb);
#pragma unroll
      for (int e = 0; e < V; ++e) o[e] = (x[e] - mean) * rstd * g[e] + (RMS ? 0.f : bb[e]);
      LnVec<T>::store(reinterpret_cast<uint4*>(Y.p[sh[i]]) + r * vps + lc[i], o);
    }
  }
  if (threadIdx.x == 0) {
    if (mean_out && !RMS) mean_out[r] = mean;
    if (rstd_out) rstd_out[r] = rstd;
  }
}



// Backward of a hidden-sharded norm in one pass over x and dy, with the rows
// staged as above (a stage holds a row of x and the same row of dy). Thread tid
// owns the same column vectors of every row, so besides dx it keeps running
// column partials dgamma = sum dy * xhat and dbeta = sum dy in registers and
// writes them once: part[b][0][col], part[b][1][col]. A second kernel sums the
// partials over b in order, so the parameter gradients are deterministic.
// RES: DRES holds a gradient to add to dx (the residual branch); a separate
// instance, so the plain one keeps its register count (and its residency).
template <typename T, int THREADS, int VPT, int STAGES, bool RMS, bool RES>
__global__ void __launch_bounds__(THREADS) norm_hsh_bwd_fused_kernel(
    const __grid_constant__ PtrArray X, const __grid_constant__ PtrArray G,
    const __grid_constant__ PtrArray DY, const __grid_constant__ MutPtrArray DX,
    const __grid_constant__ PtrArray DRES, int p, int vps, int64_t hs, int64_t h, int64_t rows,
    const float* mean_in, const float* rstd_in, float* part, unsigned* status) {
  tpd::pdl_entry();
  constexpr int V = LnVec<T>::N;
  extern __shared__ __align__(128) uint8_t sbuf[];
  __shared__ uint64_t bar[STAGES];
  __shared__ int abort_flag;
  __shared__ float2 red[THREADS / 32];
  const uint32_t shard_bytes = static_cast<uint32_t>(hs * sizeof(T));
  const size_t row_bytes = static_cast<size_t>(h) * sizeof(T);
  const size_t stage_bytes = 2 * row_bytes;
  const int vpr = static_cast<int>(h / V);
  const float inv_h = 1.f / static_cast<float>(h);
  const int64_t G0 = blockIdx.x, GS = gridDim.x;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int st = 0; st < STAGES; ++st) tpd::mbar_init(&bar[st], 1);
    tpd::fence_barrier_init();
  }
  __syncthreads();
  int64_t issued = 0;  // thread 0: rows [0, issued) of this CTA have their loads issued
  if (threadIdx.x == 0)
    for (; issued < STAGES && G0 + issued * GS < rows; ++issued)
      issue_row(X, &DY, p, G0 + issued * GS, shard_bytes, sbuf + issued * stage_bytes, &bar[issued]);
  uint4 gp[VPT];
  float pg[VPT][V], pb[VPT][V];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = threadIdx.x + i * THREADS;
    gp[i] = make_uint4(0, 0, 0, 0);
    if (c < vpr) {
      const int sh = c / vps, lc = c - sh * vps;
      gp[i] = *reinterpret_cast<const uint4*>(static_cast<const T*>(G.p[sh]) + static_cast<int64_t>(lc) * V);
    }
#pragma unroll
    for (int e = 0; e < V; ++e) pg[i][e] = pb[i][e] = 0.f;
  }
  int64_t k = 0;
  for (;; ++k) {
    const int64_t r = G0 + k * GS;
    if (r >= rows) break;
    const int st = static_cast<int>(k % STAGES);
    const float mean = RMS ? 0.f : mean_in[r], rstd = rstd_in[r];
    // a gradient to add to dx (the residual branch), read now so the loads
    // are in flight during the row's sums
    uint4 rv[VPT];
    if (RES) {
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int c = threadIdx.x + i * THREADS;
        rv[i] = make_uint4(0, 0, 0, 0);
        if (c < vpr) {
          const int sh = c / vps, lc = c - sh * vps;
          rv[i] = __ldcs(reinterpret_cast<const uint4*>(static_cast<const T*>(DRES.p[sh]) + r * hs) + lc);
        }
      }
    }
    // a thread whose wait gave up computes on an unfinished stage; the sum's
    // barrier then stops every thread before anything is written
    const bool ok = tpd::mbar_wait(&bar[st], static_cast<uint32_t>(k / STAGES) & 1u, &abort_flag, status);
    const uint4* xrow = reinterpret_cast<const uint4*>(sbuf + st * stage_bytes);
    const uint4* drow = reinterpret_cast<const uint4*>(sbuf + st * stage_bytes + row_bytes);
    float2 acc = make_float2(0.f, 0.f);  // (sum g dy, sum g dy xhat) of this thread's columns
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = threadIdx.x + i * THREADS;
      if (c < vpr) {
        float x[V], d[V], g[V];
        LnVec<T>::unpack(xrow[c], x);
        LnVec<T>::unpack(drow[c], d);
        LnVec<T>::unpack(gp[i], g);
#pragma unroll
        for (int e = 0; e < V; ++e) {
          const float xh = (x[e] - mean) * rstd;
          const float gy = d[e] * g[e];
          acc.x += gy;
          acc.y += gy * xh;
          pg[i][e] += d[e] * xh;
          pb[i][e] += d[e];
        }
      }
    }
    float2 tot = acc;
    if (!block_sum2_ok<THREADS>(tot, ok, red)) break;
    const float m1 = RMS ? 0.f : tot.x * inv_h, m2 = tot.y * inv_h;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = threadIdx.x + i * THREADS;
      if (c < vpr) {
        float x[V], d[V], g[V], o[V];
        LnVec<T>::unpack(xrow[c], x);
        LnVec<T>::unpack(drow[c], d);
        LnVec<T>::unpack(gp[i], g);
#pragma unroll
        for (int e = 0; e < V; ++e) o[e] = rstd * (d[e] * g[e] - m1 - (x[e] - mean) * rstd * m2);
        if (RES) {
          float rr[V];
          LnVec<T>::unpack(rv[i], rr);
#pragma unroll
          for (int e = 0; e < V; ++e) o[e] += rr[e];
        }
        LnVec<T>::store(const_cast<uint4*>(xrow) + c, o);  // dx replaces x in the stage
      }
    }
    tpd::fence_proxy_async_smem();
    __syncthreads();  // the stage holds the row's dx
    if (threadIdx.x == 0) {
      store_row(DX, p, r, shard_bytes, sbuf + st * stage_bytes);
      tpd::bulk_wait_read<1>();
      if (k >= 1 && G0 + (k - 1 + STAGES) * GS < rows) {
        const int s2 = static_cast<int>((k - 1) % STAGES);
        issue_row(X, &DY, p, G0 + (k - 1 + STAGES) * GS, shard_bytes, sbuf + s2 * stage_bytes, &bar[s2]);
        issued = k - 1 + STAGES + 1;
      }
    }
  }
  if (threadIdx.x == 0) {
    tpd::bulk_wait_all();  // every store has landed
    if (abort_flag)        // let loads still in flight land (bounded)
      for (int64_t kk = k; kk < issued; ++kk) {
        int again = 0;
        tpd::mbar_wait(&bar[kk % STAGES], static_cast<uint32_t>(kk / STAGES) & 1u, &again, nullptr);
      }
  }
  float* pgo = part + (static_cast<int64_t>(blockIdx.x) * 2 + 0) * h;
  float* pbo = part + (static_cast<int64_t>(blockIdx.x) * 2 + 1) * h;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = threadIdx.x + i * THREADS;
    if (c < vpr) {
#pragma unroll
      for (int e = 0; e < V; e += 4) {
        *reinterpret_cast<float4*>(pgo + static_cast<int64_t>(c) * V + e) =
            make_float4(pg[i][e], pg[i][e + 1], pg[i][e + 2], pg[i][e + 3]);
        *reinterpret_cast<float4*>(pbo + static_cast<int64_t>(c) * V + e) =
            make_float4(pb[i][e], pb[i][e + 1], pb[i][e + 2], pb[i][e + 3]);
      }
    }
  }
}

// Groups and final sum in one launch: block (x, g) sums group g of the
// partials for kPass2Cols columns into inter[g] (as param_group_sum); the last
// group block of each column block, counted on counters[x], then adds the
// groups in order (deterministic) and writes dgamma / dbeta of those columns
// (as norm_hsh_param_pass2), and sets its counter back to zero.
__global__ void __launch_bounds__(256) norm_hsh_param_groups_final(
    const float* part, int splits, int64_t hs, int64_t h, float* inter, const __grid_constant__ MutPtrArray dg,
    const __grid_constant__ MutPtrArray db, int accumulate, unsigned* counters) {
  tpd::pdl_entry();
  __shared__ int last;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kPass2Cols + (threadIdx.x & 31);
  const int g = static_cast<int>(blockIdx.y), groups = static_cast<int>(gridDim.y);
  const int k1 = min(splits, (g + 1) * kParamGroup);
  float sg, sb;
  if (param_colsum_range(part, g * kParamGroup, k1, h, c, &sg, &sb)) {
    inter[(static_cast<int64_t>(g) * 2 + 0) * h + c] = sg;
    inter[(static_cast<int64_t>(g) * 2 + 1) * h + c] = sb;
  }
  __threadfence();  // this block's group sums are visible before it is counted
  __syncthreads();
  if (threadIdx.x == 0) {
    last = atomicAdd(counters + blockIdx.x, 1u) == static_cast<unsigned>(groups - 1);
    if (last) atomicExch(counters + blockIdx.x, 0u);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (!param_colsum_range<true>(inter, 0, groups, h, c, &sg, &sb)) return;
  const int sh = static_cast<int>(c / hs);
  const int64_t lc = c - sh * hs;
  float* gp = static_cast<float*>(dg.p[sh]) + lc;
  *gp = accumulate ? *gp + sg : sg;
  if (db.p[sh]) {
    float* bp = static_cast<float*>(db.p[sh]) + lc;
    *bp = accumulate ? *bp + sb : sb;
  }
}

// dgamma[c] (and dbeta[c]) = the fixed-order sum over the CTAs' partials
// (added to the existing value when accumulate is set).
__global__ void __launch_bounds__(256) norm_hsh_param_pass2(const float* part, int splits, int64_t hs, int64_t h,
                                                            const __grid_constant__ MutPtrArray dg,
                                                            const __grid_constant__ MutPtrArray db, int accumulate) {
  tpd::pdl_entry();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kPass2Cols + (threadIdx.x & 31);
  float sg, sb;
  if (!param_colsum(part, splits, h, c, &sg, &sb)) return;
  const int sh = static_cast<int>(c / hs);
  const int64_t lc = c - sh * hs;
  float* g = static_cast<float*>(dg.p[sh]) + lc;
  *g = accumulate ? *g + sg : sg;
  if (db.p[sh]) {
    float* bp = static_cast<float*>(db.p[sh]) + lc;
    *bp = accumulate ? *bp + sb : sb;
  }
}

}  // namespace

namespace tpi {

// Threads for the sharded norms: up to 256, so a thread holds at most 4
// vectors up to 1024 vectors a row (8 beyond).
int hsh_threads(int64_t vpr) { return vpr <= 64 ? 64 : vpr <= 128 ? 128 : 256; }

// Vectors per thread for a row of vpr vectors over th threads: 1, 2, 4 or 8.
int vpt_for(int64_t vpr, int th) {
  const int64_t need = (vpr + th - 1) / th;
  return need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : 8;
}

constexpr int kNormBwdStages = 3;

#define TP_NH_DISPATCH(LAUNCH, T, R)                 \
  if (th == 64) LAUNCH(T, 64, 1, R);                 \
  else if (th == 128) LAUNCH(T, 128, 1, R);          \
  else if (vpt == 1) LAUNCH(T, 256, 1, R);           \
  else if (vpt == 2) LAUNCH(T, 256, 2, R);           \
  else if (vpt == 4) LAUNCH(T, 256, 4, R);           \
  else LAUNCH(T, 256, 8, R)
// The backward's instances also differ by whether a residual gradient is added.
#define TP_NH_BWD_DISPATCH(LAUNCH, T, R)                                 \
  if (res) { TP_NH_DISPATCH(LAUNCH##_RES, T, R); }                       \
  else { TP_NH_DISPATCH(LAUNCH##_PLAIN, T, R); }

// Persistent grid for a staged row kernel: as many CTAs as are resident at
// once (at most one per row), with its dynamic shared memory opted in.
template <typename K>
tp_status pipe_grid(K kernel, int threads, int smem, int64_t rows, int64_t* grid) {
  return persistent_grid(reinterpret_cast<const void*>(kernel), threads, smem, rows, grid);
}

tp_status launch_norm_sharded_fwd(bool rms, const PtrArray& X, const PtrArray& G,
                                  const PtrArray& B, const MutPtrArray& Y, int p, int64_t rows,
                                  int64_t h, float* mean, float* rstd, tp_dtype dt,
                                  cudaStream_t st) {
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = h / V, hs = h / p;
  if (vpr > 256 * kVptMax) return fail(TP_ERR_UNSUPPORTED, "norm row too long (%lld)", (long long)h);
  if (rows == 0) return TP_OK;
  const int vps = static_cast<int>(hs / V);
  const int th = threads_for(vpr);
#define TP_NH_FWD(T, TH, R)                                                                      \
  (void)tpi::launch(norm_hsh_row_fwd_kernel<T, TH, R>, dim3(static_cast<unsigned>(rows)), dim3(TH), 0, st, X, G, B, Y, vps, h, \
                                                                               mean, rstd)
#define TP_NH_FWD_TH(T, R)          \
  do {                              \
    if (th == 64) TP_NH_FWD(T, 64, R);       \
    else if (th == 128) TP_NH_FWD(T, 128, R); \
    else TP_NH_FWD(T, 256, R);               \
  } while (0)
  if (dt == TP_BF16) {
    if (rms) TP_NH_FWD_TH(__nv_bfloat16, true);
    else TP_NH_FWD_TH(__nv_bfloat16, false);
  } else {
    if (rms) TP_NH_FWD_TH(float, true);
    else TP_NH_FWD_TH(float, false);
  }
#undef TP_NH_FWD_TH
#undef TP_NH_FWD
  return after_launch("norm_sharded_fwd");
}

tp_status launch_norm_sharded_bwd(tp_plan* plan, bool rms, const PtrArray& X, const PtrArray& G,
                                  const PtrArray& DY, const MutPtrArray& DX, const MutPtrArray& dg,
                                  const MutPtrArray& db, int p, int64_t rows, int64_t h,
                                  const float* mean, const float* rstd, tp_dtype dt,
                                  cudaStream_t st, int accumulate, const PtrArray& DRES) {
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = h / V, hs = h / p;
  if (vpr > 256 * kVptMax) return fail(TP_ERR_UNSUPPORTED, "norm row too long (%lld)", (long long)h);
  const int vps = static_cast<int>(hs / V);
  const int th = hsh_threads(vpr);
  const int vpt = vpt_for(vpr, th);
  const int smem = static_cast<int>(kNormBwdStages * 2 * h * static_cast<int64_t>(dsize(dt)));
  unsigned* status = nullptr;
  tp_status s = device_status_word(&status);
  if (s != TP_OK) return s;
  // The grid (and so the partials' size) depends only on the kernel, not on
  // the data: size it first, then the workspace.
  int64_t grid = 1;
  const bool res = DRES.p[0] != nullptr;
#define TP_NH_GRID_(T, TH, VP, R, RES)                                                          \
  s = pipe_grid(norm_hsh_bwd_fused_kernel<T, TH, VP, kNormBwdStages, R, RES>, TH, smem,          \
                std::max<int64_t>(rows, 1), &grid)
#define TP_NH_GRID_RES(T, TH, VP, R) TP_NH_GRID_(T, TH, VP, R, true)
#define TP_NH_GRID_PLAIN(T, TH, VP, R) TP_NH_GRID_(T, TH, VP, R, false)
  if (dt == TP_BF16) {
    if (rms) { TP_NH_BWD_DISPATCH(TP_NH_GRID, __nv_bfloat16, true); }
    else { TP_NH_BWD_DISPATCH(TP_NH_GRID, __nv_bfloat16, false); }
  } else {
    if (rms) { TP_NH_BWD_DISPATCH(TP_NH_GRID, float, true); }
    else { TP_NH_BWD_DISPATCH(TP_NH_GRID, float, false); }
  }
#undef TP_NH_GRID_PLAIN
#undef TP_NH_GRID_RES
#undef TP_NH_GRID_
  if (s != TP_OK) return s;
  const int groups = grid > 2 * kParamGroup ? static_cast<int>((grid + kParamGroup - 1) / kParamGroup) : 0;
  void* ws = nullptr;
  s = workspace(plan, static_cast<size_t>(grid + groups) * 2 * h * sizeof(float), &ws);
  if (s != TP_OK) return s;
  float* part = static_cast<float*>(ws);
  float* inter = part + grid * 2 * h;
  if (rows > 0) {
#define TP_NH_BWD_(T, TH, VP, R, RES)                                                                 \
  (void)tpi::launch(norm_hsh_bwd_fused_kernel<T, TH, VP, kNormBwdStages, R, RES>,                    \
                    dim3(static_cast<unsigned>(grid)), dim3(TH), smem, st, X, G, DY, DX, DRES, p, vps, \
                    hs, h, rows, mean, rstd, part, status)
#define TP_NH_BWD_RES(T, TH, VP, R) TP_NH_BWD_(T, TH, VP, R, true)
#define TP_NH_BWD_PLAIN(T, TH, VP, R) TP_NH_BWD_(T, TH, VP, R, false)
    if (dt == TP_BF16) {
      if (rms) { TP_NH_BWD_DISPATCH(TP_NH_BWD, __nv_bfloat16, true); }
      else { TP_NH_BWD_DISPATCH(TP_NH_BWD, __nv_bfloat16, false); }
    } else {
      if (rms) { TP_NH_BWD_DISPATCH(TP_NH_BWD, float, true); }
      else { TP_NH_BWD_DISPATCH(TP_NH_BWD, float, false); }
    }
#undef TP_NH_BWD_PLAIN
#undef TP_NH_BWD_RES
#undef TP_NH_BWD_
    s = after_launch("norm_sharded_bwd");
    if (s != TP_OK) return s;
  }
  const unsigned cblocks = static_cast<unsigned>((h + kPass2Cols - 1) / kPass2Cols);
  if (rows > 0 && groups > 0 && cblocks <= static_cast<unsigned>(kPlanCounters)) {
    unsigned* ctr = nullptr;
    s = plan_counters(plan, st, &ctr);
    if (s != TP_OK) return s;
    (void)tpi::launch(norm_hsh_param_groups_final, dim3(cblocks, static_cast<unsigned>(groups)), dim3(256), 0, st,
                      part, static_cast<int>(grid), hs, h, inter, dg, db, accumulate, ctr);
  } else if (rows > 0 && groups > 0) {
    (void)tpi::launch(param_group_sum, dim3(dim3(cblocks, static_cast<unsigned>(groups))), dim3(256), 0, st, 
        part, static_cast<int>(grid), h, inter);
    s = after_launch("norm_sharded_bwd/param groups");
    if (s != TP_OK) return s;
    (void)tpi::launch(norm_hsh_param_pass2, dim3(cblocks), dim3(256), 0, st, inter, groups, hs, h, dg, db, accumulate);
  } else {
    (void)tpi::launch(norm_hsh_param_pass2, dim3(cblocks), dim3(256), 0, st, part, rows > 0 ? static_cast<int>(grid) : 0, hs, h, dg,
                                                  db, accumulate);
  }
  return after_launch("norm_sharded_bwd/param");
}

#undef TP_NH_BWD_DISPATCH
#undef TP_NH_DISPATCH

}  // namespace tpi
