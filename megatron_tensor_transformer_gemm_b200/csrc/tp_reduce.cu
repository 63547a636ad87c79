// HBM-streaming kernels of the TP path: the local all-reduce of the row-layer
// partials (sum in fixed order + bias once + residual), its sequence-parallel
// reduce-scatter form, the sequence all-gather, the bit-exact 2-D copies used
// for sharding, and deterministic column sums (bias gradients).
//
// Layout: a thread owns one 16-byte column vector (8 bf16 or 4 fp32) of a row
// and walks down the rows with a grid stride, so the column index, the bias
// vector and the output pointer arithmetic are computed once per thread and
// every warp touches 512 contiguous bytes per row: coalesced 128-bit traffic.
#include <algorithm>
#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {

using tpi::MutPtrArray;
using tpi::PtrArray;

constexpr int kThreads = 256;

// SM count of the current device, queried once per device and cached.
int sm_count() {
  constexpr int kMaxDev = 64;
  static int cached[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return 148;
  }
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

// 16-byte vector <-> 8 (bf16) or 4 (fp32) floats.
template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const uint4& u, float* f) {
    float2 a = tpd::unpack_bf16x2(u.x), b = tpd::unpack_bf16x2(u.y);
    float2 c = tpd::unpack_bf16x2(u.z), d = tpd::unpack_bf16x2(u.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
  }
  __device__ static uint4 store(const float* f) {
    return make_uint4(tpd::pack_bf16x2(f[0], f[1]), tpd::pack_bf16x2(f[2], f[3]),
                      tpd::pack_bf16x2(f[4], f[5]), tpd::pack_bf16x2(f[6], f[7]));
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 store(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));  // read once: evict-first
}
__device__ __forceinline__ uint4 ld_keep(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Finish one output vector: + bias, + residual, store (to the full output, or
// in the reduce-scatter (scatter != 0) to the sequence shard that owns row rr).
template <typename T>
__device__ __forceinline__ void reduce_finish(float (&a)[Vec<T>::N], const float (&b)[Vec<T>::N],
                                              int64_t rr, int64_t cols, int64_t cv,
                                              const T* residual, const PtrArray& res_seq,
                                              int res_is_seq, const MutPtrArray& out,
                                              int scatter, int64_t rows_per_out) {
  constexpr int V = Vec<T>::N;
#pragma unroll
  for (int k = 0; k < V; ++k) a[k] += b[k];
  T* dst;
  const T* res = nullptr;
  if (!scatter) {
    dst = static_cast<T*>(out.p[0]) + rr * cols + cv * V;
    if (residual) res = residual + rr * cols + cv * V;
  } else {
    const int j = static_cast<int>(rr / rows_per_out);
    const int64_t lr = rr - static_cast<int64_t>(j) * rows_per_out;
    dst = static_cast<T*>(out.p[j]) + lr * cols + cv * V;
    if (res_is_seq) res = static_cast<const T*>(res_seq.p[j]) + lr * cols + cv * V;
  }
  if (res) {
    float f[V];
    Vec<T>::load(ld_stream(res), f);
#pragma unroll
    for (int k = 0; k < V; ++k) a[k] += f[k];
  }
  *reinterpret_cast<uint4*>(dst) = Vec<T>::store(a);
}

// Y[rows] = sum_{i<n} P[i] in order 0..n-1 (fp32), + bias once, + residual.
// out.p[0] is the full output when scatter == 0, else out.p[j] holds rows
// [j*rows_per_out, (j+1)*rows_per_out) (the sequence-parallel reduce-scatter).
// A thread owns one 16-byte vector of the output (V elements of OT); the
// partials are of type PT, so each contributes W = V * sizeof(PT) / 16
// 16-byte loads per row (W = 2 for fp32 partials of a bf16 output). Each
// thread walks two rows per step and issues all 2nW loads before using any.
template <typename PT, typename OT, int NMAX>
__global__ void __launch_bounds__(kThreads) reduce_kernel(const __grid_constant__ PtrArray P, int n,
                                                          const OT* bias, const OT* residual,
                                                          const __grid_constant__ PtrArray res_seq,
                                                          int res_is_seq,
                                                          const __grid_constant__ MutPtrArray out,
                                                          int scatter, int64_t rows, int64_t vpr,
                                                          int64_t rows_per_out) {
  tpd::pdl_entry();
  constexpr int V = Vec<OT>::N;
  constexpr int W = V * static_cast<int>(sizeof(PT)) / 16;
  constexpr int VP = Vec<PT>::N;  // partial elements per 16-byte load
  static_assert(W * VP == V, "a partial vector spans whole 16-byte loads");
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (cv >= vpr) return;
  const int64_t cols = vpr * V;
  float b[V];
#pragma unroll
  for (int k = 0; k < V; ++k) b[k] = 0.f;
  if (bias) Vec<OT>::load(ld_keep(bias + cv * V), b);
  const int64_t stride = static_cast<int64_t>(gridDim.y) * blockDim.y;
  for (int64_t r = static_cast<int64_t>(blockIdx.y) * blockDim.y + threadIdx.y; r < rows;
       r += 2 * stride) {
    const int64_t r2 = r + stride;
    const bool two = r2 < rows;
    const int64_t off1 = r * cols + cv * V, off2 = (two ? r2 : r) * cols + cv * V;
    uint4 u1[NMAX][W], u2[NMAX][W];
#pragma unroll
    for (int i = 0; i < NMAX; ++i) {
      if (i < n) {
        const PT* base = static_cast<const PT*>(P.p[i]);
#pragma unroll
        for (int w = 0; w < W; ++w) {
          u1[i][w] = ld_stream(base + off1 + w * VP);
          if (two) u2[i][w] = ld_stream(base + off2 + w * VP);
        }
      }
    }
    float a1[V], a2[V];
#pragma unroll
    for (int k = 0; k < V; ++k) a1[k] = a2[k] = 0.f;
#pragma unroll
    for (int i = 0; i < NMAX; ++i) {
      if (i < n) {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          float f[VP];
          Vec<PT>::load(u1[i][w], f);
#pragma unroll
          for (int k = 0; k < VP; ++k) a1[w * VP + k] += f[k];
          if (two) {
            Vec<PT>::load(u2[i][w], f);
#pragma unroll
            for (int k = 0; k < VP; ++k) a2[w * VP + k] += f[k];
          }
        }
      }
    }
    reduce_finish<OT>(a1, b, r, cols, cv, residual, res_seq, res_is_seq, out, scatter, rows_per_out);
    if (two)
      reduce_finish<OT>(a2, b, r2, cols, cv, residual, res_seq, res_is_seq, out, scatter, rows_per_out);
  }
}

// X_full rows [j*rows_per_src, ...) = src.p[j] rows; 16-byte vectors. A thread
// owns one column vector and walks the rows of the full output with the grid's
// row stride, reading each from the shard that holds it (streaming loads: the
// shards are read once).
__global__ void __launch_bounds__(kThreads) gather_kernel(const __grid_constant__ PtrArray src, void* dst,
                                                          int64_t rows, int64_t vpr, int64_t rows_per_src) {
  tpd::pdl_entry();
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (cv >= vpr) return;
  const int64_t stride = static_cast<int64_t>(gridDim.y) * blockDim.y;
  uint4* D = static_cast<uint4*>(dst);
  for (int64_t r = static_cast<int64_t>(blockIdx.y) * blockDim.y + threadIdx.y; r < rows; r += stride) {
    const int j = static_cast<int>(r / rows_per_src);
    const int64_t lr = r - static_cast<int64_t>(j) * rows_per_src;
    D[r * vpr + cv] = ld_stream(static_cast<const uint4*>(src.p[j]) + lr * vpr + cv);
  }
}

// Strided 2-D copy of 16-byte vectors.
__global__ void copy2d_vec_kernel(const uint4* src, int64_t sld, uint4* dst, int64_t dld,
                                  int64_t rows, int64_t vpr) {
  tpd::pdl_entry();
  const int64_t total = rows * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vpr, c = i - r * vpr;
    dst[r * dld + c] = src[r * sld + c];
  }
}

// Strided 2-D copy, element by element (any element size that is 2 or 4 bytes).
template <typename E>
__global__ void copy2d_elem_kernel(const E* src, int64_t sld, E* dst, int64_t dld, int64_t rows,
                                   int64_t cols) {
  tpd::pdl_entry();
  const int64_t total = rows * cols;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / cols, c = i - r * cols;
    dst[r * dld + c] = src[r * sld + c];
  }
}

// Column sums, pass 1: block (32 column vectors x 8 row lanes) sums rows
// [split*rows_per_split, ...) of 32*V columns; lanes are combined in a fixed
// order and the result written to part[split][col].
template <typename T>
__global__ void __launch_bounds__(256) colsum_pass1(const T* x, int64_t ld, int64_t rows,
                                                    int64_t vpr, int64_t rows_per_split,
                                                    float* part, int64_t cols) {
  tpd::pdl_entry();
  constexpr int V = Vec<T>::N;
  __shared__ float red[8][32 * V + 1];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(rows, r0 + rows_per_split);
  float acc[V];
#pragma unroll
  for (int k = 0; k < V; ++k) acc[k] = 0.f;
  if (cv < vpr) {
    for (int64_t r = r0 + ty; r < r1; r += 8) {
      float f[V];
      Vec<T>::load(ld_stream(x + r * ld + cv * V), f);
#pragma unroll
      for (int k = 0; k < V; ++k) acc[k] += f[k];
    }
  }
#pragma unroll
  for (int k = 0; k < V; ++k) red[ty][tx * V + k] = acc[k];
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * V; c += 256) {
    float s = 0.f;
#pragma unroll
    for (int y = 0; y < 8; ++y) s += red[y][c];
    const int64_t col = static_cast<int64_t>(blockIdx.x) * 32 * V + c;
    if (col < cols) part[static_cast<int64_t>(blockIdx.y) * cols + col] = s;
  }
}

// Column sums, pass 2: out[c] (+)= sum over splits in order.
__global__ void colsum_pass2(const float* part, int splits, int64_t cols, float* out,
                             int accumulate) {
  tpd::pdl_entry();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float s = 0.f;
#pragma unroll 8
  for (int k = 0; k < splits; ++k) s += part[static_cast<int64_t>(k) * cols + c];
  out[c] = accumulate ? out[c] + s : s;
}

// Column sums of n same-shape inputs in one launch (blockIdx.z = input):
// pass 1 as colsum_pass1 over X.p[z], partials at part + z * splits * cols.
template <typename T>
__global__ void __launch_bounds__(256) colsum_grouped_pass1(const __grid_constant__ PtrArray X,
                                                            int64_t ld, int64_t rows, int64_t vpr,
                                                            int64_t rows_per_split, float* part,
                                                            int64_t cols) {
  tpd::pdl_entry();
  constexpr int V = Vec<T>::N;
  __shared__ float red[8][32 * V + 1];
  const T* x = static_cast<const T*>(X.p[blockIdx.z]);
  float* pz = part + static_cast<int64_t>(blockIdx.z) * gridDim.y * cols;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(rows, r0 + rows_per_split);
  float acc[V];
#pragma unroll
  for (int k = 0; k < V; ++k) acc[k] = 0.f;
  if (cv < vpr) {
    for (int64_t r = r0 + ty; r < r1; r += 8) {
      float f[V];
      Vec<T>::load(ld_stream(x + r * ld + cv * V), f);
#pragma unroll
      for (int k = 0; k < V; ++k) acc[k] += f[k];
    }
  }
#pragma unroll
  for (int k = 0; k < V; ++k) red[ty][tx * V + k] = acc[k];
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * V; c += 256) {
    float sum = 0.f;
#pragma unroll
    for (int y = 0; y < 8; ++y) sum += red[y][c];
    const int64_t col = static_cast<int64_t>(blockIdx.x) * 32 * V + c;
    if (col < cols) pz[static_cast<int64_t>(blockIdx.y) * cols + col] = sum;
  }
}

// Pass 2 of the grouped sums: out.p[blockIdx.y][c] (+)= sum over splits in order.
__global__ void colsum_grouped_pass2(const float* part, int splits, int64_t cols,
                                     const __grid_constant__ MutPtrArray out, int accumulate) {
  tpd::pdl_entry();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const float* pz = part + static_cast<int64_t>(blockIdx.y) * splits * cols;
  float sum = 0.f;
#pragma unroll 8
  for (int k = 0; k < splits; ++k) sum += pz[static_cast<int64_t>(k) * cols + c];
  float* o = static_cast<float*>(out.p[blockIdx.y]);
  o[c] = accumulate ? o[c] + sum : sum;
}

// Column sums of n same-shape inputs in one launch: every block sums its split
// of rows for 32*V columns of input blockIdx.z into part (as pass 1 above),
// and the last block to finish a (column slab, input) pair, counted on
// counters[z * gridDim.x + x], adds that slab's partials over the splits in
// split order and writes out.p[z] (so the sums are deterministic), then sets
// its counter back to zero.
template <typename T>
__global__ void __launch_bounds__(256) colsum_fused(const __grid_constant__ PtrArray X, int64_t ld,
                                                    int64_t rows, int64_t vpr, int64_t rows_per_split,
                                                    float* part, int64_t cols,
                                                    const __grid_constant__ MutPtrArray out,
                                                    int accumulate, unsigned* counters) {
  tpd::pdl_entry();
  constexpr int V = Vec<T>::N;
  __shared__ float red[8][32 * V + 1];
  __shared__ int last;
  const int splits = static_cast<int>(gridDim.y);
  const T* x = static_cast<const T*>(X.p[blockIdx.z]);
  float* pz = part + static_cast<int64_t>(blockIdx.z) * splits * cols;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(rows, r0 + rows_per_split);
  float acc[V];
#pragma unroll
  for (int k = 0; k < V; ++k) acc[k] = 0.f;
  if (cv < vpr) {
    for (int64_t r = r0 + ty; r < r1; r += 8) {
      float f[V];
      Vec<T>::load(ld_stream(x + r * ld + cv * V), f);
#pragma unroll
      for (int k = 0; k < V; ++k) acc[k] += f[k];
    }
  }
#pragma unroll
  for (int k = 0; k < V; ++k) red[ty][tx * V + k] = acc[k];
  __syncthreads();
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * 32 * V;
  for (int c = threadIdx.x; c < 32 * V; c += 256) {
    float sum = 0.f;
#pragma unroll
    for (int y = 0; y < 8; ++y) sum += red[y][c];
    if (col0 + c < cols) pz[static_cast<int64_t>(blockIdx.y) * cols + col0 + c] = sum;
  }
  __threadfence();  // this block's partials are visible before it is counted
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned* ctr = counters + static_cast<int64_t>(blockIdx.z) * gridDim.x + blockIdx.x;
    last = atomicAdd(ctr, 1u) == static_cast<unsigned>(splits - 1);
    if (last) atomicExch(ctr, 0u);  // no other block of this slab counts again
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  float* o = static_cast<float*>(out.p[blockIdx.z]);
  for (int c = threadIdx.x; c < 32 * V; c += 256) {
    const int64_t col = col0 + c;
    if (col >= cols) continue;
    float sum = 0.f;
#pragma unroll 16
    for (int k = 0; k < splits; ++k) sum += __ldcg(pz + static_cast<int64_t>(k) * cols + col);
    o[col] = accumulate ? o[col] + sum : sum;
  }
}

// Block shape for row-walking kernels: x covers column vectors, y rows.
void row_walk_shape(int64_t vpr, int64_t rows, dim3* grid, dim3* block) {
  int bx = static_cast<int>(std::min<int64_t>(kThreads, ((vpr + 31) / 32) * 32));
  int by = kThreads / bx;
  int gx = static_cast<int>((vpr + bx - 1) / bx);
  int64_t want = static_cast<int64_t>(sm_count()) * 8;  // 8 blocks per SM
  int64_t gy = std::max<int64_t>(1, want / gx);
  gy = std::min<int64_t>(gy, (rows + by - 1) / by);
  gy = std::min<int64_t>(gy, 65535);
  *block = dim3(bx, by);
  *grid = dim3(gx, static_cast<unsigned>(std::max<int64_t>(gy, 1)));
}

}  // namespace

namespace tpi {

tp_status launch_copy_2d(const void* src, int64_t src_ld, void* dst, int64_t dst_ld, int64_t rows,
                         int64_t cols, size_t esize, cudaStream_t st) {
  if (rows <= 0 || cols <= 0) return TP_OK;
  const bool vec = aligned16(src) && aligned16(dst) && (cols * esize) % 16 == 0 &&
                   (src_ld * esize) % 16 == 0 && (dst_ld * esize) % 16 == 0;
  if (vec) {
    const int64_t vpr = cols * esize / 16;
    const int64_t total = rows * vpr;
    int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, sm_count() * 16LL));
    (void)tpi::launch(copy2d_vec_kernel, dim3(blocks), dim3(256), 0, st, static_cast<const uint4*>(src),
                                              src_ld * esize / 16, static_cast<uint4*>(dst),
                                              dst_ld * esize / 16, rows, vpr);
  } else {
    const int64_t total = rows * cols;
    int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, sm_count() * 16LL));
    if (esize == 2)
      (void)tpi::launch(copy2d_elem_kernel<uint16_t>, dim3(blocks), dim3(256), 0, st, static_cast<const uint16_t*>(src),
                                                           src_ld, static_cast<uint16_t*>(dst),
                                                           dst_ld, rows, cols);
    else if (esize == 4)
      (void)tpi::launch(copy2d_elem_kernel<uint32_t>, dim3(blocks), dim3(256), 0, st, static_cast<const uint32_t*>(src),
                                                           src_ld, static_cast<uint32_t*>(dst),
                                                           dst_ld, rows, cols);
    else
      return fail(TP_ERR_ARG, "copy of %zu-byte elements", esize);
  }
  return after_launch("copy_2d");
}

tp_status launch_reduce(const PtrArray& P, int n, const void* bias, const void* residual,
                        const PtrArray& residual_seq, bool res_seq, const MutPtrArray& out,
                        bool out_is_seq, int nout, int64_t T, int64_t cols, tp_dtype pt,
                        tp_dtype dt, cudaStream_t st) {
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = cols / V;
  dim3 grid, block;
  row_walk_shape(vpr, T, &grid, &block);
  const int64_t rows_per_out = T / nout;
  const int rs = res_seq ? 1 : 0;
  const int scatter = out_is_seq ? 1 : 0;
  const int64_t T_rows = T;
#define TP_REDUCE_LAUNCH(PT, OT, NM)                                                            \
  (void)tpi::launch(reduce_kernel<PT, OT, NM>, dim3(grid), dim3(block), 0, st, P, n, static_cast<const OT*>(bias),          \
                                                    static_cast<const OT*>(residual),            \
                                                    residual_seq, rs, out, scatter, T_rows, vpr, \
                                                    rows_per_out)
#define TP_REDUCE_BY_N(PT, OT)                    \
  do {                                            \
    if (n <= 4) TP_REDUCE_LAUNCH(PT, OT, 4);      \
    else if (n <= 8) TP_REDUCE_LAUNCH(PT, OT, 8); \
    else TP_REDUCE_LAUNCH(PT, OT, TP_MAX_SHARDS); \
  } while (0)
  if (dt == TP_BF16 && pt == TP_BF16) TP_REDUCE_BY_N(__nv_bfloat16, __nv_bfloat16);
  else if (dt == TP_BF16 && pt == TP_F32) TP_REDUCE_BY_N(float, __nv_bfloat16);
  else if (dt == TP_F32 && pt == TP_F32) TP_REDUCE_BY_N(float, float);
  else return fail(TP_ERR_DTYPE, "reduce of partials of dtype %d into dtype %d", pt, dt);
#undef TP_REDUCE_BY_N
#undef TP_REDUCE_LAUNCH
  return after_launch("reduce_partials");
}

tp_status launch_gather(const PtrArray& src, int n, void* dst, int64_t T, int64_t cols,
                        tp_dtype dt, cudaStream_t st) {
  const int64_t vpr = cols * static_cast<int64_t>(dsize(dt)) / 16;
  dim3 grid, block;
  row_walk_shape(vpr, T, &grid, &block);
  (void)tpi::launch(gather_kernel, dim3(grid), dim3(block), 0, st, src, dst, T, vpr, T / n);
  return after_launch("all_gather_seq");
}

tp_status launch_column_sum(tp_plan* plan, const void* x, int64_t rows, int64_t cols, int64_t ld,
                            float* out, int accumulate, tp_dtype dt, cudaStream_t st, size_t ws_offset) {
  if (rows > 0) {  // one launch: the grouped form with one input
    PtrArray X{};
    MutPtrArray O{};
    X.p[0] = x;
    O.p[0] = out;
    return launch_column_sum_grouped(plan, X, 1, rows, cols, ld, O, accumulate, dt, st, ws_offset);
  }
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = cols / V;
  const int gx = static_cast<int>((vpr + 31) / 32);
  int64_t splits = std::max<int64_t>(1, (static_cast<int64_t>(sm_count()) * 8) / gx);
  splits = std::min<int64_t>(splits, std::max<int64_t>(1, (rows + 63) / 64));
  splits = std::min<int64_t>(splits, 1024);
  const int64_t rps = rows > 0 ? (rows + splits - 1) / splits : 1;
  splits = rows > 0 ? (rows + rps - 1) / rps : 1;
  void* ws = nullptr;
  tp_status s = workspace(plan, ws_offset + static_cast<size_t>(splits) * cols * sizeof(float), &ws);
  if (s != TP_OK) return s;
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ws_offset);
  if (rows > 0) {
    dim3 grid(gx, static_cast<unsigned>(splits));
    if (dt == TP_BF16)
      (void)tpi::launch(colsum_pass1<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x), ld,
                                                        rows, vpr, rps, part, cols);
    else
      (void)tpi::launch(colsum_pass1<float>, dim3(grid), dim3(256), 0, st, static_cast<const float*>(x), ld, rows, vpr, rps,
                                                part, cols);
    s = after_launch("column_sum/pass1");
    if (s != TP_OK) return s;
  } else {
    splits = 0;
  }
  (void)tpi::launch(colsum_pass2, dim3(static_cast<unsigned>((cols + 255) / 256)), dim3(256), 0, st, 
      part, static_cast<int>(splits), cols, out, accumulate);
  return after_launch("column_sum/pass2");
}

// The grouped column sums with their scratch chosen by the caller: `deferred`
// takes the side workspace and the upper half of the plan's counters.
static tp_status column_sum_grouped_impl(tp_plan* plan, const PtrArray& x, int n, int64_t rows, int64_t cols,
                                         int64_t ld, const MutPtrArray& out, int accumulate, tp_dtype dt,
                                         cudaStream_t st, size_t ws_offset, bool deferred) {
  if (n < 1 || n > TP_MAX_SHARDS) return fail(TP_ERR_ARG, "column sums of %d inputs", n);
  const int V = dt == TP_BF16 ? 8 : 4;
  const int64_t vpr = cols / V;
  const int gx = static_cast<int>((vpr + 31) / 32);
  int64_t splits = std::max<int64_t>(1, (static_cast<int64_t>(sm_count()) * 8) / (gx * n));
  splits = std::min<int64_t>(splits, std::max<int64_t>(1, (rows + 63) / 64));
  splits = std::min<int64_t>(splits, 1024);
  const int64_t rps = rows > 0 ? (rows + splits - 1) / splits : 1;
  splits = rows > 0 ? (rows + rps - 1) / rps : 0;
  const size_t bytes = ws_offset + static_cast<size_t>(std::max<int64_t>(splits, 1)) * cols * n * sizeof(float);
  void* ws = nullptr;
  tp_status s = deferred ? workspace2(plan, bytes, &ws) : workspace(plan, bytes, &ws);
  if (s != TP_OK) return s;
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ws_offset);
  if (rows > 0 && static_cast<int64_t>(gx) * n <= kPlanCounters) {
    // one launch: the last block of each column slab finishes it
    unsigned* ctr = nullptr;
    s = plan_counters(plan, st, &ctr);
    if (s != TP_OK) return s;
    if (deferred) ctr += kPlanCounters;
    dim3 grid(gx, static_cast<unsigned>(splits), static_cast<unsigned>(n));
    if (dt == TP_BF16)
      (void)tpi::launch(colsum_fused<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, x, ld, rows, vpr, rps, part, cols,
                        out, accumulate, ctr);
    else
      (void)tpi::launch(colsum_fused<float>, dim3(grid), dim3(256), 0, st, x, ld, rows, vpr, rps, part, cols, out,
                        accumulate, ctr);
    return after_launch("column_sum_grouped");
  }
  if (rows > 0) {
    dim3 grid(gx, static_cast<unsigned>(splits), static_cast<unsigned>(n));
    if (dt == TP_BF16)
      (void)tpi::launch(colsum_grouped_pass1<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, x, ld, rows, vpr, rps, part, cols);
    else
      (void)tpi::launch(colsum_grouped_pass1<float>, dim3(grid), dim3(256), 0, st, x, ld, rows, vpr, rps, part, cols);
    s = after_launch("column_sum_grouped/pass1");
    if (s != TP_OK) return s;
  }
  (void)tpi::launch(colsum_grouped_pass2, dim3(dim3(static_cast<unsigned>((cols + 255) / 256), static_cast<unsigned>(n))), dim3(256), 0, st, part, static_cast<int>(splits), cols, out, accumulate);
  return after_launch("column_sum_grouped/pass2");
}

tp_status launch_column_sum_grouped(tp_plan* plan, const PtrArray& x, int n, int64_t rows,
                                    int64_t cols, int64_t ld, const MutPtrArray& out, int accumulate,
                                    tp_dtype dt, cudaStream_t st, size_t ws_offset) {
  return column_sum_grouped_impl(plan, x, n, rows, cols, ld, out, accumulate, dt, st, ws_offset, false);
}

tp_status launch_column_sum_deferred(tp_plan* plan, const PtrArray& x, int n, int64_t rows,
                                     int64_t cols, int64_t ld, const MutPtrArray& out, tp_dtype dt,
                                     cudaStream_t st) {
  return column_sum_grouped_impl(plan, x, n, rows, cols, ld, out, 0, dt, st, 0, true);
}

}  // namespace tpi

// ---------------------------------------------------------------------------
// Column sums without any allocation: the scratch of the two-pass sum lives in
// a fixed file-scope device array instead of a cudaMalloc'd workspace.
// ---------------------------------------------------------------------------
namespace {

// Capacity of the static scratch in floats (2 MiB). Every GPU that loads the
// library holds this array until the process exits.
constexpr int64_t kStaticScratchFloats = 512 * 1024;
static __device__ __align__(256) float g_colsum_scratch[kStaticScratchFloats];

constexpr int kMaxDevicesStatic = 64;
float* g_scratch_addr[kMaxDevicesStatic] = {};
std::mutex g_scratch_mu;

// Device address of g_colsum_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
tp_status static_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesStatic) {
    cudaGetLastError();
    return tpi::fail(TP_ERR_NO_DEVICE, "no current CUDA device");
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    float* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_colsum_scratch);
    if (e != cudaSuccess || !ptr)
      return tpi::cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                              "cudaGetSymbolAddress(static column-sum scratch)");
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return TP_OK;
}

}  // namespace

extern "C" tp_status tp_column_sum_static(int64_t rows, int64_t cols, tp_dtype dtype,
                                          const void* x, float* out, int accumulate,
                                          void* stream) {
  using namespace tpi;
  if (dtype != TP_F32 && dtype != TP_BF16) return fail(TP_ERR_DTYPE, "unknown dtype %d", dtype);
  if (rows < 0 || rows > 0x7fffffffLL) return fail(TP_ERR_ARG, "rows = %lld", (long long)rows);
  if (cols <= 0 || cols > 0x7fffffffLL) return fail(TP_ERR_ARG, "cols = %lld", (long long)cols);
  if (cols > kStaticScratchFloats)
    return fail(TP_ERR_UNSUPPORTED,
                "cols = %lld exceeds the static scratch of tp_column_sum_static (%lld columns max)",
                (long long)cols, (long long)kStaticScratchFloats);
  if (rows > 0) {
    tp_status s = check_ptr(x, "x");
    if (s != TP_OK) return s;
  }
  tp_status s = check_ptr(out, "out");
  if (s != TP_OK) return s;
  s = check_row_bytes(cols, dtype, "cols");
  if (s != TP_OK) return s;
  float* part = nullptr;
  s = static_scratch(&part);
  if (s != TP_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int V = dtype == TP_BF16 ? 8 : 4;
  const int64_t vpr = cols / V;
  const int gx = static_cast<int>((vpr + 31) / 32);
  // Same split heuristic as the workspace version, capped so that
  // splits x cols floats fit in the static scratch.
  int64_t splits = std::max<int64_t>(1, (static_cast<int64_t>(sm_count()) * 8) / gx);
  splits = std::min<int64_t>(splits, std::max<int64_t>(1, (rows + 63) / 64));
  splits = std::min<int64_t>(splits, kStaticScratchFloats / cols);
  const int64_t rps = rows > 0 ? (rows + splits - 1) / splits : 1;
  splits = rows > 0 ? (rows + rps - 1) / rps : 0;
  if (rows > 0) {
    // Pass 1 writes every scratch entry pass 2 reads (splits x cols), so
    // nothing left from an earlier call is ever read.
    dim3 grid(gx, static_cast<unsigned>(splits));
    if (dtype == TP_BF16)
      (void)tpi::launch(colsum_pass1<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x),
                                                        cols, rows, vpr, rps, part, cols);
    else
      (void)tpi::launch(colsum_pass1<float>, dim3(grid), dim3(256), 0, st, static_cast<const float*>(x), cols, rows, vpr,
                                                rps, part, cols);
    s = after_launch("column_sum_static/pass1");
    if (s != TP_OK) return s;
  }
  (void)tpi::launch(colsum_pass2, dim3(static_cast<unsigned>((cols + 255) / 256)), dim3(256), 0, st, 
      part, static_cast<int>(splits), cols, out, accumulate);
  return after_launch("column_sum_static/pass2");
}
