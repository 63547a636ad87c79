// fp32 path: a shared-memory tiled FFMA GEMM (exact fp32 products and sums,
// k in increasing order) for plans whose dtype is fp32, and the element-wise
// activation kernels that follow it (GELU / SwiGLU forward and backward).
// The tensor cores have no fp32-exact mode, so fp32 plans run on the FMA pipes.
#include <algorithm>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {

using tpi::GemmBatch;

constexpr int TM = 64, TN = 64, TK = 16;

struct F32Problem {
  int M, N, K;
  const float* A;
  int64_t lda;
  const float* B;
  int64_t ldb;
  float* D;
  int64_t ldd;
  const float* bias;
};

// 256 threads; each computes a 4x4 block of the 64x64 output tile.
__global__ void __launch_bounds__(256) sgemm_kernel(F32Problem p, int a_mn, int b_mn) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += TK) {
    for (int i = threadIdx.x; i < TK * TM; i += 256) {
      const int kk = i / TM, mm = i % TM;
      const int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < p.M && k < p.K) v = a_mn ? p.A[static_cast<int64_t>(k) * p.lda + m] : p.A[static_cast<int64_t>(m) * p.lda + k];
      As[kk][mm] = v;
    }
    for (int i = threadIdx.x; i < TK * TN; i += 256) {
      const int kk = i / TN, nn = i % TN;
      const int n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < p.N && k < p.K) v = b_mn ? p.B[static_cast<int64_t>(k) * p.ldb + n] : p.B[static_cast<int64_t>(n) * p.ldb + k];
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= p.N) continue;
      float v = acc[i][j];
      if (p.bias) v += p.bias[n];
      p.D[static_cast<int64_t>(m) * p.ldd + n] = v;
    }
  }
}

__global__ void act_fwd_kernel(int act, const float* Z, int64_t T, int64_t nh, int64_t ldz,
                               float* H, int64_t ldh) {
  const int64_t total = T * nh;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / nh, j = i - t * nh;
    const float z = Z[t * ldz + j];
    H[t * ldh + j] = act == TP_ACT_GELU ? tpd::gelu_f(z) : tpd::silu_f(z) * Z[t * ldz + nh + j];
  }
}

__global__ void act_bwd_kernel(int act, const float* dH, int64_t T, int64_t nh, const float* Z,
                               int64_t ldz, float* dZ, int64_t lddz) {
  const int64_t total = T * nh;
  const int64_t ldh = act == TP_ACT_GELU ? lddz : nh;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / nh, j = i - t * nh;
    const float dh = dH[t * ldh + j];
    const float z = Z[t * ldz + j];
    if (act == TP_ACT_GELU) {
      dZ[t * lddz + j] = dh * tpd::gelu_grad_f(z);
    } else {
      const float u = Z[t * ldz + nh + j];
      dZ[t * lddz + j] = dh * u * tpd::silu_grad_f(z);
      dZ[t * lddz + nh + j] = dh * tpd::silu_f(z);
    }
  }
}

int grid_for(int64_t total) {
  return static_cast<int>(std::min<int64_t>((total + 255) / 256, 148 * 16));
}

}  // namespace

namespace tpi {

tp_status launch_gemm_f32(const GemmBatch& b, cudaStream_t st) {
  if (b.epi != EPI_STORE) return fail(TP_ERR_DTYPE, "fp32 GEMM supports the plain epilogue only");
  for (int i = 0; i < b.n; ++i) {
    const GemmProblem& g = b.g[i];
    F32Problem p{g.M, g.N, g.K, static_cast<const float*>(g.A), g.lda,
                 static_cast<const float*>(g.B), g.ldb, static_cast<float*>(g.D), g.ldd,
                 static_cast<const float*>(g.bias)};
    dim3 grid((g.N + TN - 1) / TN, (g.M + TM - 1) / TM);
    sgemm_kernel<<<grid, 256, 0, st>>>(p, b.a_mn ? 1 : 0, b.b_mn ? 1 : 0);
    tp_status s = after_launch("gemm_f32");
    if (s != TP_OK) return s;
  }
  return TP_OK;
}

tp_status launch_act_fwd(tp_act act, const float* Z, int64_t T, int64_t nh, int64_t ldz, float* H,
                         int64_t ldh, cudaStream_t st) {
  act_fwd_kernel<<<grid_for(T * nh), 256, 0, st>>>(static_cast<int>(act), Z, T, nh, ldz, H, ldh);
  return after_launch("act_fwd");
}

tp_status launch_act_bwd(tp_act act, const float* dH, int64_t T, int64_t nh, const float* Z,
                         int64_t ldz, float* dZ, int64_t lddz, cudaStream_t st) {
  act_bwd_kernel<<<grid_for(T * nh), 256, 0, st>>>(static_cast<int>(act), dH, T, nh, Z, ldz, dZ,
                                                   lddz);
  return after_launch("act_bwd");
}

}  // namespace tpi
