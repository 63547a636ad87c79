// fp32 path: a shared-memory tiled FFMA GEMM (exact fp32 products, sums in
// increasing k) for plans whose dtype is fp32, with the same fused epilogues
// and grouping as the tensor-core kernel: one launch covers every shard
// (grid.z), and the epilogue adds the bias, applies GELU / SwiGLU or their
// derivatives, or adds the residual of a K-concatenated shard sum.
//   EPI_STORE      D = acc (+ bias) (+ residual)
//   EPI_BIAS_GELU  Z = acc + bias (D, optional); H = GELU(Z) (D2)
//   EPI_SWIGLU     two accumulators per output unit j: gate row j and up row
//                  nh + j of B; Z = [g | u] (D, optional); H = SiLU(g) * u (D2)
//   EPI_DGELU      dZ = acc * GELU'(Z)                        (Z = aux)
//   EPI_DSWIGLU    dZ = [acc * u * SiLU'(g) | acc * SiLU(g)]  (Z = [g | u] = aux)
// K-concatenated (kcat): one output, the K loop runs over every shard's
// (A_s, B_s), so the sum over shards happens in the accumulator (TP
// walkthrough §2.2: the row layer's partials summed); an optional row scatter
// writes row r to the sequence shard that owns it (§4.3).
// The tensor cores have no fp32-exact mode, so fp32 plans run on the FMA pipes.
#include <algorithm>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {

using tpi::GemmBatch;

constexpr int TM = 64, TN = 64, TK = 16;

struct F32Group {
  int M, N, K;
  int nh;
  const float* A;
  int64_t lda;
  const float* B;
  int64_t ldb;
  float* D;
  int64_t ldd;
  float* D2;
  int64_t ldd2;
  const float* bias;
  const float* aux;
  int64_t ldaux;
};

struct F32Params {
  F32Group g[TP_MAX_SHARDS];
  int ngroups;
  int kcat;  // > 0: g[0..kcat) are K segments of the single output g[0]
  int epi;
  int a_mn, b_mn;
  int scatter;
  int rows_per_out;
  float* out_seq[TP_MAX_SHARDS];
  const float* res_seq[TP_MAX_SHARDS];
};

__device__ __forceinline__ float load_a(const F32Group& g, int a_mn, int m, int k) {
  if (m >= g.M || k >= g.K) return 0.f;
  return a_mn ? g.A[static_cast<int64_t>(k) * g.lda + m] : g.A[static_cast<int64_t>(m) * g.lda + k];
}
__device__ __forceinline__ float load_b(const F32Group& g, int b_mn, int n, int k, int nmax) {
  if (n >= nmax || k >= g.K) return 0.f;
  return b_mn ? g.B[static_cast<int64_t>(k) * g.ldb + n] : g.B[static_cast<int64_t>(n) * g.ldb + k];
}

// 256 threads; each computes a 4x4 block of the 64x64 output tile (two
// blocks, gate and up, for SwiGLU). blockIdx.z = group (shard).
__global__ void __launch_bounds__(256) sgemm_kernel(const __grid_constant__ F32Params p) {
  tpd::pdl_entry();
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  __shared__ float Us[TK][TN + 4];
  const int gi = p.kcat ? 0 : static_cast<int>(blockIdx.z);
  const F32Group& out = p.g[gi];
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  if (m0 >= out.M || n0 >= out.N) return;
  const bool swiglu = p.epi == tpi::EPI_SWIGLU;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  float accu[4][4] = {};
  const int nseg = p.kcat ? p.kcat : 1;
  for (int sg = 0; sg < nseg; ++sg) {
    const F32Group& g = p.g[p.kcat ? sg : gi];
    for (int k0 = 0; k0 < g.K; k0 += TK) {
      for (int i = threadIdx.x; i < TK * TM; i += 256) {
        const int kk = i / TM, mm = i % TM;
        As[kk][mm] = load_a(g, p.a_mn, m0 + mm, k0 + kk);
      }
      for (int i = threadIdx.x; i < TK * TN; i += 256) {
        const int kk = i / TN, nn = i % TN;
        const int n = n0 + nn;
        Bs[kk][nn] = load_b(g, p.b_mn, n, k0 + kk, out.N);
        // SwiGLU: up row nh + n of the [G_i; U_i] shard beside gate row n
        if (swiglu) Us[kk][nn] = load_b(g, p.b_mn, out.nh + n, k0 + kk, 2 * out.nh);
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
        if (swiglu) {
#pragma unroll
          for (int j = 0; j < 4; ++j) b[j] = Us[kk][tx * 4 + j];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) accu[i][j] = fmaf(a[i], b[j], accu[i][j]);
        }
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= out.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= out.N) continue;
      float v = acc[i][j];
      const int64_t mm = m;
      switch (p.epi) {
        case tpi::EPI_STORE: {
          if (out.bias) v += out.bias[n];
          float* dst = out.D + mm * out.ldd;
          const float* res = out.aux ? out.aux + mm * out.ldaux : nullptr;
          if (p.scatter) {
            const int js = m / p.rows_per_out;
            const int64_t lr = m - static_cast<int64_t>(js) * p.rows_per_out;
            dst = p.out_seq[js] + lr * out.ldd;
            res = p.res_seq[js] ? p.res_seq[js] + lr * out.ldaux : nullptr;
          }
          if (res) v += res[n];
          dst[n] = v;
          break;
        }
        case tpi::EPI_BIAS_GELU:
          if (out.bias) v += out.bias[n];
          if (out.D) out.D[mm * out.ldd + n] = v;
          out.D2[mm * out.ldd2 + n] = tpd::gelu_f(v);
          break;
        case tpi::EPI_SWIGLU: {
          const float u = accu[i][j];
          if (out.D) {
            out.D[mm * out.ldd + n] = v;
            out.D[mm * out.ldd + out.nh + n] = u;
          }
          out.D2[mm * out.ldd2 + n] = tpd::silu_f(v) * u;
          break;
        }
        case tpi::EPI_DGELU:
          out.D[mm * out.ldd + n] = v * tpd::gelu_grad_f(out.aux[mm * out.ldaux + n]);
          break;
        case tpi::EPI_DSWIGLU: {
          const float zg = out.aux[mm * out.ldaux + n];
          const float zu = out.aux[mm * out.ldaux + out.nh + n];
          out.D[mm * out.ldd + n] = v * zu * tpd::silu_grad_f(zg);
          out.D[mm * out.ldd + out.nh + n] = v * tpd::silu_f(zg);
          break;
        }
        default:
          break;
      }
    }
  }
}

}  // namespace

namespace tpi {

tp_status launch_gemm_f32(const GemmBatch& b, cudaStream_t st) {
  if (b.n < 1 || b.n > TP_MAX_SHARDS) return fail(TP_ERR_ARG, "GEMM group count %d", b.n);
  if (b.kcat && b.epi != EPI_STORE)
    return fail(TP_ERR_ARG, "K-concatenated GEMM supports the plain epilogue only");
  F32Params p{};
  int mmax = 0, nmax = 0;
  const int nout = b.kcat ? 1 : b.n;
  for (int i = 0; i < b.n; ++i) {
    const GemmProblem& g = b.g[i];
    const GemmProblem& o = b.kcat ? b.g[0] : g;
    if (o.M <= 0 || o.N <= 0 || g.K <= 0)
      return fail(TP_ERR_ARG, "GEMM %d has an empty extent (%d x %d x %d)", i, o.M, o.N, g.K);
    F32Group& f = p.g[i];
    f.M = o.M;
    f.N = o.N;
    f.K = g.K;
    f.nh = o.nh;
    f.A = static_cast<const float*>(g.A);
    f.lda = g.lda;
    f.B = static_cast<const float*>(g.B);
    f.ldb = g.ldb;
    f.D = static_cast<float*>(o.D);
    f.ldd = o.ldd;
    f.D2 = static_cast<float*>(o.D2);
    f.ldd2 = o.ldd2;
    f.bias = static_cast<const float*>(o.bias);
    f.aux = static_cast<const float*>(o.aux);
    f.ldaux = o.ldaux;
    if (i < nout) {
      mmax = std::max(mmax, o.M);
      nmax = std::max(nmax, o.N);
    }
  }
  p.ngroups = nout;
  p.kcat = b.kcat ? b.n : 0;
  p.epi = b.epi;
  p.a_mn = b.a_mn ? 1 : 0;
  p.b_mn = b.b_mn ? 1 : 0;
  if (b.scatter_n > 0) {
    if (!b.kcat && b.n != 1) return fail(TP_ERR_ARG, "row scatter needs a single output");
    p.scatter = 1;
    p.rows_per_out = static_cast<int>(b.rows_per_out);
    for (int j = 0; j < b.scatter_n; ++j) {
      p.out_seq[j] = static_cast<float*>(b.out_seq[j]);
      p.res_seq[j] = static_cast<const float*>(b.res_seq[j]);
    }
  }
  dim3 grid((nmax + TN - 1) / TN, (mmax + TM - 1) / TM, nout);
  (void)tpi::launch(sgemm_kernel, dim3(grid), dim3(256), 0, st, p);
  return after_launch("gemm_f32");
}

}  // namespace tpi
