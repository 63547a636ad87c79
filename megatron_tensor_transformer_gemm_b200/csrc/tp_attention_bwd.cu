// Causal attention backward on each shard's local heads, on the sm_100a
// tensor cores. From the forward's Q, K, V, O, the row log-sum-exp and dO:
//   P  = exp(Q K^T / sqrt(d) - lse)         (recomputed, masked)
//   dV = P^T dO;  dP = dO V^T;  dS = P * (dP - D),  D = rowsum(dO * O)
//   dQ = dS K / sqrt(d);  dK = dS^T Q / sqrt(d)
// Three launches, deterministic (no atomics):
//   attn_bwd_prep   D for every query row (one warp per row)
//   attn_bwd_dkdv   one CTA per 128-key block: loops over the query blocks that
//                   see it; S and dP in TMEM, P and dS written to shared memory
//                   (128B-swizzled, query rows), then read back MN-major as P^T
//                   and dS^T for dV += P^T dO and dK += dS^T Q (TMEM accumulators)
//   attn_bwd_dq     one CTA per 128-query block: loops over its key blocks;
//                   dS to shared memory (K-major) for dQ += dS K (TMEM)
// Warp roles in both main kernels: warp 0 TMA, warp 1 TMEM + MMA issue, warps
// 2..9 the element-wise work (softmax recompute, dS, epilogue), two warps per
// TMEM lane quarter, each on half of the 128 columns. Waits are bounded.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"
#include "tp_tma.h"

namespace {

using namespace tpd;
using tpi::MutPtrArray;
using tpi::PtrArray;

constexpr int BQ = 128, BKV = 128;
// Warp 0 TMA, warp 1 TMEM + MMA issue, warps 2..9 the element-wise work:
// warp w takes TMEM lane quarter w % 4 and column half (w - 2) / 4.
constexpr int kThreads = 320;
constexpr int CHUNK = 128 * 128;  // 128 rows x 128 bytes
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
  CUtensorMap tm_qkv[TP_MAX_SHARDS];  // {3*Hl*d, batch, seq}, box {64, 1, 128}
  CUtensorMap tm_do[TP_MAX_SHARDS];   // {Hl*d, batch, seq}, box {64, 1, 128}
  void* dqkv[TP_MAX_SHARDS];
  const float* lse[TP_MAX_SHARDS];
  const float* dvec[TP_MAX_SHARDS];
  int p, batch, seq, hl, nq, nkv;
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
  unsigned* status;
};

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Write 32 bf16 values (keys c*32 .. c*32+31 of row r) into a [128 x 128] bf16
// tile stored as two 128B-swizzled chunks of 64 columns.
__device__ __forceinline__ void store_row32_sw128(uint8_t* tile, int r, int c, const uint32_t (&pk)[16]) {
  uint8_t* rowp = tile + (c / 2) * CHUNK + r * 128;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int qv = (c % 2) * 4 + v;
    *reinterpret_cast<uint4*>(rowp + ((qv ^ (r & 7)) << 4)) =
        make_uint4(pk[v * 4 + 0], pk[v * 4 + 1], pk[v * 4 + 2], pk[v * 4 + 3]);
  }
}

// Store a row of D fp32 values (TMEM lane row, columns [col0, col0 + D)) scaled, as bf16.
template <int D>
__device__ __forceinline__ void tmem_row_to_global(uint32_t taddr, __nv_bfloat16* dst, float scale,
                                                   bool store) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    tc_wait_ld();
    if (store) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(dst + c * 32 + q * 8) = make_uint4(
            pack_bf16x2(v[q * 8 + 0] * scale, v[q * 8 + 1] * scale),
            pack_bf16x2(v[q * 8 + 2] * scale, v[q * 8 + 3] * scale),
            pack_bf16x2(v[q * 8 + 4] * scale, v[q * 8 + 5] * scale),
            pack_bf16x2(v[q * 8 + 6] * scale, v[q * 8 + 7] * scale));
    }
  }
}

// D[row] = sum_c dO[row, c] * O[row, c] for every (shard, b, head, q).
__global__ void attn_bwd_prep(const __grid_constant__ PtrArray O, const __grid_constant__ PtrArray dO,
                              const __grid_constant__ MutPtrArray dvec, int p, int batch, int seq,
                              int hl, int d) {
  const int64_t rows_per_shard = static_cast<int64_t>(batch) * hl * seq;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows_per_shard * p) return;
  const int shard = static_cast<int>(row / rows_per_shard);
  int64_t rest = row - shard * rows_per_shard;
  const int q = static_cast<int>(rest % seq);
  rest /= seq;
  const int hh = static_cast<int>(rest % hl);
  const int b = static_cast<int>(rest / hl);
  const int64_t off = (static_cast<int64_t>(q) * batch + b) * hl * d + static_cast<int64_t>(hh) * d;
  const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(O.p[shard]) + off;
  const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(dO.p[shard]) + off;
  float s = 0.f;
  for (int c = lane * 2; c < d; c += 64) {
    const float2 a = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(o + c));
    const float2 bb = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(g + c));
    s += a.x * bb.x + a.y * bb.y;
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) s += __shfl_xor_sync(0xffffffffu, s, k);
  if (lane == 0) static_cast<float*>(dvec.p[shard])[(static_cast<int64_t>(b) * hl + hh) * seq + q] = s;
}

// Row r of this CTA's 128 x 128 (query x key) block, 32-column chunks
// [c0, c0 + 2): P and dS recomputed from S and dP in TMEM. Writes P (if sP)
// and dS as bf16 into 128B-swizzled tiles.
__device__ __forceinline__ void p_ds_row(uint32_t tS, uint32_t tdP, uint32_t lane_off, int r, int q,
                                         int k0, int seq, float scale_log2, float lse2, float Dq,
                                         uint8_t* sP, uint8_t* sdS, int c0) {
#pragma unroll 1
  for (int c = c0; c < c0 + 2; ++c) {
    float s[32], dp[32];
    tmem_ld32(tS + lane_off + c * 32, s);
    tmem_ld32(tdP + lane_off + c * 32, dp);
    tc_wait_ld();
    uint32_t pk[16], dk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int key0 = k0 + c * 32 + e;
      const bool v0 = key0 <= q && key0 < seq && q < seq;
      const bool v1 = key0 + 1 <= q && key0 + 1 < seq && q < seq;
      const float p0 = v0 ? exp2f(s[e] * scale_log2 - lse2) : 0.f;
      const float p1 = v1 ? exp2f(s[e + 1] * scale_log2 - lse2) : 0.f;
      pk[e / 2] = pack_bf16x2(p0, p1);
      dk[e / 2] = pack_bf16x2(p0 * (dp[e] - Dq), p1 * (dp[e + 1] - Dq));
    }
    if (sP) store_row32_sw128(sP, r, c, pk);
    store_row32_sw128(sdS, r, c, dk);
  }
}

template <int D, int ST>
struct DkdvSmem {
  static constexpr int T = BQ * D * 2;  // one [128 x D] bf16 tile
  static constexpr int TOTAL = 1024 + 2 * T + 2 * ST * T + 2 * CHUNK * 2 + 256;
};

template <int D, int ST>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dkdv(const __grid_constant__ BwdParams p) {
  using SM = DkdvSmem<D, ST>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sK = smem;
  uint8_t* sV = sK + SM::T;
  uint8_t* sQ = sV + SM::T;          // [ST]
  uint8_t* sdO = sQ + ST * SM::T;    // [ST]
  uint8_t* sP = sdO + ST * SM::T;    // 2 chunks
  uint8_t* sdS = sP + 2 * CHUNK;     // 2 chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(sdS + 2 * CHUNK);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;   // [ST]
  uint64_t* q_empty = q_full + ST;  // [ST]
  uint64_t* s_full = q_empty + ST;
  uint64_t* p_full = s_full + 1;
  uint64_t* pds_empty = p_full + 1;
  uint64_t* acc_full = pds_empty + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = p.p * p.batch * p.hl;
  const int j = static_cast<int>(blockIdx.x) / per;  // key block; j = 0 has the most work
  int rest = static_cast<int>(blockIdx.x) % per;
  const int hh = rest % p.hl;
  rest /= p.hl;
  const int b = rest % p.batch;
  const int shard = rest / p.batch;
  const int k0 = j * BKV;
  const int n_iter = p.nq - j;  // query blocks j .. nq-1 see this key block
  const int hl_d = p.hl * D;
  const CUtensorMap* tq = &p.tm_qkv[shard];
  const CUtensorMap* tdo = &p.tm_do[shard];

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    mbar_init(pds_empty, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tq);
    tma_prefetch_desc(tdo);
    mbar_arrive_expect_tx(kv_full, 2 * SM::T);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sK + c * CHUNK, tq, kv_full, hl_d + hh * D + c * 64, b, k0);
      tma_load_3d(sV + c * CHUNK, tq, kv_full, 2 * hl_d + hh * D + c * 64, b, k0);
    }
    int last_par[ST];
    for (int s = 0; s < ST; ++s) last_par[s] = -1;
    for (int it = 0; it < n_iter; ++it) {
      const int st = it % ST;
      const uint32_t ph = static_cast<uint32_t>(it / ST) & 1u;
      if (!mbar_wait(&q_empty[st], ph ^ 1u, abort_flag, p.status)) break;
      const int q0 = (j + it) * BQ;
      mbar_arrive_expect_tx(&q_full[st], 2 * SM::T);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(sQ + st * SM::T + c * CHUNK, tq, &q_full[st], hh * D + c * 64, b, q0);
        tma_load_3d(sdO + st * SM::T + c * CHUNK, tdo, &q_full[st], hh * D + c * 64, b, q0);
      }
      last_par[st] = static_cast<int>(ph);
    }
    mbar_wait(kv_full, 0, abort_flag, p.status);
    for (int s = 0; s < ST; ++s)
      if (last_par[s] >= 0) mbar_wait(&q_full[s], static_cast<uint32_t>(last_par[s]), abort_flag, p.status);
  } else if (warp == 1 && lane == 0) {
    const uint32_t id_s = idesc_bf16(BQ, BKV, false, false);
    const uint32_t id_acc = idesc_bf16(BKV, D, true, true);
    const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
    const uint32_t p_base = smem_u32(sP), ds_base = smem_u32(sdS);
    bool ok = mbar_wait(kv_full, 0, abort_flag, p.status);
    for (int it = 0; ok && it < n_iter; ++it) {
      const int st = it % ST;
      if (!mbar_wait(&q_full[st], static_cast<uint32_t>(it / ST) & 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t q_base = smem_u32(sQ + st * SM::T), do_base = smem_u32(sdO + st * SM::T);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * CHUNK + (kk % 4) * 32;
        tc_mma_bf16(tS, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(k_base + off, 16, 1024),
                    id_s, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * CHUNK + (kk % 4) * 32;
        tc_mma_bf16(tdP, smem_desc_sw128(do_base + off, 16, 1024), smem_desc_sw128(v_base + off, 16, 1024),
                    id_s, kk > 0 ? 1u : 0u);
      }
      tc_commit(s_full);
      if (!mbar_wait(p_full, static_cast<uint32_t>(it) & 1u, abort_flag, p.status)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BQ / 16; ++kk) {  // K = queries
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        tc_mma_bf16(tdV, smem_desc_sw128(p_base + kk * 2048, CHUNK, 1024),
                    smem_desc_sw128(do_base + kk * 2048, CHUNK, 1024), id_acc, acc);
        tc_mma_bf16(tdK, smem_desc_sw128(ds_base + kk * 2048, CHUNK, 1024),
                    smem_desc_sw128(q_base + kk * 2048, CHUNK, 1024), id_acc, acc);
      }
      tc_commit(&q_empty[st]);
      tc_commit(pds_empty);
    }
    tc_commit(acc_full);
    tc_commit(drain);
    mbar_wait(drain, 0, abort_flag, p.status);
  } else if (warp >= 2) {
    const int lg = warp & 3;
    const int half = (warp - 2) / 4;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    const float* lse = p.lse[shard] + (static_cast<int64_t>(b) * p.hl + hh) * p.seq;
    const float* dv = p.dvec[shard] + (static_cast<int64_t>(b) * p.hl + hh) * p.seq;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int q = (j + it) * BQ + r;
      const float lse2 = q < p.seq ? lse[q] * kLog2e : 0.f;
      const float Dq = q < p.seq ? dv[q] : 0.f;
      // warp-uniform: p_ds_row's tcgen05.ld is warp-collective
      const bool got = mbar_wait(s_full, static_cast<uint32_t>(it) & 1u, abort_flag, p.status) &&
                       mbar_wait(pds_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      p_ds_row(tS, tdP, lane_off, r, q, k0, p.seq, p.scale_log2, lse2, Dq, sP, sdS, 2 * half);
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.status))) {
      tc_fence_after();
      const int key = k0 + r;  // accumulator lane = key row
      __nv_bfloat16* base = static_cast<__nv_bfloat16*>(p.dqkv[shard]) +
                            (static_cast<int64_t>(key) * p.batch + b) * (3 * hl_d) + hh * D;
      const bool st_ok = key < p.seq;
      if (half == 0) tmem_row_to_global<D>(tdV + lane_off, base + 2 * hl_d, 1.f, st_ok);
      else tmem_row_to_global<D>(tdK + lane_off, base + hl_d, p.scale, st_ok);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int ST>
struct DqSmem {
  static constexpr int T = BQ * D * 2;
  static constexpr int TOTAL = 1024 + 2 * T + 2 * ST * T + 2 * CHUNK + 256;
};

template <int D, int ST>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dq(const __grid_constant__ BwdParams p) {
  using SM = DqSmem<D, ST>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + SM::T;
  uint8_t* sK = sdO + SM::T;        // [ST]
  uint8_t* sV = sK + ST * SM::T;    // [ST]
  uint8_t* sdS = sV + ST * SM::T;   // 2 chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(sdS + 2 * CHUNK);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 1;    // [ST]
  uint64_t* kv_empty = kv_full + ST; // [ST]
  uint64_t* s_full = kv_empty + ST;
  uint64_t* p_full = s_full + 1;
  uint64_t* ds_empty = p_full + 1;
  uint64_t* acc_full = ds_empty + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = p.p * p.batch * p.hl;
  const int i = p.nq - 1 - static_cast<int>(blockIdx.x) / per;  // heaviest query blocks first
  int rest = static_cast<int>(blockIdx.x) % per;
  const int hh = rest % p.hl;
  rest /= p.hl;
  const int b = rest % p.batch;
  const int shard = rest / p.batch;
  const int q0 = i * BQ;
  const int n_iter = min(i + 1, p.nkv);
  const int hl_d = p.hl * D;
  const CUtensorMap* tq = &p.tm_qkv[shard];
  const CUtensorMap* tdo = &p.tm_do[shard];

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    mbar_init(ds_empty, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tq);
    tma_prefetch_desc(tdo);
    mbar_arrive_expect_tx(q_full, 2 * SM::T);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sQ + c * CHUNK, tq, q_full, hh * D + c * 64, b, q0);
      tma_load_3d(sdO + c * CHUNK, tdo, q_full, hh * D + c * 64, b, q0);
    }
    int last_par[ST];
    for (int s = 0; s < ST; ++s) last_par[s] = -1;
    for (int it = 0; it < n_iter; ++it) {
      const int st = it % ST;
      const uint32_t ph = static_cast<uint32_t>(it / ST) & 1u;
      if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag, p.status)) break;
      const int kb0 = it * BKV;
      mbar_arrive_expect_tx(&kv_full[st], 2 * SM::T);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(sK + st * SM::T + c * CHUNK, tq, &kv_full[st], hl_d + hh * D + c * 64, b, kb0);
        tma_load_3d(sV + st * SM::T + c * CHUNK, tq, &kv_full[st], 2 * hl_d + hh * D + c * 64, b, kb0);
      }
      last_par[st] = static_cast<int>(ph);
    }
    mbar_wait(q_full, 0, abort_flag, p.status);
    for (int s = 0; s < ST; ++s)
      if (last_par[s] >= 0) mbar_wait(&kv_full[s], static_cast<uint32_t>(last_par[s]), abort_flag, p.status);
  } else if (warp == 1 && lane == 0) {
    const uint32_t id_s = idesc_bf16(BQ, BKV, false, false);
    const uint32_t id_dq = idesc_bf16(BQ, D, false, true);
    const uint32_t q_base = smem_u32(sQ), do_base = smem_u32(sdO), ds_base = smem_u32(sdS);
    bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
    for (int it = 0; ok && it < n_iter; ++it) {
      const int st = it % ST;
      if (!mbar_wait(&kv_full[st], static_cast<uint32_t>(it / ST) & 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t k_base = smem_u32(sK + st * SM::T), v_base = smem_u32(sV + st * SM::T);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * CHUNK + (kk % 4) * 32;
        tc_mma_bf16(tS, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(k_base + off, 16, 1024),
                    id_s, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * CHUNK + (kk % 4) * 32;
        tc_mma_bf16(tdP, smem_desc_sw128(do_base + off, 16, 1024), smem_desc_sw128(v_base + off, 16, 1024),
                    id_s, kk > 0 ? 1u : 0u);
      }
      tc_commit(s_full);
      if (!mbar_wait(p_full, static_cast<uint32_t>(it) & 1u, abort_flag, p.status)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BKV / 16; ++kk) {  // K = keys
        const uint32_t aoff = (kk / 4) * CHUNK + (kk % 4) * 32;
        tc_mma_bf16(tdQ, smem_desc_sw128(ds_base + aoff, 16, 1024),
                    smem_desc_sw128(k_base + kk * 2048, CHUNK, 1024), id_dq,
                    (it > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(&kv_empty[st]);
      tc_commit(ds_empty);
    }
    tc_commit(acc_full);
    tc_commit(drain);
    mbar_wait(drain, 0, abort_flag, p.status);
  } else if (warp >= 2) {
    const int lg = warp & 3;
    const int half = (warp - 2) / 4;
    const int r = lg * 32 + lane;
    const int q = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    const float* lse = p.lse[shard] + (static_cast<int64_t>(b) * p.hl + hh) * p.seq;
    const float* dv = p.dvec[shard] + (static_cast<int64_t>(b) * p.hl + hh) * p.seq;
    const float lse2 = q < p.seq ? lse[q] * kLog2e : 0.f;
    const float Dq = q < p.seq ? dv[q] : 0.f;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      // warp-uniform: p_ds_row's tcgen05.ld is warp-collective
      const bool got = mbar_wait(s_full, static_cast<uint32_t>(it) & 1u, abort_flag, p.status) &&
                       mbar_wait(ds_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      p_ds_row(tS, tdP, lane_off, r, q, it * BKV, p.seq, p.scale_log2, lse2, Dq, nullptr, sdS, 2 * half);
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.status))) {
      tc_fence_after();
      __nv_bfloat16* base = static_cast<__nv_bfloat16*>(p.dqkv[shard]) +
                            (static_cast<int64_t>(q) * p.batch + b) * (3 * hl_d) + hh * D;
      // each column half of warps stores half of dQ's D columns
      tmem_row_to_global<D / 2>(tdQ + lane_off + half * (D / 2), base + half * (D / 2), p.scale, q < p.seq);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// STK / STQ: stages of the streamed Q, dO blocks (dK/dV kernel) and K, V
// blocks (dQ kernel); as many as fit the 227 KB of shared memory.
template <int D, int STK, int STQ>
tp_status launch_bwd_d(const BwdParams& prm, cudaStream_t st) {
  static_assert(DkdvSmem<D, STK>::TOTAL <= 232448 && DqSmem<D, STQ>::TOTAL <= 232448,
                "shared memory of the backward kernels");
  static bool attr = false;
  if (!attr) {
    tp_status s = tpi::cuda_status(
        cudaFuncSetAttribute(attn_bwd_dkdv<D, STK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkdvSmem<D, STK>::TOTAL), "cudaFuncSetAttribute(attention dkdv)");
    if (s != TP_OK) return s;
    s = tpi::cuda_status(cudaFuncSetAttribute(attn_bwd_dq<D, STQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              DqSmem<D, STQ>::TOTAL), "cudaFuncSetAttribute(attention dq)");
    if (s != TP_OK) return s;
    attr = true;
  }
  const int per = prm.p * prm.batch * prm.hl;
  attn_bwd_dkdv<D, STK><<<prm.nkv * per, kThreads, DkdvSmem<D, STK>::TOTAL, st>>>(prm);
  tp_status s = tpi::after_launch("attention_bwd dK/dV (tcgen05)");
  if (s != TP_OK) return s;
  attn_bwd_dq<D, STQ><<<prm.nq * per, kThreads, DqSmem<D, STQ>::TOTAL, st>>>(prm);
  return tpi::after_launch("attention_bwd dQ (tcgen05)");
}

}  // namespace

namespace tpi {

tp_status launch_attention_bwd(tp_plan* plan, int batch, int seq, const PtrArray& qkv,
                               const PtrArray& o, const PtrArray& dO, const float* const* lse,
                               const MutPtrArray& dqkv, cudaStream_t st) {
  const int p = plan->p, d = plan->head_dim, hl = plan->heads / plan->p;
  const int64_t rows_per_shard = static_cast<int64_t>(batch) * hl * seq;
  void* ws = nullptr;
  tp_status s = workspace(plan, static_cast<size_t>(rows_per_shard * p) * sizeof(float), &ws);
  if (s != TP_OK) return s;
  static BwdParams prm;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&prm, 0, sizeof(prm));
  MutPtrArray dvec{};
  const int64_t C = 3LL * hl * d;
  for (int i = 0; i < p; ++i) {
    dvec.p[i] = static_cast<float*>(ws) + i * rows_per_shard;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(batch), static_cast<cuuint64_t>(seq)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(C) * 2 * batch};
    cuuint32_t box[3] = {64, 1, 128};
    s = encode_bf16(&prm.tm_qkv[i], qkv.p[i], 3, dims, strides, box, "QKV (bwd)");
    if (s != TP_OK) return s;
    cuuint64_t dims2[3] = {static_cast<cuuint64_t>(hl) * d, static_cast<cuuint64_t>(batch), static_cast<cuuint64_t>(seq)};
    cuuint64_t strides2[2] = {static_cast<cuuint64_t>(hl) * d * 2, static_cast<cuuint64_t>(hl) * d * 2 * batch};
    s = encode_bf16(&prm.tm_do[i], dO.p[i], 3, dims2, strides2, box, "dO");
    if (s != TP_OK) return s;
    prm.dqkv[i] = dqkv.p[i];
    prm.lse[i] = lse[i];
    prm.dvec[i] = static_cast<const float*>(dvec.p[i]);
  }
  prm.p = p;
  prm.batch = batch;
  prm.seq = seq;
  prm.hl = hl;
  prm.nq = (seq + BQ - 1) / BQ;
  prm.nkv = (seq + BKV - 1) / BKV;
  prm.scale = 1.f / sqrtf(static_cast<float>(d));
  prm.scale_log2 = kLog2e * prm.scale;
  s = device_status_word(&prm.status);
  if (s != TP_OK) return s;
  const int64_t warps = rows_per_shard * p;
  if (warps * 32 / 256 + 1 > 0x7fffffffLL || static_cast<int64_t>(prm.nq) * p * batch * hl > 0x7fffffffLL)
    return fail(TP_ERR_UNSUPPORTED, "attention backward grid too large");
  attn_bwd_prep<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(o, dO, dvec, p, batch, seq, hl, d);
  s = after_launch("attention_bwd prep");
  if (s != TP_OK) return s;
  if (d == 64) return launch_bwd_d<64, 2, 2>(prm, st);
  if (d == 128) return launch_bwd_d<128, 1, 2>(prm, st);
  return fail(TP_ERR_UNSUPPORTED, "head_dim %d", d);
}

}  // namespace tpi
