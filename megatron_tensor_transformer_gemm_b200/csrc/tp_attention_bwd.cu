// Causal attention backward on each shard's local heads, on the sm_100a
// tensor cores. From the forward's Q, K, V, O, the row log-sum-exp and dO:
//   P  = exp(Q K^T / sqrt(d) - lse)         (recomputed, masked)
//   dV = P^T dO;  dP = dO V^T;  dS = P * (dP - D),  D = rowsum(dO * O)
//   dQ = dS K / sqrt(d);  dK = dS^T Q / sqrt(d)
// Three launches, deterministic (no atomics):
//   attn_bwd_prep     D and lse * log2(e) for every query row (d / 8 threads per row)
//   attn_bwd_dkdv_st  one CTA per 128-key block, keys as the MMA rows: loops
//                     over the 64-query sub-tiles that see it, S^T and dP^T in
//                     TMEM (two sub-tiles in flight), P^T and dS^T written to
//                     shared memory for dV += P^T dO and dK += dS^T Q (TMEM)
//   attn_bwd_dq       one CTA per 128-query block: loops over its key blocks;
//                     dS to shared memory (K-major) for dQ += dS K (TMEM)
// Warp roles in both main kernels: warp 0 TMA, warp 1 TMEM + MMA issue, warps
// 2..9 the element-wise work (softmax recompute, dS, epilogue), two warps per
// TMEM lane quarter, each on half of the 128 columns. Waits are bounded.
#include <cuda.h>

#include <algorithm>
#include <cstdlib>
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
  CUtensorMap tm_q64[TP_MAX_SHARDS];  // the same QKV, box {64, 1, 64}
  CUtensorMap tm_do64[TP_MAX_SHARDS]; // the same dO, box {64, 1, 64}
  void* dqkv[TP_MAX_SHARDS];
  const float* lse[TP_MAX_SHARDS];
  const float* dvec[TP_MAX_SHARDS];   // D, [batch * hl][seq_pad]
  const float* lse2[TP_MAX_SHARDS];   // lse * log2(e), [batch * hl][seq_pad]
  int p, batch, seq, hl, nq, nkv;
  int seq_pad;                        // seq rounded up to a multiple of 64
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
  // store_ds: the dK/dV kernel also stores dS^T to the workspace, viewed as
  // {queries, keys, shard * batch * hl} (query rows padded to seq_pad), and
  // dQ = dS K runs as a GEMM over it (attn_bwd_dq_gemm) instead of recomputing
  // S and dP (attn_bwd_dq).
  int store_ds;
  CUtensorMap tm_ds_st;  // box {64, 32, 1}: one warp pair's 32 key rows of a sub-tile
  CUtensorMap tm_ds_ld;  // box {64, 64, 1}
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

// D[row] = sum_c dO[row, c] * O[row, c] for every (shard, b, head, q), and
// lse2[row] = lse[row] * log2(e); both into [batch * hl][seq_pad] arrays.
// A row is G = d / 8 threads, each loading 16 bytes of O and of dO; the G
// products are summed by shuffles in a fixed order.
template <int G>
__global__ void attn_bwd_prep(const __grid_constant__ PtrArray O, const __grid_constant__ PtrArray dO,
                              const __grid_constant__ PtrArray LSE, const __grid_constant__ MutPtrArray dvec,
                              const __grid_constant__ MutPtrArray lse2, int p, int batch, int seq,
                              int seq_pad, int hl) {
  tpd::pdl_entry();
  constexpr int d = 8 * G;
  const int64_t rows_per_shard = static_cast<int64_t>(batch) * hl * seq;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = t / G;
  const int part = static_cast<int>(t % G);
  const bool live = row < rows_per_shard * p;  // whole groups share one row
  float s = 0.f;
  int shard = 0, q = 0;
  int64_t bh = 0;
  if (live) {
    shard = static_cast<int>(row / rows_per_shard);
    int64_t rest = row - shard * rows_per_shard;
    q = static_cast<int>(rest % seq);
    rest /= seq;
    const int hh = static_cast<int>(rest % hl);
    const int b = static_cast<int>(rest / hl);
    bh = static_cast<int64_t>(b) * hl + hh;
    const int64_t off = (static_cast<int64_t>(q) * batch + b) * hl * d + static_cast<int64_t>(hh) * d + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(O.p[shard]) + off);
    const uint4 g = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(dO.p[shard]) + off);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x = unpack_bf16x2(av[k]), y = unpack_bf16x2(gv[k]);
      s += x.x * y.x + x.y * y.y;
    }
  }
#pragma unroll
  for (int k = G / 2; k > 0; k >>= 1) s += __shfl_xor_sync(0xffffffffu, s, k, G);
  if (live && part == 0) {
    static_cast<float*>(dvec.p[shard])[bh * seq_pad + q] = s;
    static_cast<float*>(lse2.p[shard])[bh * seq_pad + q] = static_cast<const float*>(LSE.p[shard])[bh * seq + q] * kLog2e;
  }
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

// ---------------------------------------------------------------------------
// dK / dV with keys as the MMA rows and 64-query sub-tiles, two in flight.
// One CTA per 128-key block of one (shard, batch, head). For each sub-tile of
// 64 queries that sees the block:
//   S^T = K Q_s^T and dP^T = V dO_s^T      (M = 128 keys, N = 64 queries)
//   P^T = exp2(S^T * scale * log2e - lse2), dS^T = P^T * (dP^T - D)  (element-wise)
//   dV += P^T dO_s, dK += dS^T Q_s         (M = 128 keys, N = d, K = 64 queries)
// TMEM holds dV and dK (d columns each) and two (S^T, dP^T) pairs of 64
// columns each, so the MMAs of sub-tile i + 1 (and the dV / dK MMAs of i - 1)
// run while the element-wise warps turn sub-tile i into P^T and dS^T.
// Q_s, dO_s and their 64 values of lse2 and D stream through ST stages.
template <int D, int ST>
struct DkdvStSmem {
  static constexpr int KV = 128 * D * 2;    // one [128 x D] bf16 tile
  static constexpr int QS = 64 * D * 2;     // one [64 x D] bf16 sub-tile
  static constexpr int CH = 64 * 128;       // a 64-row 128B-swizzle column chunk of a sub-tile
  static constexpr int PT = 128 * 128;      // [128 keys x 64 queries] bf16 (one swizzle chunk)
  static constexpr int TOTAL = 1024 + 2 * KV + 2 * ST * QS + 4 * PT + ST * 512 + 256;
};

template <int D, int ST>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dkdv_st(const __grid_constant__ BwdParams p) {
  tpd::pdl_entry();
  using SM = DkdvStSmem<D, ST>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sK = smem;
  uint8_t* sV = sK + SM::KV;
  uint8_t* sQ = sV + SM::KV;           // [ST]
  uint8_t* sdO = sQ + ST * SM::QS;     // [ST]
  uint8_t* sP = sdO + ST * SM::QS;     // [2] P^T buffers
  uint8_t* sdS = sP + 2 * SM::PT;      // [2] dS^T buffers
  float* sL = reinterpret_cast<float*>(sdS + 2 * SM::PT);  // [ST][64] lse2 then [ST][64] D
  uint64_t* bars = reinterpret_cast<uint64_t*>(sL + ST * 128);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;      // [ST]
  uint64_t* q_empty = q_full + ST;     // [ST]
  uint64_t* s_full = q_empty + ST;     // [2]
  uint64_t* p_full = s_full + 2;       // [2]
  uint64_t* pds_empty = p_full + 2;    // [2]
  uint64_t* acc_full = pds_empty + 2;
  uint64_t* drain = acc_full + 1;
  uint64_t* ds_written = drain + 1;    // [4] per lane quarter: both column halves written
  uint64_t* ds_read = ds_written + 4;  // [4] per lane quarter: the slab's earlier store has read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ds_read + 4);
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
  const int nsub = (p.seq + 63) / 64 - 2 * j;  // 64-query sub-tiles 2j .. that see this key block
  const int hl_d = p.hl * D;
  const int64_t bh = static_cast<int64_t>(b) * p.hl + hh;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 8);
      mbar_init(&pds_empty[x], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&ds_written[q], 2);  // lane 0 of each of the two warps
      mbar_init(&ds_read[q], 1);
    }
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
  const uint32_t tdV = tmem, tdK = tmem + D;
  const uint32_t tS0 = tmem + 2 * D;  // buffer x: S^T at tS0 + 128 x, dP^T at tS0 + 128 x + 64

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    const CUtensorMap* tq = &p.tm_qkv[shard];
    const CUtensorMap* tq64 = &p.tm_q64[shard];
    const CUtensorMap* tdo64 = &p.tm_do64[shard];
    tma_prefetch_desc(tq);
    tma_prefetch_desc(tq64);
    tma_prefetch_desc(tdo64);
    mbar_arrive_expect_tx(kv_full, 2 * SM::KV);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sK + c * 128 * 128, tq, kv_full, hl_d + hh * D + c * 64, b, k0);
      tma_load_3d(sV + c * 128 * 128, tq, kv_full, 2 * hl_d + hh * D + c * 64, b, k0);
    }
    const float* lse2 = p.lse2[shard] + bh * p.seq_pad;
    const float* dv = p.dvec[shard] + bh * p.seq_pad;
    int last_par[ST];
    for (int s = 0; s < ST; ++s) last_par[s] = -1;
    for (int it = 0; it < nsub; ++it) {
      const int st = it % ST;
      const uint32_t ph = static_cast<uint32_t>(it / ST) & 1u;
      if (!mbar_wait(&q_empty[st], ph ^ 1u, abort_flag, p.status)) break;
      const int q0 = (2 * j + it) * 64;
      mbar_arrive_expect_tx(&q_full[st], 2 * SM::QS + 512);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(sQ + st * SM::QS + c * SM::CH, tq64, &q_full[st], hh * D + c * 64, b, q0);
        tma_load_3d(sdO + st * SM::QS + c * SM::CH, tdo64, &q_full[st], hh * D + c * 64, b, q0);
      }
      bulk_load(sL + st * 128, lse2 + q0, 256, &q_full[st]);
      bulk_load(sL + st * 128 + 64, dv + q0, 256, &q_full[st]);
      last_par[st] = static_cast<int>(ph);
    }
    mbar_wait(kv_full, 0, abort_flag, p.status);
    for (int s = 0; s < ST; ++s)
      if (last_par[s] >= 0) mbar_wait(&q_full[s], static_cast<uint32_t>(last_par[s]), abort_flag, p.status);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t id_s = idesc_bf16(BKV, 64, false, false);  // M = 128 keys, N = 64 queries
    const uint32_t id_acc = idesc_bf16(BKV, D, false, true);  // M = 128 keys, N = d, B MN-major
    const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
    bool ok = mbar_wait(kv_full, 0, abort_flag, p.status);
    // dV += P^T dO_s and dK += dS^T Q_s of sub-tile `it` (buffer it & 1)
    auto acc_mmas = [&](int it) -> bool {
      const int x = it & 1, st = it % ST;
      if (!mbar_wait(&p_full[x], static_cast<uint32_t>(it >> 1) & 1u, abort_flag, p.status)) return false;
      tc_fence_after();
      const uint32_t p_base = smem_u32(sP + x * SM::PT), ds_base = smem_u32(sdS + x * SM::PT);
      const uint32_t q_base = smem_u32(sQ + st * SM::QS), do_base = smem_u32(sdO + st * SM::QS);
#pragma unroll
      for (int kk = 0; kk < 64 / 16; ++kk) {  // K = the sub-tile's 64 queries
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        tc_mma_bf16(tdV, smem_desc_sw128(p_base + kk * 32, 16, 1024),
                    smem_desc_sw128(do_base + kk * 2048, SM::CH, 1024), id_acc, acc);
        tc_mma_bf16(tdK, smem_desc_sw128(ds_base + kk * 32, 16, 1024),
                    smem_desc_sw128(q_base + kk * 2048, SM::CH, 1024), id_acc, acc);
      }
      tc_commit(&q_empty[st]);
      tc_commit(&pds_empty[x]);
      return true;
    };
    for (int it = 0; ok && it < nsub; ++it) {
      const int st = it % ST, x = it & 1;
      if (!mbar_wait(&q_full[st], static_cast<uint32_t>(it / ST) & 1u, abort_flag, p.status)) break;
      tc_fence_after();
      // buffer x was last read by the element-wise pass of it - 2, whose
      // completion acc_mmas(it - 2) already waited for
      const uint32_t q_base = smem_u32(sQ + st * SM::QS), do_base = smem_u32(sdO + st * SM::QS);
      const uint32_t tS = tS0 + 128 * x, tdP = tS + 64;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t aoff = (kk / 4) * (128 * 128) + (kk % 4) * 32;
        const uint32_t boff = (kk / 4) * SM::CH + (kk % 4) * 32;
        tc_mma_bf16(tS, smem_desc_sw128(k_base + aoff, 16, 1024), smem_desc_sw128(q_base + boff, 16, 1024),
                    id_s, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t aoff = (kk / 4) * (128 * 128) + (kk % 4) * 32;
        const uint32_t boff = (kk / 4) * SM::CH + (kk % 4) * 32;
        tc_mma_bf16(tdP, smem_desc_sw128(v_base + aoff, 16, 1024), smem_desc_sw128(do_base + boff, 16, 1024),
                    id_s, kk > 0 ? 1u : 0u);
      }
      tc_commit(&s_full[x]);
      if (it > 0 && !acc_mmas(it - 1)) {
        ok = false;
        break;
      }
    }
    if (ok && nsub > 0) ok = acc_mmas(nsub - 1);
    tc_commit(acc_full);
    tc_commit(drain);
    mbar_wait(drain, 0, abort_flag, p.status);
  } else if (warp >= 2) {
    // --------------------------------------------------------- element-wise
    const int lg = warp & 3;
    const int half = (warp - 2) / 4;  // query columns [32 half, 32 half + 32) of a sub-tile
    const int r = lg * 32 + lane;     // key row of the block
    const int key = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    bool ok = true;
    for (int it = 0; it < nsub; ++it) {
      const int x = it & 1, st = it % ST;
      const uint32_t ph2 = static_cast<uint32_t>(it >> 1) & 1u;
      // warp-uniform: the tcgen05.ld below is warp-collective
      const bool got = mbar_wait(&s_full[x], ph2, abort_flag, p.status) &&
                       mbar_wait(&pds_empty[x], ph2 ^ 1u, abort_flag, p.status) &&
                       mbar_wait(&q_full[st], static_cast<uint32_t>(it / ST) & 1u, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tS0 + 128 * x, tdP = tS + 64;
      float sv[32], dp[32];
      tmem_ld32(tS + lane_off + half * 32, sv);
      tmem_ld32(tdP + lane_off + half * 32, dp);
      tc_wait_ld();
      const float* l2 = sL + st * 128 + half * 32;
      const float* dd = l2 + 64;
      const int qb = (2 * j + it) * 64 + half * 32;  // query of column 0 of this half
      uint32_t pk[16], dk[16];
      // below the diagonal and inside the sequence for the whole warp (every
      // key <= the first query, the last query < seq): no masks
      if (__all_sync(0xffffffffu, key <= qb && qb + 31 < p.seq)) {
        const float sc = p.scale_log2;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 L = *reinterpret_cast<const float4*>(l2 + e);
          const float4 Dq = *reinterpret_cast<const float4*>(dd + e);
          // pairs of columns in packed fp32 (one instruction per pair)
          const float2 x01 = fma2(sv[e], sv[e + 1], sc, sc, -L.x, -L.y);
          const float2 x23 = fma2(sv[e + 2], sv[e + 3], sc, sc, -L.z, -L.w);
          const float p0 = ex2(x01.x), p1 = ex2(x01.y), p2 = ex2(x23.x), p3 = ex2(x23.y);
          pk[e / 2] = pack_bf16x2(p0, p1);
          pk[e / 2 + 1] = pack_bf16x2(p2, p3);
          const float2 d01 = submul2(dp[e], dp[e + 1], Dq.x, Dq.y, p0, p1);
          const float2 d23 = submul2(dp[e + 2], dp[e + 3], Dq.z, Dq.w, p2, p3);
          dk[e / 2] = pack_bf16x2(d01.x, d01.y);
          dk[e / 2 + 1] = pack_bf16x2(d23.x, d23.y);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int qa = qb + e;
          const bool v0 = key <= qa && qa < p.seq && key < p.seq;
          const bool v1 = key <= qa + 1 && qa + 1 < p.seq && key < p.seq;
          const float p0 = v0 ? ex2(fmaf(sv[e], p.scale_log2, -l2[e])) : 0.f;
          const float p1 = v1 ? ex2(fmaf(sv[e + 1], p.scale_log2, -l2[e + 1])) : 0.f;
          pk[e / 2] = pack_bf16x2(p0, p1);
          dk[e / 2] = pack_bf16x2(v0 ? p0 * (dp[e] - dd[e]) : 0.f, v1 ? p1 * (dp[e + 1] - dd[e + 1]) : 0.f);
        }
      }
      if (p.store_ds && it >= 2) {
        // buffer x's dS^T slab was stored at it - 2; that store must have
        // read it before the rewrite (the half-0 warp's lane 0 issued it)
        bool rd = true;
        if (half == 0) {
          if (lane == 0) {
            bulk_wait_read<1>();
            mbar_arrive(&ds_read[lg]);
          }
          __syncwarp();
        } else {
          rd = mbar_wait(&ds_read[lg], static_cast<uint32_t>(it & 1), abort_flag, p.status);
        }
        if (!__all_sync(0xffffffffu, rd)) {
          ok = false;
          break;
        }
      }
      // row r of the [128 keys x 64 queries] K-major tiles: 16-byte chunks
      // 4 half .. 4 half + 3 of its 128-byte swizzled row
      uint8_t* prow = sP + x * SM::PT + r * 128;
      uint8_t* drow = sdS + x * SM::PT + r * 128;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int qv = half * 4 + v;
        *reinterpret_cast<uint4*>(prow + ((qv ^ (r & 7)) << 4)) =
            make_uint4(pk[v * 4 + 0], pk[v * 4 + 1], pk[v * 4 + 2], pk[v * 4 + 3]);
        *reinterpret_cast<uint4*>(drow + ((qv ^ (r & 7)) << 4)) =
            make_uint4(dk[v * 4 + 0], dk[v * 4 + 1], dk[v * 4 + 2], dk[v * 4 + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[x]);
      if (p.store_ds) {
        // rows [32 lg, 32 lg + 32) of dS^T, both column halves written: the
        // half-0 warp's lane 0 stores them (keys k0 + 32 lg.., this sub-tile's 64 queries)
        if (lane == 0) mbar_arrive(&ds_written[lg]);
        if (half == 0 && lane == 0 &&
            mbar_wait(&ds_written[lg], static_cast<uint32_t>(it & 1), abort_flag, p.status)) {
          tma_store_3d(&p.tm_ds_st, sdS + x * SM::PT + lg * 32 * 128, (2 * j + it) * 64, k0 + lg * 32,
                       static_cast<int>((static_cast<int64_t>(shard) * p.batch + b) * p.hl + hh));
          bulk_commit();
        }
      }
    }
    if (p.store_ds && half == 0 && lane == 0) bulk_wait_all();  // every dS^T store has landed
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.status))) {
      tc_fence_after();
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
  tpd::pdl_entry();
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
    const float* dv = p.dvec[shard] + (static_cast<int64_t>(b) * p.hl + hh) * p.seq_pad;
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

// ---------------------------------------------------------------------------
// dQ = dS K / sqrt(d) as a GEMM over the dS^T the dK/dV kernel stored: one CTA
// per 128-query block of one (shard, batch, head), looping over the 64-key
// blocks that reach it (causal: keys < q0 + 128). Per key block, dS (two
// 64-query blocks of dS^T, read MN-major) and K (D/64 blocks, MN-major) arrive
// by TMA into one of ST stages, and dQ += dS K accumulates in TMEM (M = 128
// queries, N = d, K = 64 keys); the epilogue scales and stores dQ. Entries of
// dS^T above the diagonal inside a stored tile are zeros (P is masked there).
template <int D, int ST>
struct DqgSmem {
  static constexpr int A = 64 * BQ * 2;  // dS^T [64 keys x 128 queries]
  static constexpr int B = 64 * D * 2;   // K [64 keys x D]
  static constexpr int STAGE = A + B;
  static constexpr int TOTAL = 1024 + ST * STAGE + 256;
};

template <int D, int ST>
__global__ void __launch_bounds__(kThreads, 2) attn_bwd_dq_gemm(const __grid_constant__ BwdParams p) {
  tpd::pdl_entry();
  using SM = DqgSmem<D, ST>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sA = smem;                 // [ST]
  uint8_t* sB = sA + ST * SM::A;      // [ST]
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + ST * SM::B);  // [ST]
  uint64_t* empty = full + ST;        // [ST]
  uint64_t* acc_full = empty + ST;
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
  const int n_kb = min(2 * i + 2, (p.seq + 63) / 64);  // 64-key blocks with keys < q0 + 128
  const int hl_d = p.hl * D;
  const int bhg = static_cast<int>((static_cast<int64_t>(shard) * p.batch + b) * p.hl + hh);
  constexpr uint32_t kCols = D < 32 ? 32 : D;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tdQ = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    const CUtensorMap* tk = &p.tm_q64[shard];  // QKV, box {64, 1, 64}: 64 keys x 64 of K's columns
    tma_prefetch_desc(tk);
    tma_prefetch_desc(&p.tm_ds_ld);
    int last_par[ST];
    for (int s = 0; s < ST; ++s) last_par[s] = -1;
    for (int kb = 0; kb < n_kb; ++kb) {
      const int st = kb % ST;
      const uint32_t ph = static_cast<uint32_t>(kb / ST) & 1u;
      if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) break;
      mbar_arrive_expect_tx(&full[st], SM::A + SM::B);
#pragma unroll
      for (int c = 0; c < BQ / 64; ++c)
        tma_load_3d(sA + st * SM::A + c * (64 * 128), &p.tm_ds_ld, &full[st], q0 + c * 64, kb * 64, bhg);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sB + st * SM::B + c * (64 * 128), tk, &full[st], hl_d + hh * D + c * 64, b, kb * 64);
      last_par[st] = static_cast<int>(ph);
    }
    for (int s = 0; s < ST; ++s)
      if (last_par[s] >= 0) mbar_wait(&full[s], static_cast<uint32_t>(last_par[s]), abort_flag, p.status);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t id = idesc_bf16(BQ, D, true, true);  // A = dS (MN-major), B = K (MN-major)
    bool ok = true;
    for (int kb = 0; kb < n_kb; ++kb) {
      const int st = kb % ST;
      if (!mbar_wait(&full[st], static_cast<uint32_t>(kb / ST) & 1u, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a_base = smem_u32(sA + st * SM::A), b_base = smem_u32(sB + st * SM::B);
#pragma unroll
      for (int kk = 0; kk < 64 / 16; ++kk)  // K = 64 keys, 16 per MMA: 16 rows of 128 bytes
        tc_mma_bf16(tdQ, smem_desc_sw128(a_base + kk * 2048, 64 * 128, 1024),
                    smem_desc_sw128(b_base + kk * 2048, 64 * 128, 1024), id, (kb | kk) != 0 ? 1u : 0u);
      tc_commit(&empty[st]);
    }
    (void)ok;
    tc_commit(acc_full);
    tc_commit(drain);
    mbar_wait(drain, 0, abort_flag, p.status);
  } else if (warp >= 2) {
    // ------------------------------------------------------------- epilogue
    const int lg = warp & 3;
    const int half = (warp - 2) / 4;
    const int q = q0 + lg * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    if (n_kb > 0 && __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.status))) {
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
    tmem_dealloc(tdQ, kCols);
  }
}

// STS: stages of the streamed 64-query Q, dO sub-tiles (dK/dV kernel); STQ:
// stages of the streamed 128-key K, V blocks (dQ kernel); as many as fit the
// 227 KB of shared memory.
template <int D, int STS, int STQ, int STG>
tp_status launch_bwd_d(const BwdParams& prm, cudaStream_t st) {
  static_assert(DkdvStSmem<D, STS>::TOTAL <= 232448 && DqSmem<D, STQ>::TOTAL <= 232448 &&
                    2 * DqgSmem<D, STG>::TOTAL <= 232448,
                "shared memory of the backward kernels");
  constexpr int kMaxDev = 64;
  static bool attr[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return tpi::fail(TP_ERR_NO_DEVICE, "no current CUDA device");
  }
  if (!attr[dev]) {
    tp_status s = tpi::cuda_status(
        cudaFuncSetAttribute(attn_bwd_dkdv_st<D, STS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkdvStSmem<D, STS>::TOTAL), "cudaFuncSetAttribute(attention dkdv)");
    if (s != TP_OK) return s;
    s = tpi::cuda_status(cudaFuncSetAttribute(attn_bwd_dq<D, STQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              DqSmem<D, STQ>::TOTAL), "cudaFuncSetAttribute(attention dq)");
    if (s != TP_OK) return s;
    s = tpi::cuda_status(cudaFuncSetAttribute(attn_bwd_dq_gemm<D, STG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              DqgSmem<D, STG>::TOTAL), "cudaFuncSetAttribute(attention dq gemm)");
    if (s != TP_OK) return s;
    attr[dev] = true;
  }
  const int per = prm.p * prm.batch * prm.hl;
  (void)tpi::launch(attn_bwd_dkdv_st<D, STS>, dim3(prm.nkv * per), dim3(kThreads), DkdvStSmem<D, STS>::TOTAL, st,
                    prm);
  tp_status s = tpi::after_launch("attention_bwd dK/dV (tcgen05)");
  if (s != TP_OK) return s;
  if (prm.store_ds)
    (void)tpi::launch(attn_bwd_dq_gemm<D, STG>, dim3(prm.nq * per), dim3(kThreads), DqgSmem<D, STG>::TOTAL, st,
                      prm);
  else
    (void)tpi::launch(attn_bwd_dq<D, STQ>, dim3(prm.nq * per), dim3(kThreads), DqSmem<D, STQ>::TOTAL, st, prm);
  return tpi::after_launch("attention_bwd dQ (tcgen05)");
}

}  // namespace

namespace tpi {

tp_status launch_attention_bwd(tp_plan* plan, int batch, int seq, const PtrArray& qkv,
                               const PtrArray& o, const PtrArray& dO, const float* const* lse,
                               const MutPtrArray& dqkv, cudaStream_t st) {
  const int p = plan->p, d = plan->head_dim, hl = plan->heads / plan->p;
  const int64_t rows_per_shard = static_cast<int64_t>(batch) * hl * seq;
  const int seq_pad = (seq + 63) / 64 * 64;
  const int64_t padded_per_shard = static_cast<int64_t>(batch) * hl * seq_pad;
  // workspace: D and lse2 ([p][batch * hl][seq_pad] fp32 each), then, when dQ
  // runs as a GEMM over the stored dS^T, dS^T [p * batch * hl][seq_pad keys][seq_pad queries]
  // bf16 (up to kDsBytesMax; longer sequences recompute S and dP in attn_bwd_dq).
  constexpr size_t kDsBytesMax = size_t(8) << 30;
  const size_t vec_bytes = (static_cast<size_t>(2 * padded_per_shard * p) * sizeof(float) + 1023) / 1024 * 1024;
  const size_t ds_bytes = static_cast<size_t>(p) * batch * hl * seq_pad * seq_pad * 2;
  const char* e_ds = getenv("TP_ATTN_BWD_DS");
  const bool store_ds = !(e_ds && e_ds[0] == '0') && ds_bytes <= kDsBytesMax;
  void* ws = nullptr;
  tp_status s = workspace(plan, vec_bytes + (store_ds ? ds_bytes : 0), &ws);
  if (s != TP_OK) return s;
  static BwdParams prm;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&prm, 0, sizeof(prm));
  MutPtrArray dvec{}, lse2{};
  PtrArray lse_in{};
  const int64_t C = 3LL * hl * d;
  for (int i = 0; i < p; ++i) {
    dvec.p[i] = static_cast<float*>(ws) + i * padded_per_shard;
    lse2.p[i] = static_cast<float*>(ws) + (p + i) * padded_per_shard;
    lse_in.p[i] = lse[i];
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(batch), static_cast<cuuint64_t>(seq)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(C) * 2 * batch};
    cuuint32_t box[3] = {64, 1, 128};
    s = encode_bf16(&prm.tm_qkv[i], qkv.p[i], 3, dims, strides, box, "QKV (bwd)");
    if (s != TP_OK) return s;
    cuuint64_t dims2[3] = {static_cast<cuuint64_t>(hl) * d, static_cast<cuuint64_t>(batch), static_cast<cuuint64_t>(seq)};
    cuuint64_t strides2[2] = {static_cast<cuuint64_t>(hl) * d * 2, static_cast<cuuint64_t>(hl) * d * 2 * batch};
    s = encode_bf16(&prm.tm_do[i], dO.p[i], 3, dims2, strides2, box, "dO");
    if (s != TP_OK) return s;
    cuuint32_t box64[3] = {64, 1, 64};
    s = encode_bf16(&prm.tm_q64[i], qkv.p[i], 3, dims, strides, box64, "QKV (bwd, 64 rows)");
    if (s != TP_OK) return s;
    s = encode_bf16(&prm.tm_do64[i], dO.p[i], 3, dims2, strides2, box64, "dO (64 rows)");
    if (s != TP_OK) return s;
    prm.lse2[i] = static_cast<const float*>(lse2.p[i]);
    prm.dqkv[i] = dqkv.p[i];
    prm.lse[i] = lse[i];
    prm.dvec[i] = static_cast<const float*>(dvec.p[i]);
  }
  prm.store_ds = store_ds ? 1 : 0;
  if (store_ds) {
    void* ds = static_cast<uint8_t*>(ws) + vec_bytes;
    cuuint64_t dd[3] = {static_cast<cuuint64_t>(seq), static_cast<cuuint64_t>(seq),
                        static_cast<cuuint64_t>(p) * batch * hl};
    cuuint64_t ds_str[2] = {static_cast<cuuint64_t>(seq_pad) * 2, static_cast<cuuint64_t>(seq_pad) * seq_pad * 2};
    cuuint32_t box_st[3] = {64, 32, 1}, box_ld[3] = {64, 64, 1};
    s = encode_bf16(&prm.tm_ds_st, ds, 3, dd, ds_str, box_st, "dS^T (stores)");
    if (s != TP_OK) return s;
    s = encode_bf16(&prm.tm_ds_ld, ds, 3, dd, ds_str, box_ld, "dS^T (loads)");
    if (s != TP_OK) return s;
  }
  prm.p = p;
  prm.batch = batch;
  prm.seq = seq;
  prm.hl = hl;
  prm.nq = (seq + BQ - 1) / BQ;
  prm.nkv = (seq + BKV - 1) / BKV;
  prm.seq_pad = seq_pad;
  prm.scale = 1.f / sqrtf(static_cast<float>(d));
  prm.scale_log2 = kLog2e * prm.scale;
  s = device_status_word(&prm.status);
  if (s != TP_OK) return s;
  const int64_t warps = rows_per_shard * p;
  if (warps * 32 / 256 + 1 > 0x7fffffffLL || static_cast<int64_t>(prm.nq) * p * batch * hl > 0x7fffffffLL)
    return fail(TP_ERR_UNSUPPORTED, "attention backward grid too large");
  const int G = d / 8;  // threads per row
  const unsigned pblocks = static_cast<unsigned>((rows_per_shard * p * G + 255) / 256);
  if (d == 64)
    (void)tpi::launch(attn_bwd_prep<8>, dim3(pblocks), dim3(256), 0, st, o, dO, lse_in, dvec, lse2, p, batch, seq,
                      seq_pad, hl);
  else
    (void)tpi::launch(attn_bwd_prep<16>, dim3(pblocks), dim3(256), 0, st, o, dO, lse_in, dvec, lse2, p, batch, seq,
                      seq_pad, hl);
  s = after_launch("attention_bwd prep");
  if (s != TP_OK) return s;
  if (d == 64) return launch_bwd_d<64, 4, 2, 4>(prm, st);
  if (d == 128) return launch_bwd_d<128, 3, 2, 3>(prm, st);
  return fail(TP_ERR_UNSUPPORTED, "head_dim %d", d);
}

}  // namespace tpi
