// Causal attention on each shard's local heads, forward, on the sm_100a
// tensor cores (TP walkthrough 2kiu.com §3.1: every shard runs full-sequence
// attention on its own whole heads, with no cross-shard step).
//
// One CTA computes one 128-query tile of one (shard, batch, head):
//   warp 0      TMA producer: the Q tile once, then K and V blocks of 128 keys
//               into a 2-stage ring (3-D tensor map over the sequence-major
//               [seq, batch, 3*heads_local*d] QKV buffer of the shard)
//   warp 1      TMEM allocator + MMA issuer: S = Q K^T (128 x 128, fp32 in
//               TMEM), then O_j = P V_j (128 x d, fp32 in TMEM)
//   warps 2..5  softmax: thread r owns query row r; two passes over its row of
//               S in TMEM (row max, then exp2 and the row sum), P rounded to
//               bf16 and written to shared memory in the 128-byte-swizzled
//               K-major layout the PV MMA reads; O and the online-softmax
//               state (m, l) stay in registers and are rescaled per block.
// Blocks are causal: the tile's last key block is the diagonal one and is
// masked (key > query -> probability 0); keys and queries past seq are masked.
// The backward (tp_attention_bwd.cu) recomputes P from the saved row log-sum-exp.
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

constexpr int BQ = 128;        // queries per tile
constexpr int BKV = 128;       // keys per block
constexpr int KV_STAGES = 2;
constexpr int kThreads = 192;
constexpr int CHUNK_BYTES = 128 * 128;  // 128 rows x 64 bf16 (one swizzle-atom column)
constexpr float kLog2e = 1.4426950408889634f;

struct AttnParams {
  CUtensorMap tm[TP_MAX_SHARDS];  // QKV_i as {3*Hl*d, batch, seq}, box {64, 1, 128}
  void* O[TP_MAX_SHARDS];
  float* lse[TP_MAX_SHARDS];
  int p, batch, seq, heads_local, d;
  int n_qtiles;
  float scale_log2;  // log2(e) / sqrt(d)
  unsigned* status;
};

template <int D>
struct AttnSmem {
  static constexpr int Q_BYTES = BQ * D * 2;
  static constexpr int KV_BYTES = BKV * D * 2;
  static constexpr int P_BYTES = BQ * BKV * 2;
  static constexpr int TOTAL = 1024 + Q_BYTES + 2 * KV_STAGES * KV_BYTES + P_BYTES + 256;
};

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using SM = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + SM::Q_BYTES;
  uint8_t* sV = sK + KV_STAGES * SM::KV_BYTES;
  uint8_t* sP = sV + KV_STAGES * SM::KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + SM::P_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                  // [KV_STAGES]
  uint64_t* v_full = k_full + KV_STAGES;        // [KV_STAGES]
  uint64_t* kv_empty = v_full + KV_STAGES;      // [KV_STAGES]
  uint64_t* s_full = kv_empty + KV_STAGES;
  uint64_t* p_full = s_full + 1;
  uint64_t* o_full = p_full + 1;
  uint64_t* o_empty = o_full + 1;
  uint64_t* drain = o_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Tile decode: heaviest (last) query tiles first.
  const int per_qt = p.p * p.batch * p.heads_local;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / per_qt;
  int rest = static_cast<int>(blockIdx.x) % per_qt;
  const int hh = rest % p.heads_local;
  rest /= p.heads_local;
  const int b = rest % p.batch;
  const int shard = rest / p.batch;
  const int q0 = qt * BQ;
  const int n_kv_total = (p.seq + BKV - 1) / BKV;
  const int nb = min(qt + 1, n_kv_total);  // causal: key blocks 0..qt
  const int hl_d = p.heads_local * D;
  const CUtensorMap* tm = &p.tm[shard];

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;        // columns [0, 128)
  const uint32_t tO = tmem + 128;  // columns [128, 128 + D)

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------- producer
    tma_prefetch_desc(tm);
    mbar_arrive_expect_tx(q_full, SM::Q_BYTES);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_load_3d(sQ + c * CHUNK_BYTES, tm, q_full, hh * D + c * 64, b, q0);
    int last_par[KV_STAGES];
    for (int s = 0; s < KV_STAGES; ++s) last_par[s] = -1;
    for (int j = 0; j < nb; ++j) {
      const int st = j % KV_STAGES;
      const uint32_t ph = static_cast<uint32_t>(j / KV_STAGES) & 1u;
      if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag, p.status)) break;
      const int k0 = j * BKV;
      mbar_arrive_expect_tx(&k_full[st], SM::KV_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sK + st * SM::KV_BYTES + c * CHUNK_BYTES, tm, &k_full[st],
                    hl_d + hh * D + c * 64, b, k0);
      mbar_arrive_expect_tx(&v_full[st], SM::KV_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sV + st * SM::KV_BYTES + c * CHUNK_BYTES, tm, &v_full[st],
                    2 * hl_d + hh * D + c * 64, b, k0);
      last_par[st] = static_cast<int>(ph);
    }
    mbar_wait(q_full, 0, abort_flag, p.status);
    for (int s = 0; s < KV_STAGES; ++s)
      if (last_par[s] >= 0) {
        mbar_wait(&k_full[s], static_cast<uint32_t>(last_par[s]), abort_flag, p.status);
        mbar_wait(&v_full[s], static_cast<uint32_t>(last_par[s]), abort_flag, p.status);
      }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc_s = idesc_bf16(BQ, BKV, false, false);
    const uint32_t idesc_o = idesc_bf16(BQ, D, false, true);
    const uint32_t q_base = smem_u32(sQ), p_base = smem_u32(sP);
    bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
    auto issue_s = [&](int j) -> bool {
      const int st = j % KV_STAGES;
      if (!mbar_wait(&k_full[st], static_cast<uint32_t>(j / KV_STAGES) & 1u, abort_flag, p.status))
        return false;
      tc_fence_after();
      const uint32_t k_base = smem_u32(sK + st * SM::KV_BYTES);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * CHUNK_BYTES + (kk % 4) * 32;
        tc_mma_bf16(tS, smem_desc_sw128(q_base + off, 16, 1024),
                    smem_desc_sw128(k_base + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
      }
      tc_commit(s_full);
      return true;
    };
    if (ok && nb > 0) ok = issue_s(0);
    for (int j = 0; ok && j < nb; ++j) {
      const int st = j % KV_STAGES;
      const uint32_t ph = static_cast<uint32_t>(j) & 1u;
      if (!mbar_wait(p_full, ph, abort_flag, p.status)) break;
      if (!mbar_wait(&v_full[st], static_cast<uint32_t>(j / KV_STAGES) & 1u, abort_flag, p.status)) break;
      if (!mbar_wait(o_empty, ph ^ 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t v_base = smem_u32(sV + st * SM::KV_BYTES);
#pragma unroll
      for (int kk = 0; kk < BKV / 16; ++kk) {
        const uint64_t adesc = smem_desc_sw128(p_base + (kk / 4) * CHUNK_BYTES + (kk % 4) * 32, 16, 1024);
        const uint64_t bdesc = smem_desc_sw128(v_base + kk * 2048, CHUNK_BYTES, 1024);
        tc_mma_bf16(tO, adesc, bdesc, idesc_o, kk > 0 ? 1u : 0u);
      }
      tc_commit(o_full);
      tc_commit(&kv_empty[st]);
      if (j + 1 < nb) ok = issue_s(j + 1);
    }
    tc_commit(drain);
    mbar_wait(drain, 0, abort_flag, p.status);
  } else if (warp >= 2) {
    // ------------------------------------------------------------- softmax
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const int q = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    float o[D];
#pragma unroll
    for (int i = 0; i < D; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nb && ok; ++j) {
      const uint32_t ph = static_cast<uint32_t>(j) & 1u;
      if (!mbar_wait(s_full, ph, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = j * BKV;
      // keys visible to this row: k <= q and k < seq
      const int kmax = min(q, p.seq - 1) - k0;  // last visible column in this block
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < BKV / 32; ++c) {
        float s[32];
        tmem_ld32(tS + lane_off + c * 32, s);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c * 32 + i <= kmax) mx = fmaxf(mx, s[i] * p.scale_log2);
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m - m_new);
      const float msub = (m_new == -INFINITY) ? 0.f : m_new;
      float rs = 0.f;
#pragma unroll 1
      for (int c = 0; c < BKV / 32; ++c) {
        float s[32];
        tmem_ld32(tS + lane_off + c * 32, s);
        tc_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float a = (c * 32 + i <= kmax) ? exp2f(s[i] * p.scale_log2 - msub) : 0.f;
          const float bb = (c * 32 + i + 1 <= kmax) ? exp2f(s[i + 1] * p.scale_log2 - msub) : 0.f;
          const uint32_t u = pack_bf16x2(a, bb);
          pk[i / 2] = u;
          // the row sum uses the rounded probabilities the PV product sees
          const float2 f = unpack_bf16x2(u);
          rs += f.x + f.y;
        }
        // 4 16-byte vectors: keys c*32 .. c*32+31 -> chunk (c/2), vectors (c%2)*4 .. +3
        uint8_t* rowp = sP + (c / 2) * CHUNK_BYTES + r * 128;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int qv = (c % 2) * 4 + v;
          *reinterpret_cast<uint4*>(rowp + ((qv ^ (r & 7)) << 4)) =
              make_uint4(pk[v * 4 + 0], pk[v * 4 + 1], pk[v * 4 + 2], pk[v * 4 + 3]);
        }
      }
      l = l * alpha + rs;
      m = m_new;
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      // O_j = P_j V_j is ready: O <- alpha * O + O_j
      if (!mbar_wait(o_full, ph, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32(tO + lane_off + c * 32, ov);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c * 32 + i] = o[c * 32 + i] * alpha + ov[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
    }
    if (ok && q < p.seq) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.O[shard]) +
                           (static_cast<int64_t>(q) * p.batch + b) * hl_d + hh * D;
#pragma unroll
      for (int v = 0; v < D / 8; ++v)
        *reinterpret_cast<uint4*>(dst + v * 8) = make_uint4(
            pack_bf16x2(o[v * 8 + 0] * inv, o[v * 8 + 1] * inv),
            pack_bf16x2(o[v * 8 + 2] * inv, o[v * 8 + 3] * inv),
            pack_bf16x2(o[v * 8 + 4] * inv, o[v * 8 + 5] * inv),
            pack_bf16x2(o[v * 8 + 6] * inv, o[v * 8 + 7] * inv));
      if (p.lse[shard])
        p.lse[shard][(static_cast<int64_t>(b) * p.heads_local + hh) * p.seq + q] =
            (m + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
tp_status launch_fwd_d(AttnParams& prm, cudaStream_t st) {
  static bool attr = false;
  const int smem = AttnSmem<D>::TOTAL;
  if (!attr) {
    tp_status s = tpi::cuda_status(
        cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
        "cudaFuncSetAttribute(attention)");
    if (s != TP_OK) return s;
    attr = true;
  }
  const int grid = prm.n_qtiles * prm.p * prm.batch * prm.heads_local;
  attn_fwd_kernel<D><<<grid, kThreads, smem, st>>>(prm);
  return tpi::after_launch("attention_fwd (tcgen05)");
}

}  // namespace

namespace tpi {

tp_status launch_attention_fwd(const tp_plan* plan, int batch, int seq, const PtrArray& qkv,
                               const MutPtrArray& o, float* const* lse, cudaStream_t st) {
  const int p = plan->p, d = plan->head_dim, hl = plan->heads / plan->p;
  const int64_t C = 3LL * hl * d;
  tp_status s = TP_OK;
  static AttnParams prm;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&prm, 0, sizeof(prm));
  for (int i = 0; i < p; ++i) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(batch),
                          static_cast<cuuint64_t>(seq)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(C) * 2 * batch};
    cuuint32_t box[3] = {64, 1, 128};
    s = encode_bf16(&prm.tm[i], qkv.p[i], 3, dims, strides, box, "QKV");
    if (s != TP_OK) return s;
    prm.O[i] = o.p[i];
    prm.lse[i] = lse ? lse[i] : nullptr;
  }
  prm.p = p;
  prm.batch = batch;
  prm.seq = seq;
  prm.heads_local = hl;
  prm.d = d;
  prm.n_qtiles = (seq + BQ - 1) / BQ;
  prm.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  s = device_status_word(&prm.status);
  if (s != TP_OK) return s;
  if (static_cast<int64_t>(prm.n_qtiles) * p * batch * hl > 0x7fffffffLL)
    return fail(TP_ERR_UNSUPPORTED, "attention grid too large");
  if (d == 64) return launch_fwd_d<64>(prm, st);
  if (d == 128) return launch_fwd_d<128>(prm, st);
  return fail(TP_ERR_UNSUPPORTED, "head_dim %d", d);
}

}  // namespace tpi
