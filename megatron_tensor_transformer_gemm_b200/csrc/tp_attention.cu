// Causal attention on each shard's local heads, forward, on the sm_100a
// tensor cores (TP walkthrough 2kiu.com §3.1: every shard runs full-sequence
// attention on its own whole heads, with no cross-shard step).
//
// One CTA computes two adjacent 128-query tiles (A = 2i, B = 2i + 1) of one
// (shard, batch, head); both read every K/V block once from shared memory:
//   warp 8      TMA producer: both Q tiles, then K_0, V_0, K_1, V_1, ... into a
//               ring of K/V buffers (five with P in TMEM, three with P in shared
//               memory; item n waits only for item n - slots to be released, so
//               V_j lands while block j - 1 is still in flight) from a 3-D
//               tensor map over the sequence-major [seq, batch, 3*heads_local*d]
//               QKV of the shard
//   warp 9      TMEM allocator + MMA issuer, ping-pong order: S_A(0), S_B(0),
//               then per block PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so one
//               tile's MMAs run while the other tile's softmax works
//   warps 0..3  softmax of tile A, warps 4..7 of tile B: thread r owns query
//               row r; its 128 scores of a block come from TMEM in one read
//               (row max, then exp2 and the row sum), P rounded to bf16 and written back
//               into the first 64 columns of the tile's S in TMEM (two keys per column),
//               where the PV MMA reads it as its A operand, so P takes no shared-memory
//               bandwidth from the MMAs' Q, K and V operands (PT = false, selected with
//               TP_ATTN_P_SMEM=1, keeps the earlier form: P in shared memory,
//               128-byte-swizzled K-major). Only the diagonal block (and a ragged last
//               block) is masked.
// O accumulates in TMEM across key blocks. P is taken relative to a reference
// max m that is raised (and O, l rescaled in place) only when a row's max
// exceeds it by more than 2^8; P <= 2^8 stays exact in fp32/bf16 range and the
// final O / l is independent of the reference, so this is exact, not an
// approximation. Blocks are causal: the diagonal block of each tile is masked
// (key > query -> probability 0); keys and queries past seq are masked.
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

constexpr int BQ = 128;   // queries per tile
constexpr int BKV = 128;  // keys per block
// Warps 0-3 softmax of tile A, 4-7 of tile B (warp w reads TMEM lanes
// 32 (w % 4) ..), warp 8 TMA producer, warp 9 TMEM owner and MMA issuer.
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int CHUNK_BYTES = 128 * 128;  // 128 rows x 64 bf16 (one swizzle-atom column)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;  // raise the reference max when exceeded by > 2^8

struct AttnParams {
  CUtensorMap tm[TP_MAX_SHARDS];  // QKV_i as {3*Hl*d, batch, seq}, box {64, 1, 128}
  void* O[TP_MAX_SHARDS];
  float* lse[TP_MAX_SHARDS];
  int p, batch, seq, heads_local, d;
  int n_qtiles, n_pairs;
  float scale_log2;  // log2(e) / sqrt(d)
  unsigned* status;
};

template <int D, bool PT>
struct AttnSmem {
  static constexpr int Q_BYTES = BQ * D * 2;
  static constexpr int KV_BYTES = BKV * D * 2;
  static constexpr int P_BYTES = PT ? 0 : BQ * BKV * 2;
  static constexpr int KV_SLOTS = PT ? 5 : 3;  // the shared memory P no longer takes
  static constexpr int TOTAL = 1024 + 2 * Q_BYTES + KV_SLOTS * KV_BYTES + 2 * P_BYTES + 256;
  static_assert(TOTAL <= 232448, "attention forward shared memory");
  static_assert((1 + 2 * KV_SLOTS + 7) * 8 + 8 <= 256, "barrier area");
};

// tcgen05.st of 16 raw 32-bit words per lane (two bf16 packed per column).
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// D[tmem] (+)= A[tmem] . B[smem desc]^T, kind::f16, with A read from tensor
// memory: row m of A in lane m, its K elements two per 32-bit column (element
// 2c in the low half of column c), so a K = 16 step spans 8 columns.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}


template <int D, bool PT>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  tpd::pdl_entry();
  using SM = AttnSmem<D, PT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sQ = smem;                     // [2] tiles
  uint8_t* sKV = sQ + 2 * SM::Q_BYTES;    // [KV_SLOTS] K or V blocks
  uint8_t* sP = sKV + SM::KV_SLOTS * SM::KV_BYTES;  // [2] tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * SM::P_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;                  // [KV_SLOTS]
  uint64_t* kv_empty = kv_full + SM::KV_SLOTS;   // [KV_SLOTS]
  uint64_t* s_full = kv_empty + SM::KV_SLOTS;    // [2]
  uint64_t* p_full = s_full + 2;                 // [2]
  uint64_t* o_done = p_full + 2;                 // [2]
  uint64_t* drain = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work decode: heaviest (last) tile pairs first.
  const int per = p.p * p.batch * p.heads_local;
  const int pair = p.n_pairs - 1 - static_cast<int>(blockIdx.x) / per;
  int rest = static_cast<int>(blockIdx.x) % per;
  const int hh = rest % p.heads_local;
  rest /= p.heads_local;
  const int b = rest % p.batch;
  const int shard = rest / p.batch;
  const int n_kv_total = (p.seq + BKV - 1) / BKV;
  int nbt[2];
  int q0t[2];
  for (int t = 0; t < 2; ++t) {
    const int qt = 2 * pair + t;
    q0t[t] = qt * BQ;
    nbt[t] = qt < p.n_qtiles ? min(qt + 1, n_kv_total) : 0;  // causal: key blocks 0..qt
  }
  const int nb = max(nbt[0], nbt[1]);
  const int hl_d = p.heads_local * D;
  const CUtensorMap* tm = &p.tm[shard];

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int k = 0; k < SM::KV_SLOTS; ++k) {
      mbar_init(&kv_full[k], 1);
      mbar_init(&kv_empty[k], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // S of tile t in columns [128 t, 128 t + 128) (PT: its P in the first 64 of them, written
  // after S is read; the MMAs issue PV(j) before S(j + 1), and tcgen05.mma executes in issue
  // order, so S(j + 1) overwrites P(j) only after PV(j) has read it); O of tile t in
  // [256 + D t, 256 + D (t + 1)).

  if (warp == kProducerWarp && lane == 0) {
    // ------------------------------------------------------------- producer
    tma_prefetch_desc(tm);
    mbar_arrive_expect_tx(q_full, (nbt[1] > 0 ? 2 : 1) * SM::Q_BYTES);
    for (int t = 0; t < 2; ++t) {
      if (nbt[t] == 0) continue;
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sQ + t * SM::Q_BYTES + c * CHUNK_BYTES, tm, q_full, hh * D + c * 64, b, q0t[t]);
    }
    // Ring items: 2j = K_j, 2j + 1 = V_j, in slot n % KV_SLOTS.
    const int n_items = 2 * nb;
    int issued = 0;
    for (int n = 0; n < n_items; ++n) {
      const int slot = n % SM::KV_SLOTS, use = n / SM::KV_SLOTS;
      if (use > 0 && !mbar_wait(&kv_empty[slot], static_cast<uint32_t>(use - 1) & 1u, abort_flag,
                                p.status))
        break;
      mbar_arrive_expect_tx(&kv_full[slot], SM::KV_BYTES);
      const int col0 = ((n & 1) ? 2 * hl_d : hl_d) + hh * D;
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sKV + slot * SM::KV_BYTES + c * CHUNK_BYTES, tm, &kv_full[slot], col0 + c * 64, b,
                    (n >> 1) * BKV);
      issued = n + 1;
    }
    // Drain: every copy issued has landed before the CTA exits.
    mbar_wait(q_full, 0, abort_flag, p.status);
    for (int k = 0; k < SM::KV_SLOTS; ++k) {
      const int uses = issued > k ? (issued - 1 - k) / SM::KV_SLOTS + 1 : 0;
      if (uses > 0) mbar_wait(&kv_full[k], static_cast<uint32_t>(uses - 1) & 1u, abort_flag, p.status);
    }
  } else if (warp == kMmaWarp && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc_s = idesc_bf16(BQ, BKV, false, false);
    const uint32_t idesc_o = idesc_bf16(BQ, D, false, true);
    auto slot_of = [](int n) { return n % SM::KV_SLOTS; };
    auto full_parity = [](int n) { return static_cast<uint32_t>(n / SM::KV_SLOTS) & 1u; };
    auto issue_s = [&](int t, int j) {
      const uint32_t q_base = smem_u32(sQ + t * SM::Q_BYTES);
      const uint32_t k_base = smem_u32(sKV + slot_of(2 * j) * SM::KV_BYTES);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * CHUNK_BYTES + (kk % 4) * 32;
        tc_mma_bf16(tmem + 128 * t, smem_desc_sw128(q_base + off, 16, 1024),
                    smem_desc_sw128(k_base + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
      }
      tc_commit(&s_full[t]);
    };
    auto issue_pv = [&](int t, int j) {
      const bool first = j == 0;
      const uint32_t p_base = smem_u32(sP + t * SM::P_BYTES);
      const uint32_t v_base = smem_u32(sKV + slot_of(2 * j + 1) * SM::KV_BYTES);
#pragma unroll
      for (int kk = 0; kk < BKV / 16; ++kk) {
        const uint64_t bdesc = smem_desc_sw128(v_base + kk * 2048, CHUNK_BYTES, 1024);
        if (PT) {  // A = P from TMEM: keys 16 kk .. 16 kk + 15 in columns 8 kk .. 8 kk + 7
          tc_mma_bf16_ts(tmem + 256 + D * t, tmem + 128 * t + 8 * kk, bdesc, idesc_o,
                         (first && kk == 0) ? 0u : 1u);
        } else {
          const uint64_t adesc = smem_desc_sw128(p_base + (kk / 4) * CHUNK_BYTES + (kk % 4) * 32, 16, 1024);
          tc_mma_bf16(tmem + 256 + D * t, adesc, bdesc, idesc_o, (first && kk == 0) ? 0u : 1u);
        }
      }
      tc_commit(&o_done[t]);
    };
    bool ok = mbar_wait(q_full, 0, abort_flag, p.status) &&
              mbar_wait(&kv_full[slot_of(0)], full_parity(0), abort_flag, p.status);
    if (ok) {
      tc_fence_after();
      for (int t = 0; t < 2; ++t)
        if (nbt[t] > 0) issue_s(t, 0);
      tc_commit(&kv_empty[slot_of(0)]);  // K_0 free once both S MMAs finish
    }
    for (int j = 0; ok && j < nb; ++j) {
      if (!mbar_wait(&kv_full[slot_of(2 * j + 1)], full_parity(2 * j + 1), abort_flag, p.status)) break;
      tc_fence_after();
      bool have_k_next = false;
      for (int t = 0; t < 2 && ok; ++t) {
        if (j >= nbt[t]) continue;
        if (!mbar_wait(&p_full[t], static_cast<uint32_t>(j) & 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(t, j);
        if (j + 1 < nbt[t]) {
          if (!have_k_next) {
            if (!mbar_wait(&kv_full[slot_of(2 * j + 2)], full_parity(2 * j + 2), abort_flag,
                           p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            have_k_next = true;
          }
          issue_s(t, j + 1);
        }
      }
      if (!ok) break;
      tc_commit(&kv_empty[slot_of(2 * j + 1)]);                 // V_j free after both P.V MMAs
      if (have_k_next) tc_commit(&kv_empty[slot_of(2 * j + 2)]);  // K_{j+1} after both S MMAs
    }
    tc_commit(drain);
    mbar_wait(drain, 0, abort_flag, p.status);
  } else if (warp < 8) {
    // ------------------------------------------------------------- softmax
    const int t = warp / 4;  // query tile of this warpgroup
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    // this tile's first query and key-block count as scalars (an index by t
    // into the two-entry arrays would place them in local memory)
    const int my_q0 = t ? q0t[1] : q0t[0];
    const int my_nb = t ? nbt[1] : nbt[0];
    const int q = my_q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    const uint32_t tS = tmem + 128 * t + lane_off;
    const uint32_t tO = tmem + 256 + D * t + lane_off;
    uint8_t* sPt = sP + t * SM::P_BYTES;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < my_nb && ok; ++j) {
      // The whole warp proceeds together (tcgen05.ld below is warp-collective).
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], static_cast<uint32_t>(j) & 1u, abort_flag,
                                              p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = j * BKV;
      const int kmax = min(q, p.seq - 1) - k0;  // last visible column of this block
      // No column of this block is masked for any row of the warp (every block
      // but the diagonal one and a ragged last one): skip the per-column tests.
      const bool full = k0 + BKV - 1 <= min(my_q0 + lg * 32, p.seq - 1);
      // The whole 128-column row of S into registers with one wait; both
      // passes below work from there.
      float sv[BKV / 32][32];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c) tmem_ld32(tS + c * 32, sv[c]);
      tc_wait_ld();
      float mx = -INFINITY;
      if (full) {
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 2) mx = max3(mx, sv[c][i], sv[c][i + 1]);
      } else {
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i <= kmax) mx = fmaxf(mx, sv[c][i]);
      }
      mx *= p.scale_log2;  // the scale is positive: max of the scaled scores
      if (j > 0) {
        // P.V of the previous block done: the P buffer is free and O is stable.
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done[t], static_cast<uint32_t>(j - 1) & 1u,
                                                abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // Raise the reference max only when some row of the warp outgrew it by
      // more than 2^kRescale (warp-uniform: the O rescale below is a
      // warp-collective TMEM access); rows whose max did not move get alpha 1.
      float alpha = 1.f;
      const bool rescale = j > 0 && __any_sync(0xffffffffu, mx > m + kRescale);
      if (j == 0) {
        m = mx;
      } else if (rescale) {
        const float m_new = fmaxf(m, mx);
        alpha = exp2f(m - m_new);
        m = m_new;
      }
      float rs = 0.f;
      const float sc = p.scale_log2;
#pragma unroll
      for (int cc = 0; cc < BKV / 32; ++cc) {  // 32 keys -> 16 packed words
        uint32_t pw[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 x = fma2_bcast(sv[cc][i], sv[cc][i + 1], sc, -m);  // scaled score - m
          float a = ex2(x.x);
          float bb = ex2(x.y);
          if (!full) {
            a = (cc * 32 + i <= kmax) ? a : 0.f;
            bb = (cc * 32 + i + 1 <= kmax) ? bb : 0.f;
          }
          const uint32_t w = pack_bf16x2(a, bb);
          pw[i / 2] = w;
          // the row sum uses the rounded P of the PV MMA (bf16 widening is exact)
          const float2 f = unpack_bf16x2(w);
          rs += f.x + f.y;
        }
        if (PT) {
          tmem_st16u(tS + 16 * cc, pw);
        } else {
          uint8_t* rowp = sPt + (cc / 2) * CHUNK_BYTES + r * 128;
#pragma unroll
          for (int v = 0; v < 4; ++v) {  // 8 keys -> one 16-byte store of P
            const int qv = (cc % 2) * 4 + v;
            *reinterpret_cast<uint4*>(rowp + ((qv ^ (r & 7)) << 4)) =
                make_uint4(pw[4 * v], pw[4 * v + 1], pw[4 * v + 2], pw[4 * v + 3]);
          }
        }
      }
      if (PT) tc_wait_st();  // P is in TMEM before the MMA warp is told
      if (rescale) {
        // O of the previous blocks (stable: their P.V is done) to the new reference.
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tmem_ld32(tO + c * 32, ov);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tO + c * 32, ov);
        }
        tc_wait_st();
      }
      l = l * alpha + rs;
      if (!PT) fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok && my_nb > 0 &&
        __all_sync(0xffffffffu, mbar_wait(&o_done[t], static_cast<uint32_t>(my_nb - 1) & 1u,
                                          abort_flag, p.status))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.O[shard]) +
                           (static_cast<int64_t>(q) * p.batch + b) * hl_d + hh * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32(tO + c * 32, ov);
        tc_wait_ld();
        if (q < p.seq) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(dst + c * 32 + v * 8) = make_uint4(
                pack_bf16x2(ov[v * 8 + 0] * inv, ov[v * 8 + 1] * inv),
                pack_bf16x2(ov[v * 8 + 2] * inv, ov[v * 8 + 3] * inv),
                pack_bf16x2(ov[v * 8 + 4] * inv, ov[v * 8 + 5] * inv),
                pack_bf16x2(ov[v * 8 + 6] * inv, ov[v * 8 + 7] * inv));
        }
      }
      if (q < p.seq && p.lse[shard])
        p.lse[shard][(static_cast<int64_t>(b) * p.heads_local + hh) * p.seq + q] =
            (m + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool PT>
tp_status launch_fwd_d(AttnParams& prm, cudaStream_t st) {
  static bool attr = false;
  const int smem = AttnSmem<D, PT>::TOTAL;
  if (!attr) {
    tp_status s = tpi::cuda_status(
        cudaFuncSetAttribute(attn_fwd_kernel<D, PT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
        "cudaFuncSetAttribute(attention)");
    if (s != TP_OK) return s;
    attr = true;
  }
  const int grid = prm.n_pairs * prm.p * prm.batch * prm.heads_local;
  (void)tpi::launch(attn_fwd_kernel<D, PT>, dim3(grid), dim3(kThreads), smem, st, prm);
  return tpi::after_launch("attention_fwd (tcgen05)");
}

// P in TMEM (default) or, with TP_ATTN_P_SMEM=1, in shared memory.
bool p_in_tmem() {
  static const bool on = [] {
    const char* e = getenv("TP_ATTN_P_SMEM");
    return !(e && e[0] == '1');
  }();
  return on;
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
  prm.n_pairs = (prm.n_qtiles + 1) / 2;
  prm.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  s = device_status_word(&prm.status);
  if (s != TP_OK) return s;
  if (static_cast<int64_t>(prm.n_pairs) * p * batch * hl > 0x7fffffffLL)
    return fail(TP_ERR_UNSUPPORTED, "attention grid too large");
  if (d == 64) return p_in_tmem() ? launch_fwd_d<64, true>(prm, st) : launch_fwd_d<64, false>(prm, st);
  if (d == 128) return p_in_tmem() ? launch_fwd_d<128, true>(prm, st) : launch_fwd_d<128, false>(prm, st);
  return fail(TP_ERR_UNSUPPORTED, "head_dim %d", d);
}

}  // namespace tpi
