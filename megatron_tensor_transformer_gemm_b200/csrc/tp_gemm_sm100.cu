// Grouped, persistent bf16 GEMM on the sm_100a 5th-generation tensor cores.
//
// One launch computes every shard's GEMM of a column- or row-parallel layer
// (the p shards are separate buffers on this GPU): D_g = A_g . B_g^T for
// g < p, with a fused epilogue:
//   EPI_STORE      D = acc (+ column bias)              QKV, row partials, grads
//   EPI_BIAS_GELU  Z = acc + bias, H = GELU(Z)           column layer, GELU MLP
//   EPI_SWIGLU     Z = [g|u], H = SiLU(g) * u            column layer, SwiGLU MLP
//   EPI_DGELU      dZ = acc * GELU'(Z)                   row layer backward
//   EPI_DSWIGLU    dZ = [acc*u*SiLU'(g) | acc*SiLU(g)]   row layer backward
// (TP walkthrough 2kiu.com §2.1-§2.2 and §3.2; 张量并行 wiki, 两种切法.)
//
// Tile layouts: a CTA pair (cta_group::2) on a 256 x 256 tile by default; for
// problems whose 256 x 256 tiles would leave SMs idle, the host may instead
// run 128-column tiles, one CTA per 128-row tile, or both (choose_layout).
//
// Design (per CTA, one CTA per SM, persistent; tiles drawn in order from an
// atomic counter, see the tile ring below):
//   warp 0      TMA producer: 128B-swizzled A and B tiles into a 4-stage ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..9  epilogue: tcgen05.ld TMEM -> registers -> fused math -> HBM;
//               two warps per TMEM lane quarter, each taking half of the columns
// The 128x256 fp32 accumulator lives in TMEM (256 columns); two accumulators
// (all 512 columns) let the epilogue of one tile overlap the MMAs of the next.
// Operands may be K-major or MN-major (the backward GEMMs read dY^T, X^T and
// W without transposes); SwiGLU stacks 128 gate rows and the 128 matching up
// rows into one 256-wide B tile, so one accumulator holds both halves.
// Every mbarrier wait is bounded (tp_device.cuh); on a time-out the CTA drains
// its in-flight copies and MMAs, frees TMEM and returns with the status set.
#include <cuda.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"
#include "tp_tma.h"

namespace {

using namespace tpd;
using tpi::GemmBatch;
using tpi::GemmProblem;

constexpr int BM = 128;  // accumulator rows per CTA
constexpr int BN = 256;
constexpr int BK = 64;  // one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int TMEM_COLS = 512;
constexpr int kBarBytes = 512;  // barriers, TMEM slot, abort flag, tile ring
constexpr int MN_BLOCK_BYTES = 64 * BK * 2;  // one 64-wide MN block of an MN-major tile
// TMA epilogue staging: per epilogue warp two [32 rows x 32 bf16] tiles.
constexpr int kEpiTile = 32 * 64;
constexpr int kEpiBuf = 2 * kEpiTile;
constexpr int kEpiBytes = kEpiWarps * kEpiBuf;

// Per-CTA tile geometry. PAIR = 1: one CTA computes a 128 x 256 tile.
// PAIR = 2: a (2,1,1) cluster computes a 256 x 256 tile with cta_group::2
// MMAs; each CTA loads its 128 rows of A and its 128 rows of B.
template <int PAIR>
struct Cfg {
  static constexpr int TILE_M = BM * PAIR;
  static constexpr int B_ROWS = BN / PAIR;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = PAIR == 1 ? 4 : 6;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + kEpiBytes + kBarBytes;
  static_assert(SMEM_BYTES <= 232448, "shared memory of the GEMM kernel");
};

struct GroupArgs {
  int M, N, K;
  int tiles_n;
  int tile_begin;
  int num_kb;
  int nh;
  int pad;
  void* D;
  int64_t ldd;
  void* D2;
  int64_t ldd2;
  const void* bias;
  const void* aux;
  int64_t ldaux;
};

struct alignas(64) GemmParams {
  CUtensorMap tmA[TP_MAX_SHARDS];
  CUtensorMap tmB[TP_MAX_SHARDS];
  GroupArgs g[TP_MAX_SHARDS];
  int ngroups;
  int total_tiles;
  int tile_n;      // output columns per tile: BN, or BN / 2 (SwiGLU pairs; narrow launches)
  int narrow_all;  // every tile runs as an N = BN / 2 MMA (small problems: twice the tiles)
  int a_mn;
  int b_mn;
  int epi;
  int out_f32;
  // K-concatenated mode (kcat > 0): one output problem (g[0]) whose K loop runs
  // over kcat segments, segment s reading tmA[s] / tmB[s] for seg_kb[s] blocks:
  // D = sum_s A_s B_s^T, i.e. the sum over shards happens in the accumulator.
  int kcat;
  int seg_kb[TP_MAX_SHARDS];
  // Row scatter (scatter > 0): output row r goes to out_seq[r / rows_per_out]
  // at row r % rows_per_out, with residual rows from res_seq (if non-NULL).
  int scatter;
  int rows_per_out;
  void* out_seq[TP_MAX_SHARDS];
  const void* res_seq[TP_MAX_SHARDS];
  // Split K (ksplit > 1, EPI_STORE with fp32 outputs): every output tile runs
  // ksplit times, split s over K blocks [s * kb_per_split, ...) writing its
  // fp32 partial at D + s * split_stride; a reduce kernel sums the splits.
  int ksplit;
  int base_tiles;
  int kb_per_split;
  int64_t split_stride;
  // Dynamic tile schedule: {draws, pairs done drawing}, zero at launch. Pair c
  // (or CTA c) starts on tile c; its leader then draws tile clusters + n with
  // n = atomicAdd(draws, 1) until one comes back past the end, and the last
  // pair to get there sets both words back to zero.
  unsigned* sched;
  int dyn_sched;  // 1: draw tiles from *sched; 0: cluster c takes c, c + clusters, ...
  // TMA epilogue (tma_epi = 1; bf16 outputs, no scatter, no split K): per
  // output problem, tmE views D and tmX the staged input (Z of the dGELU /
  // dSwiGLU epilogues, or the residual) as {columns, halves, rows} with a
  // {32, 1, 32} box and 64-byte swizzle; halves = 2 splits [gate | up] at nh.
  // With the row scatter, tmE[j] / tmX[j] view sequence shard j's output /
  // residual ({N, 1, rows_per_out}) and scatter_res says whether residuals come.
  int tma_epi;
  int scatter_res;
  // Plain stores through the stage (plain_staged = 1): outputs that may be
  // another GPU's memory, EPI_STORE, bf16, no bias, residual or split.
  int plain_staged;
  CUtensorMap tmE[TP_MAX_SHARDS];
  CUtensorMap tmX[TP_MAX_SHARDS];
  unsigned* status;
};
static_assert(sizeof(GemmParams) <= 32764, "kernel parameter space");

__device__ __forceinline__ void decode_tile(const GemmParams& p, int t, int& g, int& mt, int& nt,
                                            int& ks) {
  ks = 0;
  if (p.ksplit > 1) {
    ks = t / p.base_tiles;
    t -= ks * p.base_tiles;
  }
  g = 0;
#pragma unroll 1
  for (int i = 1; i < p.ngroups; ++i)
    if (t >= p.g[i].tile_begin) g = i;
  const int local = t - p.g[g].tile_begin;
  mt = local / p.g[g].tiles_n;
  nt = local - mt * p.g[g].tiles_n;
}

// K blocks of a tile: [kb0, kb0 + nkb) of its problem (the split's share
// under split K, else all of them).
__device__ __forceinline__ void kb_range(const GemmParams& p, const GroupArgs& ga, int ks, int& kb0,
                                         int& nkb) {
  if (p.ksplit > 1) {
    kb0 = ks * p.kb_per_split;
    nkb = min(p.kb_per_split, ga.num_kb - kb0);
  } else {
    kb0 = 0;
    nkb = ga.num_kb;
  }
}

// A tile with at most BN / 2 valid columns left (the ragged last N tile of a
// problem, e.g. N = 1376 = 5 x 256 + 96) runs narrow: an N = BN / 2 MMA over
// the first BN / 2 rows of B, so the tensor cores skip the empty half. In a
// CTA pair each CTA then supplies BN / 4 rows of B (its half of the narrow N).
// SwiGLU tiles (gate and up halves of one B tile) never run narrow.
__device__ __forceinline__ bool narrow_tile(const GemmParams& p, const GroupArgs& ga, int n0) {
  return p.epi != tpi::EPI_SWIGLU && (p.narrow_all || ga.N - n0 <= BN / 2);
}

// ------------------------------------------------------------- epilogue math
__device__ __forceinline__ void store_row_chunk_bf16(void* base, int64_t ld, int row, int col0,
                                                     int N, const float (&v)[32]) {
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(base) + static_cast<int64_t>(row) * ld + col0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (col0 + q * 8 < N) {
      uint4 u = make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]),
                           pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                           pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]),
                           pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]));
      *reinterpret_cast<uint4*>(dst + q * 8) = u;
    }
  }
}

__device__ __forceinline__ void store_row_chunk_f32(void* base, int64_t ld, int row, int col0,
                                                    int N, const float (&v)[32]) {
  float* dst = static_cast<float*>(base) + static_cast<int64_t>(row) * ld + col0;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (col0 + q * 4 < N)
      *reinterpret_cast<float4*>(dst + q * 4) =
          make_float4(v[q * 4 + 0], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
}

__device__ __forceinline__ void load_row_chunk_bf16(const void* base, int64_t ld, int row,
                                                    int col0, int N, float (&v)[32]) {
  const __nv_bfloat16* src =
      static_cast<const __nv_bfloat16*>(base) + static_cast<int64_t>(row) * ld + col0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u = make_uint4(0, 0, 0, 0);
    if (col0 + q * 8 < N) u = *reinterpret_cast<const uint4*>(src + q * 8);
    float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y), c = unpack_bf16x2(u.z),
           d = unpack_bf16x2(u.w);
    v[q * 8 + 0] = a.x; v[q * 8 + 1] = a.y; v[q * 8 + 2] = b.x; v[q * 8 + 3] = b.y;
    v[q * 8 + 4] = c.x; v[q * 8 + 5] = c.y; v[q * 8 + 6] = d.x; v[q * 8 + 7] = d.y;
  }
}

// Columns [half * BN/2, (half + 1) * BN/2) of the accumulator row this thread owns.
__device__ void epilogue_tile(const GemmParams& p, const GroupArgs& ga, uint32_t taddr, int row,
                              int n0, int half, bool narrow, int ks) {
  const bool row_ok = row < ga.M;
  if (p.epi == tpi::EPI_SWIGLU) {
    // Accumulator columns [0,128) = gate units n0.., [128,256) = the same up units;
    // this thread handles gate/up pairs [half * 64, half * 64 + 64).
#pragma unroll 1
    for (int c = half * 2; c < half * 2 + 2; ++c) {
      float g[32], u[32];
      tmem_ld32(taddr + c * 32, g);
      tmem_ld32(taddr + 128 + c * 32, u);
      tc_wait_ld();
      const int j0 = n0 + c * 32;
      if (row_ok && j0 < ga.N) {
        if (ga.D) {
          store_row_chunk_bf16(ga.D, ga.ldd, row, j0, ga.N, g);
          store_row_chunk_bf16(static_cast<__nv_bfloat16*>(ga.D) + ga.nh, ga.ldd, row, j0, ga.N, u);
        }
        float h[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) h[i] = g[i] * sigmoid_fast(g[i]) * u[i];
        store_row_chunk_bf16(ga.D2, ga.ldd2, row, j0, ga.N, h);
      }
    }
    return;
  }
  const int cpw = narrow ? BN / 128 : BN / 64;  // 32-column chunks per warp half
#pragma unroll 1
  for (int c = half * cpw; c < (half + 1) * cpw; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    tc_wait_ld();
    const int j0 = n0 + c * 32;
    if (!row_ok || j0 >= ga.N) continue;
    switch (p.epi) {
      case tpi::EPI_STORE: {
        if (ga.bias) {
          float b[32];
          load_row_chunk_bf16(ga.bias, 0, 0, j0, ga.N, b);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += b[i];
        }
        void* dst = ga.D;
        if (ks) dst = static_cast<float*>(dst) + ks * p.split_stride;  // split K: fp32 partials
        const void* res = ga.aux;
        int orow = row;
        if (p.scatter) {
          const int j = row / p.rows_per_out;
          orow = row - j * p.rows_per_out;
          dst = p.out_seq[j];
          res = p.res_seq[j];
        }
        if (res) {
          float r[32];
          load_row_chunk_bf16(res, ga.ldaux, orow, j0, ga.N, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += r[i];
        }
        if (p.out_f32) store_row_chunk_f32(dst, ga.ldd, orow, j0, ga.N, v);
        else store_row_chunk_bf16(dst, ga.ldd, orow, j0, ga.N, v);
        break;
      }
      case tpi::EPI_BIAS_GELU: {
        if (ga.bias) {
          float b[32];
          load_row_chunk_bf16(ga.bias, 0, 0, j0, ga.N, b);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += b[i];
        }
        if (ga.D) store_row_chunk_bf16(ga.D, ga.ldd, row, j0, ga.N, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = gelu_f(v[i]);
        store_row_chunk_bf16(ga.D2, ga.ldd2, row, j0, ga.N, v);
        break;
      }
      case tpi::EPI_DGELU: {
        float z[32];
        load_row_chunk_bf16(ga.aux, ga.ldaux, row, j0, ga.N, z);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= gelu_grad_f(z[i]);
        store_row_chunk_bf16(ga.D, ga.ldd, row, j0, ga.N, v);
        break;
      }
      case tpi::EPI_DSWIGLU: {
        float zg[32], zu[32], dg[32];
        load_row_chunk_bf16(ga.aux, ga.ldaux, row, j0, ga.N, zg);
        load_row_chunk_bf16(static_cast<const __nv_bfloat16*>(ga.aux) + ga.nh, ga.ldaux, row, j0,
                            ga.N, zu);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          // one sigmoid per element: SiLU(g) = g s, SiLU'(g) = s (1 + g (1 - s))
          const float sg = sigmoid_fast(zg[i]);
          dg[i] = v[i] * zu[i] * (sg * (1.0f + zg[i] * (1.0f - sg)));
          v[i] = v[i] * (zg[i] * sg);
        }
        store_row_chunk_bf16(ga.D, ga.ldd, row, j0, ga.N, dg);
        store_row_chunk_bf16(static_cast<__nv_bfloat16*>(ga.D) + ga.nh, ga.ldd, row, j0, ga.N, v);
        break;
      }
      default:
        break;
    }
  }
}

// ------------------------------------------------------ TMA epilogue
// Each epilogue warp stages its 32 rows x 32 columns of a chunk in its own two
// [32 x 64 B] tiles of shared memory, 64-byte swizzled: the 16-byte piece q of
// row r sits at r * 64 + ((q ^ ((r >> 1) & 3)) << 4), so a warp reading or
// writing one piece of each of its rows touches every bank once per 128 bytes.
// Inputs (the aux Z, or the residual) arrive by TMA load, outputs leave by TMA
// store (clipped at the tensor's edges), and a thread touches only its own
// row. Global memory sees whole 64-byte row segments instead of the 16-byte
// pieces of 32 rows that one vector store per row gives.
__device__ __forceinline__ uint32_t sw64(uint32_t tile, int r, int q) {
  return tile + static_cast<uint32_t>(r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
}
__device__ __forceinline__ void stage_read(uint32_t tile, int r, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = ld_shared_v4(sw64(tile, r, q));
    const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y), c = unpack_bf16x2(u.z),
                 d = unpack_bf16x2(u.w);
    v[q * 8 + 0] = a.x; v[q * 8 + 1] = a.y; v[q * 8 + 2] = b.x; v[q * 8 + 3] = b.y;
    v[q * 8 + 4] = c.x; v[q * 8 + 5] = c.y; v[q * 8 + 6] = d.x; v[q * 8 + 7] = d.y;
  }
}
__device__ __forceinline__ void stage_write(uint32_t tile, int r, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_shared_v4(sw64(tile, r, q), make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]),
                                              pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                                              pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]),
                                              pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7])));
}

// Plain-store epilogue through the stage (outputs that may be another GPU's
// memory take no TMA): each 32 x 32 chunk of the warp's rows is written to
// the stage by row, then read back four lanes to a row, so that one warp
// store writes eight whole 64-byte row segments instead of 16-byte pieces of
// 32 rows. EPI_STORE with bf16 outputs, no bias or residual, optionally
// scattered by row to out_seq (any rows_per_out).
__device__ void epilogue_plain_staged(const GemmParams& p, const GroupArgs& ga, uint32_t taddr, int row0,
                                      int n0, int half, bool narrow, int lane, uint32_t tile) {
  const int cpw = narrow ? BN / 128 : BN / 64;  // 32-column chunks per warp half
  const int q = lane & 3, rsub = lane >> 2;     // this lane's piece and row within each group of 8
#pragma unroll 1
  for (int c = half * cpw; c < (half + 1) * cpw; ++c) {
    const int j0 = n0 + c * 32;
    if (j0 >= ga.N) break;  // warp-uniform
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    tc_wait_ld();
    stage_write(tile, lane, v);
    __syncwarp();
    const int col = j0 + q * 8;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int r = it * 8 + rsub, row = row0 + r;
      const uint4 u = ld_shared_v4(sw64(tile, r, q));
      if (row < ga.M && col < ga.N) {
        __nv_bfloat16* base;
        if (p.scatter) {
          const int jb = row / p.rows_per_out;
          base = static_cast<__nv_bfloat16*>(p.out_seq[jb]) +
                 static_cast<int64_t>(row - jb * p.rows_per_out) * ga.ldd;
        } else {
          base = static_cast<__nv_bfloat16*>(ga.D) + static_cast<int64_t>(row) * ga.ldd;
        }
        *reinterpret_cast<uint4*>(base + col) = u;
      }
    }
    __syncwarp();  // every lane has read the stage before the next chunk rewrites it
  }
}

// Staged inputs per chunk: Z's gate and up halves (dSwiGLU), Z (dGELU), the
// residual (plain store with aux), or none.
__device__ __forceinline__ int epi_inputs(const GemmParams& p, const GroupArgs& ga) {
  if (p.epi == tpi::EPI_DSWIGLU) return 2;
  if (p.epi == tpi::EPI_DGELU) return 1;
  if (p.epi == tpi::EPI_STORE) return (p.scatter ? p.scatter_res : ga.aux != nullptr) ? 1 : 0;
  return 0;  // the forward activations stage outputs only
}

// Per-warp state of the TMA epilogue (lane 0 issues every copy).
struct EpiStage {
  uint8_t* buf;   // kEpiBuf bytes: tiles 0 and 1
  uint64_t* bar;  // completes the staged inputs of a chunk
  uint32_t phase;
  int slot;       // plain stores alternate between the two tiles
};

// Lane 0: load chunk j0's inputs into the stage (the tiles are free once this
// thread's earlier stores have read them).
__device__ __forceinline__ void epi_issue_inputs(const GemmParams& p, int gi, int nin, int j0, int row0,
                                                 EpiStage& es) {
  const bool plain = p.epi == tpi::EPI_STORE;
  uint8_t* t = es.buf + (plain ? es.slot * kEpiTile : 0);
  // plain stores alternate tiles: the store two chunks back must have read this one
  if (plain) bulk_wait_read<1>();
  else bulk_wait_read<0>();
  mbar_arrive_expect_tx(es.bar, static_cast<uint32_t>(nin * kEpiTile));
  tma_load_3d(t, &p.tmX[gi], es.bar, j0, 0, row0);
  if (nin == 2) tma_load_3d(t + kEpiTile, &p.tmX[gi], es.bar, j0, 1, row0);
}

// Forward activation epilogues through the stage (nothing staged in): SwiGLU
// stores Z = [g | u] (when requested, through tmE) and H = SiLU(g) u (tmX);
// bias + GELU stores Z (when requested, tmE) and H = GELU(Z) (tmX).
__device__ void epilogue_fwd_tma(const GemmParams& p, const GroupArgs& ga, int gi, uint32_t taddr, int row0,
                                 int n0, int half, bool narrow, int lane, EpiStage& es) {
  uint8_t* t = es.buf;
  const uint32_t t0 = smem_u32(t), t1 = t0 + kEpiTile;
  if (p.epi == tpi::EPI_SWIGLU) {
    // accumulator columns [0, 128) = gate units n0.., [128, 256) = the same up
    // units; this warp takes units [half * 64, half * 64 + 64)
#pragma unroll 1
    for (int c = half * 2; c < half * 2 + 2; ++c) {
      const int j0 = n0 + c * 32;
      if (j0 >= ga.N) break;  // warp-uniform
      float g[32], u[32];
      tmem_ld32(taddr + c * 32, g);
      tmem_ld32(taddr + 128 + c * 32, u);
      tc_wait_ld();
      if (lane == 0) bulk_wait_read<0>();  // the last chunk's stores have read both tiles
      __syncwarp();
      if (ga.D) {
        stage_write(t0, lane, g);
        stage_write(t1, lane, u);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&p.tmE[gi], t, j0, 0, row0);
          bulk_commit();
          tma_store_3d(&p.tmE[gi], t + kEpiTile, j0, 1, row0);
          bulk_commit();
          bulk_wait_read<1>();  // tile 0 has been read
        }
        __syncwarp();
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = g[i] * sigmoid_fast(g[i]) * u[i];
      stage_write(t0, lane, g);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(&p.tmX[gi], t, j0, 0, row0);
        bulk_commit();
      }
    }
    return;
  }
  // bias + GELU: Z to tile 0, H to tile 1
  const int cpw = narrow ? BN / 128 : BN / 64;
#pragma unroll 1
  for (int c = half * cpw; c < (half + 1) * cpw; ++c) {
    const int j0 = n0 + c * 32;
    if (j0 >= ga.N) break;  // warp-uniform
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    tc_wait_ld();
    if (ga.bias) {
      float bb[32];
      load_row_chunk_bf16(ga.bias, 0, 0, j0, ga.N, bb);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] += bb[i];
    }
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
    if (ga.D) stage_write(t0, lane, v);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gelu_f(v[i]);
    stage_write(t1, lane, v);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (ga.D) tma_store_3d(&p.tmE[gi], t, j0, 0, row0);
      tma_store_3d(&p.tmX[gi], t + kEpiTile, j0, 0, row0);
      bulk_commit();
    }
  }
}

// The tile's epilogue through the stage; `pre`: the first chunk's inputs are
// already in flight. Returns false if a bounded wait gave up.
__device__ bool epilogue_tile_tma(const GemmParams& p, const GroupArgs& ga, int gi, uint32_t taddr, int row0,
                                  int n0, int half, bool narrow, bool pre, int lane, EpiStage& es,
                                  volatile int* abort, unsigned* status) {
  const int cpw = narrow ? BN / 128 : BN / 64;  // 32-column chunks per warp half
  const int nin = epi_inputs(p, ga);
  const bool plain = p.epi == tpi::EPI_STORE;
  bool first = true;
#pragma unroll 1
  for (int c = half * cpw; c < (half + 1) * cpw; ++c) {
    const int j0 = n0 + c * 32;
    if (j0 >= ga.N) break;  // warp-uniform
    uint8_t* t = es.buf + (plain ? es.slot * kEpiTile : 0);
    if (lane == 0) {
      if (nin > 0) {
        if (!(first && pre)) epi_issue_inputs(p, gi, nin, j0, row0, es);
      } else {
        bulk_wait_read<1>();  // the store issued from this tile two chunks ago has read it
      }
    }
    __syncwarp();  // the tile is free before any lane writes it
    first = false;
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    tc_wait_ld();
    if (nin > 0) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(es.bar, es.phase, abort, status));
      es.phase ^= 1u;
      if (!ok) {
        if (lane == 0) {  // let the copies in flight land before the CTA may exit (bounded)
          volatile int none = 0;
          mbar_wait(es.bar, es.phase ^ 1u, &none, nullptr, 1000000ull);
        }
        return false;
      }
    }
    const uint32_t t0 = smem_u32(t), t1 = t0 + kEpiTile;
    switch (p.epi) {
      case tpi::EPI_DSWIGLU: {
        float zg[32], zu[32];
        stage_read(t0, lane, zg);
        stage_read(t1, lane, zu);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          // one sigmoid per element: SiLU(g) = g s, SiLU'(g) = s (1 + g (1 - s))
          const float sg = sigmoid_fast(zg[i]);
          const float dg = v[i] * zu[i] * (sg * (1.0f + zg[i] * (1.0f - sg)));
          zu[i] = v[i] * (zg[i] * sg);
          zg[i] = dg;
        }
        stage_write(t0, lane, zg);
        stage_write(t1, lane, zu);
        break;
      }
      case tpi::EPI_DGELU: {
        float z[32];
        stage_read(t0, lane, z);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= gelu_grad_f(z[i]);
        stage_write(t0, lane, v);
        break;
      }
      default: {  // plain store: + bias, + residual
        if (ga.bias) {
          float bb[32];
          load_row_chunk_bf16(ga.bias, 0, 0, j0, ga.N, bb);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += bb[i];
        }
        if (nin > 0) {
          float r[32];
          stage_read(t0, lane, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += r[i];
        }
        stage_write(t0, lane, v);
        break;
      }
    }
    fence_proxy_async_smem();  // this lane's writes are visible to the TMA store
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(&p.tmE[gi], t, j0, 0, row0);
      if (nin == 2) tma_store_3d(&p.tmE[gi], t + kEpiTile, j0, 1, row0);
      bulk_commit();
    }
    if (plain) es.slot ^= 1;
  }
  return true;
}

// ------------------------------------------------------------ tile ring
// The persistent CTAs take tiles in order from one atomic counter, so the
// tiles in flight at any moment are a window of consecutive indices (the
// operands they share stay in L2) and a CTA that drew narrow or short tiles
// simply takes more: no pair waits at the end for one whose static share
// held more work. The leader CTA's producer draws each tile and publishes it
// through a ring of kRing slots in both CTAs of the pair; every consumer (the
// MMA issuer, the epilogue warps, the peer's producer) reads each entry once
// and arrives on the leader's `empty` barrier of that slot. -1 ends the list.
constexpr int kRing = 8;
struct TileRing {
  volatile int* slot;
  uint64_t* full;
  uint64_t* empty;
};
// Consumers of each entry: per CTA of the pair, the MMA issuer (leader) or
// the producer (peer), plus the epilogue warps.
constexpr int kRingConsumers = 1 + kEpiWarps;

// Called once by each leader that drew (a draw returned past the end, or it
// gave up): the last of the pairs that draw sets the slot back to zero. Every
// draw of every pair has returned by then, since each pair's last draw
// returned before it counted itself out.
__device__ __forceinline__ void sched_done_drawing(const GemmParams& p, int clusters) {
  const unsigned drawers = static_cast<unsigned>(min(clusters, p.total_tiles));
  __threadfence();  // this pair's draws are performed before it counts itself out
  if (atomicAdd(p.sched + 1, 1u) == drawers - 1) {
    atomicExch(p.sched, 0u);
    atomicExch(p.sched + 1, 0u);
  }
}

template <int PAIR>
__device__ __forceinline__ bool ring_put(const TileRing& r, int k, int v, volatile int* abort,
                                         unsigned* status) {
  const int s = k % kRing;
  const uint32_t par = static_cast<uint32_t>(k / kRing) & 1u;
  if (!mbar_wait_cl(&r.empty[s], par ^ 1u, abort, status)) return false;
  r.slot[s] = v;
  if (PAIR == 2) {
    st_shared_cluster_u32(map_shared(smem_u32(const_cast<int*>(&r.slot[s])), 1), static_cast<uint32_t>(v));
    mbar_arrive_cluster(map_shared(smem_u32(&r.full[s]), 1));
  }
  mbar_arrive_release_cluster(&r.full[s]);
  return true;
}
// One consumer thread: entry k (-2 when the wait gave up).
template <int PAIR>
__device__ __forceinline__ int ring_take(const TileRing& r, int k, uint32_t rank, volatile int* abort,
                                         unsigned* status) {
  const int s = k % kRing;
  const uint32_t par = static_cast<uint32_t>(k / kRing) & 1u;
  if (!mbar_wait_cl(&r.full[s], par, abort, status)) return -2;
  const int v = r.slot[s];
  if (PAIR == 2 && rank != 0) mbar_arrive_cluster(map_shared(smem_u32(&r.empty[s]), 0));
  else mbar_arrive_release_cluster(&r.empty[s]);
  return v;
}
// A whole warp: every lane reads entry k, lane 0 arrives once for the warp.
template <int PAIR>
__device__ __forceinline__ int ring_take_warp(const TileRing& r, int k, uint32_t rank, int lane,
                                              volatile int* abort, unsigned* status) {
  const int s = k % kRing;
  const uint32_t par = static_cast<uint32_t>(k / kRing) & 1u;
  if (!__all_sync(0xffffffffu, mbar_wait_cl(&r.full[s], par, abort, status))) return -2;
  const int v = r.slot[s];
  __syncwarp();
  if (lane == 0) {
    if (PAIR == 2 && rank != 0) mbar_arrive_cluster(map_shared(smem_u32(&r.empty[s]), 0));
    else mbar_arrive_release_cluster(&r.empty[s]);
  }
  return v;
}

// -------------------------------------------------------------------- kernel
template <int PAIR>
__global__ void __launch_bounds__(kThreads, 1) tp_gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<PAIR>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint8_t* sE = smem + STAGES * C::STAGE_BYTES;  // TMA epilogue stages, kEpiBuf per epilogue warp
  uint64_t* full = reinterpret_cast<uint64_t*>(sE + kEpiBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  TileRing ring;
  ring.full = drain + 2;
  ring.empty = ring.full + kRing;
  ring.slot = reinterpret_cast<volatile int*>(ring.empty + kRing);
  uint64_t* ebar = reinterpret_cast<uint64_t*>(const_cast<int*>(ring.slot) + kRing);  // [kEpiWarps]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR == 2 ? cluster_ctarank() : 0u;  // 0 = MMA leader of the pair

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], PAIR * kEpiWarps);  // one arrival per epilogue warp of the pair
    }
    mbar_init(drain, 1);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&ring.full[r], 1);
      mbar_init(&ring.empty[r], PAIR * kRingConsumers);
    }
    for (int w = 0; w < kEpiWarps; ++w) mbar_init(&ebar[w], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    const int nmaps = p.kcat ? p.kcat : p.ngroups;
    for (int g = 0; g < nmaps; ++g) {
      tma_prefetch_desc(&p.tmA[g]);
      tma_prefetch_desc(&p.tmB[g]);
    }
    if (p.tma_epi && p.scatter) {
      for (int j = 0; j * p.rows_per_out < p.g[0].M && j < TP_MAX_SHARDS; ++j) {
        tma_prefetch_desc(&p.tmE[j]);
        if (p.scatter_res) tma_prefetch_desc(&p.tmX[j]);
      }
    } else if (p.tma_epi) {
      const bool fwd = p.epi == tpi::EPI_SWIGLU || p.epi == tpi::EPI_BIAS_GELU;
      for (int g = 0; g < p.ngroups; ++g) {  // only the views the launch encoded
        if (!fwd || p.g[g].D) tma_prefetch_desc(&p.tmE[g]);
        if (fwd || epi_inputs(p, p.g[g]) > 0) tma_prefetch_desc(&p.tmX[g]);
      }
    }
  }
  if (warp == 1) {
    if (PAIR == 2) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR == 2) cluster_sync_all();  // the peer's barriers are initialised before any signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touched only shared memory, TMEM and the kernel
  // parameters, so it overlapped the previous kernel's tail.
  pdl_entry();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------- producer
    int stage = 0;
    uint32_t phase = 0;
    int last_parity[STAGES];
#pragma unroll
    for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
    bool ok = true;
    int kseq = 0;
    const int cluster = static_cast<int>(blockIdx.x) / PAIR, clusters = static_cast<int>(gridDim.x) / PAIR;
    // The first tile needs no draw, so the first copies start at once; each
    // draw is issued a tile ahead and its result first read one tile later.
    int next = cluster;
    bool drawing = false;  // a draw of this pair is outstanding or came back empty
    bool done_drawing = !p.dyn_sched || cluster >= p.total_tiles;
    for (;;) {
      int t;
      if (rank == 0) {  // draw the next tile and publish it (or the end)
        t = next;
        if (t < p.total_tiles) {
          if (p.dyn_sched) {
            next = clusters + static_cast<int>(atomicAdd(p.sched, 1u));
            drawing = true;
          } else {
            next += clusters;
          }
        } else if (drawing && !done_drawing) {
          sched_done_drawing(p, clusters);
          done_drawing = true;
        }
        if (!ring_put<PAIR>(ring, kseq, t < p.total_tiles ? t : -1, abort_flag, p.status)) break;
      } else {
        t = ring_take<PAIR>(ring, kseq, rank, abort_flag, p.status);
      }
      ++kseq;
      if (t < 0 || t >= p.total_tiles) break;
      int g, mt, nt, ks;
      decode_tile(p, t, g, mt, nt, ks);
      const GroupArgs& ga = p.g[g];
      int kb_first, kb_count;
      kb_range(p, ga, ks, kb_first, kb_count);
      const int m0 = mt * C::TILE_M + static_cast<int>(rank) * BM;  // this CTA's A rows
      const int n0 = nt * p.tile_n;
      // this CTA's B rows (in a narrow tile of a pair, each CTA's first BN / 4)
      const int nb0 = n0 + static_cast<int>(rank) * (narrow_tile(p, ga, n0) ? BN / (2 * PAIR) : C::B_ROWS);
      // A narrow tile loads only the B rows its MMAs read (half a B stage):
      // always for MN-major B (64-column blocks, one copy each); for K-major
      // B only in a narrow launch, whose tensor map has the half-height box
      // (a ragged narrow tile of a full-width launch loads the full box).
      const bool half_b = p.narrow_all || (p.b_mn && narrow_tile(p, ga, n0));
      const uint32_t b_bytes = half_b ? C::B_BYTES / 2 : C::B_BYTES;
      const int b_blocks = (half_b ? C::B_ROWS / 2 : C::B_ROWS) / 64;  // MN-major 64-column blocks
      const int nseg = p.kcat ? p.kcat : 1;
      for (int sg = 0; sg < nseg && ok; ++sg) {
        const int gi = p.kcat ? sg : g;  // tensor maps of this K segment
        const int nkb = p.kcat ? p.seg_kb[sg] : kb_count;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const int k0 = (p.kcat ? kb : kb_first + kb) * BK;
          uint8_t* a_dst = sA + stage * C::A_BYTES;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          if (PAIR == 1) {
            mbar_arrive_expect_tx(&full[stage], C::A_BYTES + b_bytes);
            if (!p.a_mn) {
              tma_load_2d(a_dst, &p.tmA[gi], &full[stage], k0, m0);
            } else {
#pragma unroll
              for (int c = 0; c < BM / 64; ++c)
                tma_load_2d(a_dst + c * MN_BLOCK_BYTES, &p.tmA[gi], &full[stage], m0 + c * 64, k0);
            }
            if (p.epi == tpi::EPI_SWIGLU) {
              tma_load_3d(b_dst, &p.tmB[gi], &full[stage], k0, n0, 0);
              tma_load_3d(b_dst + C::B_BYTES / 2, &p.tmB[gi], &full[stage], k0, n0, 1);
            } else if (!p.b_mn) {
              tma_load_2d(b_dst, &p.tmB[gi], &full[stage], k0, n0);
            } else {
              for (int c = 0; c < b_blocks; ++c)
                tma_load_2d(b_dst + c * MN_BLOCK_BYTES, &p.tmB[gi], &full[stage], n0 + c * 64, k0);
            }
          } else {
            // Both CTAs' copies complete on the leader's full barrier, which
            // expects the bytes of the whole pair.
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], PAIR * (C::A_BYTES + b_bytes));
            const uint32_t fb = map_shared(smem_u32(&full[stage]), 0);
            if (!p.a_mn) {
              tma_load_2d_pair(a_dst, &p.tmA[gi], fb, k0, m0);
            } else {
#pragma unroll
              for (int c = 0; c < BM / 64; ++c)
                tma_load_2d_pair(a_dst + c * MN_BLOCK_BYTES, &p.tmA[gi], fb, m0 + c * 64, k0);
            }
            if (p.epi == tpi::EPI_SWIGLU) {
              // rank 0 holds the 128 gate rows, rank 1 the matching 128 up rows
              tma_load_3d_pair(b_dst, &p.tmB[gi], fb, k0, n0, static_cast<int>(rank));
            } else if (!p.b_mn) {
              tma_load_2d_pair(b_dst, &p.tmB[gi], fb, k0, nb0);
            } else {
              for (int c = 0; c < b_blocks; ++c)
                tma_load_2d_pair(b_dst + c * MN_BLOCK_BYTES, &p.tmB[gi], fb, nb0 + c * 64, k0);
            }
          }
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) break;
    }
    // A leader that left early (bounded wait gave up) still counts itself out,
    // so the counters of this slot return to zero.
    if (rank == 0 && !done_drawing) sched_done_drawing(p, clusters);
    // Drain: every copy of this CTA (and, for the leader, of the pair) has
    // landed before the CTA exits. The peer's copies complete on the leader's
    // barriers, which the leader drains.
    if (rank == 0)
      for (int s = 0; s < STAGES; ++s)
        if (last_parity[s] >= 0)
          mbar_wait(&full[s], static_cast<uint32_t>(last_parity[s]), abort_flag, p.status);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc_full = idesc_bf16(C::TILE_M, BN, p.a_mn != 0, p.b_mn != 0);
    const uint32_t idesc_narrow = idesc_bf16(C::TILE_M, BN / 2, p.a_mn != 0, p.b_mn != 0);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int kseq = 0;; ++kseq) {
      const int t = ring_take<PAIR>(ring, kseq, rank, abort_flag, p.status);
      if (t < 0) break;
      int g, mt, nt, ks;
      decode_tile(p, t, g, mt, nt, ks);
      const uint32_t idesc =
          narrow_tile(p, p.g[g], nt * p.tile_n) ? idesc_narrow : idesc_full;
      int kb_first, num_kb;
      kb_range(p, p.g[g], ks, kb_first, num_kb);
      if (p.kcat) {
        num_kb = 0;
        for (int sg = 0; sg < p.kcat; ++sg) num_kb += p.seg_kb[sg];
      }
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
        const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k) {
          const uint64_t adesc =
              p.a_mn ? smem_desc_sw128(a_base + k * (UMMA_K * 128), MN_BLOCK_BYTES, 1024)
                     : smem_desc_sw128(a_base + k * (UMMA_K * 2), 16, 1024);
          const uint64_t bdesc =
              p.b_mn ? smem_desc_sw128(b_base + k * (UMMA_K * 128), MN_BLOCK_BYTES, 1024)
                     : smem_desc_sw128(b_base + k * (UMMA_K * 2), 16, 1024);
          if (PAIR == 2) tc_mma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          else tc_mma_bf16(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
        }
        // frees the smem stage (in both CTAs of a pair) when these MMAs finish
        if (PAIR == 2) tc_commit_pair_mc(&empty[stage], 0x3);
        else tc_commit(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      // accumulator ready for the epilogue (of both CTAs of a pair)
      if (PAIR == 2) tc_commit_pair_mc(&tfull[acc], 0x3);
      else tc_commit(&tfull[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // Drain: no MMA of this CTA (pair) is in flight when TMEM is released.
    if (PAIR == 2) tc_commit_pair_mc(drain, 0x1);
    else tc_commit(drain);
    mbar_wait(drain, 0, abort_flag, p.status);
  } else if (warp >= 2) {
    // ------------------------------------------------------------- epilogue
    const int lg = warp & 3;          // TMEM lane quarter this warp may access
    const int half = (warp - 2) / 4;  // which half of the tile's columns
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t tempty_leader = PAIR == 2 ? map_shared(smem_u32(&tempty[0]), 0) : 0u;
    EpiStage es{sE + (warp - 2) * kEpiBuf, &ebar[warp - 2], 0u, 0};
    bool ok = true;
    for (int kseq = 0;; ++kseq) {
      const int t = ring_take_warp<PAIR>(ring, kseq, rank, lane, abort_flag, p.status);
      if (t < 0) break;
      int g, mt, nt, ks;
      decode_tile(p, t, g, mt, nt, ks);
      const GroupArgs& ga = p.g[g];
      const int row0 = mt * C::TILE_M + static_cast<int>(rank) * BM + lg * 32;
      const int n0 = nt * p.tile_n;
      const bool narrow = narrow_tile(p, ga, n0);
      // TMA views: the output problem's, or with the row scatter the view of
      // the sequence shard holding these 32 rows (whole: rows_per_out is a
      // multiple of 32), at its local row; warps past the last row store nothing
      int gi = p.kcat ? 0 : g, trow = row0;
      bool tma_rows = true;
      if (p.scatter) {
        tma_rows = row0 < ga.M;
        gi = tma_rows ? row0 / p.rows_per_out : 0;
        trow = row0 - gi * p.rows_per_out;
      }
      // TMA epilogue: the first chunk's inputs load while the MMAs finish
      const bool pre = p.tma_epi && tma_rows && epi_inputs(p, ga) > 0 &&
                       n0 + half * (narrow ? BN / 4 : BN / 2) < ga.N;
      if (pre && lane == 0) epi_issue_inputs(p, gi, epi_inputs(p, ga), n0 + half * (narrow ? BN / 4 : BN / 2), trow, es);
      // warp-uniform: the epilogue's tcgen05.ld is warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status))) {
        if (pre && lane == 0) {  // the prefetched copies land before the CTA may exit (bounded)
          volatile int none = 0;
          mbar_wait(es.bar, es.phase, &none, nullptr, 1000000ull);
        }
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(lg * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      if (p.tma_epi && !tma_rows) {
        // past the last row of a scattered launch: nothing to store
      } else if (p.tma_epi && (p.epi == tpi::EPI_SWIGLU || p.epi == tpi::EPI_BIAS_GELU)) {
        epilogue_fwd_tma(p, ga, gi, taddr, trow, n0, half, narrow, lane, es);
      } else if (p.tma_epi) {
        ok = epilogue_tile_tma(p, ga, gi, taddr, trow, n0, half, narrow, pre, lane, es, abort_flag, p.status);
      } else if (p.plain_staged) {
        epilogue_plain_staged(p, ga, taddr, row0, n0, half, narrow, lane, smem_u32(es.buf));
      } else {
        epilogue_tile(p, ga, taddr, row0 + lane, n0, half, narrow, ks);
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR == 2) mbar_arrive_cluster(tempty_leader + static_cast<uint32_t>(acc * 8));
        else mbar_arrive(&tempty[acc]);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (p.tma_epi && lane == 0) bulk_wait_all();  // every store of this warp has landed
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR == 2) cluster_sync_all();  // neither CTA leaves while its pair may still signal it
  if (warp == 1) {
    tc_fence_after();
    if (PAIR == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------- host
using tpi::EncodeTiledFn;

// 2-D bf16 tensor [outer, inner] (row stride ld elements), box {64, box_outer}.
tp_status encode_2d(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, uint64_t inner,
                    uint64_t outer, int64_t ld, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return tpi::fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(2d, %llu x %llu, ld %lld) failed: %d",
                     (unsigned long long)inner, (unsigned long long)outer, (long long)ld, (int)r);
  return TP_OK;
}

// [2][nh][K] view of a SwiGLU column shard [G_i; U_i], box {64, 128, 1}.
tp_status encode_gateup(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, uint64_t K,
                        uint64_t nh, int64_t ld) {
  cuuint64_t dims[3] = {K, nh, 2};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2, static_cast<cuuint64_t>(ld) * 2 * nh};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return tpi::fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(3d gate/up) failed: %d", (int)r);
  return TP_OK;
}

// {cols, halves, rows} view of a bf16 epilogue output or staged input with a
// {32, 1, 32} box and 64-byte swizzle (the TMA epilogue's staging tiles).
// halves = 2 views [gate | up] of width cols = nh at a column offset of nh.
tp_status encode_epi(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t halves,
                     uint64_t half_stride, uint64_t rows, int64_t ld) {
  cuuint64_t dims[3] = {cols, halves, rows};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(half_stride) * 2, static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[3] = {32, 1, 32};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TP_OK : TP_ERR_CUDA;
}

// The TMA epilogue serves bf16 outputs of the plain, dGELU and dSwiGLU
// epilogues without row scatter or split K, on 16-byte aligned outputs and
// inputs (and, for dSwiGLU, halves of a multiple of 8 columns).
// TP_GEMM_TMA_EPI=0 keeps every launch on the direct epilogue.
bool tma_epilogue_ok(const GemmBatch& b, int nout, int ksplit) {
  const char* e = getenv("TP_GEMM_TMA_EPI");
  if (e && e[0] == '0') return false;
  if (b.out_f32 || ksplit > 1 || b.plain_stores) return false;
  if (b.scatter_n > 0) {  // plain stores into sequence shards of whole 32-row warp slabs
    if (b.epi != tpi::EPI_STORE || b.rows_per_out % 32 || b.scatter_n > TP_MAX_SHARDS ||
        static_cast<int64_t>(b.scatter_n) * b.rows_per_out != b.g[0].M)
      return false;
    const bool res = b.res_seq[0] != nullptr;
    for (int j = 0; j < b.scatter_n; ++j) {
      if (!b.out_seq[j] || reinterpret_cast<uintptr_t>(b.out_seq[j]) % 16) return false;
      if ((b.res_seq[j] != nullptr) != res) return false;
      if (res && reinterpret_cast<uintptr_t>(b.res_seq[j]) % 16) return false;
    }
    return true;
  }
  const bool fwd = b.epi == tpi::EPI_SWIGLU || b.epi == tpi::EPI_BIAS_GELU;
  const bool bwd = b.epi == tpi::EPI_DGELU || b.epi == tpi::EPI_DSWIGLU;
  if (!fwd && !bwd && b.epi != tpi::EPI_STORE) return false;
  const bool halves = b.epi == tpi::EPI_SWIGLU || b.epi == tpi::EPI_DSWIGLU;
  for (int i = 0; i < nout; ++i) {
    const GemmProblem& o = b.g[i];
    const void* out = fwd ? o.D2 : o.D;  // the output every tile writes
    if (!out || reinterpret_cast<uintptr_t>(out) % 16) return false;
    if (fwd && o.D && reinterpret_cast<uintptr_t>(o.D) % 16) return false;
    if (bwd && !o.aux) return false;
    if (!fwd && o.aux && reinterpret_cast<uintptr_t>(o.aux) % 16) return false;
    if (halves && (o.nh % 8 || o.N != o.nh)) return false;
  }
  return true;
}

// CTA pairing forced by the environment variable TP_GEMM_CTA_PAIR ("1": one
// CTA per 128-row tile, "2": CTA pairs with 256-row tiles); 0 = chosen per launch.
int forced_pair() {
  const char* e = getenv("TP_GEMM_CTA_PAIR");
  if (e && e[0] == '1') return 1;
  if (e && e[0] == '2') return 2;
  return 0;
}

// Tile width forced by TP_GEMM_NARROW ("0": 256-column tiles, "1": 128-column
// tiles everywhere); -1 = chosen per launch. SwiGLU launches ignore it.
int forced_narrow() {
  const char* e = getenv("TP_GEMM_NARROW");
  if (e && e[0] == '0') return 0;
  if (e && e[0] == '1') return 1;
  return -1;
}

// Tile layout of one launch: CTA pairing and tile width.
struct Layout {
  int pair;     // 1 or 2 CTAs per tile
  bool narrow;  // every tile N = BN / 2 (SwiGLU tiles are always 128 gate/up pairs)
};

// The layout with the least estimated time. A launch lasts as long as its
// busiest SM: ceil(tiles / units) waves of the average tile, where a tile's
// cost on each of its SMs is its MMA width times its K blocks. Layouts that
// move more operand bytes per FLOP (one CTA instead of a pair, N = 128
// instead of 256) carry a factor, so they win only when they fill more SMs:
// small problems, whose 256 x 256 tiles leave most of the GPU idle.
// CTA pairs are considered only for launches of at least one 256 x 256 tile
// per SM (two waves of pairs): below that the launch is a wave or two of
// short tiles, where what a pair saves in operand reads is less than what it
// costs to start and to keep two SMs in step. Measured on the 12-layer stack
// at hidden 512 (every GEMM 16-128 such tiles): single CTAs took the step
// from 3.63 to 3.51 ms; the larger workloads' launches (512 and more tiles)
// keep their pairs.
Layout choose_layout(const GemmBatch& b, int sms, double* cost_out = nullptr) {
  const bool swiglu = b.epi == tpi::EPI_SWIGLU;
  const int ks = b.ksplit > 1 ? b.ksplit : 1;
  const int nout = b.kcat ? 1 : b.n;
  int64_t kb_cat = 0;
  if (b.kcat)
    for (int i = 0; i < b.n; ++i) kb_cat += (b.g[i].K + BK - 1) / BK;
  const int fp = forced_pair();
  const int fn = swiglu ? 0 : forced_narrow();
  int64_t pair_tiles = 0;  // 256 x 256 tiles of the launch
  for (int i = 0; i < nout; ++i)
    pair_tiles += static_cast<int64_t>((b.g[i].M + 2 * BM - 1) / (2 * BM)) * ((b.g[i].N + BN - 1) / BN) * ks;
  Layout best{2, false};
  double best_cost = -1.0;
  for (int pair = 2; pair >= 1; --pair) {
    if (fp && pair != fp) continue;
    if (!fp && pair == 2 && pair_tiles < sms) continue;
    for (int nar = 0; nar <= (swiglu ? 0 : 1); ++nar) {
      if (fn >= 0 && nar != fn) continue;
      const int tile_m = BM * pair;
      const int tn = (swiglu || nar) ? BN / 2 : BN;
      double work = 0.0;
      int64_t tiles = 0;
      for (int i = 0; i < nout; ++i) {
        const GemmProblem& o = b.g[i];
        const int64_t mt = (o.M + tile_m - 1) / tile_m;
        const int64_t nt = (o.N + tn - 1) / tn;
        const int64_t kb_all = b.kcat ? kb_cat : (o.K + BK - 1) / BK;
        const int64_t kb = (kb_all + ks - 1) / ks;  // K blocks of one split
        const int last = o.N - static_cast<int>(nt - 1) * tn;  // columns of the last N tile
        const int mma_n = swiglu ? BN : (nar ? BN / 2 : BN);
        const int last_n = (!swiglu && last <= BN / 2) ? BN / 2 : mma_n;
        tiles += mt * nt * ks;
        work += static_cast<double>(mt) * ks * kb * ((nt - 1) * mma_n + last_n);
      }
      const int64_t units = std::max(1, sms / pair);
      const double waves = static_cast<double>((tiles + units - 1) / units);
      const double factor = (pair == 2 ? 1.0 : 1.08) * (nar ? 1.10 : 1.0);
      const double cost = waves * (work / static_cast<double>(std::max<int64_t>(tiles, 1))) * factor;
      if (best_cost < 0.0 || cost < best_cost) {
        best_cost = cost;
        best = Layout{pair, nar != 0};
      }
    }
  }
  if (cost_out) *cost_out = best_cost;
  return best;
}

template <int PAIR>
tp_status launch_kernel(const GemmParams& p, int tiles, int sms, cudaStream_t st) {
  using C = Cfg<PAIR>;
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return tpi::fail(TP_ERR_NO_DEVICE, "no current CUDA device");
  }
  if (!attr_set[dev][PAIR - 1]) {
    tp_status s = tpi::cuda_status(
        cudaFuncSetAttribute(tp_gemm_kernel<PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES),
        "cudaFuncSetAttribute(gemm smem)");
    if (s != TP_OK) return s;
    attr_set[dev][PAIR - 1] = true;
  }
  const int clusters = std::max(1, std::min(tiles, sms / PAIR));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(clusters * PAIR);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = tpi::pdl_enabled() ? 2 : 1;
  tp_status s = tpi::cuda_status(cudaLaunchKernelEx(&cfg, tp_gemm_kernel<PAIR>, p),
                                 "cudaLaunchKernelEx(gemm)");
  if (s != TP_OK) return s;
  return tpi::after_launch(PAIR == 2 ? "gemm_bf16 (tcgen05, CTA pair)" : "gemm_bf16 (tcgen05)");
}

// Dynamic-schedule counters: two words per launch, zero at rest (each launch
// sets its pair back to zero as it ends). Eager launches take slots
// [0, kEagerSlots) in turn; launches recorded into a CUDA graph take slots
// from [kEagerSlots, kSchedSlots), so a replayed graph never shares a counter
// with an eager launch. Two launches running at the same time must not share
// a slot: eager launches are kEagerSlots launches apart before one repeats,
// and a captured graph must not run concurrently with another replay of
// itself.
constexpr int kSchedSlots = 4096, kEagerSlots = 1024;
__device__ unsigned g_sched[2 * kSchedSlots];

tp_status sched_slot(cudaStream_t st, unsigned** out) {
  constexpr int kMaxDev = 64;
  static unsigned* base[kMaxDev] = {};
  static unsigned next_eager[kMaxDev] = {}, next_graph[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return tpi::fail(TP_ERR_NO_DEVICE, "no current CUDA device");
  }
  if (!base[dev]) {
    void* ptr = nullptr;
    tp_status s = tpi::cuda_status(cudaGetSymbolAddress(&ptr, g_sched), "cudaGetSymbolAddress(scheduler)");
    if (s != TP_OK) return s;
    base[dev] = static_cast<unsigned*>(ptr);
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    cs = cudaStreamCaptureStatusNone;
  }
  unsigned slot;
  if (cs == cudaStreamCaptureStatusActive)
    slot = kEagerSlots + next_graph[dev]++ % (kSchedSlots - kEagerSlots);
  else
    slot = next_eager[dev]++ % kEagerSlots;
  *out = base[dev] + 2 * slot;
  return TP_OK;
}

// Dynamic tile schedule for a launch of `tiles` tiles on `units` CTA pairs (or
// CTAs): on when some unit takes more than one tile (with one tile each, the
// first tiles are the whole schedule). TP_GEMM_SCHED=static / dynamic forces it.
bool dynamic_schedule(int tiles, int units) {
  const char* e = getenv("TP_GEMM_SCHED");
  if (e && e[0] == 's') return false;
  if (e && e[0] == 'd') return true;
  return tiles > units;
}

int device_sms() {
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

tp_status launch_gemm_bf16(const GemmBatch& b, cudaStream_t st) {
  if (b.n < 1 || b.n > TP_MAX_SHARDS) return fail(TP_ERR_ARG, "GEMM group count %d", b.n);
  EncodeTiledFn enc = nullptr;
  tp_status s = tma_encoder(&enc);
  if (s != TP_OK) return s;
  static GemmParams p;  // host staging (large); launches copy it into the parameter buffer
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&p, 0, sizeof(p));
  const bool swiglu = b.epi == EPI_SWIGLU;
  if (b.kcat && b.epi != EPI_STORE)
    return fail(TP_ERR_ARG, "K-concatenated GEMM supports the plain epilogue only");
  const int nout = b.kcat ? 1 : b.n;
  for (int i = 0; i < nout; ++i)
    if (b.g[i].M <= 0 || b.g[i].N <= 0)
      return fail(TP_ERR_ARG, "GEMM %d has an empty output (%d x %d)", i, b.g[i].M, b.g[i].N);
  const int sms = device_sms();
  int ksplit = b.ksplit > 1 ? b.ksplit : 1;
  if (ksplit > 1) {
    if (b.kcat || b.scatter_n || b.epi != EPI_STORE || !b.out_f32)
      return fail(TP_ERR_ARG, "split K needs plain fp32 outputs (no K concatenation or scatter)");
    for (int i = 1; i < b.n; ++i)
      if (b.g[i].K != b.g[0].K) return fail(TP_ERR_ARG, "split K needs every problem with the same K");
  }
  const Layout lay = choose_layout(b, sms);
  const int pair = lay.pair;
  const int tile_n = (swiglu || lay.narrow) ? BN / 2 : BN;
  const int tile_m = BM * pair;
  const int b_box = (lay.narrow ? BN / 2 : BN) / pair;  // K-major B rows per CTA
  int tiles = 0;
  for (int i = 0; i < b.n; ++i) {
    const GemmProblem& g = b.g[i];
    const GemmProblem& o = b.kcat ? b.g[0] : g;  // the output this segment feeds
    if (o.M <= 0 || o.N <= 0 || g.K <= 0)
      return fail(TP_ERR_ARG, "GEMM %d has an empty extent (%d x %d x %d)", i, o.M, o.N, g.K);
    // TMA needs 16-byte row strides; the epilogue stores 8-column vectors, so N
    // and the output strides must be multiples of 8. K and M may be ragged.
    if (o.N % 8 || g.lda % 8 || g.ldb % 8 || (o.D && o.ldd % 8) || (o.D2 && o.ldd2 % 8) ||
        (o.aux && o.ldaux % 8))
      return fail(TP_ERR_ALIGN, "GEMM %d: N and every leading dimension must be multiples of 8 "
                  "(N=%d lda=%lld ldb=%lld ldd=%lld)", i, o.N, (long long)g.lda, (long long)g.ldb,
                  (long long)o.ldd);
    if (i < nout) {
      GroupArgs& a = p.g[i];
      a.M = o.M;
      a.N = o.N;
      a.K = g.K;
      a.tiles_n = (o.N + tile_n - 1) / tile_n;
      a.tile_begin = tiles;
      a.num_kb = (g.K + BK - 1) / BK;
      a.nh = o.nh;
      a.D = o.D;
      a.ldd = o.ldd;
      a.D2 = o.D2;
      a.ldd2 = o.ldd2;
      a.bias = o.bias;
      a.aux = o.aux;
      a.ldaux = o.ldaux;
      const int64_t t = static_cast<int64_t>((o.M + tile_m - 1) / tile_m) * a.tiles_n;
      if (tiles + t > 0x7fffffffLL) return fail(TP_ERR_UNSUPPORTED, "too many GEMM tiles");
      tiles += static_cast<int>(t);
    }
    if (b.kcat) p.seg_kb[i] = (g.K + BK - 1) / BK;
    // A operand: [M, K] (K-major) or [K, M] (MN-major)
    if (!b.a_mn) s = encode_2d(enc, &p.tmA[i], g.A, g.K, o.M, g.lda, BM);
    else s = encode_2d(enc, &p.tmA[i], g.A, o.M, g.K, g.lda, BK);
    if (s != TP_OK) return s;
    // B operand
    if (swiglu) s = encode_gateup(enc, &p.tmB[i], g.B, g.K, o.nh, g.ldb);
    else if (!b.b_mn) s = encode_2d(enc, &p.tmB[i], g.B, g.K, o.N, g.ldb, b_box);
    else s = encode_2d(enc, &p.tmB[i], g.B, o.N, g.K, g.ldb, BK);
    if (s != TP_OK) return s;
  }
  p.kcat = b.kcat ? b.n : 0;
  if (b.scatter_n > 0) {
    if (!b.kcat && b.n != 1) return fail(TP_ERR_ARG, "row scatter needs a single output");
    p.scatter = 1;
    p.rows_per_out = static_cast<int>(b.rows_per_out);
    for (int j = 0; j < b.scatter_n; ++j) {
      p.out_seq[j] = b.out_seq[j];
      p.res_seq[j] = b.res_seq[j];
    }
  }
  if (ksplit > 1) {
    const int nkb = (b.g[0].K + BK - 1) / BK;
    const int kbps = (nkb + ksplit - 1) / ksplit;
    if ((nkb + kbps - 1) / kbps != ksplit)
      return fail(TP_ERR_ARG, "split K of %d over %d K blocks leaves a split empty", ksplit, nkb);
    if (static_cast<int64_t>(tiles) * ksplit > 0x7fffffffLL) return fail(TP_ERR_UNSUPPORTED, "too many GEMM tiles");
    p.ksplit = ksplit;
    p.base_tiles = tiles;
    p.kb_per_split = kbps;
    p.split_stride = b.split_stride;
    tiles *= ksplit;
  }
  if (b.plain_stores && b.epi == tpi::EPI_STORE && !b.out_f32 && ksplit <= 1) {
    bool plain = true;
    for (int i = 0; i < nout; ++i)
      if (b.g[i].bias || b.g[i].aux || b.g[i].ldd % 8) plain = false;
    for (int j = 0; j < b.scatter_n; ++j)
      if (b.res_seq[j] || reinterpret_cast<uintptr_t>(b.out_seq[j]) % 16) plain = false;
    p.plain_staged = plain ? 1 : 0;
  }
  if (b.scatter_n > 0 && tma_epilogue_ok(b, nout, ksplit)) {
    p.tma_epi = 1;
    p.scatter_res = b.res_seq[0] != nullptr ? 1 : 0;
    const GemmProblem& o = b.g[0];
    for (int j = 0; j < b.scatter_n && p.tma_epi; ++j) {
      bool good = encode_epi(enc, &p.tmE[j], b.out_seq[j], o.N, 1, o.ldd, b.rows_per_out, o.ldd) == TP_OK;
      if (good && p.scatter_res)
        good = encode_epi(enc, &p.tmX[j], b.res_seq[j], o.N, 1, o.ldaux, b.rows_per_out, o.ldaux) == TP_OK;
      if (!good) p.tma_epi = 0;
    }
  } else if (tma_epilogue_ok(b, nout, ksplit)) {
    p.tma_epi = 1;
    const bool sw = b.epi == tpi::EPI_DSWIGLU || b.epi == tpi::EPI_SWIGLU;
    const bool fwd = b.epi == tpi::EPI_SWIGLU || b.epi == tpi::EPI_BIAS_GELU;
    const uint64_t halves = sw ? 2 : 1;
    for (int i = 0; i < nout && p.tma_epi; ++i) {
      const GemmProblem& o = b.g[i];
      bool good = true;
      // tmE: D (Z in the forward activations, where it may be absent)
      if (o.D) good = encode_epi(enc, &p.tmE[i], o.D, o.N, halves, sw ? o.nh : o.ldd, o.M, o.ldd) == TP_OK;
      // tmX: H (forward activations) or the staged input
      if (good && fwd) good = encode_epi(enc, &p.tmX[i], o.D2, o.N, 1, o.ldd2, o.M, o.ldd2) == TP_OK;
      else if (good && o.aux)
        good = encode_epi(enc, &p.tmX[i], o.aux, o.N, halves, sw ? o.nh : o.ldaux, o.M, o.ldaux) == TP_OK;
      if (!good) p.tma_epi = 0;  // a view the encoder refuses: the direct epilogue serves
    }
  }
  p.ngroups = nout;
  p.total_tiles = tiles;
  p.tile_n = tile_n;
  p.narrow_all = lay.narrow ? 1 : 0;
  p.a_mn = b.a_mn;
  p.b_mn = b.b_mn;
  p.epi = b.epi;
  p.out_f32 = b.out_f32;
  s = device_status_word(&p.status);
  if (s != TP_OK) return s;
  p.dyn_sched = dynamic_schedule(tiles, sms / pair) ? 1 : 0;
  if (p.dyn_sched) {
    s = sched_slot(st, &p.sched);
    if (s != TP_OK) return s;
  }
  if (pair == 2) return launch_kernel<2>(p, tiles, sms, st);
  return launch_kernel<1>(p, tiles, sms, st);
}

bool gemm_fills_gpu(const GemmBatch& b) {
  const int sms = device_sms();
  const Layout lay = choose_layout(b, sms);
  const bool swiglu = b.epi == EPI_SWIGLU;
  const int tile_m = BM * lay.pair, tn = (swiglu || lay.narrow) ? BN / 2 : BN;
  const int nout = b.kcat ? 1 : b.n;
  int64_t tiles = 0;
  for (int i = 0; i < nout; ++i)
    tiles += static_cast<int64_t>((b.g[i].M + tile_m - 1) / tile_m) * ((b.g[i].N + tn - 1) / tn);
  return tiles * (b.ksplit > 1 ? b.ksplit : 1) >= sms / lay.pair;
}

int gemm_split_k(const GemmBatch& b) {
  if (b.kcat || b.scatter_n || b.epi != EPI_STORE || b.n < 1) return 1;
  for (int i = 1; i < b.n; ++i)
    if (b.g[i].K != b.g[0].K || b.g[i].M != b.g[0].M || b.g[i].N != b.g[0].N) return 1;
  const int sms = device_sms();
  const int nkb = (b.g[0].K + BK - 1) / BK;
  if (const char* e = getenv("TP_GEMM_SPLITK")) {  // forced split (tests): 1..16
    const int f = std::max(1, std::min(16, std::min(nkb, atoi(e))));
    const int kbps = (nkb + f - 1) / f;
    return (nkb + kbps - 1) / kbps;
  }
  // Cost units of choose_layout: one K block of one column on a 128-row slab
  // of one SM (16 KFLOP, about 1.25 ns at the clocks seen under load). The
  // reduce reads the fp32 partials once and writes the outputs once at about
  // 6 KB per unit, plus about 2 us of launch and ramp.
  const double out_bytes = static_cast<double>(b.n) * b.g[0].M * b.g[0].N;
  GemmBatch t = b;
  t.out_f32 = true;
  t.ksplit = 1;
  double best_cost = 0.0;
  choose_layout(t, sms, &best_cost);
  int best = 1;
  for (int s = 2; s <= 16; s *= 2) {
    if (nkb < 4 * s) break;  // at least four K blocks per split
    t.ksplit = s;
    double c = 0.0;
    choose_layout(t, sms, &c);
    c += (out_bytes * (4.0 * s + 2.0)) / 6000.0 + 1600.0;
    if (c < 0.9 * best_cost) {
      best_cost = c;
      best = s;
    }
  }
  const int kbps = (nkb + best - 1) / best;
  return (nkb + kbps - 1) / kbps;  // every split gets at least one K block
}

}  // namespace tpi

namespace tpi {

tp_status tma_encoder(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  if (!fn)
    return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *out = fn;
  return TP_OK;
}

tp_status encode_bf16(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims,
                      const cuuint64_t* strides, const cuuint32_t* box, const char* what) {
  EncodeTiledFn enc = nullptr;
  tp_status s = tma_encoder(&enc);
  if (s != TP_OK) return s;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                   const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
  return TP_OK;
}

}  // namespace tpi
