// Vocab-parallel embedding and cross-entropy (TP walkthrough 2kiu.com §6.2;
// 张量并行 wiki, 工程实践): the padded vocab Vp is split into p shards of
// Vs = Vp / p rows; shard i owns vocab ids [i*Vs, (i+1)*Vs).
//
//  embed_fwd   Y[t] = E_{s}[id - s*Vs] with s the owning shard: the sum over
//              shards of the partial lookups (zero outside a shard's range) has
//              exactly one non-zero term, so the kernel reads it directly.
//  embed_bwd   dE[v] = sum over tokens with id == v of dY[t], deterministic: a
//              CTA owns 32 vocab rows x 512 columns, walks the ids in token
//              order and accumulates the matching dY rows in fp32 in shared
//              memory (no atomics), then writes its rows to the owning shard.
//  ce          per token row: max, sum of exp and the target logit over the
//              real (non-padding) columns of all shards -- the shards' local
//              max / sum / target reduced over shards, here merged as running
//              (max, sum) pairs in one streaming pass -- then loss = lse - z_t
//              and the gradient of the scaled loss, (softmax - onehot) * scale,
//              written to dlogits (which may alias the logits).
#include <algorithm>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace {

using tpi::MutPtrArray;
using tpi::PtrArray;

constexpr unsigned kStatusBadIndex = 2u;

__global__ void embed_fwd_kernel(const int32_t* ids, const __grid_constant__ PtrArray E, int vocab,
                                 int64_t Vs, int64_t T, int64_t vpr, uint4* Y,
                                 unsigned* status) {
  tpd::pdl_entry();
  const int64_t total = T * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vpr, c = i - t * vpr;
    const int id = ids[t];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (id >= 0 && id < vocab) {
      const int s = static_cast<int>(id / Vs);
      v = reinterpret_cast<const uint4*>(E.p[s])[(id - s * Vs) * vpr + c];
    } else if (c == 0) {
      atomicOr(status, kStatusBadIndex);
    }
    Y[t * vpr + c] = v;
  }
}

// Embedding gradient as a stable bucket sort of the tokens, then a gather-sum:
//   count    per 1024-token block, how many of its tokens fall in each bucket of
//            16 vocab ids (cnt[block][bucket], block-major);
//   scan     per bucket, the exclusive prefix of its counts over the blocks
//            (in place) and the bucket's total; then one CTA turns the totals
//            into each bucket's start in the sorted list (tot[bucket], with
//            tot[nb] the number of listed tokens);
//   scatter  each token's slot = its bucket's start + its block's prefix + the
//            number of earlier tokens of its block in the same bucket, so
//            every bucket lists its tokens in token order;
//   accum    one CTA per bucket, one warp per vocab row: each warp sums its
//            row's listed dY rows in that order in fp32 registers and writes
//            the row of dE (zeros if none; a copy if one).
// No atomics touch the sums, so the result is deterministic.
constexpr int kEmbRows = 16;    // vocab ids per bucket
constexpr int kTokBlock = 1024; // tokens per count / scatter CTA
constexpr int kEmbMaxBuckets = 12288;  // 48 KB of shared counters (padded vocab <= 196608)
constexpr int kListChunk = 512;

__device__ __forceinline__ bool valid_id(int id, int vocab) { return id >= 0 && id < vocab; }

__global__ void __launch_bounds__(kTokBlock) emb_bucket_count(const int32_t* ids, int64_t ntok,
                                                              int vocab, int nb, int nblk,
                                                              int* cnt) {
  tpd::pdl_entry();
  __shared__ int hist[kEmbMaxBuckets];
  for (int i = threadIdx.x; i < nb; i += kTokBlock) hist[i] = 0;
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kTokBlock + threadIdx.x;
  if (t < ntok) {
    const int id = ids[t];
    if (valid_id(id, vocab)) atomicAdd(&hist[id / kEmbRows], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nb; i += kTokBlock) cnt[static_cast<int64_t>(blockIdx.x) * nb + i] = hist[i];
}

// Thread b: bucket b's counts over the blocks become their exclusive prefix
// (in place); tot[b] = the bucket's total.
__global__ void __launch_bounds__(256) emb_bucket_prefix(int* cnt, int nb, int nblk, int* tot) {
  tpd::pdl_entry();
  const int b = blockIdx.x * 256 + threadIdx.x;
  if (b >= nb) return;
  int run = 0;
  for (int k0 = 0; k0 < nblk; k0 += 8) {  // eight loads in flight, then their stores
    int c[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) c[j] = k0 + j < nblk ? cnt[static_cast<int64_t>(k0 + j) * nb + b] : 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (k0 + j < nblk) cnt[static_cast<int64_t>(k0 + j) * nb + b] = run;
      run += c[j];
    }
  }
  tot[b] = run;
}

// One CTA: a[0..n) <- exclusive prefix sums, a[n] <- the total. Thread tid
// owns the contiguous chunk [tid * C, (tid + 1) * C), C a multiple of 4, read
// and written as 16-byte vectors (a is 16-byte aligned).
__global__ void __launch_bounds__(1024) emb_scan(int* a, int64_t n) {
  tpd::pdl_entry();
  __shared__ int wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t C = ((n + 1023) / 1024 + 3) / 4 * 4;
  const int64_t lo = tid * C < n ? tid * C : n;
  const int64_t hi = lo + C < n ? lo + C : n;
  const int64_t hv = lo + (hi - lo) / 4 * 4;  // [lo, hv) as int4
  int sum = 0;
#pragma unroll 16
  for (int64_t i = lo; i < hv; i += 4) {
    const int4 v = *reinterpret_cast<const int4*>(a + i);
    sum += v.x + v.y + v.z + v.w;
  }
  for (int64_t i = hv; i < hi; ++i) sum += a[i];
  // exclusive scan of the per-thread sums: within the warp, then over warps
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int run = (warp > 0 ? wsum[warp - 1] : 0) + incl - sum;
#pragma unroll 16
  for (int64_t i = lo; i < hv; i += 4) {
    int4 v = *reinterpret_cast<const int4*>(a + i);
    const int4 o = make_int4(run, run + v.x, run + v.x + v.y, run + v.x + v.y + v.z);
    run += v.x + v.y + v.z + v.w;
    *reinterpret_cast<int4*>(a + i) = o;
  }
  for (int64_t i = hv; i < hi; ++i) {
    const int v = a[i];
    a[i] = run;
    run += v;
  }
  if (tid == 1023) a[n] = wsum[31];
}

// sorted[k] = (token, id - bucket * kEmbRows) of the k-th entry of the sorted list.
__global__ void __launch_bounds__(kTokBlock) emb_bucket_scatter(const int32_t* ids, int64_t ntok,
                                                                int vocab, int nb, const int* off,
                                                                const int* tot, int2* sorted) {
  tpd::pdl_entry();
  __shared__ int seen[kEmbMaxBuckets];
  for (int i = threadIdx.x; i < nb; i += kTokBlock) seen[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kTokBlock + threadIdx.x;
  const int id = t < ntok ? ids[t] : -1;
  const bool valid = valid_id(id, vocab);
  const int b = valid ? id / kEmbRows : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, b);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  int base = 0;
  // Warps in order: each reads how many tokens of its bucket earlier warps
  // placed, then the first lane of each bucket group adds its group's size.
  for (int w = 0; w < kTokBlock / 32; ++w) {
    if (warp == w) {
      if (valid) base = seen[b];
      __syncwarp();
      if (valid && rank == 0) seen[b] += __popc(peers);
    }
    __syncthreads();
  }
  if (valid)
    sorted[tot[b] + off[static_cast<int64_t>(blockIdx.x) * nb + b] + base + rank] =
        make_int2(static_cast<int>(t), id - b * kEmbRows);
}

// 16 bytes as floats (8 bf16, widened exactly by shifts, or 4 fp32) and back.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4 u, float (&x)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 2) {
    x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
    x[4] = __uint_as_float(u.z << 16); x[5] = __uint_as_float(u.z & 0xffff0000u);
    x[6] = __uint_as_float(u.w << 16); x[7] = __uint_as_float(u.w & 0xffff0000u);
  } else {
    x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z); x[3] = __uint_as_float(u.w);
  }
}
template <typename T>
__device__ __forceinline__ uint4 pack16(const float (&x)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 2) {
    return make_uint4(tpd::pack_bf16x2(x[0], x[1]), tpd::pack_bf16x2(x[2], x[3]),
                      tpd::pack_bf16x2(x[4], x[5]), tpd::pack_bf16x2(x[6], x[7]));
  } else {
    return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                      __float_as_uint(x[3]));
  }
}

// One CTA per bucket of 16 vocab rows, all h columns: warp w owns vocab row
// v0 + w. The bucket's token list comes into shared memory once; each warp
// counts its own entries (ballots over the list) and then
//   - no token: writes a zero row;
//   - one token: copies that token's dY row (a sum of one term in fp32,
//     rounded back to the same type, is that term), 8 vectors per lane in
//     flight;
//   - more: passes of kAccCols columns, lane l owning vectors l, l + 32, ...
//     of the pass (each load and store of the warp covers 512 contiguous
//     bytes), summing the listed dY rows in list (token) order in fp32
//     registers.
// A bucket listed by more than kListChunk tokens takes the list in chunks,
// pass by pass, with every warp summing.
constexpr int kAccCols = 1024;                 // columns per accumulation pass
constexpr int kAccThreads = 32 * kEmbRows;     // one warp per vocab row of the bucket
constexpr int kCopyVec = 8;                    // vectors per lane in flight when copying a row

template <typename T>
__device__ __forceinline__ void emb_accum_pass(const int* ltok, const int* lrow, int n, int warp, int lane,
                                               const T* dY, int64_t h, int64_t cs, float (&acc)[32]) {
  constexpr int E = 16 / sizeof(T);   // elements per 16-byte vector
  constexpr int NV = 32 / E;          // vectors per lane in a pass
  constexpr int STRIDE = 32 * E;      // columns between a lane's vectors
  const int64_t c0 = cs + lane * E;
  for (int k = 0; k < n; ++k) {
    if (lrow[k] != warp) continue;  // warp-uniform
    const T* src = dY + static_cast<int64_t>(ltok[k]) * h + c0;
    uint4 u[NV];
#pragma unroll
    for (int q = 0; q < NV; ++q)
      u[q] = c0 + q * STRIDE < h ? *reinterpret_cast<const uint4*>(src + q * STRIDE) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      float x[E];
      unpack16<T>(u[q], x);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[q * E + e] += x[e];
    }
  }
}

template <typename T>
__device__ __forceinline__ void emb_store_pass(T* dst, int64_t h, int64_t cs, int lane, const float (&acc)[32]) {
  constexpr int E = 16 / sizeof(T);
  constexpr int NV = 32 / E;
  constexpr int STRIDE = 32 * E;
  const int64_t c0 = cs + lane * E;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    if (c0 + q * STRIDE < h) {
      float x[E];
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = acc[q * E + e];
      *reinterpret_cast<uint4*>(dst + c0 + q * STRIDE) = pack16<T>(x);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kAccThreads, 2) emb_bucket_accum(
    const int2* sorted, const int* tot, const T* dY, int64_t h, int64_t Vs, int64_t Vp,
    const __grid_constant__ MutPtrArray dE) {
  tpd::pdl_entry();
  constexpr int E = 16 / sizeof(T);
  __shared__ int ltok[kListChunk];
  __shared__ int lrow[kListChunk];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t v = static_cast<int64_t>(b) * kEmbRows + warp;
  const bool has_row = v < Vp;
  T* dst = nullptr;
  if (has_row) {
    const int s = static_cast<int>(v / Vs);
    dst = static_cast<T*>(dE.p[s]) + (v - s * Vs) * h;
  }
  const int start = tot[b];
  const int n = tot[b + 1] - start;  // tot[nb] is the number of listed tokens
  float acc[32];
  if (n <= kListChunk) {
    for (int k = threadIdx.x; k < n; k += kAccThreads) {
      const int2 e = sorted[start + k];
      ltok[k] = e.x;
      lrow[k] = e.y;
    }
    __syncthreads();
    if (!has_row) return;
    int cnt = 0, first = 0;
    for (int k0 = 0; k0 < n; k0 += 32) {
      const int k = k0 + lane;
      const unsigned m = __ballot_sync(0xffffffffu, k < n && lrow[k] == warp);
      if (cnt == 0 && m) first = k0 + __ffs(m) - 1;
      cnt += __popc(m);
    }
    const int vpr = static_cast<int>(h / E);
    uint4* dv = reinterpret_cast<uint4*>(dst);
    if (cnt == 0) {
      for (int c = lane; c < vpr; c += 32) dv[c] = make_uint4(0, 0, 0, 0);
    } else if (cnt == 1) {
      const uint4* sv = reinterpret_cast<const uint4*>(dY + static_cast<int64_t>(ltok[first]) * h);
      for (int c0 = lane; c0 < vpr; c0 += 32 * kCopyVec) {
        uint4 u[kCopyVec];
#pragma unroll
        for (int j = 0; j < kCopyVec; ++j) u[j] = c0 + 32 * j < vpr ? sv[c0 + 32 * j] : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < kCopyVec; ++j)
          if (c0 + 32 * j < vpr) dv[c0 + 32 * j] = u[j];
      }
    } else {
      for (int64_t cs = 0; cs < h; cs += kAccCols) {
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
        emb_accum_pass<T>(ltok, lrow, n, warp, lane, dY, h, cs, acc);
        emb_store_pass<T>(dst, h, cs, lane, acc);
      }
    }
    return;
  }
  for (int64_t cs = 0; cs < h; cs += kAccCols) {
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int k0 = 0; k0 < n; k0 += kListChunk) {
      const int nn = n - k0 < kListChunk ? n - k0 : kListChunk;
      __syncthreads();  // the previous chunk's list is consumed
      for (int k = threadIdx.x; k < nn; k += kAccThreads) {
        const int2 e = sorted[start + k0 + k];
        ltok[k] = e.x;
        lrow[k] = e.y;
      }
      __syncthreads();
      emb_accum_pass<T>(ltok, lrow, nn, warp, lane, dY, h, cs, acc);
    }
    if (has_row) emb_store_pass<T>(dst, h, cs, lane, acc);
  }
}

template <typename T>
__device__ __forceinline__ float ld_logit(const void* p, int64_t i) {
  if constexpr (sizeof(T) == 2) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  else return static_cast<const float*>(p)[i];
}

// 2^x by the hardware approximation (denormal results flush to 0).
__device__ __forceinline__ float ex2f_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Running (max, sum of exp2) pair in the log2 domain: the pair (m, s) stands
// for s * 2^m. Merging rescales the smaller side; an empty side is (-inf, 0).
struct MaxSum {
  float m, s;
};

// CTA-wide max or sum: warp shuffles, then warp 0 combines the warps' values;
// every thread gets the result. red holds THREADS / 32 + 1 floats.
template <int THREADS, bool MAX>
__device__ __forceinline__ float block_reduce(float v, float* red) {
  constexpr int W = THREADS / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, o);
    v = MAX ? fmaxf(v, u) : v + u;
  }
  __syncthreads();  // red may still be read from the previous use
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float x = lane < W ? red[lane] : (MAX ? -INFINITY : 0.f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float u = __shfl_xor_sync(0xffffffffu, x, o);
      x = MAX ? fmaxf(x, u) : x + u;
    }
    if (lane == 0) red[W] = x;
  }
  __syncthreads();
  return red[W];
}

// Merge of every thread's (max m, sum s of 2^(x - m)): the CTA max M, then
// the sum of s * 2^(m - M) (threads that saw no column hold (-inf, 0)).
template <int THREADS>
__device__ __forceinline__ MaxSum block_merge(MaxSum v, float* red) {
  const float M = block_reduce<THREADS, true>(v.m, red);
  const float s = v.m == -INFINITY ? 0.f : v.s * exp2f(v.m - M);
  return {M, block_reduce<THREADS, false>(s, red)};
}

// The same merge with one barrier, which also carries every thread's wait
// result: each warp merges its threads' pairs by shuffles, one pair per warp
// goes through shared memory, and every warp merges those pairs again by
// shuffles. Returns false (for every thread) if any thread's ok is false.
// red2 holds THREADS / 32 pairs; it is written again only after the caller's
// next barrier.
template <int THREADS>
__device__ __forceinline__ bool block_merge_ok(MaxSum& v, bool ok, float2* red2) {
  constexpr int W = THREADS / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float M = v.m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float S = v.m == -INFINITY ? 0.f : v.s * ex2f_fast(v.m - M);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
  if (lane == 0) red2[warp] = make_float2(M, S);
  if (!__syncthreads_and(ok)) return false;
  const float2 w = lane < W ? red2[lane] : make_float2(-INFINITY, 0.f);
  float M2 = w.x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M2 = fmaxf(M2, __shfl_xor_sync(0xffffffffu, M2, o));
  float S2 = w.x == -INFINITY ? 0.f : w.y * ex2f_fast(w.x - M2);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S2 += __shfl_xor_sync(0xffffffffu, S2, o);
  v = MaxSum{M2, S2};
  return true;
}



// 16 bytes of logits as floats (8 bf16 or 4 fp32).
template <typename T>
struct Vec {
  static constexpr int N = 16 / sizeof(T);
  float v[N];
  __device__ __forceinline__ void load(const void* base, int64_t i) {
    // plain load: the gradient may overwrite the logits in place
    unpack(reinterpret_cast<const uint4*>(base)[i]);
  }
  __device__ __forceinline__ void unpack(const uint4 u) {
    if constexpr (sizeof(T) == 2) {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = tpd::unpack_bf16x2(w[k]);
        v[2 * k] = f.x;
        v[2 * k + 1] = f.y;
      }
    } else {
      v[0] = __uint_as_float(u.x);
      v[1] = __uint_as_float(u.y);
      v[2] = __uint_as_float(u.z);
      v[3] = __uint_as_float(u.w);
    }
  }
  __device__ __forceinline__ void store(void* base, int64_t i) const {
    uint4 u;
    if constexpr (sizeof(T) == 2) {
      u.x = tpd::pack_bf16x2(v[0], v[1]);
      u.y = tpd::pack_bf16x2(v[2], v[3]);
      u.z = tpd::pack_bf16x2(v[4], v[5]);
      u.w = tpd::pack_bf16x2(v[6], v[7]);
    } else {
      u = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                     __float_as_uint(v[3]));
    }
    reinterpret_cast<uint4*>(base)[i] = u;
  }
};

// One CTA per token row t. Pass 1 streams every shard's slice of the row once
// in 16-byte vectors and keeps a running (max, sum of exp) per thread; pass 2
// re-reads it (mostly from L2) to write the gradient. Exponentials are taken
// as exp2 of logits scaled by log2(e). Vs is a multiple of 8 (the vocab is
// padded to a multiple of 8 p), so every shard row starts on 16 bytes.
template <typename T, int THREADS>
__global__ void __launch_bounds__(THREADS) vocab_ce_kernel(
    const __grid_constant__ PtrArray L, const __grid_constant__ MutPtrArray G, int p, int64_t Vs,
    int vocab, const int32_t* labels, float scale, float* loss, float* lse_out,
    unsigned* status) {
  tpd::pdl_entry();
  constexpr int N = Vec<T>::N;
  constexpr float kLog2e = 1.4426950408889634f;
  __shared__ float red[THREADS / 32 + 1];
  __shared__ float ztarget;
  const int64_t t = blockIdx.x;
  const int label = labels[t];
  const bool ignore = label < 0 || label >= vocab;
  if (threadIdx.x == 0) {
    ztarget = 0.f;
    if (label >= vocab) atomicOr(status, kStatusBadIndex);
    if (!ignore) {
      const int s = static_cast<int>(label / Vs);
      ztarget = ld_logit<T>(L.p[s], t * Vs + (label - s * Vs));
    }
  }
  const int64_t nv = Vs / N;  // vectors per shard row
  MaxSum acc{-INFINITY, 0.f};
  for (int s = 0; s < p; ++s) {
    const int64_t col0 = static_cast<int64_t>(s) * Vs;
    if (col0 >= vocab) break;
    const int64_t row = t * nv;
    for (int64_t j = threadIdx.x; j < nv; j += THREADS) {
      Vec<T> x;
      x.load(L.p[s], row + j);
      const int64_t c = col0 + j * N;
      float lm = -INFINITY;
#pragma unroll
      for (int k = 0; k < N; ++k) {
        x.v[k] = (c + k < vocab) ? x.v[k] * kLog2e : -INFINITY;
        lm = fmaxf(lm, x.v[k]);
      }
      if (lm == -INFINITY) continue;  // all padding
      if (lm > acc.m) {
        acc.s *= exp2f(acc.m - lm);
        acc.m = lm;
      }
#pragma unroll
      for (int k = 0; k < N; ++k) acc.s += exp2f(x.v[k] - acc.m);
    }
  }
  const MaxSum tot = block_merge<THREADS>(acc, red);
  const float lse2 = tot.m + log2f(tot.s);  // log2 of the sum of exp
  if (threadIdx.x == 0) {
    const float lse = lse2 * 0.6931471805599453f;
    loss[t] = ignore ? 0.f : lse - ztarget;
    if (lse_out) lse_out[t] = lse;
  }
  // pass 2: gradient of scale * loss (zero for ignored tokens and padding columns)
  if (G.p[0] == nullptr) return;
  for (int s = 0; s < p; ++s) {
    const int64_t col0 = static_cast<int64_t>(s) * Vs;
    const int64_t row = t * nv;
    for (int64_t j = threadIdx.x; j < nv; j += THREADS) {
      Vec<T> x;
      const int64_t c = col0 + j * N;
      if (!ignore && c < vocab) x.load(L.p[s], row + j);
#pragma unroll
      for (int k = 0; k < N; ++k) {
        float g = 0.f;
        if (!ignore && c + k < vocab)
          g = (exp2f(fmaf(x.v[k], kLog2e, -lse2)) - (c + k == label ? 1.f : 0.f)) * scale;
        x.v[k] = g;
      }
      x.store(G.p[s], row + j);
    }
  }
}

// thread 0: start loading token row t (the CTA's k-th row) into stage
// k % STAGES, one bulk copy per shard slice. False if t is past the rows.
template <int STAGES>
__device__ __forceinline__ bool ce_issue_row(const PtrArray& L, int p, int64_t t, int64_t T_rows,
                                             uint32_t shard_bytes, uint8_t* sbuf, uint32_t stage_bytes,
                                             uint64_t* bar, int64_t k) {
  if (t >= T_rows) return false;
  const int st = static_cast<int>(k % STAGES);
  uint8_t* dst = sbuf + static_cast<size_t>(st) * stage_bytes;
  tpd::mbar_arrive_expect_tx(&bar[st], shard_bytes * static_cast<uint32_t>(p));
  for (int s = 0; s < p; ++s)
    tpd::bulk_load(dst + static_cast<size_t>(s) * shard_bytes,
                   static_cast<const uint8_t*>(L.p[s]) + t * shard_bytes, shard_bytes, &bar[st]);
  return true;
}

// Rows of up to kCeSmemMax / 2 bytes, persistent CTAs: CTA b takes rows
// b, b + G, b + 2G, ... and keeps STAGES of them in flight in shared memory.
// Each row's p shard slices arrive by bulk copy (one per shard, completing on
// the stage's mbarrier) while the CTA works on the rows before it; each
// thread takes its max and sum of exp2 from the shared copy, the CTA merges
// the (max, sum) pairs, the gradient overwrites the shared copy and leaves by
// bulk copies too (a stage is reloaded once its store has read it), so the
// logits cross HBM exactly once each way and the SM's load/store units stay
// out of the stream. The
// shards are contiguous slices of the padded vocab, so 16-byte vector i of
// a row holds columns [i * N, (i + 1) * N).
//
// VPT > 0: every thread's vectors of a row (at most VPT) are held in registers
// through the row: its own max first, then one exp2 per logit relative to it,
// kept for the gradient, which is that exp2 times 2^(own max - lse2) * scale:
// one exponential per logit instead of two.
template <typename T, int THREADS, int STAGES, int VPT>
__global__ void __launch_bounds__(THREADS) vocab_ce_pipe_kernel(
    const __grid_constant__ PtrArray L, const __grid_constant__ MutPtrArray G, int p, int64_t Vs,
    int vocab, int64_t T_rows, uint32_t stage_bytes, const int32_t* labels, float scale,
    float* loss, float* lse_out, unsigned* status) {
  tpd::pdl_entry();
  constexpr int N = Vec<T>::N;
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ __align__(128) uint8_t sbuf[];
  __shared__ uint64_t bar[STAGES];
  __shared__ int abort_flag;
  __shared__ float2 red2[THREADS / 32];
  // the label's logit, handed to thread 0 by the thread that owns its vector
  // (before the merge's barrier: after it, the owner may overwrite the stage)
  __shared__ float s_zt;
  const uint32_t shard_bytes = static_cast<uint32_t>(Vs * sizeof(T));
  const int64_t G0 = blockIdx.x, GS = gridDim.x;
  int64_t issued = 0;  // thread 0: rows [0, issued) of this CTA have their loads issued
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int st = 0; st < STAGES; ++st) tpd::mbar_init(&bar[st], 1);
    tpd::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int k = 0; k < STAGES; ++k)
      if (ce_issue_row<STAGES>(L, p, G0 + k * GS, T_rows, shard_bytes, sbuf, stage_bytes, bar, k)) issued = k + 1;
  const int nv = static_cast<int>(Vs / N);
  const int total = p * nv;
  int next_label = G0 < T_rows ? labels[G0] : 0;  // the next row's label, loaded a row early
  int64_t k = 0;
  for (;; ++k) {
    const int64_t t = G0 + k * GS;
    if (t >= T_rows) break;
    const int label = next_label;
    if (t + GS < T_rows) next_label = labels[t + GS];
    const int st = static_cast<int>(k % STAGES);
    // A thread whose wait gave up reads a stage that may not have landed; its
    // values are discarded: the merge's barrier tells every thread to stop.
    const bool ok = tpd::mbar_wait(&bar[st], static_cast<uint32_t>(k / STAGES) & 1u, &abort_flag, status);
    const uint4* row = reinterpret_cast<const uint4*>(sbuf + static_cast<size_t>(st) * stage_bytes);
    const bool ignore = label < 0 || label >= vocab;
    const int lab_vec = ignore ? -1 : label / N;
    // a bit test per element, not an index into x (which would put x in local memory)
    const uint32_t lab_bit = ignore ? 0u : 1u << (label % N);
    // Vectors below nfull hold no padding column: no per-column tests there.
    const int nfull = vocab / N;
    float e[VPT > 0 ? VPT : 1][N];  // VPT > 0: 2^(x log2e - m) of this thread's columns
    float m = -INFINITY, sum = 0.f;
    if constexpr (VPT > 0) {
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int i = threadIdx.x + j * THREADS;
        if (i < total) {
          unpack16<T>(row[i], e[j]);
          if (i == lab_vec) {
            float z = 0.f;
#pragma unroll
            for (int q = 0; q < N; ++q) z += ((lab_bit >> q) & 1u) ? e[j][q] : 0.f;
            s_zt = z;
          }
          if (i >= nfull) {
#pragma unroll
            for (int q = 0; q < N; ++q)
              if (i * N + q >= vocab) e[j][q] = -INFINITY;
          }
        } else {
#pragma unroll
          for (int q = 0; q < N; ++q) e[j][q] = -INFINITY;
        }
#pragma unroll
        for (int q = 0; q < N; ++q) m = fmaxf(m, e[j][q]);
      }
      m *= kLog2e;
      const float mo = m == -INFINITY ? 0.f : m;  // no column: every term is 2^-inf = 0
#pragma unroll
      for (int j = 0; j < VPT; ++j)
#pragma unroll
        for (int q = 0; q < N; ++q) {
          e[j][q] = ex2f_fast(fmaf(e[j][q], kLog2e, -mo));
          sum += e[j][q];
        }
    } else {
      // One pass: this thread's running max (log2 domain) and sum of 2^(x - max).
      for (int i = threadIdx.x; i < total; i += THREADS) {
        float x[N];
        unpack16<T>(row[i], x);
        if (i == lab_vec) {
          float z = 0.f;
#pragma unroll
          for (int q = 0; q < N; ++q) z += ((lab_bit >> q) & 1u) ? x[q] : 0.f;
          s_zt = z;
        }
        if (i >= nfull) {
#pragma unroll
          for (int q = 0; q < N; ++q)
            if (i * N + q >= vocab) x[q] = -INFINITY;
        }
        float lm = x[0];
#pragma unroll
        for (int q = 1; q < N; ++q) lm = fmaxf(lm, x[q]);
        lm *= kLog2e;
        if (lm > m) {  // (an all-padding vector has lm = -inf and adds nothing below)
          sum *= ex2f_fast(m - lm);
          m = lm;
        }
        if (lm != -INFINITY) {
#pragma unroll
          for (int q = 0; q < N; ++q) sum += ex2f_fast(fmaf(x[q], kLog2e, -m));
        }
      }
    }
    const float m_own = m;
    MaxSum tot{m, sum};
    if (!block_merge_ok<THREADS>(tot, ok, red2)) break;
    const float lse2 = tot.m + log2f(tot.s);
    if (threadIdx.x == 0) {
      if (label >= vocab) atomicOr(status, kStatusBadIndex);
      const float lse = lse2 * 0.6931471805599453f;
      loss[t] = ignore ? 0.f : lse - s_zt;
      if (lse_out) lse_out[t] = lse;
    }
    const bool grad = G.p[0] != nullptr;
    if (grad && VPT > 0) {
      // scale * softmax = e * 2^(m_own - lse2) * scale (the scale in the
      // exponent when it is positive); padding columns hold e = 0
      const float f = ignore || m_own == -INFINITY
                          ? 0.f
                          : (scale > 0.f ? ex2f_fast(m_own - lse2 + log2f(scale)) : ex2f_fast(m_own - lse2) * scale);
      uint4* out = const_cast<uint4*>(row);  // the gradient replaces the staged row
#pragma unroll
      for (int j = 0; j < (VPT > 0 ? VPT : 1); ++j) {
        const int i = threadIdx.x + j * THREADS;
        if (i < total) {
          float g[N];
#pragma unroll
          for (int q = 0; q < N; ++q) g[q] = e[j][q] * f;
          if (i == lab_vec) {  // minus the one-hot target
#pragma unroll
            for (int q = 0; q < N; ++q) g[q] -= ((lab_bit >> q) & 1u) ? scale : 0.f;
          }
          out[i] = pack16<T>(g);
        }
      }
      tpd::fence_proxy_async_smem();
    } else if (grad) {
      // scale * softmax = 2^(x log2e - lse2 + log2 scale): the scale rides in
      // the exponent when it is positive.
      const bool fold = scale > 0.f;
      const float bias = fold ? lse2 - log2f(scale) : lse2;
      const float mul = fold ? 1.f : scale;
      uint4* out = const_cast<uint4*>(row);  // the gradient replaces the staged row
      for (int i = threadIdx.x; i < total; i += THREADS) {
        float x[N];
        unpack16<T>(row[i], x);
        if (ignore) {
#pragma unroll
          for (int e = 0; e < N; ++e) x[e] = 0.f;
        } else if (i < nfull) {
#pragma unroll
          for (int e = 0; e < N; ++e) x[e] = ex2f_fast(fmaf(x[e], kLog2e, -bias));
          if (!fold) {
#pragma unroll
            for (int e = 0; e < N; ++e) x[e] *= mul;
          }
        } else {
#pragma unroll
          for (int e = 0; e < N; ++e)
            x[e] = i * N + e < vocab ? ex2f_fast(fmaf(x[e], kLog2e, -bias)) * mul : 0.f;
        }
        if (i == lab_vec) {  // minus the one-hot target
#pragma unroll
          for (int q = 0; q < N; ++q) x[q] -= ((lab_bit >> q) & 1u) ? scale : 0.f;
        }
        out[i] = pack16<T>(x);
      }
      tpd::fence_proxy_async_smem();
    }
    __syncthreads();  // every thread is done with this stage (and its gradient is in it)
    if (threadIdx.x == 0) {
      if (grad) {
        // Store the row's gradient from shared memory, one bulk copy per shard;
        // then reload the stage of the previous row once its store has read it.
        const uint8_t* src = sbuf + static_cast<size_t>(st) * stage_bytes;
        for (int s = 0; s < p; ++s)
          tpd::bulk_store(static_cast<uint8_t*>(G.p[s]) + t * shard_bytes, src + static_cast<size_t>(s) * shard_bytes,
                          shard_bytes);
        tpd::bulk_commit();
        tpd::bulk_wait_read<1>();
        if (k >= 1 && ce_issue_row<STAGES>(L, p, G0 + (k - 1 + STAGES) * GS, T_rows, shard_bytes, sbuf,
                                           stage_bytes, bar, k - 1 + STAGES))
          issued = k + STAGES;
      } else if (ce_issue_row<STAGES>(L, p, G0 + (k + STAGES) * GS, T_rows, shard_bytes, sbuf, stage_bytes,
                                      bar, k + STAGES)) {
        issued = k + STAGES + 1;
      }
    }
  }
  if (threadIdx.x == 0) tpd::bulk_wait_all();  // every gradient store has landed
  // On a time-out, let the loads still in flight land (bounded) before exit.
  if (threadIdx.x == 0 && abort_flag) {
    for (int64_t kk = k; kk < issued; ++kk) {
      int again = 0;
      tpd::mbar_wait(&bar[kk % STAGES], static_cast<uint32_t>(kk / STAGES) & 1u, &again, nullptr);
    }
  }
}

constexpr int kCeSmemMax = 200 * 1024;  // shared memory for the staged rows
constexpr int kCeVpt = 4;                // vectors per thread of the register-resident rows

template <typename E, int THREADS, int STAGES, int VPT>
tp_status launch_ce_pipe(const PtrArray& L, const MutPtrArray& G, int p, int64_t Vs, int vocab,
                         const int32_t* labels, float scale, float* loss, float* lse, int64_t T,
                         uint32_t stage_bytes, unsigned* status, cudaStream_t st) {
  auto fn = vocab_ce_pipe_kernel<E, THREADS, STAGES, VPT>;
  const int smem = static_cast<int>(stage_bytes) * STAGES;
  int64_t grid = 1;
  tp_status r = tpi::persistent_grid(reinterpret_cast<const void*>(fn), THREADS, smem, T, &grid);
  if (r != TP_OK) return r;
  (void)tpi::launch(fn, dim3(static_cast<unsigned>(grid)), dim3(THREADS), smem, st, L, G, p, Vs, vocab, T, stage_bytes, labels,
                                                         scale, loss, lse, status);
  return TP_OK;
}

int sms() {
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

tp_status launch_embedding_fwd(const int32_t* ids, const PtrArray& E, int vocab, int64_t Vs,
                               int64_t T, int64_t h, tp_dtype dt, void* Y, cudaStream_t st) {
  unsigned* status = nullptr;
  tp_status s = device_status_word(&status);
  if (s != TP_OK) return s;
  const int64_t vpr = h * static_cast<int64_t>(dsize(dt)) / 16;
  const int64_t total = T * vpr;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, sms() * 16LL));
  (void)tpi::launch(embed_fwd_kernel, dim3(blocks), dim3(256), 0, st, ids, E, vocab, Vs, T, vpr, static_cast<uint4*>(Y), status);
  return after_launch("embedding_fwd");
}

static int64_t round4(int64_t n) { return (n + 3) / 4 * 4; }

tp_status embedding_bwd_workspace(int64_t T, int64_t Vp, size_t* bytes) {
  const int64_t nb = (Vp + kEmbRows - 1) / kEmbRows;
  const int64_t nblk = (T + kTokBlock - 1) / kTokBlock;
  if (nb > kEmbMaxBuckets)
    return fail(TP_ERR_UNSUPPORTED, "embedding backward supports a padded vocab of at most %d rows",
                kEmbMaxBuckets * kEmbRows);
  if (T > 0x7fffffffLL || nb * nblk + 1 > 0x7fffffffLL)
    return fail(TP_ERR_UNSUPPORTED, "embedding backward: %lld tokens is too many", (long long)T);
  // cnt[nblk][nb], tot[nb + 1], sorted[T] (int2), each starting on 16 bytes
  *bytes = static_cast<size_t>(round4(nb * nblk) + round4(nb + 1) + 2 * T) * sizeof(int);
  return TP_OK;
}

tp_status launch_embedding_bwd(const int32_t* ids, int64_t T, const void* dY, int64_t h, int vocab,
                               int64_t Vp, int64_t Vs, const MutPtrArray& dE, tp_dtype dt,
                               void* ws, cudaStream_t st) {
  const int nb = static_cast<int>((Vp + kEmbRows - 1) / kEmbRows);
  const int nblk = static_cast<int>((T + kTokBlock - 1) / kTokBlock);
  int* cnt = static_cast<int*>(ws);
  int* tot = cnt + round4(static_cast<int64_t>(nb) * nblk);
  int2* sorted = reinterpret_cast<int2*>(tot + round4(nb + 1));
  tp_status s = TP_OK;
  if (T > 0) {
    (void)tpi::launch(emb_bucket_count, dim3(nblk), dim3(kTokBlock), 0, st, ids, T, vocab, nb, nblk, cnt);
    s = after_launch("embedding_bwd count");
    if (s != TP_OK) return s;
    (void)tpi::launch(emb_bucket_prefix, dim3((nb + 255) / 256), dim3(256), 0, st, cnt, nb, nblk, tot);
    s = after_launch("embedding_bwd prefix");
    if (s != TP_OK) return s;
    (void)tpi::launch(emb_scan, dim3(1), dim3(1024), 0, st, tot, nb);
    s = after_launch("embedding_bwd scan");
    if (s != TP_OK) return s;
    (void)tpi::launch(emb_bucket_scatter, dim3(nblk), dim3(kTokBlock), 0, st, ids, T, vocab, nb, cnt, tot, sorted);
    s = after_launch("embedding_bwd scatter");
    if (s != TP_OK) return s;
  } else {
    s = cuda_status(cudaMemsetAsync(tot, 0, static_cast<size_t>(nb + 1) * sizeof(int), st), "embedding_bwd");
    if (s != TP_OK) return s;
  }
  const unsigned grid = static_cast<unsigned>(nb);
  if (dt == TP_BF16)
    (void)tpi::launch(emb_bucket_accum<__nv_bfloat16>, dim3(grid), dim3(kAccThreads), 0, st, 
        sorted, tot, static_cast<const __nv_bfloat16*>(dY), h, Vs, Vp, dE);
  else
    (void)tpi::launch(emb_bucket_accum<float>, dim3(grid), dim3(kAccThreads), 0, st, sorted, tot, static_cast<const float*>(dY), h, Vs,
                                                         Vp, dE);
  return after_launch("embedding_bwd accumulate");
}

tp_status launch_vocab_ce(const PtrArray& L, const MutPtrArray& G, int p, int64_t Vs, int vocab,
                          const int32_t* labels, float scale, float* loss, float* lse, int64_t T,
                          tp_dtype dt, cudaStream_t st) {
  unsigned* status = nullptr;
  tp_status s = device_status_word(&status);
  if (s != TP_OK) return s;
  const int64_t row_bytes = static_cast<int64_t>(p) * Vs * static_cast<int64_t>(dsize(dt));
  const uint32_t sb = static_cast<uint32_t>((row_bytes + 127) / 128 * 128);
  const int64_t vecs = row_bytes / 16;  // 16-byte vectors per row
  if (3 * row_bytes <= kCeSmemMax && vecs <= kCeVpt * 1024) {
    s = dt == TP_BF16 ? launch_ce_pipe<__nv_bfloat16, 1024, 3, kCeVpt>(L, G, p, Vs, vocab, labels, scale, loss, lse, T, sb, status, st)
                      : launch_ce_pipe<float, 1024, 3, kCeVpt>(L, G, p, Vs, vocab, labels, scale, loss, lse, T, sb, status, st);
  } else if (3 * row_bytes <= kCeSmemMax) {
    s = dt == TP_BF16 ? launch_ce_pipe<__nv_bfloat16, 1024, 3, 0>(L, G, p, Vs, vocab, labels, scale, loss, lse, T, sb, status, st)
                      : launch_ce_pipe<float, 1024, 3, 0>(L, G, p, Vs, vocab, labels, scale, loss, lse, T, sb, status, st);
  } else if (2 * row_bytes <= kCeSmemMax) {
    s = dt == TP_BF16 ? launch_ce_pipe<__nv_bfloat16, 1024, 2, 0>(L, G, p, Vs, vocab, labels, scale, loss, lse, T, sb, status, st)
                      : launch_ce_pipe<float, 1024, 2, 0>(L, G, p, Vs, vocab, labels, scale, loss, lse, T, sb, status, st);
  } else if (dt == TP_BF16) {
    (void)tpi::launch(vocab_ce_kernel<__nv_bfloat16, 256>, dim3(static_cast<unsigned>(T)), dim3(256), 0, st, 
        L, G, p, Vs, vocab, labels, scale, loss, lse, status);
  } else {
    (void)tpi::launch(vocab_ce_kernel<float, 256>, dim3(static_cast<unsigned>(T)), dim3(256), 0, st, L, G, p, Vs, vocab, labels,
                                                                         scale, loss, lse, status);
  }
  if (s != TP_OK) return s;
  return after_launch("vocab_cross_entropy");
}

}  // namespace tpi
