// Stage 2: per (batch, head, round) the stable order of positions by bucket,
// i.e. the key (round, bucket, position) ("Reformer: The Efficient
// Transformer", section 2 "LSH attention": queries and keys are sorted by
// bucket; "Causal masking": positions follow the same permutation; Appendix
// A "Implementation").
//
// Positions already increase in input order, so one stable counting pass on
// the bucket id gives the full key order (a single radix digit).  Each
// segment of L keys is cut into tiles of kTileKeys keys, so the work spreads
// over every SM:
//   1. count: one CTA per tile counts its keys per bucket (shared-memory
//      histogram) into cnt[segment][tile][bucket];
//   2. scan: one CTA per segment: per bucket an exclusive scan over the
//      tiles (in place), the bucket totals (the `counts` output) and the
//      buckets' first slots (their exclusive scan, into base[segment][bucket]);
//   3. scatter: one CTA of eight warps per tile; each warp takes a
//      contiguous eighth of the tile, counts it per bucket into its own row
//      of shared memory, the rows are turned into each warp's first slot per
//      bucket (base + tile prefix + the counts of the warps before it), and
//      each warp then walks its keys in order, 32 at a time, ranking equal
//      keys inside the warp (equal-key lane masks built from one ballot per
//      bit of the bucket id): equal buckets keep position order (stability)
//      without global atomics.  Above 192
//      buckets (where eight rows of counts cost more than they save) one
//      warp walks the whole tile instead.
#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kTileKeys = 2048;
constexpr int kCountThreads = 256;
constexpr int kScanThreads = 1024;
constexpr int kBatch = 16;  // rows of 32 keys loaded ahead in the scatter
constexpr int kScanBatch = 16;  // tiles loaded ahead in the scan
constexpr int kScatterWarps = 8;
constexpr int kSubKeys = kTileKeys / kScatterWarps;  // keys per scatter warp
// The eight-warp scatter keeps eight rows of n_b counts per tile; its
// per-bucket work (8 n_b) outgrows the tile's 2048 keys as n_b grows.
// Measured in the pass on a B200 (old one-warp walk -> eight warps, µs):
// n_b = 64: 31.7 -> 21.5; 192: 33.8 -> 27.6; 256: 29.7 -> 35.8; 1024:
// 60.4 -> 87.0.  So eight warps up to n_b = 192, one warp above.
constexpr int kScatterWideMaxBuckets = 192;

// Lanes of the warp holding the same key as this lane: built from one ballot
// per bit of the key (keys below 2^bits; invalid lanes form their own
// group).  Cheaper than __match_any_sync for the ten bits of 1024 buckets.
__device__ __forceinline__ unsigned same_key(bool valid, int b, int bits) {
  const unsigned v = __ballot_sync(0xffffffffu, valid);
  unsigned m = valid ? v : ~v;
  for (int k = 0; k < bits; ++k) {
    const bool bit = valid && ((b >> k) & 1);
    const unsigned x = __ballot_sync(0xffffffffu, bit);
    m &= bit ? x : ~x;
  }
  return m;
}

__global__ void __launch_bounds__(kCountThreads)
sort_count_kernel(const int16_t* __restrict__ buckets, int32_t* __restrict__ cnt, int L,
                  int n_b, int T) {
  extern __shared__ int32_t hist[];  // [n_b]
  const int seg = blockIdx.x, tile = blockIdx.y;
  for (int b = threadIdx.x; b < n_b; b += blockDim.x) hist[b] = 0;
  wait_prior_grid();
  __syncthreads();
  const int16_t* keys = buckets + (size_t)seg * L;
  const int beg = tile * kTileKeys, end = min(L, beg + kTileKeys);
  int kb[kTileKeys / kCountThreads];
#pragma unroll
  for (int i = 0; i < kTileKeys / kCountThreads; ++i) {
    const int e = beg + i * kCountThreads + threadIdx.x;
    kb[i] = e < end ? (int)keys[e] : -1;
  }
#pragma unroll
  for (int i = 0; i < kTileKeys / kCountThreads; ++i)
    if ((unsigned)kb[i] < (unsigned)n_b) atomicAdd(&hist[kb[i]], 1);
  __syncthreads();
  int32_t* out = cnt + ((size_t)seg * T + tile) * n_b;
  for (int b = threadIdx.x; b < n_b; b += blockDim.x) out[b] = hist[b];
}

// Exclusive scan of a[0..n) in place by the whole block.
__device__ void block_exclusive_scan(int32_t* a, int n) {
  __shared__ int32_t warp_tot[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int32_t local = 0;
  for (int t = lo; t < hi; ++t) local += a[t];
  int32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int32_t w = lane < nw ? warp_tot[lane] : 0;
    int32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < nw) warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
  }
  __syncthreads();
  int32_t run = warp_tot[warp] + incl - local;
  for (int t = lo; t < hi; ++t) {
    const int32_t x = a[t];
    a[t] = run;
    run += x;
  }
  __syncthreads();
}

// cnt[seg][t][b] -> the number of keys of bucket b in tiles before t;
// counts[seg][b] and base[seg][b] (first slot of bucket b) from the totals.
__global__ void __launch_bounds__(kScanThreads)
sort_scan_kernel(int32_t* __restrict__ cnt, int32_t* __restrict__ counts,
                 int32_t* __restrict__ base_out, int n_b, int T) {
  extern __shared__ int32_t base[];  // [n_b]
  const int seg = blockIdx.x;
  int32_t* c = cnt + (size_t)seg * T * n_b;
  wait_prior_grid();
  // The tiles are walked kScanBatch at a time with all of a batch's loads
  // issued before any is used, so a thread waits on memory once per batch.
  for (int b = threadIdx.x; b < n_b; b += blockDim.x) {
    int32_t run = 0;
    for (int t0 = 0; t0 < T; t0 += kScanBatch) {
      int32_t x[kScanBatch];
#pragma unroll
      for (int k = 0; k < kScanBatch; ++k)
        x[k] = t0 + k < T ? c[(size_t)(t0 + k) * n_b + b] : 0;
#pragma unroll
      for (int k = 0; k < kScanBatch; ++k) {
        if (t0 + k < T) c[(size_t)(t0 + k) * n_b + b] = run;
        run += x[k];
      }
    }
    base[b] = run;
    if (counts) counts[(size_t)seg * n_b + b] = run;
  }
  __syncthreads();
  block_exclusive_scan(base, n_b);  // base[b] = first slot of bucket b
  for (int b = threadIdx.x; b < n_b; b += blockDim.x) base_out[(size_t)seg * n_b + b] = base[b];
}

// Eight warps per tile: per-warp counts, then per-warp first slots, then the
// scatter (see the file comment).
__global__ void __launch_bounds__(kScatterWarps * 32)
sort_scatter8_kernel(const int16_t* __restrict__ buckets, const int32_t* __restrict__ cnt,
                     const int32_t* __restrict__ base, int32_t* __restrict__ perm,
                     int32_t* __restrict__ undo, int L, int n_b, int T) {
  extern __shared__ int32_t off[];  // [kScatterWarps][n_b]
  const int seg = blockIdx.x, tile = blockIdx.y;
  wait_prior_grid();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* mine = off + (size_t)warp * n_b;
  for (int b = lane; b < n_b; b += 32) mine[b] = 0;
  const int16_t* keys = buckets + (size_t)seg * L;
  const int beg = tile * kTileKeys + warp * kSubKeys;
  const int end = min(L, min(tile * kTileKeys + kTileKeys, beg + kSubKeys));
  constexpr int kRowsW = kSubKeys / 32;
  const int bits = 32 - __clz(max(n_b - 1, 1));
  int kb[kRowsW];
  unsigned peers[kRowsW];
#pragma unroll
  for (int i = 0; i < kRowsW; ++i) {
    const int e = beg + 32 * i + lane;
    kb[i] = (e < end) ? (int)keys[e] : -1 - lane;
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < kRowsW; ++i) {
    const int e = beg + 32 * i + lane;
    const int b = kb[i];
    const bool valid = (e < end) && (unsigned)b < (unsigned)n_b;
    peers[i] = same_key(valid, b, bits);
    if (valid && lane == 31 - __clz(peers[i])) mine[b] += __popc(peers[i]);
    __syncwarp();
  }
  __syncthreads();
  const int32_t* c = cnt + ((size_t)seg * T + tile) * n_b;
  const int32_t* bs = base + (size_t)seg * n_b;
  for (int b = threadIdx.x; b < n_b; b += kScatterWarps * 32) {
    int32_t run = bs[b] + c[b];
#pragma unroll
    for (int w = 0; w < kScatterWarps; ++w) {
      const int32_t x = off[(size_t)w * n_b + b];
      off[(size_t)w * n_b + b] = run;
      run += x;
    }
  }
  __syncthreads();
  int32_t* P = perm + (size_t)seg * L;
  int32_t* U = undo ? undo + (size_t)seg * L : nullptr;
#pragma unroll
  for (int i = 0; i < kRowsW; ++i) {
    const int e = beg + 32 * i + lane;
    const int b = kb[i];
    const bool valid = (e < end) && (unsigned)b < (unsigned)n_b;
    const int rank = __popc(peers[i] & ((1u << lane) - 1u));
    int slot = 0;
    if (valid) slot = mine[b] + rank;
    __syncwarp();
    if (valid) {
      P[slot] = e;
      if (U) U[e] = slot;
      if (lane == 31 - __clz(peers[i])) mine[b] += __popc(peers[i]);
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(32)
sort_scatter_kernel(const int16_t* __restrict__ buckets, const int32_t* __restrict__ cnt,
                    const int32_t* __restrict__ base, int32_t* __restrict__ perm,
                    int32_t* __restrict__ undo, int L, int n_b, int T) {
  extern __shared__ int32_t off[];  // [n_b]
  const int seg = blockIdx.x, tile = blockIdx.y, lane = threadIdx.x;
  wait_prior_grid();
  const int32_t* c = cnt + ((size_t)seg * T + tile) * n_b;
  const int32_t* bs = base + (size_t)seg * n_b;
  for (int b = lane; b < n_b; b += 32) off[b] = c[b] + bs[b];
  __syncwarp();
  const int16_t* keys = buckets + (size_t)seg * L;
  int32_t* P = perm + (size_t)seg * L;
  int32_t* U = undo ? undo + (size_t)seg * L : nullptr;
  const int beg = tile * kTileKeys, end = min(L, beg + kTileKeys);
  const int bits = 32 - __clz(max(n_b - 1, 1));
  for (int base0 = beg; base0 < end; base0 += 32 * kBatch) {
    int kb[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int e = base0 + 32 * i + lane;
      kb[i] = (e < end) ? (int)keys[e] : -1 - lane;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int e = base0 + 32 * i + lane;
      const int b = kb[i];
      const bool valid = (e < end) && (unsigned)b < (unsigned)n_b;
      const unsigned peers = same_key(valid, b, bits);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int slot = 0;
      if (valid) slot = off[b] + rank;
      __syncwarp();
      if (valid) {
        P[slot] = e;
        if (U) U[e] = slot;
        if (lane == 31 - __clz(peers)) off[b] += __popc(peers);
      }
      __syncwarp();
    }
  }
}

}  // namespace

// Per-tile counts [segments][tiles][n_b], then each bucket's first slot
// [segments][n_b] (the second part 256-byte aligned).
size_t sort_scratch_bytes(const Problem& p) {
  const size_t T = (size_t)(p.L + kTileKeys - 1) / kTileKeys;
  const size_t segs = (size_t)p.BH() * p.n_h;
  const size_t cnt = (segs * T * p.n_b * sizeof(int32_t) + 255) & ~(size_t)255;
  return cnt + segs * p.n_b * sizeof(int32_t);
}

cudaError_t launch_sort(const Problem& p, const int16_t* buckets, int32_t* perm, int32_t* undo,
                        int32_t* counts, void* scratch, cudaStream_t st) {
  const int n_b = p.n_b;
  const size_t hist_bytes = (size_t)n_b * sizeof(int32_t);
  if (hist_bytes > 200 * 1024) return cudaErrorInvalidValue;
  const int T = (p.L + kTileKeys - 1) / kTileKeys;
  const unsigned segs = (unsigned)((long long)p.BH() * p.n_h);
  if (T > 65535) return cudaErrorInvalidValue;
  int32_t* cnt = static_cast<int32_t*>(scratch);
  const size_t cnt_bytes = ((size_t)segs * T * n_b * sizeof(int32_t) + 255) & ~(size_t)255;
  int32_t* base = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + cnt_bytes);
  const size_t scatter8_bytes = (size_t)kScatterWarps * n_b * sizeof(int32_t);
  const bool wide = n_b <= kScatterWideMaxBuckets;
  cudaError_t e;
  if (wide && scatter8_bytes > 48 * 1024 &&
      (e = cudaFuncSetAttribute(sort_scatter8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)scatter8_bytes)))
    return e;
  if (hist_bytes > 48 * 1024) {
    if ((e = cudaFuncSetAttribute(sort_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)hist_bytes)))
      return e;
    if ((e = cudaFuncSetAttribute(sort_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)hist_bytes)))
      return e;
    if ((e = cudaFuncSetAttribute(sort_scatter_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hist_bytes)))
      return e;
  }
  if ((e = launch_dependent(sort_count_kernel, dim3(segs, T), dim3(kCountThreads), hist_bytes, st,
                            buckets, cnt, p.L, n_b, T)))
    return e;
  note_launch();
  if ((e = launch_dependent(sort_scan_kernel, dim3(segs), dim3(kScanThreads), hist_bytes, st, cnt,
                            counts, base, n_b, T)))
    return e;
  note_launch();
  if (wide) {
    e = launch_dependent(sort_scatter8_kernel, dim3(segs, T), dim3(kScatterWarps * 32),
                         scatter8_bytes, st, buckets, static_cast<const int32_t*>(cnt),
                         static_cast<const int32_t*>(base), perm, undo, p.L, n_b, T);
  } else {
    e = launch_dependent(sort_scatter_kernel, dim3(segs, T), dim3(32), hist_bytes, st, buckets,
                         static_cast<const int32_t*>(cnt), static_cast<const int32_t*>(base),
                         perm, undo, p.L, n_b, T);
  }
  if (e) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
