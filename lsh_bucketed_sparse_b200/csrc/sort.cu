// Stage 2: per (batch, head, round) the stable order of positions by bucket,
// i.e. the key (round, bucket, position) ("Reformer: The Efficient
// Transformer", section 2 "LSH attention": queries and keys are sorted by
// bucket; "Causal masking": positions follow the same permutation; Appendix
// A "Implementation").
//
// Positions already increase in input order, so one stable counting pass on
// the bucket id gives the full key order (a single radix digit).  One CTA
// sorts one segment of L keys:
//   1. the segment is split into W contiguous owner ranges (one per warp);
//      a shared-memory histogram counts each owner's keys per bucket;
//   2. per bucket, an exclusive scan over owners, then an exclusive scan of
//      the bucket totals, gives every (owner, bucket) its first output slot;
//   3. each owner warp walks its range in order, 32 keys at a time; equal
//      keys inside the warp are ranked with __match_any_sync, so equal
//      buckets keep position order (stability) without global atomics.
#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kThreads = 1024;
constexpr int kBatch = 16;  // keys per thread loaded ahead
constexpr int kMaxSmem = 227 * 1024 - 1024;  // leave room for static shared memory

// Exclusive scan of a[0..n) in place by the whole block; returns nothing.
__device__ void block_exclusive_scan(int32_t* a, int n) {
  __shared__ int32_t warp_tot[kThreads / 32];
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

__global__ void __launch_bounds__(kThreads)
sort_kernel(const int16_t* __restrict__ buckets, int32_t* __restrict__ perm,
            int32_t* __restrict__ undo, int32_t* __restrict__ counts, int L, int n_b, int W) {
  extern __shared__ int32_t sh[];  // [W][n_b] owner offsets, then [n_b] totals if W > 1
  const size_t seg = blockIdx.x;
  const int16_t* keys = buckets + seg * L;
  int32_t* P = perm + seg * L;
  int32_t* U = undo ? undo + seg * L : nullptr;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* tot = (W > 1) ? sh + (size_t)W * n_b : sh;
  const int len = (((L + W - 1) / W) + 31) & ~31;  // owner range, a multiple of 32

  for (int t = tid; t < W * n_b; t += blockDim.x) sh[t] = 0;
  __syncthreads();
  // kBatch loads in flight per thread before their counts, so the loop pays
  // the memory latency once per batch rather than once per key
  for (int e0 = tid; e0 < L; e0 += kBatch * blockDim.x) {
    int kb[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int e = e0 + i * blockDim.x;
      kb[i] = e < L ? (int)keys[e] : -1;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int e = e0 + i * blockDim.x;
      if ((unsigned)kb[i] < (unsigned)n_b) atomicAdd(&sh[(e / len) * n_b + kb[i]], 1);
    }
  }
  __syncthreads();
  if (W > 1) {
    for (int b = tid; b < n_b; b += blockDim.x) {
      int32_t run = 0;
      for (int o = 0; o < W; ++o) {
        const int32_t t = sh[o * n_b + b];
        sh[o * n_b + b] = run;
        run += t;
      }
      tot[b] = run;
    }
    __syncthreads();
  }
  if (counts)
    for (int b = tid; b < n_b; b += blockDim.x) counts[seg * n_b + b] = tot[b];
  __syncthreads();
  block_exclusive_scan(tot, n_b);  // tot[b] = first slot of bucket b
  if (W > 1) {
    for (int t = tid; t < W * n_b; t += blockDim.x) sh[t] += tot[t % n_b];
    __syncthreads();
  }

  if (warp < W) {
    int32_t* off = sh + (size_t)warp * n_b;
    const int beg = warp * len, end = min(L, beg + len);
    for (int base0 = beg; base0 < end; base0 += 32 * kBatch) {
      // the next kBatch rows of 32 keys, loaded ahead of their ranking
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
        const unsigned peers = __match_any_sync(0xffffffffu, b);
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
}

}  // namespace

cudaError_t launch_sort(const Problem& p, const int16_t* buckets, int32_t* perm, int32_t* undo,
                        int32_t* counts, cudaStream_t st) {
  const int n_b = p.n_b;
  const long long per = (long long)n_b * 4;
  int W = (int)((kMaxSmem - per) / per);
  if (W > kThreads / 32) W = kThreads / 32;
  const int max_owners = (p.L + 31) / 32;
  if (W > max_owners) W = max_owners;
  if (W < 2) W = 1;
  const size_t smem = (size_t)(W > 1 ? W + 1 : 1) * per;
  if (smem > (size_t)kMaxSmem) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned segs = (unsigned)((long long)p.BH() * p.n_h);
  sort_kernel<<<segs, kThreads, smem, st>>>(buckets, perm, undo, counts, p.L, n_b, W);
  return cudaGetLastError();
}

}  // namespace lsh
