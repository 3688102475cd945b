// Stage 3 on CUDA cores: chunked shared-QK attention of every hashing round
// ("Reformer: The Efficient Transformer", section 2 "LSH attention" and
// "Causal masking"; section 5 "Shared query-key space"; Appendix A
// "Implementation" and "Masking").
//
// Used for float32 inputs and shapes the tensor-core kernel does not take.
// One CTA per (b*h, round, chunk, group of kWarps queries of the chunk),
// flattened into grid.x; one warp per query.  The keys of the window (chunk
// k-1 when k > 0, and chunk k, in sorted order) are staged 32 at a time in
// shared memory by the whole CTA (coalesced row loads; key rows padded by one
// float so that 32 lanes reading 32 rows hit 32 banks); each warp then scores
// its query against them, one key per lane, with an online softmax, and
// accumulates the values with each lane owning output dimensions lane,
// lane + 32, ...  The result is stored at the query's original position.
//
// With `undo` (the duplicate-count correction of Appendix A "Multi-round LSH
// attention"), the score of key j for query i loses log N_ij, N_ij = the
// number of rounds r' in which j sits in i's window, i.e. in which
// chunk(undo_r'[i]) - chunk(undo_r'[j]) is 0 or 1; the self pair keeps its
// replacement score.  With `buckets` (the bucket-equality mask, section 2
// "LSH attention": a query attends only to targets in its own bucket), keys
// whose bucket in this round differs from the query's are left out.
#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxD = 256;
constexpr int kKB = 32;  // keys staged per block

// Shared memory (floats): keys [kKB][d + 1], values [kKB][d], queries
// [kWarps][d], then the block's positions, key scales and buckets.
__host__ __device__ inline size_t portable_smem_floats(int d) {
  return (size_t)kKB * (d + 1) + (size_t)kKB * d + (size_t)kWarps * d + 3 * kKB;
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
attn_portable_kernel(const T* __restrict__ qk, const T* __restrict__ v,
                     const float* __restrict__ inv_norm, const int32_t* __restrict__ perm,
                     const int32_t* __restrict__ undo, const int16_t* __restrict__ bkt,
                     T* __restrict__ o_rounds,
                     float* __restrict__ lse_rounds, int L, int d, int n_h, int c, int causal,
                     float scale) {
  wait_prior_grid();
  extern __shared__ float smem[];
  float* ks = smem;                              // [kKB][d + 1]
  float* vs = ks + (size_t)kKB * (d + 1);        // [kKB][d]
  float* q_all = vs + (size_t)kKB * d;           // [kWarps][d]
  int* kpos = reinterpret_cast<int*>(q_all + (size_t)kWarps * d);  // [kKB]
  float* kin = reinterpret_cast<float*>(kpos + kKB);               // [kKB]
  int* kbk = reinterpret_cast<int*>(kin + kKB);                     // [kKB]
  const int n_c = (L + c - 1) / c;  // the last chunk may be short
  const int qparts = (c + kWarps - 1) / kWarps;
  const int qp = (int)(blockIdx.x % qparts);
  const size_t chunk_id = blockIdx.x / qparts;
  const int k = (int)(chunk_id % n_c);
  const int r = (int)((chunk_id / n_c) % n_h);
  const size_t bh = chunk_id / ((size_t)n_c * n_h);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t* P = perm + (bh * n_h + r) * (size_t)L;
  const T* X = qk + bh * (size_t)L * d;
  const T* V = v + bh * (size_t)L * d;
  const float* IN = inv_norm + bh * (size_t)L;
  const int32_t* UD = undo ? undo + bh * (size_t)n_h * L : nullptr;  // [n_h][L]
  const int16_t* BK = bkt ? bkt + (bh * n_h + r) * (size_t)L : nullptr;  // this round
  float* qs = q_all + warp * d;
  const int k0 = k > 0 ? (k - 1) * c : 0, k1 = min((k + 1) * c, L);
  constexpr int kPer = kMaxD / 32;

  const int qslot = k * c + qp * kWarps + warp;
  const bool has_q = qslot < min(k * c + (qp + 1) * kWarps, k1);
  const int i = has_q ? P[qslot] : 0;
  if (has_q)
    for (int e = lane; e < d; e += 32) qs[e] = to_f32(X[(size_t)i * d + e]);
  const int bq = (BK && has_q) ? (int)BK[i] : 0;
  float m = -INFINITY, l = 0.f;
  float acc[kPer];
#pragma unroll
  for (int t = 0; t < kPer; ++t) acc[t] = 0.f;

  for (int t0 = k0; t0 < k1; t0 += kKB) {
    __syncthreads();  // the previous block is consumed (and qs is written)
    if (tid < kKB) {
      const int js = t0 + tid;
      const int j = js < k1 ? P[js] : -1;
      kpos[tid] = j;
      kin[tid] = j >= 0 ? IN[j] : 0.f;
      kbk[tid] = (BK && j >= 0) ? (int)BK[j] : -1;
    }
    __syncthreads();
    for (int idx = tid; idx < kKB * d; idx += kWarps * 32) {
      const int rr = idx / d, e = idx - rr * d;
      const int j = kpos[rr];
      float kv = 0.f, vv = 0.f;
      if (j >= 0) {
        kv = to_f32(X[(size_t)j * d + e]);
        vv = to_f32(V[(size_t)j * d + e]);
      }
      ks[rr * (d + 1) + e] = kv;
      vs[rr * d + e] = vv;
    }
    __syncthreads();
    if (!has_q) continue;

    const int j = kpos[lane];
    const bool in_window = j >= 0;
    float s = -INFINITY;
    const bool other_bucket = BK && in_window && kbk[lane] != bq;
    if (in_window && !(causal && j > i) && !other_bucket) {
      if (j == i) {
        s = kSelfScore;
      } else {
        const float* kr = ks + lane * (d + 1);
        float dot = 0.f;
#pragma unroll 8
        for (int e = 0; e < d; ++e) dot = fmaf(qs[e], kr[e], dot);
        s = dot * kin[lane] * scale;
        if (UD) {
          int n = 0;
          for (int rr = 0; rr < n_h; ++rr) {
            const int dc = UD[(size_t)rr * L + i] / c - UD[(size_t)rr * L + j] / c;
            n += (dc == 0 || dc == 1) ? 1 : 0;
          }
          s -= logf((float)n);
        }
      }
    }
    const float mnew = fmaxf(m, warp_max(s));
    if (mnew == -INFINITY) continue;  // nothing valid yet (warp-uniform)
    const float alpha = expf(m - mnew);
    const float pj = (s == -INFINITY) ? 0.f : expf(s - mnew);
    l = l * alpha + warp_sum(pj);
#pragma unroll
    for (int t = 0; t < kPer; ++t) acc[t] *= alpha;
    for (int src = 0; src < kKB; ++src) {
      const float ps = __shfl_sync(0xffffffffu, pj, src);
      if (ps == 0.f) continue;  // masked or underflowed: adds nothing
      const float* vr = vs + src * d;
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const int e = lane + 32 * t;
        if (e < d) acc[t] = fmaf(ps, vr[e], acc[t]);
      }
    }
    m = mnew;
  }
  if (!has_q) return;
  const float inv_l = 1.f / l;
  T* orow = o_rounds + ((bh * n_h + r) * (size_t)L + i) * d;
#pragma unroll
  for (int t = 0; t < kPer; ++t) {
    const int e = lane + 32 * t;
    if (e < d) orow[e] = from_f32<T>(acc[t] * inv_l);
  }
  if (lane == 0) lse_rounds[(bh * n_h + r) * (size_t)L + i] = m + logf(l);
}

}  // namespace

cudaError_t launch_attn_portable(const Problem& p, const void* qk, const void* v,
                                 const float* inv_norm, const int32_t* perm,
                                 const int32_t* undo, const int16_t* buckets, void* o_rounds,
                                 float* lse_rounds, cudaStream_t st) {
  if (!p.dedup) undo = nullptr;
  if (!p.bucket_mask) buckets = nullptr;
  if (p.d > kMaxD) return cudaErrorInvalidValue;
  const long long qparts = (p.c + kWarps - 1) / kWarps;
  const long long grid_ll = (long long)p.n_chunks() * p.n_h * p.BH() * qparts;
  if (grid_ll > 0x7fffffffLL) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)grid_ll;
  const size_t smem = portable_smem_floats(p.d) * sizeof(float);
  const float scale = 1.0f / sqrtf((float)p.d);
  cudaError_t e = p.bf16 ? cudaFuncSetAttribute(attn_portable_kernel<__nv_bfloat16>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem)
                         : cudaFuncSetAttribute(attn_portable_kernel<float>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 b(kWarps * 32);
  e = p.bf16 ? launch_dependent(attn_portable_kernel<__nv_bfloat16>, grid, b, smem, st,
                                (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, inv_norm, perm,
                                undo, buckets, (__nv_bfloat16*)o_rounds, lse_rounds, p.L, p.d,
                                p.n_h, p.c, p.causal ? 1 : 0, scale)
             : launch_dependent(attn_portable_kernel<float>, grid, b, smem, st, (const float*)qk,
                                (const float*)v, inv_norm, perm, undo, buckets, (float*)o_rounds,
                                lse_rounds, p.L, p.d, p.n_h, p.c, p.causal ? 1 : 0, scale);
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
