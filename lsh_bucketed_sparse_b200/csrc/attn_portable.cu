// Stage 3 on CUDA cores: chunked shared-QK attention of every hashing round
// ("Reformer: The Efficient Transformer", section 2 "LSH attention" and
// "Causal masking"; section 5 "Shared query-key space"; Appendix A
// "Implementation" and "Masking").
//
// Used for float32 inputs and shapes the tensor-core kernel does not take.
// One CTA per (b*h, round, chunk, group of kWarps queries of the chunk),
// flattened into grid.x; one warp per query.  Keys of the window
// (chunk k-1 when k > 0, and chunk k, in sorted order) are visited 32 at a
// time, one key per lane for the score, with an online softmax; the value
// accumulation gives each lane the output dimensions lane, lane + 32, ...
// The result is stored at the query's original position.
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

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
attn_portable_kernel(const T* __restrict__ qk, const T* __restrict__ v,
                     const float* __restrict__ inv_norm, const int32_t* __restrict__ perm,
                     const int32_t* __restrict__ undo, const int16_t* __restrict__ bkt,
                     T* __restrict__ o_rounds,
                     float* __restrict__ lse_rounds, int L, int d, int n_h, int c, int causal,
                     float scale) {
  extern __shared__ float q_all[];  // [kWarps][d]
  const int n_c = (L + c - 1) / c;  // the last chunk may be short
  const int qparts = (c + kWarps - 1) / kWarps;
  const int qp = (int)(blockIdx.x % qparts);
  const size_t chunk_id = blockIdx.x / qparts;
  const int k = (int)(chunk_id % n_c);
  const int r = (int)((chunk_id / n_c) % n_h);
  const size_t bh = chunk_id / ((size_t)n_c * n_h);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* P = perm + (bh * n_h + r) * (size_t)L;
  const T* X = qk + bh * (size_t)L * d;
  const T* V = v + bh * (size_t)L * d;
  const float* IN = inv_norm + bh * (size_t)L;
  const int32_t* UD = undo ? undo + bh * (size_t)n_h * L : nullptr;  // [n_h][L]
  const int16_t* BK = bkt ? bkt + (bh * n_h + r) * (size_t)L : nullptr;  // this round
  float* qs = q_all + warp * d;
  const int k0 = k > 0 ? (k - 1) * c : 0, k1 = min((k + 1) * c, L);
  constexpr int kPer = kMaxD / 32;

  const int q_end = min(k * c + (qp + 1) * kWarps, k1);
  for (int qslot = k * c + qp * kWarps + warp; qslot < q_end; qslot += kWarps) {
    const int i = P[qslot];
    for (int e = lane; e < d; e += 32) qs[e] = to_f32(X[(size_t)i * d + e]);
    __syncwarp();
    float m = -INFINITY, l = 0.f;
    float acc[kPer];
#pragma unroll
    for (int t = 0; t < kPer; ++t) acc[t] = 0.f;

    for (int t0 = k0; t0 < k1; t0 += 32) {
      const int js = t0 + lane;
      const bool in_window = js < k1;
      const int j = in_window ? P[js] : 0;
      float s = -INFINITY;
      const bool other_bucket = BK && in_window && BK[j] != BK[i];
      if (in_window && !(causal && j > i) && !other_bucket) {
        if (j == i) {
          s = kSelfScore;
        } else {
          float dot = 0.f;
          const T* xj = X + (size_t)j * d;
          for (int e = 0; e < d; ++e) dot = fmaf(qs[e], to_f32(xj[e]), dot);
          s = dot * IN[j] * scale;
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
      for (int src = 0; src < 32; ++src) {
        const float ps = __shfl_sync(0xffffffffu, pj, src);
        const int jj = __shfl_sync(0xffffffffu, j, src);
        if (ps == 0.f) continue;  // masked or underflowed: adds nothing
        const T* vj = V + (size_t)jj * d;
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
          const int e = lane + 32 * t;
          if (e < d) acc[t] = fmaf(ps, to_f32(vj[e]), acc[t]);
        }
      }
      m = mnew;
    }
    const float inv_l = 1.f / l;
    T* orow = o_rounds + ((bh * n_h + r) * (size_t)L + i) * d;
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int e = lane + 32 * t;
      if (e < d) orow[e] = from_f32<T>(acc[t] * inv_l);
    }
    if (lane == 0) lse_rounds[(bh * n_h + r) * (size_t)L + i] = m + logf(l);
    __syncwarp();
  }
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
  const size_t smem = (size_t)kWarps * p.d * sizeof(float);
  const float scale = 1.0f / sqrtf((float)p.d);
  if (p.bf16)
    attn_portable_kernel<__nv_bfloat16><<<grid, kWarps * 32, smem, st>>>(
        (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, inv_norm, perm, undo, buckets,
        (__nv_bfloat16*)o_rounds, lse_rounds, p.L, p.d, p.n_h, p.c, p.causal ? 1 : 0, scale);
  else
    attn_portable_kernel<float><<<grid, kWarps * 32, smem, st>>>(
        (const float*)qk, (const float*)v, inv_norm, perm, undo, buckets, (float*)o_rounds, lse_rounds, p.L,
        p.d, p.n_h, p.c, p.causal ? 1 : 0, scale);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
