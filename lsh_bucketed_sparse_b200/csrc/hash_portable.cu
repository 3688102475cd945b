// Stage 1 on CUDA cores: random-rotation hash h(x) = argmax([xR; -xR]) for
// every round ("Reformer: The Efficient Transformer", section 2 "LSH
// attention"; Appendix A, one rotation per round), plus 1/||x|| for the key
// normalisation of section 5 ("Shared query-key space").
//
// Used for float32 inputs (projections in float32 FMA, no TF32) and for
// shapes the tensor-core kernel does not take.  One warp per token row: the
// row is staged in shared memory, each lane owns projection columns
// j = lane, lane + 32, ..., accumulates x . R[:, j] in float32 in order
// k = 0..d-1, tracks its best (|p|, z-index) and the warp reduces them.
//
// With `kmeans` (routing-style assignment) the n_b columns of the round's
// matrix are centroids and the bucket is argmax_j x . mu_j (lowest j on
// ties): the same loop over signed values instead of |p|.
#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
hash_portable_kernel(const T* __restrict__ qk, const T* __restrict__ rot,
                     int16_t* __restrict__ buckets, float* __restrict__ inv_norm, int BH, int L,
                     int d, int n_h, int half, int n_cent) {
  extern __shared__ float xs_all[];  // [kWarps][d]
  wait_prior_grid();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* xs = xs_all + warp * d;
  const long long rows = (long long)BH * L;
  for (long long row = (long long)blockIdx.x * kWarps + warp; row < rows;
       row += (long long)gridDim.x * kWarps) {
    const T* x = qk + row * d;
    float ss = 0.f;
    for (int k = lane; k < d; k += 32) {
      const float t = to_f32(x[k]);
      xs[k] = t;
      ss = fmaf(t, t, ss);
    }
    ss = warp_sum(ss);
    __syncwarp();
    const long long bh = row / L, i = row % L;
    if (lane == 0) inv_norm[row] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
    for (int r = 0; r < n_h; ++r) {
      float best_a = -1.f;
      int best_z = 0x7fffffff;
      if (n_cent > 0) {
        best_a = -INFINITY;
        const T* C = rot + (size_t)r * d * n_cent;
        for (int j = lane; j < n_cent; j += 32) {
          float p = 0.f;
          for (int k = 0; k < d; ++k) p = fmaf(xs[k], to_f32(C[(size_t)k * n_cent + j]), p);
          if (z_better(p, j, best_a, best_z)) { best_a = p; best_z = j; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const float oa = __shfl_xor_sync(0xffffffffu, best_a, o);
          const int oz = __shfl_xor_sync(0xffffffffu, best_z, o);
          if (z_better(oa, oz, best_a, best_z)) { best_a = oa; best_z = oz; }
        }
      } else if (half > 0) {
        const T* R = rot + (size_t)r * d * half;
        for (int j = lane; j < half; j += 32) {
          float p = 0.f;
          for (int k = 0; k < d; ++k) p = fmaf(xs[k], to_f32(R[(size_t)k * half + j]), p);
          const float a = fabsf(p);
          const int z = (p >= 0.f) ? j : half + j;  // -0.0 >= 0 holds: index j
          if (z_better(a, z, best_a, best_z)) { best_a = a; best_z = z; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const float oa = __shfl_xor_sync(0xffffffffu, best_a, o);
          const int oz = __shfl_xor_sync(0xffffffffu, best_z, o);
          if (z_better(oa, oz, best_a, best_z)) { best_a = oa; best_z = oz; }
        }
      } else {
        best_z = 0;  // one bucket: every token in bucket 0
      }
      if (lane == 0) buckets[((size_t)bh * n_h + r) * L + i] = (int16_t)best_z;
    }
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_hash_portable(const Problem& p, const void* qk, const void* rot,
                                 int16_t* buckets, float* inv_norm, cudaStream_t st) {
  const long long rows = (long long)p.BH() * p.L;
  long long blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > 148 * 16) blocks = 148 * 16;
  const size_t smem = (size_t)kWarps * p.d * sizeof(float);
  const dim3 g((unsigned)blocks), b(kWarps * 32);
  const int half = p.kmeans ? 0 : p.half(), n_cent = p.kmeans ? p.n_b : 0;
  const cudaError_t e =
      p.bf16 ? launch_dependent(hash_portable_kernel<__nv_bfloat16>, g, b, smem, st,
                                (const __nv_bfloat16*)qk, (const __nv_bfloat16*)rot, buckets,
                                inv_norm, p.BH(), p.L, p.d, p.n_h, half, n_cent)
             : launch_dependent(hash_portable_kernel<float>, g, b, smem, st, (const float*)qk,
                                (const float*)rot, buckets, inv_norm, p.BH(), p.L, p.d, p.n_h,
                                half, n_cent);
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
