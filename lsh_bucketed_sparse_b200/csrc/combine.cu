// Stage 4: combine the per-round outputs ("Reformer: The Efficient
// Transformer", Appendix A "Multi-round attention": every round gives an
// independently computable output; they are combined after unsorting):
//   LSE_i = logsumexp_r lse_r,i,   out_i = sum_r exp(lse_r,i - LSE_i) o_r,i.
//
// Pure streaming: o_rounds is stored at original positions, so for a fixed
// round consecutive threads read consecutive 16-byte pieces of consecutive
// rows (coalesced), and out is written the same way.
#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kThreads = 256;

template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static uint4 raw(const float* p) { return *reinterpret_cast<const uint4*>(p); }
  __device__ static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static void load(const float* p, float* f) { unpack(raw(p), f); }
  __device__ static void store(float* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static uint4 raw(const __nv_bfloat16* p) {
    return *reinterpret_cast<const uint4*>(p);
  }
  __device__ static void unpack(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 x = __bfloat1622float2(h[t]);
      f[2 * t] = x.x; f[2 * t + 1] = x.y;
    }
  }
  __device__ static void load(const __nv_bfloat16* p, float* f) { unpack(raw(p), f); }
  __device__ static void store(__nv_bfloat16* p, const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(f[2 * t], f[2 * t + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};

// NH > 0: the number of rounds as a compile-time constant, so every round's
// lse and 16-byte piece are loaded before any is used (all loads in flight
// at once); NH == 0: any n_h.
template <typename T, int NH>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const T* __restrict__ o_rounds, const float* __restrict__ lse_rounds,
               T* __restrict__ out, float* __restrict__ lse, long long rows, int L, int d,
               int n_h_rt) {
  wait_prior_grid();
  using V = Vec16<T>;
  const int n_h = NH > 0 ? NH : n_h_rt;
  const int per_row = d / V::N;
  // blocks run in roughly increasing index order: the last rows first, since
  // the attention wrote the last heads' rounds last and they may still be in L2
  const long long tid = (long long)(gridDim.x - 1 - blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = tid / per_row;
  const int part = (int)(tid % per_row);
  if (row >= rows) return;
  const long long bh = row / L, i = row % L;
  const float* lr = lse_rounds + bh * n_h * (long long)L + i;
  const T* orow = o_rounds + (bh * n_h * (long long)L + i) * d + part * V::N;
  float acc[V::N];
#pragma unroll
  for (int t = 0; t < V::N; ++t) acc[t] = 0.f;
  float LSE;
  if constexpr (NH > 0) {
    float l[NH];
    uint4 u[NH];
#pragma unroll
    for (int r = 0; r < NH; ++r) {
      l[r] = lr[(long long)r * L];
      u[r] = V::raw(orow + (long long)r * L * d);
    }
    float m = l[0];
#pragma unroll
    for (int r = 1; r < NH; ++r) m = fmaxf(m, l[r]);
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < NH; ++r) {
      l[r] = expf(l[r] - m);
      s += l[r];
    }
    LSE = m + logf(s);
    // exp(lse_r - LSE) evaluated as exp(lse_r - m) / s: the differences to
    // the maximum stay exact even where |lse| is ~1e5 (a token that saw only
    // itself).
    const float inv_s = 1.f / s;
#pragma unroll
    for (int r = 0; r < NH; ++r) {
      const float w = l[r] * inv_s;
      float f[V::N];
      V::unpack(u[r], f);
#pragma unroll
      for (int t = 0; t < V::N; ++t) acc[t] = fmaf(w, f[t], acc[t]);
    }
  } else {
    float m = -INFINITY;
    for (int r = 0; r < n_h; ++r) m = fmaxf(m, lr[(long long)r * L]);
    float s = 0.f;
    for (int r = 0; r < n_h; ++r) s += expf(lr[(long long)r * L] - m);
    LSE = m + logf(s);
    const float inv_s = 1.f / s;
    for (int r = 0; r < n_h; ++r) {
      const float w = expf(lr[(long long)r * L] - m) * inv_s;
      float f[V::N];
      V::load(orow + (long long)r * L * d, f);
#pragma unroll
      for (int t = 0; t < V::N; ++t) acc[t] = fmaf(w, f[t], acc[t]);
    }
  }
  V::store(out + row * d + part * V::N, acc);
  if (part == 0) lse[row] = LSE;
}

template <typename T>
void launch_t(const Problem& p, const void* o_rounds, const float* lse_rounds, void* out,
              float* lse, unsigned blocks, long long rows, cudaStream_t st) {
  const T* o = static_cast<const T*>(o_rounds);
  T* y = static_cast<T*>(out);
  // launch errors surface through the caller's cudaGetLastError
  const int nh = p.n_h;
  const dim3 g(blocks), b(kThreads);
  switch (nh) {
    case 1: (void)launch_dependent(combine_kernel<T, 1>, g, b, 0, st, o, lse_rounds, y, lse, rows,
                                   p.L, p.d, 1); break;
    case 2: (void)launch_dependent(combine_kernel<T, 2>, g, b, 0, st, o, lse_rounds, y, lse, rows,
                                   p.L, p.d, 2); break;
    case 4: (void)launch_dependent(combine_kernel<T, 4>, g, b, 0, st, o, lse_rounds, y, lse, rows,
                                   p.L, p.d, 4); break;
    case 8: (void)launch_dependent(combine_kernel<T, 8>, g, b, 0, st, o, lse_rounds, y, lse, rows,
                                   p.L, p.d, 8); break;
    default: (void)launch_dependent(combine_kernel<T, 0>, g, b, 0, st, o, lse_rounds, y, lse,
                                    rows, p.L, p.d, nh);
  }
  note_launch();
}

}  // namespace

cudaError_t launch_combine(const Problem& p, const void* o_rounds, const float* lse_rounds,
                           void* out, float* lse, cudaStream_t st) {
  const long long rows = (long long)p.BH() * p.L;
  const int per_row = p.d / (p.bf16 ? 8 : 4);
  const long long threads = rows * per_row;
  const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
  if (p.bf16)
    launch_t<__nv_bfloat16>(p, o_rounds, lse_rounds, out, lse, blocks, rows, st);
  else
    launch_t<float>(p, o_rounds, lse_rounds, out, lse, blocks, rows, st);
  return cudaGetLastError();
}

}  // namespace lsh
