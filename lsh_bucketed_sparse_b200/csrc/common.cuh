// Small device helpers shared by the kernel translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsh {

// Score that replaces q_i . k_i: a token attends to itself only when it has
// no other target ("Reformer: The Efficient Transformer", section 2 "Causal
// masking"; Appendix A "Masking").  The finite value is a reading: the page
// gives no constant.
constexpr float kSelfScore = -1.0e5f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Programmatic dependent launch: the forward path's kernels are launched
// so that one may be set up (launch, shared-memory and tensor-memory
// allocation, barrier initialisation) while the kernel before it on the
// stream finishes; every thread waits here for that kernel to complete,
// with its writes visible, before it touches global memory.  No kernel
// triggers its successor early: when the short kernels did, the next
// kernel's CTAs sat beside them and the long-text pass got slower.
__device__ __forceinline__ void wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Order used by the hash argmax over z = [p; -p]: larger |p| first; among
// equal magnitudes, the smaller index into z.  Column j contributes the
// entry p_j (index j) when p_j >= 0, else -p_j (index half + j); either way
// the entry's value is |p_j|.
__device__ __forceinline__ bool z_better(float a, int z, float best_a, int best_z) {
  return a > best_a || (a == best_a && z < best_z);
}

}  // namespace lsh
