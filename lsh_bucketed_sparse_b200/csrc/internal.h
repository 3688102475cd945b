// Internal interface between the C ABI layer (lsh_attn_api.cu) and the
// kernel translation units.  Not installed; the public boundary is
// include/lsh_attn.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "lsh_attn.h"

namespace lsh {

// Validated copy of lsh_shape with the derived sizes every launcher needs.
struct Problem {
  int B, H, L, d, n_h, n_b, c;
  bool causal;
  bool bf16;         // element type of qk, v, rotations, out, o_rounds
  bool portable;     // LSH_FLAG_PORTABLE: CUDA-core kernels only
  bool dedup;        // LSH_FLAG_DEDUP: duplicate-count correction
  bool bucket_mask;  // LSH_FLAG_BUCKET_MASK: bucket-equality mask
  bool kmeans;       // LSH_FLAG_KMEANS: argmax over n_b given centroids
  int BH() const { return B * H; }
  int half() const { return n_b / 2; }  // projections per round, 0 when n_b == 1
  int n_chunks() const { return (L + c - 1) / c; }  // the last one may be short
  size_t elem() const { return bf16 ? 2 : 4; }
};

// ---- shared by the C ABI entry points (lsh_attn_api.cu) ------------------
// Record a failure message for lsh_attn_last_error() and return `st`.
lsh_status fail(lsh_status st, const char* fmt, ...);
lsh_status cuda_fail(cudaError_t e, const char* what);
// Validate the public shape into a Problem.
lsh_status to_problem(const lsh_shape* s, Problem* p);
// NULL (unless may_be_null) or not 16-byte aligned -> LSH_ERR_INVALID_ARG.
lsh_status check_ptr(const void* ptr, const char* name, bool may_be_null = false);
// rotations must be NULL exactly when n_buckets == 1.
lsh_status check_rotations(const Problem& p, const void* rot);
// Byte offsets of the fused pass's intermediates inside its workspace.
struct Workspace {
  size_t buckets, inv_norm, perm, undo, o_rounds, lse_rounds, sort_scratch, total;
};
Workspace workspace_layout(const Problem& p);
// Stages 1-4 into a checked workspace of workspace_layout(p).total bytes.
lsh_status forward_body(const Problem& p, const void* qk, const void* v, const void* rot,
                        void* out, float* lse, void* ws, cudaStream_t st);

// ---- backward (hash and sort held fixed) ------------------------------------
size_t backward_workspace_bytes(const Problem& p);
cudaError_t launch_backward(const Problem& p, const void* qk, const void* v,
                            const float* inv_norm, const int32_t* perm, const void* out,
                            const float* lse, const void* dout, float* dqk, float* dv,
                            void* workspace, cudaStream_t st);

// Counts one kernel launch of this library (every launch site calls it right
// after its launch); read through lsh_attn_kernel_launches().
void note_launch();

// Launch with programmatic stream serialisation allowed (the kernel calls
// wait_prior_grid before its first global-memory access).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Streaming multiprocessors of the current device (148 on B200; 148 if the
// query fails), cached per device.
int sm_count();

// Address of the device word that kernels set when a bounded wait runs out.
// Resolved for the current device (cudaGetSymbolAddress); nullptr on error.
unsigned int* device_error_word();

// ---- stage 1: hash -------------------------------------------------------
cudaError_t launch_hash_portable(const Problem& p, const void* qk, const void* rot,
                                 int16_t* buckets, float* inv_norm, cudaStream_t st);
bool hash_tc_supported(const Problem& p);
// Sets the limit of the tensor-core hash's first MMA wait (test hook); returns
// the previous limit.
unsigned long long set_hash_first_wait_ns(unsigned long long ns);
cudaError_t launch_hash_tc(const Problem& p, const void* qk, const void* rot, int16_t* buckets,
                           float* inv_norm, cudaStream_t st);

// ---- stage 2: sort -------------------------------------------------------
// Device scratch the sort needs (per-tile bucket counts), in bytes.
size_t sort_scratch_bytes(const Problem& p);
cudaError_t launch_sort(const Problem& p, const int16_t* buckets, int32_t* perm, int32_t* undo,
                        int32_t* counts, void* scratch, cudaStream_t st);

// ---- stage 3: chunked attention --------------------------------------------
// undo: every round's inverse permutation when p.dedup, else ignored;
// buckets: the bucket ids when p.bucket_mask, else ignored.
cudaError_t launch_attn_portable(const Problem& p, const void* qk, const void* v,
                                 const float* inv_norm, const int32_t* perm,
                                 const int32_t* undo, const int16_t* buckets, void* o_rounds,
                                 float* lse_rounds, cudaStream_t st);
// chunks of 64 with d_k = 64 (bf16): P kept in tensor memory
bool attn_tc64_supported(const Problem& p);
cudaError_t launch_attn_tc64(const Problem& p, const void* qk, const void* v,
                             const float* inv_norm, const int32_t* perm, const int16_t* buckets,
                             const int32_t* undo, void* o_rounds, float* lse_rounds,
                             cudaStream_t st);
bool attn_tc_supported(const Problem& p);
cudaError_t launch_attn_tc(const Problem& p, const void* qk, const void* v, const float* inv_norm,
                           const int32_t* perm, const int16_t* buckets, const int32_t* undo,
                           void* o_rounds, float* lse_rounds, cudaStream_t st);

// ---- stage 4: combine ------------------------------------------------------
cudaError_t launch_combine(const Problem& p, const void* o_rounds, const float* lse_rounds,
                           void* out, float* lse, cudaStream_t st);

}  // namespace lsh
