// lsh_attn_forward_noalloc: the fused forward pass for callers that cannot
// allocate device memory.
//
// lsh_attn_forward needs a caller-provided workspace for its intermediates
// (bucket ids, 1/||x||, the sort permutation and the per-round outputs).  Some
// callers have no way to provide one: a plugin inside a host framework that
// owns all device memory through its own pool and hands the plugin nothing
// but its input and output buffers, or a latency-critical path that must not
// call cudaMalloc because it can synchronise the whole device and take an
// unpredictable time.  This entry point keeps the intermediates in a fixed
// scratch array that is part of the library itself, so it needs nothing from
// the caller beyond inputs and outputs and allocates nothing.
#include <mutex>

#include "internal.h"
#include "lsh_attn.h"

namespace lsh {
namespace {

constexpr size_t kScratchBytes = (size_t)LSH_ATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch lives in device memory of every GPU whose context has loaded
// this library's device code, until the process exits.  Under lazy module
// loading (CUDA's default, CUDA_MODULE_LOADING=LAZY) that is the GPUs on
// which a kernel of this translation unit's module has been needed, i.e.
// where this entry point has run; with CUDA_MODULE_LOADING=EAGER it is every
// GPU on which the process creates a context after loading the library.  In host code `g_noalloc_scratch` names a host-side stand-in,
// not a device address: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch[kMaxDevices];  // non-null once resolved on that device

// Device address of the scratch on the current device, looked up with that
// device current.  Only a successful lookup is kept: a failed one (say, a
// transient error) is tried again on the next call.
lsh_status scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LSH_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    g_scratch[dev] = ptr;
  }
  *out = g_scratch[dev];
  return LSH_OK;
}

}  // namespace
}  // namespace lsh

using namespace lsh;

extern "C" lsh_status lsh_attn_forward_noalloc(const lsh_shape* shape, const void* qk,
                                               const void* v, const void* rotations,
                                               void* out, float* lse, void* stream) {
  Problem p;
  lsh_status s;
  if ((s = to_problem(shape, &p)) != LSH_OK) return s;
  if ((s = check_ptr(qk, "qk")) != LSH_OK) return s;
  if ((s = check_ptr(v, "v")) != LSH_OK) return s;
  if ((s = check_rotations(p, rotations)) != LSH_OK) return s;
  if ((s = check_ptr(out, "out")) != LSH_OK) return s;
  if ((s = check_ptr(lse, "lse")) != LSH_OK) return s;
  const size_t need = workspace_layout(p).total;
  if (need > kScratchBytes)
    return fail(LSH_ERR_WORKSPACE,
                "lsh_attn_forward_noalloc: this problem needs %zu bytes of scratch, the "
                "built-in scratch holds %zu; use lsh_attn_forward with a workspace",
                need, kScratchBytes);
  void* ws = nullptr;
  if ((s = scratch_for_current_device(&ws)) != LSH_OK) return s;
  // Every intermediate in the scratch is written before it is read, so the
  // previous call's contents need no clearing.
  return forward_body(p, qk, v, rotations, out, lse, ws, static_cast<cudaStream_t>(stream));
}
