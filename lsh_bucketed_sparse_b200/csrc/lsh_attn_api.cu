// C ABI of liblsh_attn.so (declared in include/lsh_attn.h): argument checks,
// kernel selection, workspace layout and the host-buffer entry point.  Every
// step of the computation runs in the kernels of this library; this file
// only validates and launches.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "internal.h"
#include "lsh_attn.h"

namespace lsh {

// Set by a kernel whose bounded wait runs out; read and cleared by
// lsh_attn_device_check().
__device__ unsigned int g_device_error_word = 0;

namespace {
thread_local char g_last_error[512] = "";
std::atomic<unsigned long long> g_launches{0};
}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

lsh_status fail(lsh_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

lsh_status cuda_fail(cudaError_t e, const char* what) {
  return fail(LSH_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

namespace {

constexpr int kMaxDevices = 64;
std::once_flag g_word_once[kMaxDevices];
unsigned int* g_word_ptr[kMaxDevices];
std::atomic<int> g_sm_count[kMaxDevices];

}  // namespace

lsh_status to_problem(const lsh_shape* s, Problem* p) {
  if (!s) return fail(LSH_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 1 || s->heads < 1 || s->seq_len < 1)
    return fail(LSH_ERR_INVALID_ARG, "batch, heads and seq_len must be >= 1");
  if (s->d_k < 8 || s->d_k > 256 || s->d_k % 8)
    return fail(LSH_ERR_INVALID_ARG, "d_k=%d: must be a multiple of 8 in [8, 256]", s->d_k);
  if (s->n_hashes < 1) return fail(LSH_ERR_INVALID_ARG, "n_hashes must be >= 1");
  const bool kmeans = (s->flags & LSH_FLAG_KMEANS) != 0;
  if (kmeans && !(s->n_buckets >= 2 && s->n_buckets <= 32768))
    return fail(LSH_ERR_INVALID_ARG, "n_buckets=%d: must be in [2, 32768] with LSH_FLAG_KMEANS",
                s->n_buckets);
  if (!kmeans &&
      !(s->n_buckets == 1 || (s->n_buckets >= 2 && s->n_buckets <= 32768 && s->n_buckets % 2 == 0)))
    return fail(LSH_ERR_INVALID_ARG, "n_buckets=%d: must be 1 or even in [2, 32768]",
                s->n_buckets);
  if (s->chunk_len < 1) return fail(LSH_ERR_INVALID_ARG, "chunk_len=%d must be >= 1", s->chunk_len);
  if (s->causal != 0 && s->causal != 1) return fail(LSH_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (s->dtype != LSH_F32 && s->dtype != LSH_BF16)
    return fail(LSH_ERR_INVALID_ARG, "dtype=%d: must be LSH_F32 or LSH_BF16", s->dtype);
  if (s->flags & ~(LSH_FLAG_PORTABLE | LSH_FLAG_DEDUP | LSH_FLAG_BUCKET_MASK | LSH_FLAG_KMEANS))
    return fail(LSH_ERR_INVALID_ARG, "unknown flag bits");
  const long long bh = (long long)s->batch * s->heads;
  if (bh > (1LL << 30)) return fail(LSH_ERR_INVALID_ARG, "batch*heads too large");
  const long long chunks =
      bh * s->n_hashes * ((s->seq_len + s->chunk_len - 1) / s->chunk_len);
  if (chunks >= (1LL << 31) || (long long)s->n_hashes * s->seq_len >= (1LL << 31))
    return fail(LSH_ERR_INVALID_ARG, "problem too large for 32-bit grid/slot indices");
  p->B = s->batch; p->H = s->heads; p->L = s->seq_len; p->d = s->d_k;
  p->n_h = s->n_hashes; p->n_b = s->n_buckets; p->c = s->chunk_len;
  p->causal = s->causal != 0; p->bf16 = s->dtype == LSH_BF16;
  p->portable = (s->flags & LSH_FLAG_PORTABLE) != 0;
  p->dedup = (s->flags & LSH_FLAG_DEDUP) != 0;
  p->bucket_mask = (s->flags & LSH_FLAG_BUCKET_MASK) != 0;
  p->kmeans = kmeans;
  return LSH_OK;
}

lsh_status check_ptr(const void* ptr, const char* name, bool may_be_null) {
  if (!ptr) return may_be_null ? LSH_OK : fail(LSH_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(ptr) % 16)
    return fail(LSH_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return LSH_OK;
}

namespace {

#define CHECK(x)                  \
  do {                            \
    lsh_status _s = (x);          \
    if (_s != LSH_OK) return _s;  \
  } while (0)

}  // namespace

lsh_status check_rotations(const Problem& p, const void* rot) {
  if (p.n_b == 1) {
    if (rot) return fail(LSH_ERR_INVALID_ARG, "rotations must be NULL when n_buckets == 1");
    return LSH_OK;
  }
  return check_ptr(rot, "rotations");
}

namespace {

// ---- stage bodies (arguments already checked) ---------------------------
lsh_status run_hash(const Problem& p, const void* qk, const void* rot, int16_t* buckets,
                    float* inv_norm, cudaStream_t st) {
  cudaError_t e = (!p.portable && hash_tc_supported(p))
                      ? launch_hash_tc(p, qk, rot, buckets, inv_norm, st)
                      : launch_hash_portable(p, qk, rot, buckets, inv_norm, st);
  return e == cudaSuccess ? LSH_OK : cuda_fail(e, "hash launch");
}

lsh_status run_sort(const Problem& p, const int16_t* buckets, int32_t* perm, int32_t* undo,
                    int32_t* counts, void* scratch, cudaStream_t st) {
  cudaError_t e = launch_sort(p, buckets, perm, undo, counts, scratch, st);
  return e == cudaSuccess ? LSH_OK : cuda_fail(e, "sort launch");
}

// The variants run on the tensor-core kernel where it takes them (the
// duplicate correction for n_h <= 8, not together with the bucket mask),
// else on the CUDA-core kernel.
lsh_status run_attn(const Problem& p, const void* qk, const void* v, const float* inv_norm,
                    const int32_t* perm, const int32_t* undo, const int16_t* buckets,
                    void* o_r, float* lse_r, cudaStream_t st) {
  cudaError_t e = cudaErrorNotSupported;
  // (the chunk-64 kernel writes o_rounds in 32-byte stores)
  if (!p.portable && attn_tc64_supported(p) && reinterpret_cast<uintptr_t>(o_r) % 32 == 0)
    e = launch_attn_tc64(p, qk, v, inv_norm, perm, buckets, undo, o_r, lse_r, st);
  else if (!p.portable && attn_tc_supported(p) && !(p.dedup && (p.bucket_mask || p.n_h > 8)))
    e = launch_attn_tc(p, qk, v, inv_norm, perm, buckets, undo, o_r, lse_r, st);
  if (e == cudaErrorNotSupported)  // a shape the tensor-core kernel does not plan for
    e = launch_attn_portable(p, qk, v, inv_norm, perm, undo, buckets, o_r, lse_r, st);
  return e == cudaSuccess ? LSH_OK : cuda_fail(e, "chunked attention launch");
}

lsh_status run_combine(const Problem& p, const void* o_r, const float* lse_r, void* out,
                       float* lse, cudaStream_t st) {
  cudaError_t e = launch_combine(p, o_r, lse_r, out, lse, st);
  return e == cudaSuccess ? LSH_OK : cuda_fail(e, "combine launch");
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

Workspace workspace_layout(const Problem& p) {
  const size_t slots = (size_t)p.BH() * p.n_h * p.L;
  Workspace w;
  size_t off = 0;
  w.buckets = off;    off += align256(slots * sizeof(int16_t));
  w.inv_norm = off;   off += align256((size_t)p.BH() * p.L * sizeof(float));
  w.perm = off;       off += align256(slots * sizeof(int32_t));
  w.undo = off;       off += p.dedup ? align256(slots * sizeof(int32_t)) : 0;
  w.o_rounds = off;   off += align256(slots * p.d * p.elem());
  w.lse_rounds = off; off += align256(slots * sizeof(float));
  w.sort_scratch = off; off += align256(sort_scratch_bytes(p));
  w.total = off;
  return w;
}

namespace {

// The forward pass in two halves over one workspace: hash and sort read only
// qk, so a caller whose v arrives later can start them first.
struct WsPtrs {
  int16_t* buckets;
  float* inv_norm;
  int32_t* perm;
  int32_t* undo;
  void* o_r;
  float* lse_r;
  void* sort_scratch;
};

WsPtrs ws_ptrs(const Problem& p, void* ws) {
  const Workspace w = workspace_layout(p);
  char* base = static_cast<char*>(ws);
  return {reinterpret_cast<int16_t*>(base + w.buckets),
          reinterpret_cast<float*>(base + w.inv_norm),
          reinterpret_cast<int32_t*>(base + w.perm),
          p.dedup ? reinterpret_cast<int32_t*>(base + w.undo) : nullptr,
          base + w.o_rounds,
          reinterpret_cast<float*>(base + w.lse_rounds),
          base + w.sort_scratch};
}

lsh_status forward_hash_sort(const Problem& p, const void* qk, const void* rot, void* ws,
                             cudaStream_t st) {
  const WsPtrs w = ws_ptrs(p, ws);
  CHECK(run_hash(p, qk, rot, w.buckets, w.inv_norm, st));
  return run_sort(p, w.buckets, w.perm, w.undo, nullptr, w.sort_scratch, st);
}

lsh_status forward_attend_combine(const Problem& p, const void* qk, const void* v, void* out,
                                  float* lse, void* ws, cudaStream_t st) {
  const WsPtrs w = ws_ptrs(p, ws);
  CHECK(run_attn(p, qk, v, w.inv_norm, w.perm, w.undo, w.buckets, w.o_r, w.lse_r, st));
  return run_combine(p, w.o_r, w.lse_r, out, lse, st);
}

}  // namespace

lsh_status forward_body(const Problem& p, const void* qk, const void* v, const void* rot,
                        void* out, float* lse, void* ws, cudaStream_t st) {
  CHECK(forward_hash_sort(p, qk, rot, ws, st));
  return forward_attend_combine(p, qk, v, out, lse, ws, st);
}

namespace {

// Device-buffer layout of lsh_attn_forward_host: qk, v, rotations, out, lse, workspace.
struct HostStaging {
  size_t qk, v, rot, out, lse, ws, total, in_bytes, rot_bytes, out_bytes, lse_bytes;
};

HostStaging host_layout(const Problem& p) {
  HostStaging h;
  h.in_bytes = (size_t)p.BH() * p.L * p.d * p.elem();
  h.rot_bytes = p.n_b > 1 ? (size_t)p.n_h * p.d * (p.kmeans ? p.n_b : p.half()) * p.elem() : 0;
  h.out_bytes = h.in_bytes;
  h.lse_bytes = (size_t)p.BH() * p.L * sizeof(float);
  size_t off = 0;
  h.qk = off;  off += align256(h.in_bytes);
  h.v = off;   off += align256(h.in_bytes);
  h.rot = off; off += align256(h.rot_bytes);
  h.out = off; off += align256(h.out_bytes);
  h.lse = off; off += align256(h.lse_bytes);
  h.ws = off;  off += workspace_layout(p).total;
  h.total = off;
  return h;
}

// The host-buffer pass is split into groups of (batch, head) pairs that flow
// through three streams: copies in, compute, copies out.  Group g's inputs
// cross PCIe while group g-1 is computed and group g-2's outputs come back;
// the compute stream runs the groups in order, so one workspace serves all.
// A group's qk is copied before its v, and its hash and sort (which read only
// qk) start as soon as qk has arrived.
constexpr int kMaxGroups = 8;
struct HostPipe {
  cudaStream_t in, comp, out;
  cudaEvent_t start, qk_done[kMaxGroups], in_done[kMaxGroups], comp_done[kMaxGroups], out_done;
  bool ok;
};
HostPipe g_pipe[kMaxDevices];
std::once_flag g_pipe_once[kMaxDevices];
std::mutex g_pipe_mutex[kMaxDevices];

HostPipe* host_pipe(int dev) {
  std::call_once(g_pipe_once[dev], [dev] {
    HostPipe& h = g_pipe[dev];
    h.ok = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) == cudaSuccess &&
           cudaStreamCreateWithFlags(&h.comp, cudaStreamNonBlocking) == cudaSuccess &&
           cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) == cudaSuccess &&
           cudaEventCreateWithFlags(&h.start, cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h.out_done, cudaEventDisableTiming) == cudaSuccess;
    for (int g = 0; h.ok && g < kMaxGroups; ++g)
      h.ok = cudaEventCreateWithFlags(&h.qk_done[g], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&h.in_done[g], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&h.comp_done[g], cudaEventDisableTiming) == cudaSuccess;
  });
  return g_pipe[dev].ok ? &g_pipe[dev] : nullptr;
}

// Queues every group's copy-in, forward pass and copy-out on the pipe's
// streams (host_pipe's comment gives the overlap).
lsh_status host_groups(const Problem& p, const HostStaging& h, HostPipe* hp, int G,
                       size_t row_in, size_t row_lse, const void* qk_host, const void* v_host,
                       const void* rotations_host, void* out_host, float* lse_host, char* base) {
  cudaError_t e;
  if (h.rot_bytes &&
      (e = cudaMemcpyAsync(base + h.rot, rotations_host, h.rot_bytes, cudaMemcpyHostToDevice,
                           hp->in)))
    return cuda_fail(e, "copy rotations to device");
  const int BH = p.BH();
  for (int g = 0; g < G; ++g) {
    const int b0 = (int)((long long)BH * g / G), b1 = (int)((long long)BH * (g + 1) / G);
    const size_t in_off = (size_t)b0 * row_in, in_len = (size_t)(b1 - b0) * row_in;
    const size_t l_off = (size_t)b0 * row_lse, l_len = (size_t)(b1 - b0) * row_lse;
    // one cudaMemcpyAsync per tensor slice
    if ((e = cudaMemcpyAsync(base + h.qk + in_off, static_cast<const char*>(qk_host) + in_off,
                             in_len, cudaMemcpyHostToDevice, hp->in)))
      return cuda_fail(e, "copy qk to device");
    if ((e = cudaEventRecord(hp->qk_done[g], hp->in))) return cuda_fail(e, "record copy-in");
    if ((e = cudaMemcpyAsync(base + h.v + in_off, static_cast<const char*>(v_host) + in_off,
                             in_len, cudaMemcpyHostToDevice, hp->in)))
      return cuda_fail(e, "copy v to device");
    if ((e = cudaEventRecord(hp->in_done[g], hp->in))) return cuda_fail(e, "record copy-in");
    Problem pg = p;
    pg.B = 1;
    pg.H = b1 - b0;
    // (the rotations were queued on the same stream before the first qk)
    if ((e = cudaStreamWaitEvent(hp->comp, hp->qk_done[g], 0))) return cuda_fail(e, "wait copy-in");
    CHECK(forward_hash_sort(pg, base + h.qk + in_off, h.rot_bytes ? base + h.rot : nullptr,
                            base + h.ws, hp->comp));
    if ((e = cudaStreamWaitEvent(hp->comp, hp->in_done[g], 0))) return cuda_fail(e, "wait copy-in");
    CHECK(forward_attend_combine(pg, base + h.qk + in_off, base + h.v + in_off,
                                 base + h.out + in_off,
                                 reinterpret_cast<float*>(base + h.lse + l_off), base + h.ws,
                                 hp->comp));
    if ((e = cudaEventRecord(hp->comp_done[g], hp->comp))) return cuda_fail(e, "record compute");
    if ((e = cudaStreamWaitEvent(hp->out, hp->comp_done[g], 0))) return cuda_fail(e, "wait compute");
    if ((e = cudaMemcpyAsync(static_cast<char*>(out_host) + in_off, base + h.out + in_off, in_len,
                             cudaMemcpyDeviceToHost, hp->out)))
      return cuda_fail(e, "copy out to host");
    if ((e = cudaMemcpyAsync(reinterpret_cast<char*>(lse_host) + l_off, base + h.lse + l_off,
                             l_len, cudaMemcpyDeviceToHost, hp->out)))
      return cuda_fail(e, "copy lse to host");
  }
  return LSH_OK;
}

// Makes `st` wait for everything queued on the three streams.  Each stream
// gets its own event record, so a stream whose queue ended early (a failed
// group) is joined as well; the first error is returned after all three.
cudaError_t join_pipe(HostPipe* hp, cudaStream_t st) {
  cudaError_t first = cudaSuccess;
  const cudaStream_t streams[3] = {hp->in, hp->comp, hp->out};
  for (cudaStream_t s : streams) {
    cudaError_t e = cudaEventRecord(hp->out_done, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, hp->out_done, 0);
    if (e != cudaSuccess && first == cudaSuccess) first = e;
  }
  return first;
}

}  // namespace

int sm_count() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    return 148;
  g_sm_count[dev].store(v, std::memory_order_relaxed);
  return v;
}

unsigned int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_word_once[dev], [dev] {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_device_error_word) == cudaSuccess)
      g_word_ptr[dev] = static_cast<unsigned int*>(ptr);
  });
  return g_word_ptr[dev];
}

}  // namespace lsh

using namespace lsh;

extern "C" {

lsh_status lsh_attn_hash(const lsh_shape* shape, const void* qk, const void* rotations,
                         int16_t* buckets, float* inv_norm, void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  CHECK(check_ptr(qk, "qk"));
  CHECK(check_rotations(p, rotations));
  CHECK(check_ptr(buckets, "buckets"));
  CHECK(check_ptr(inv_norm, "inv_norm"));
  return run_hash(p, qk, rotations, buckets, inv_norm, static_cast<cudaStream_t>(stream));
}

lsh_status lsh_attn_sort_workspace_size(const lsh_shape* shape, size_t* bytes) {
  Problem p;
  CHECK(to_problem(shape, &p));
  if (!bytes) return fail(LSH_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = sort_scratch_bytes(p);
  return LSH_OK;
}

lsh_status lsh_attn_sort(const lsh_shape* shape, const int16_t* buckets, int32_t* perm,
                         int32_t* undo, int32_t* counts, void* workspace, size_t workspace_bytes,
                         void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  CHECK(check_ptr(buckets, "buckets"));
  CHECK(check_ptr(perm, "perm"));
  CHECK(check_ptr(undo, "undo", true));
  CHECK(check_ptr(counts, "counts", true));
  CHECK(check_ptr(workspace, "workspace"));
  const size_t need = sort_scratch_bytes(p);
  if (workspace_bytes < need)
    return fail(LSH_ERR_WORKSPACE, "sort workspace of %zu bytes, need %zu", workspace_bytes, need);
  return run_sort(p, buckets, perm, undo, counts, workspace, static_cast<cudaStream_t>(stream));
}

lsh_status lsh_attn_chunked_fwd(const lsh_shape* shape, const void* qk, const void* v,
                                const float* inv_norm, const int32_t* perm, void* o_rounds,
                                float* lse_rounds, void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  CHECK(check_ptr(qk, "qk"));
  CHECK(check_ptr(v, "v"));
  CHECK(check_ptr(inv_norm, "inv_norm"));
  CHECK(check_ptr(perm, "perm"));
  CHECK(check_ptr(o_rounds, "o_rounds"));
  CHECK(check_ptr(lse_rounds, "lse_rounds"));
  if (p.dedup || p.bucket_mask)
    return fail(LSH_ERR_INVALID_ARG,
                "LSH_FLAG_DEDUP / LSH_FLAG_BUCKET_MASK need undo / buckets: "
                "call lsh_attn_chunked_fwd_ex");
  return run_attn(p, qk, v, inv_norm, perm, nullptr, nullptr, o_rounds, lse_rounds,
                  static_cast<cudaStream_t>(stream));
}

lsh_status lsh_attn_chunked_fwd_ex(const lsh_shape* shape, const void* qk, const void* v,
                                   const float* inv_norm, const int32_t* perm,
                                   const int32_t* undo, const int16_t* buckets, void* o_rounds,
                                   float* lse_rounds, void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  CHECK(check_ptr(qk, "qk"));
  CHECK(check_ptr(v, "v"));
  CHECK(check_ptr(inv_norm, "inv_norm"));
  CHECK(check_ptr(perm, "perm"));
  CHECK(check_ptr(undo, "undo", !p.dedup));
  CHECK(check_ptr(buckets, "buckets", !p.bucket_mask));
  CHECK(check_ptr(o_rounds, "o_rounds"));
  CHECK(check_ptr(lse_rounds, "lse_rounds"));
  return run_attn(p, qk, v, inv_norm, perm, undo, buckets, o_rounds, lse_rounds,
                  static_cast<cudaStream_t>(stream));
}

lsh_status lsh_attn_combine(const lsh_shape* shape, const void* o_rounds,
                            const float* lse_rounds, void* out, float* lse, void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  CHECK(check_ptr(o_rounds, "o_rounds"));
  CHECK(check_ptr(lse_rounds, "lse_rounds"));
  CHECK(check_ptr(out, "out"));
  CHECK(check_ptr(lse, "lse"));
  return run_combine(p, o_rounds, lse_rounds, out, lse, static_cast<cudaStream_t>(stream));
}

lsh_status lsh_attn_forward_workspace_size(const lsh_shape* shape, size_t* bytes) {
  Problem p;
  CHECK(to_problem(shape, &p));
  if (!bytes) return fail(LSH_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = workspace_layout(p).total;
  return LSH_OK;
}

lsh_status lsh_attn_forward(const lsh_shape* shape, const void* qk, const void* v,
                            const void* rotations, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  CHECK(check_ptr(qk, "qk"));
  CHECK(check_ptr(v, "v"));
  CHECK(check_rotations(p, rotations));
  CHECK(check_ptr(out, "out"));
  CHECK(check_ptr(lse, "lse"));
  CHECK(check_ptr(workspace, "workspace"));
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(LSH_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  const size_t need = workspace_layout(p).total;
  if (workspace_bytes < need)
    return fail(LSH_ERR_WORKSPACE, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  return forward_body(p, qk, v, rotations, out, lse, workspace,
                      static_cast<cudaStream_t>(stream));
}

lsh_status lsh_attn_forward_host_device_bytes(const lsh_shape* shape, size_t* bytes) {
  Problem p;
  CHECK(to_problem(shape, &p));
  if (!bytes) return fail(LSH_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = host_layout(p).total;
  return LSH_OK;
}

lsh_status lsh_attn_forward_host(const lsh_shape* shape, const void* qk_host,
                                 const void* v_host, const void* rotations_host,
                                 void* out_host, float* lse_host, void* device_buffer,
                                 size_t device_bytes, void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  if (!qk_host || !v_host || !out_host || !lse_host)
    return fail(LSH_ERR_INVALID_ARG, "a host buffer is NULL");
  if (p.n_b == 1 && rotations_host)
    return fail(LSH_ERR_INVALID_ARG, "rotations must be NULL when n_buckets == 1");
  if (p.n_b > 1 && !rotations_host) return fail(LSH_ERR_INVALID_ARG, "rotations_host is NULL");
  CHECK(check_ptr(device_buffer, "device_buffer"));
  if (reinterpret_cast<uintptr_t>(device_buffer) % 256)
    return fail(LSH_ERR_INVALID_ARG, "device_buffer is not 256-byte aligned");
  const HostStaging h = host_layout(p);
  if (device_bytes < h.total)
    return fail(LSH_ERR_WORKSPACE, "device_buffer of %zu bytes, need %zu", device_bytes, h.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(device_buffer);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LSH_ERR_UNSUPPORTED, "device %d", dev);
  HostPipe* hp = host_pipe(dev);
  if (!hp) return fail(LSH_ERR_CUDA, "could not create the copy/compute streams");
  // Calls on one device enqueue one at a time (the streams and events are shared).
  std::lock_guard<std::mutex> lock(g_pipe_mutex[dev]);
  const int BH = p.BH();
  const int G = BH < kMaxGroups ? BH : kMaxGroups;
  const size_t row_in = (size_t)p.L * p.d * p.elem();  // bytes of one (b, h) pair
  const size_t row_lse = (size_t)p.L * sizeof(float);
  // Everything starts after the work already on the caller's stream.
  if ((e = cudaEventRecord(hp->start, st))) return cuda_fail(e, "record start");
  if ((e = cudaStreamWaitEvent(hp->in, hp->start, 0))) return cuda_fail(e, "wait start");
  if ((e = cudaStreamWaitEvent(hp->comp, hp->start, 0))) return cuda_fail(e, "wait start");
  if ((e = cudaStreamWaitEvent(hp->out, hp->start, 0))) return cuda_fail(e, "wait start");
  const lsh_status r = host_groups(p, h, hp, G, row_in, row_lse, qk_host, v_host,
                                   rotations_host, out_host, lse_host, base);
  // The caller's stream continues once all three streams are done, on
  // success and on failure alike: the copies and kernels already queued
  // use the caller's buffers, which must stay alive until they finish.
  const cudaError_t je = join_pipe(hp, st);
  if (r != LSH_OK) return r;
  return je == cudaSuccess ? LSH_OK : cuda_fail(je, "join stream");
}

lsh_status lsh_attn_backward_workspace_size(const lsh_shape* shape, size_t* bytes) {
  Problem p;
  CHECK(to_problem(shape, &p));
  if (!bytes) return fail(LSH_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = backward_workspace_bytes(p);
  return LSH_OK;
}

lsh_status lsh_attn_backward(const lsh_shape* shape, const void* qk, const void* v,
                             const float* inv_norm, const int32_t* perm, const void* out,
                             const float* lse, const void* dout, float* dqk, float* dv,
                             void* workspace, size_t workspace_bytes, void* stream) {
  Problem p;
  CHECK(to_problem(shape, &p));
  if (p.dedup || p.bucket_mask)
    return fail(LSH_ERR_UNSUPPORTED, "the backward pass has no variant flags");
  CHECK(check_ptr(qk, "qk"));
  CHECK(check_ptr(v, "v"));
  CHECK(check_ptr(inv_norm, "inv_norm"));
  CHECK(check_ptr(perm, "perm"));
  CHECK(check_ptr(out, "out"));
  CHECK(check_ptr(lse, "lse"));
  CHECK(check_ptr(dout, "dout"));
  CHECK(check_ptr(dqk, "dqk"));
  CHECK(check_ptr(dv, "dv"));
  CHECK(check_ptr(workspace, "workspace"));
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(LSH_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  const size_t need = backward_workspace_bytes(p);
  if (workspace_bytes < need)
    return fail(LSH_ERR_WORKSPACE, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  cudaError_t e = launch_backward(p, qk, v, inv_norm, perm, out, lse, dout, dqk, dv, workspace,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LSH_OK : cuda_fail(e, "backward launch");
}

const char* lsh_attn_status_string(lsh_status status) {
  switch (status) {
    case LSH_OK: return "ok";
    case LSH_ERR_INVALID_ARG: return "invalid argument";
    case LSH_ERR_UNSUPPORTED: return "unsupported";
    case LSH_ERR_WORKSPACE: return "workspace too small";
    case LSH_ERR_CUDA: return "CUDA error";
    case LSH_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* lsh_attn_last_error(void) { return g_last_error; }

lsh_status lsh_attn_device_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned int* word = device_error_word();
  if (!word) return fail(LSH_ERR_CUDA, "cannot resolve the device error word");
  unsigned int v = 0;
  if ((e = cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "read device error word");
  if (v) {
    const unsigned int zero = 0;
    if ((e = cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice)) != cudaSuccess)
      return cuda_fail(e, "clear device error word");
    return fail(LSH_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait ran out (code 0x%x)", v);
  }
  return LSH_OK;
}

int lsh_attn_version(void) { return LSH_ATTN_VERSION; }

unsigned long long lsh_attn_test_hash_first_wait(unsigned long long ns) {
  return set_hash_first_wait_ns(ns);
}

unsigned long long lsh_attn_kernel_launches(void) {
  return g_launches.load(std::memory_order_relaxed);
}

}  // extern "C"
