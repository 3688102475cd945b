// Stage 3 on the 5th-generation tensor cores: chunked shared-QK attention of
// every hashing round, stored at original positions ("Reformer: The
// Efficient Transformer", section 2 "LSH attention" and "Causal masking";
// section 5 "Shared query-key space"; Appendix A "Implementation" and
// "Masking"), for bf16 inputs with d_k in {64, 128} and chunks of 64 or 128.
//
// A CTA walks a strip of consecutive 128-slot "steps" of one (b*h, round)
// segment in sorted order.  Step s has the queries of sorted slots
// [128 s, 128 s + 128) and the keys of slots [128 s - c, 128 s + 128): the
// previous c slots (look-back, none for s = 0) and the queries themselves.
// A query in chunk k sees key chunks k-1 and k; with c = 64 the first 64
// query rows (chunk 2s) see key columns [0, 128) and the last 64 (chunk
// 2s+1) see [64, 192); with c = 128 every row sees all 256 columns.
//
// Data flow per step (warp-specialised, 6 warps):
//   warp 0      producer: reads perm for the next 128 slots, gathers their
//               qk and v rows with cp.async into a ring of shared-memory
//               blocks (128B-swizzled operand layout), and stores each
//               row's position, key scale (1/||x|| * log2 e / sqrt(d)) and
//               query reference ||x|| * log2 e / sqrt(d);
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (two MMAs per
//               k-step: look-back keys and current keys live in different
//               blocks), then O = P V with P from shared memory;
//   warps 2..5  softmax: one query row per thread, straight from TMEM.
//               Keys are unit-normalised, so q . k_hat / sqrt(d) never
//               exceeds ||q|| / sqrt(d): that bound is the exponent's
//               reference (p = 2^(s' - ref) <= 1) and no row maximum is
//               needed; a row whose sum underflows is redone with its exact
//               maximum.  Masks: window, causal (key position > query
//               position), self (the key j == i is left out and a row with
//               no other key outputs v_i with lse -1e5, the value the -1e5
//               self score gives).  Then O / l and lse go to the row's
//               original position.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lsh {
namespace {

using namespace sm100;

constexpr int kQ = 128;             // queries per step = rows per block = MMA M
constexpr int kSoftWarps = 4;
constexpr int kThreads = (2 + kSoftWarps) * 32;
constexpr int kSmemLimit = 227 * 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// A row whose sum of 2^(s' - ref) falls below this is redone with its exact max.
constexpr float kTinySum = 1e-20f;

template <int C, int D>
struct Cfg {
  static constexpr int kNk = C + kQ;               // key columns per step
  static constexpr int kTile = kQ * D * 2;         // one 128-row bf16 tile
  static constexpr int kHalf = kQ * 128;           // one 64-wide atom column of a tile
  static constexpr int kPBytes = kQ * kNk * 2;     // P (bf16) of one step
  static constexpr int kNbuf = (kNk + D) * 2 <= 512 ? 2 : 1;
  static constexpr int kBufCols = kNbuf == 2 ? 256 : 512;
  static constexpr int kCpr = D / 8;               // 16-byte chunks per row
};

struct Params {
  const __nv_bfloat16* qk;
  const __nv_bfloat16* v;
  const float* inv_norm;
  const int32_t* perm;
  __nv_bfloat16* o_rounds;
  float* lse_rounds;
  unsigned int* err;
  int L, n_h, causal;
  int steps;          // ceil(L / 128) per segment
  int strip;          // steps per unit
  int n_strips;
  long long n_units;
  int slots, pbufs;   // ring depth, P buffers
  float ksc;          // log2 e / sqrt(d)
};

struct Layout {
  uint32_t qk, v, p, pos, ksc, qref, bars, misc, total;
};

template <int C, int D>
__host__ __device__ inline Layout layout(int slots, int pbufs) {
  using K = Cfg<C, D>;
  Layout l;
  uint32_t off = 0;
  l.qk = off;   off += slots * K::kTile;
  l.v = off;    off += slots * K::kTile;
  l.p = off;    off += pbufs * K::kPBytes;
  l.pos = off;  off += slots * kQ * 4;
  l.ksc = off;  off += slots * kQ * 4;
  l.qref = off; off += slots * kQ * 4;
  l.bars = off; off += (6 * slots + 4 * 2 + 2 * 2 + 2) * 8;
  l.misc = off; off += 16;
  l.total = off;
  return l;
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Shared-memory descriptor, MN-major, 128B swizzle: 64 contiguous elements
// of N per 128-byte row, K rows 128 B apart, 8-row groups `sbo` apart, the
// next 64 elements of N `lbo` bytes further.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t saddr, uint32_t lbo,
                                                        uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor with B MN-major (bit 16).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
  return idesc_bf16_f32(M, N) | (1u << 16);
}

struct Unit {
  int bh, r, s0, s1;
};

__device__ __forceinline__ Unit unit_of(const Params& p, long long u) {
  Unit x;
  const int strip = (int)(u % p.n_strips);
  const long long seg = u / p.n_strips;
  x.r = (int)(seg % p.n_h);
  x.bh = (int)(seg / p.n_h);
  x.s0 = strip * p.strip;
  x.s1 = min(p.steps, x.s0 + p.strip);
  return x;
}

template <int C, int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const Params p) {
  using K = Cfg<C, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const Layout Ly = layout<C, D>(p.slots, p.pbufs);
  uint8_t* qk_s = smem + Ly.qk;
  uint8_t* v_s = smem + Ly.v;
  uint8_t* p_s = smem + Ly.p;
  int* pos_s = reinterpret_cast<int*>(smem + Ly.pos);
  float* ksc_s = reinterpret_cast<float*>(smem + Ly.ksc);
  float* qref_s = reinterpret_cast<float*>(smem + Ly.qref);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  const int NS = p.slots, NP = p.pbufs;
  uint64_t* qk_full = bars;
  uint64_t* v_full = bars + NS;
  uint64_t* qk_empty = bars + 2 * NS;
  uint64_t* v_empty = bars + 3 * NS;
  uint64_t* s_full = bars + 6 * NS;   // [2]
  uint64_t* s_free = s_full + 2;      // [2]
  uint64_t* o_full = s_free + 2;      // [2]
  uint64_t* o_free = o_full + 2;      // [2]
  uint64_t* p_full = o_free + 2;      // [2]
  uint64_t* p_empty = p_full + 2;     // [2]
  uint64_t* done = p_empty + 2;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly.misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&qk_full[s], 32);
      mbar_init(&v_full[s], 32);
      mbar_init(&qk_empty[s], 1 + kSoftWarps);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kSoftWarps);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], kSoftWarps);
      mbar_init(&p_full[b], kSoftWarps);
      mbar_init(&p_empty[b], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const long long u_begin = blockIdx.x, u_step = gridDim.x;

  if (warp == 0) {
    // ================================================================ producer
    constexpr int RPI = 32 / K::kCpr;        // rows per warp instruction
    const int sub = lane / K::kCpr, kc = lane % K::kCpr;
    long long li = 0;  // load index (blocks loaded so far)
    bool ok = true;
    for (long long u = u_begin; ok && u < p.n_units; u += u_step) {
      const Unit U = unit_of(p, u);
      const int32_t* perm = p.perm + ((size_t)U.bh * p.n_h + U.r) * p.L;
      const __nv_bfloat16* qk = p.qk + (size_t)U.bh * p.L * D;
      const __nv_bfloat16* vv = p.v + (size_t)U.bh * p.L * D;
      const float* invn = p.inv_norm + (size_t)U.bh * p.L;
      for (int b = (U.s0 > 0 ? U.s0 - 1 : U.s0); b < U.s1; ++b, ++li) {
        const int slot = (int)(li % NS);
        const uint32_t ph = (uint32_t)((li / NS) & 1);
        if (!mbar_wait(&qk_empty[slot], ph ^ 1, abort_flag)) { ok = false; break; }
        int pos[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int row = lane + 32 * k;
          const int sl = b * kQ + row;
          const bool valid = sl < p.L;
          const int ps = valid ? perm[sl] : INT_MAX;
          pos[k] = ps;
          const float in = valid ? invn[ps] : 0.f;
          pos_s[slot * kQ + row] = ps;
          ksc_s[slot * kQ + row] = in * p.ksc;
          qref_s[slot * kQ + row] = in > 0.f ? p.ksc / in : 0.f;
        }
        const uint32_t qk_dst = smem_u32(qk_s + (size_t)slot * K::kTile);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          for (int it = 0; it < 32 / RPI; ++it) {
            const int row = k * 32 + it * RPI + sub;
            const int ps = __shfl_sync(0xffffffffu, pos[k], row & 31);
            const bool valid = ps != INT_MAX;
            const __nv_bfloat16* src = qk + (size_t)(valid ? ps : 0) * D + kc * 8;
            const uint32_t dst = qk_dst + (kc / 8) * K::kHalf + sw128_offset(row, (kc % 8) * 8);
            cp_async_16(dst, src, valid);
          }
        }
        cp_async_commit();
        if (!mbar_wait(&v_empty[slot], ph ^ 1, abort_flag)) { ok = false; cp_async_wait<0>(); break; }
        const uint32_t v_dst = smem_u32(v_s + (size_t)slot * K::kTile);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          for (int it = 0; it < 32 / RPI; ++it) {
            const int row = k * 32 + it * RPI + sub;
            const int ps = __shfl_sync(0xffffffffu, pos[k], row & 31);
            const bool valid = ps != INT_MAX;
            const __nv_bfloat16* src = vv + (size_t)(valid ? ps : 0) * D + kc * 8;
            const uint32_t dst = v_dst + (kc / 8) * K::kHalf + sw128_offset(row, (kc % 8) * 8);
            cp_async_16(dst, src, valid);
          }
        }
        cp_async_commit();
        cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(&qk_full[slot]);
        cp_async_wait<0>();
        fence_proxy_async_smem();
        mbar_arrive(&v_full[slot]);
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kErrWaitProducer);
      *abort_flag = 1;
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      long long li = 0, t = 0;  // blocks consumed, steps issued
      bool ok = true, issued = false;
      const uint32_t idesc_prev = idesc_bf16_f32(kQ, C);
      const uint32_t idesc_cur = idesc_bf16_f32(kQ, kQ);
      const uint32_t idesc_pv = idesc_bf16_f32_bmn(kQ, D);
      for (long long u = u_begin; ok && u < p.n_units; u += u_step) {
        const Unit U = unit_of(p, u);
        const bool lookback0 = U.s0 > 0;
        const long long first = li;
        li += (U.s1 - U.s0) + (lookback0 ? 1 : 0);
        for (int s = U.s0; s < U.s1; ++s, ++t) {
          const long long ci = first + (s - U.s0) + (lookback0 ? 1 : 0);  // current block
          const long long pi = ci - 1;                                    // look-back block
          const bool has_prev = s > 0;
          const int cs = (int)(ci % NS), ps = (int)(((pi % NS) + NS) % NS);
          const uint32_t cph = (uint32_t)((ci / NS) & 1), pph = (uint32_t)((pi / NS) & 1);
          const int buf = (int)(t % K::kNbuf);
          const uint32_t bph = (uint32_t)((t / K::kNbuf) & 1);
          const int pb = (int)(t % NP);
          const uint32_t pbph = (uint32_t)((t / NP) & 1);
          const uint32_t s_tmem = tmem_base + buf * K::kBufCols;
          const uint32_t o_tmem = s_tmem + K::kNk;
          // ---- S = Q K^T
          if (!mbar_wait(&s_free[buf], bph ^ 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&qk_full[cs], cph, abort_flag)) { ok = false; break; }
          if (has_prev && s == U.s0 && !mbar_wait(&qk_full[ps], pph, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t qa = smem_u32(qk_s + (size_t)cs * K::kTile);
          const uint32_t pa = smem_u32(qk_s + (size_t)ps * K::kTile) + (kQ - C) * 128;
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (uint32_t)(kk >> 2) * K::kHalf + (uint32_t)(kk & 3) * 32;
            const uint64_t a = sdesc_kmajor_sw128(qa + koff);
            if (has_prev)
              mma_bf16_ss(s_tmem, a, sdesc_kmajor_sw128(pa + koff), idesc_prev, kk > 0);
            mma_bf16_ss(s_tmem + C, a, sdesc_kmajor_sw128(qa + koff), idesc_cur, kk > 0);
          }
          issued = true;
          mma_commit(&s_full[buf]);
          if (has_prev) mma_commit(&qk_empty[ps]);
          if (s == U.s1 - 1) mma_commit(&qk_empty[cs]);
          // ---- O = P V
          if (!mbar_wait(&p_full[pb], pbph, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&o_free[buf], bph ^ 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&v_full[cs], cph, abort_flag)) { ok = false; break; }
          if (has_prev && s == U.s0 && !mbar_wait(&v_full[ps], pph, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t pbase = smem_u32(p_s + (size_t)pb * K::kPBytes);
          const uint32_t vcur = smem_u32(v_s + (size_t)cs * K::kTile);
          const uint32_t vprev = smem_u32(v_s + (size_t)ps * K::kTile) + (kQ - C) * 128;
          bool acc = false;
          for (int kk = has_prev ? 0 : C / 16; kk < K::kNk / 16; ++kk) {
            const uint64_t a =
                sdesc_kmajor_sw128(pbase + (kk >> 2) * (kQ * 128) + (kk & 3) * 32);
            const int key = kk * 16;  // key column of this k-step
            const uint32_t vb = key < C ? vprev + key * 128 : vcur + (key - C) * 128;
            const uint64_t b = sdesc_mnmajor_sw128(vb, K::kHalf, 1024);
            mma_bf16_ss(o_tmem, a, b, idesc_pv, acc ? 1u : 0u);
            acc = true;
          }
          mma_commit(&o_full[buf]);
          mma_commit(&p_empty[pb]);
          if (has_prev) mma_commit(&v_empty[ps]);
          if (s == U.s1 - 1) mma_commit(&v_empty[cs]);
        }
      }
      if (!ok) {
        atomicOr(p.err, kErrWaitMma);
        *abort_flag = 1;
      }
      if (issued) {
        mma_commit(done);
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(done, 0)) {
          if (globaltimer() - t0 > kWaitLimitNs) { atomicOr(p.err, kErrWaitDrain); break; }
        }
      }
    }
  } else {
    // ================================================================ softmax
    const int quad = warp & 3;
    const int m = quad * 32 + lane;  // query row in the step
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    // window columns of this row: c = 64 -> [0,128) or [64,192); c = 128 -> [0,256)
    const int win_lo = (C == 64 && quad >= 2) ? 64 : 0;
    const int win_hi = (C == 64 && quad < 2) ? 128 : K::kNk;
    long long li = 0, t = 0;
    bool ok = true;
    for (long long u = u_begin; ok && u < p.n_units; u += u_step) {
      const Unit U = unit_of(p, u);
      const bool lookback0 = U.s0 > 0;
      const long long first = li;
      li += (U.s1 - U.s0) + (lookback0 ? 1 : 0);
      __nv_bfloat16* o_out = p.o_rounds + ((size_t)U.bh * p.n_h + U.r) * p.L * D;
      float* lse_out = p.lse_rounds + ((size_t)U.bh * p.n_h + U.r) * p.L;
      const __nv_bfloat16* vsrc = p.v + (size_t)U.bh * p.L * D;
      for (int s = U.s0; s < U.s1; ++s, ++t) {
        const long long ci = first + (s - U.s0) + (lookback0 ? 1 : 0);
        const long long pi = ci - 1;
        const bool has_prev = s > 0;
        const int cs = (int)(ci % NS), ps = (int)(((pi % NS) + NS) % NS);
        const uint32_t cph = (uint32_t)((ci / NS) & 1);
        const int buf = (int)(t % K::kNbuf);
        const uint32_t bph = (uint32_t)((t / K::kNbuf) & 1);
        const int pb = (int)(t % NP);
        const uint32_t pbph = (uint32_t)((t / NP) & 1);
        const uint32_t s_tmem = tmem_base + lane_off + buf * K::kBufCols;
        const uint32_t o_tmem = s_tmem + K::kNk;
        // Metadata of this step's blocks is published with qk_full.
        if (!mbar_wait(&qk_full[cs], cph, abort_flag)) { ok = false; break; }
        if (has_prev && s == U.s0 &&
            !mbar_wait(&qk_full[ps], (uint32_t)((pi / NS) & 1), abort_flag)) { ok = false; break; }
        if (!mbar_wait(&s_full[buf], bph, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        const int qpos = pos_s[cs * kQ + m];
        const bool q_valid = qpos != INT_MAX;
        const float qref = qref_s[cs * kQ + m];
        const int qlim = p.causal ? qpos : INT_MAX - 1;
        const int lo = has_prev ? win_lo : max(win_lo, C);
        // Key metadata: column j < C is look-back row (128 - C + j) of block
        // ps, column j >= C is row (j - C) of block cs.
        auto kmeta = [&](int j, int& kp, float& ks) {
          const int idx = j < C ? ps * kQ + (kQ - C) + j : cs * kQ + (j - C);
          kp = pos_s[idx];
          ks = ksc_s[idx];
        };
        if (!mbar_wait(&p_empty[pb], pbph ^ 1, abort_flag)) { ok = false; break; }
        uint8_t* prow = p_s + (size_t)pb * K::kPBytes;
        float l = 0.f;
        bool any = false;
        for (int j0 = 0; j0 < K::kNk; j0 += 32) {
          uint32_t pk[16];
          if (j0 >= lo && j0 < win_hi) {
            uint32_t sv[32];
            __syncwarp();
            tmem_ld_32x32b_x32(s_tmem + j0, sv);
            tmem_ld_wait(sv);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float pr[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                int kp;
                float ks;
                kmeta(j0 + e + h, kp, ks);
                const bool valid = kp <= qlim && kp != qpos;
                any |= valid;
                const float x = fmaf(__uint_as_float(sv[e + h]), ks, -qref);
                pr[h] = valid ? ex2(x) : 0.f;
                l += pr[h];
              }
              pk[e / 2] = pack_bf16(pr[0], pr[1]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = 0u;
          }
          uint8_t* base = prow + (j0 / 64) * (kQ * 128);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int k = (j0 % 64) + q * 8;
            *reinterpret_cast<uint4*>(base + sw128_offset(m, k)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        // Underflow: redo the row with its exact maximum as the reference.
        float ref2 = qref;
        const bool redo = any && !(l >= kTinySum);
        if (__any_sync(0xffffffffu, redo)) {
          float mx = -INFINITY;
          for (int j0 = lo & ~31; j0 < win_hi; j0 += 32) {
            uint32_t sv[32];
            __syncwarp();
            tmem_ld_32x32b_x32(s_tmem + j0, sv);
            tmem_ld_wait(sv);
            for (int e = 0; e < 32; ++e) {
              int kp;
              float ks;
              kmeta(j0 + e, kp, ks);
              if (j0 + e >= lo && kp <= qlim && kp != qpos)
                mx = fmaxf(mx, __uint_as_float(sv[e]) * ks);
            }
          }
          if (redo) { ref2 = mx; l = 0.f; }
          for (int j0 = lo & ~31; j0 < win_hi; j0 += 32) {
            uint32_t sv[32];
            __syncwarp();
            tmem_ld_32x32b_x32(s_tmem + j0, sv);
            tmem_ld_wait(sv);
            if (redo) {
              uint8_t* base = prow + (j0 / 64) * (kQ * 128);
              for (int e = 0; e < 32; e += 8) {
                uint32_t w[4];
                for (int h = 0; h < 8; h += 2) {
                  float pr[2];
                  for (int g = 0; g < 2; ++g) {
                    int kp;
                    float ks;
                    kmeta(j0 + e + h + g, kp, ks);
                    const bool valid = j0 + e + h + g >= lo && kp <= qlim && kp != qpos;
                    pr[g] = valid ? ex2(fmaf(__uint_as_float(sv[e + h + g]), ks, -ref2)) : 0.f;
                    l += pr[g];
                  }
                  w[h / 2] = pack_bf16(pr[0], pr[1]);
                }
                *reinterpret_cast<uint4*>(base + sw128_offset(m, (j0 % 64) + e)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
        tc_fence_before_sync();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s_free[buf]);
          mbar_arrive(&p_full[pb]);
        }
        // ---- O / l to the row's original position
        if (!mbar_wait(&o_full[buf], bph, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        const float inv_l = any ? 1.f / l : 0.f;
        __nv_bfloat16* orow = o_out + (size_t)(q_valid ? qpos : 0) * D;
#pragma unroll
        for (int d0 = 0; d0 < D; d0 += 32) {
          uint32_t ov[32];
          __syncwarp();
          tmem_ld_32x32b_x32(o_tmem + d0, ov);
          tmem_ld_wait(ov);
          if (q_valid) {
            if (any) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 w;
                w.x = pack_bf16(__uint_as_float(ov[8 * q + 0]) * inv_l,
                                __uint_as_float(ov[8 * q + 1]) * inv_l);
                w.y = pack_bf16(__uint_as_float(ov[8 * q + 2]) * inv_l,
                                __uint_as_float(ov[8 * q + 3]) * inv_l);
                w.z = pack_bf16(__uint_as_float(ov[8 * q + 4]) * inv_l,
                                __uint_as_float(ov[8 * q + 5]) * inv_l);
                w.w = pack_bf16(__uint_as_float(ov[8 * q + 6]) * inv_l,
                                __uint_as_float(ov[8 * q + 7]) * inv_l);
                *reinterpret_cast<uint4*>(orow + d0 + 8 * q) = w;
              }
            } else {
              // nothing but itself to attend to: the -1e5 self score makes it v_i
              const uint4* vr = reinterpret_cast<const uint4*>(vsrc + (size_t)qpos * D + d0);
              uint4* dst = reinterpret_cast<uint4*>(orow + d0);
#pragma unroll
              for (int q = 0; q < 4; ++q) dst[q] = vr[q];
            }
          }
        }
        if (q_valid)
          lse_out[qpos] = any ? (redo ? ref2 * kLn2 : qref * kLn2) + logf(l) : kSelfScore;
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&o_free[buf]);
          if (has_prev) mbar_arrive(&qk_empty[ps]);
          if (s == U.s1 - 1) mbar_arrive(&qk_empty[cs]);
        }
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kErrWaitEpilogue);
      *abort_flag = 1;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

template <int C, int D>
bool plan(const Problem& pr, int* slots, int* pbufs, size_t* smem) {
  for (int ns = 3; ns >= 2; --ns)
    for (int np = 2; np >= 1; --np) {
      const size_t t = layout<C, D>(ns, np).total + 1024;
      if (t <= (size_t)kSmemLimit) {
        *slots = ns;
        *pbufs = np;
        *smem = std::max<size_t>(t, 116 * 1024);
        return true;
      }
    }
  return false;
}

}  // namespace

bool attn_tc_supported(const Problem& p) {
  return p.bf16 && (p.d == 64 || p.d == 128) && (p.c == 64 || p.c == 128);
}

template <int C, int D>
static cudaError_t launch_cd(const Problem& pr, const void* qk, const void* v,
                             const float* inv_norm, const int32_t* perm, void* o_rounds,
                             float* lse_rounds, cudaStream_t st) {
  Params p;
  size_t smem = 0;
  if (!plan<C, D>(pr, &p.slots, &p.pbufs, &smem)) return cudaErrorNotSupported;
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorUnknown;
  p.qk = static_cast<const __nv_bfloat16*>(qk);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.inv_norm = inv_norm;
  p.perm = perm;
  p.o_rounds = static_cast<__nv_bfloat16*>(o_rounds);
  p.lse_rounds = lse_rounds;
  p.err = err;
  p.L = pr.L;
  p.n_h = pr.n_h;
  p.causal = pr.causal ? 1 : 0;
  p.steps = (pr.L + kQ - 1) / kQ;
  const long long segs = (long long)pr.BH() * pr.n_h;
  const long long total = segs * p.steps;
  // About six strips per SM, each at least two steps.
  int strip = (int)std::max<long long>(2, total / (148LL * 6));
  strip = std::min(strip, p.steps);
  p.strip = strip;
  p.n_strips = (p.steps + strip - 1) / strip;
  p.n_units = segs * p.n_strips;
  p.ksc = kLog2e / sqrtf((float)pr.d);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<C, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)std::min<long long>(148, p.n_units);
  attn_tc_kernel<C, D><<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const Problem& p, const void* qk, const void* v, const float* inv_norm,
                           const int32_t* perm, void* o_rounds, float* lse_rounds,
                           cudaStream_t st) {
  if (p.c == 64 && p.d == 64)
    return launch_cd<64, 64>(p, qk, v, inv_norm, perm, o_rounds, lse_rounds, st);
  if (p.c == 64 && p.d == 128)
    return launch_cd<64, 128>(p, qk, v, inv_norm, perm, o_rounds, lse_rounds, st);
  if (p.c == 128 && p.d == 64)
    return launch_cd<128, 64>(p, qk, v, inv_norm, perm, o_rounds, lse_rounds, st);
  if (p.c == 128 && p.d == 128)
    return launch_cd<128, 128>(p, qk, v, inv_norm, perm, o_rounds, lse_rounds, st);
  return cudaErrorNotSupported;
}

}  // namespace lsh
