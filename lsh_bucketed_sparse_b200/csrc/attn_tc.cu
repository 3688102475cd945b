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
// Data flow per step (warp-specialised, 11 warps):
//   warp 0      qk producer: reads perm for the next 128 slots and gathers
//               their qk rows with TMA (tile::gather4, four rows per lane
//               and instruction) into a ring of shared-memory blocks in the
//               128B-swizzled operand layout, and stores each row's
//               position, key scale (1/||x|| * log2 e / sqrt(d)) and query
//               reference ||x|| * log2 e / sqrt(d);
//   warp 10     v producer: the same gathers from v, so that keys never wait
//               for values;
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (two MMAs per
//               k-step: look-back keys and current keys live in different
//               blocks), then O = P V with P from shared memory;
//   warps 2..9  softmax: two warps per TMEM lane quadrant (32 query rows),
//               each taking alternate 32-key chunks of the row, straight
//               from TMEM.  Keys are unit-normalised, so q . k_hat / sqrt(d)
//               never exceeds ||q|| / sqrt(d): that bound is the exponent's
//               reference (p = 2^(s' - ref) <= 1), so no row maximum is
//               needed and the two warps only add their partial sums; a row
//               whose sum underflows is redone with its exact maximum.
//               Masks: window, causal (key position > query position), self
//               (the key j == i is left out and a row with no other key
//               outputs v_i with lse -1e5, the value the -1e5 self score
//               gives).  Then O / l (each warp half of the columns) and lse
//               go to the row's original position.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lsh {
namespace {

using namespace sm100;

constexpr int kQ = 128;             // queries per step = rows per block = MMA M
constexpr int kSoftWarps = 8;
constexpr int kThreads = (3 + kSoftWarps) * 32;   // qk producer, MMA, softmax, v producer
constexpr int kVWarp = 2 + kSoftWarps;
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
  uint32_t qk, v, p, pos, ksc, qref, xch, bars, misc, total;
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
  l.xch = off;  off += (2 * 2 + 2 + 2) * kQ * 4;   // partial sums [2][2], maxima [2], redo sums [2]
  l.bars = off; off += (4 * slots + 6 * 2 + 2 + 4 + 1) * 8;
  l.misc = off; off += 16;
  l.total = off;
  return l;
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

// Positions of sorted slots sl .. sl+3 (INT_MAX past the end of the segment).
__device__ __forceinline__ void load_positions(const int32_t* perm, int sl, int L, int* pos) {
  if (sl + 3 < L) {
    const int4 v = *reinterpret_cast<const int4*>(perm + sl);
    pos[0] = v.x; pos[1] = v.y; pos[2] = v.z; pos[3] = v.w;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) pos[k] = sl + k < L ? perm[sl + k] : INT_MAX;
  }
}

// Row of the [B*H*L, d] view that holds position `pos`; a row past the end
// of the tensor for a missing position, which the gather fills with zeros.
__device__ __forceinline__ int gather_row(int rowbase, int pos) {
  return pos == INT_MAX ? INT_MAX : rowbase + pos;
}

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
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap vmap,
               const Params p) {
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
  uint64_t* s_full = bars + 4 * NS;   // [2]
  uint64_t* s_free = s_full + 2;      // [2]
  uint64_t* o_full = s_free + 2;      // [2]
  uint64_t* o_free = o_full + 2;      // [2]
  uint64_t* p_full = o_free + 2;      // [2]
  uint64_t* p_empty = p_full + 2;     // [2]
  uint64_t* xbar = p_empty + 2;       // [2] partial-sum exchange, all softmax warps
  uint64_t* rbar = xbar + 2;          // [4] redo exchange, the two warps of a quadrant
  uint64_t* done = rbar + 4;          // [1]
  float* xl = reinterpret_cast<float*>(smem + Ly.xch);   // [2 buf][2 half][kQ]
  float* xm = xl + 4 * kQ;                               // [2 half][kQ]
  float* xl2 = xm + 2 * kQ;                              // [2 half][kQ]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly.misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&qk_full[s], 32);
      mbar_init(&v_full[s], 32);
      // released by the MMA (keys used) and the softmax warps (metadata used)
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
      mbar_init(&xbar[b], kSoftWarps);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&rbar[q], 2);
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
    // ================================================================ qk producer
    // Lane l owns rows 4l .. 4l+3 of every block.
    long long li = 0;  // load index (blocks loaded so far)
    bool ok = true;
    if (lane == 0) tma_prefetch_desc(&qmap);
    for (long long u = u_begin; ok && u < p.n_units; u += u_step) {
      const Unit U = unit_of(p, u);
      const int32_t* perm = p.perm + ((size_t)U.bh * p.n_h + U.r) * p.L;
      const float* invn = p.inv_norm + (size_t)U.bh * p.L;
      const int rowbase = U.bh * p.L;
      for (int b = (U.s0 > 0 ? U.s0 - 1 : U.s0); b < U.s1; ++b, ++li) {
        const int slot = (int)(li % NS);
        const uint32_t ph = (uint32_t)((li / NS) & 1);
        int pos[4];
        load_positions(perm, b * kQ + 4 * lane, p.L, pos);
        if (!mbar_wait(&qk_empty[slot], ph ^ 1, abort_flag)) { ok = false; break; }
        if (lane == 0) mbar_expect_tx(&qk_full[slot], K::kTile);
        __syncwarp();
        uint8_t* dst = qk_s + (size_t)slot * K::kTile + lane * 512;
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_gather4(dst + h * K::kHalf, &qmap, &qk_full[slot], h * 64,
                      gather_row(rowbase, pos[0]), gather_row(rowbase, pos[1]),
                      gather_row(rowbase, pos[2]), gather_row(rowbase, pos[3]));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int row = 4 * lane + k;
          const float in = pos[k] != INT_MAX ? invn[pos[k]] : 0.f;
          pos_s[slot * kQ + row] = pos[k];
          ksc_s[slot * kQ + row] = in * p.ksc;
          qref_s[slot * kQ + row] = in > 0.f ? p.ksc / in : 0.f;
        }
        mbar_arrive(&qk_full[slot]);
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
      // Block load index of step s of a unit whose first block has index `first`.
      auto cur_index = [](const Unit& U, long long first, int s) {
        return first + (s - U.s0) + (U.s0 > 0 ? 1 : 0);
      };
      // S(s) = Q K^T into the step's TMEM buffer.
      auto issue_qk = [&](const Unit& U, long long first, int s, long long ts) -> bool {
        const long long ci = cur_index(U, first, s), pi = ci - 1;
        const bool has_prev = s > 0;
        const int cs = (int)(ci % NS), ps = (int)(((pi % NS) + NS) % NS);
        const int buf = (int)(ts % K::kNbuf);
        const uint32_t bph = (uint32_t)((ts / K::kNbuf) & 1);
        if (!mbar_wait(&s_free[buf], bph ^ 1, abort_flag)) return false;
        if (!mbar_wait(&qk_full[cs], (uint32_t)((ci / NS) & 1), abort_flag)) return false;
        if (has_prev && s == U.s0 &&
            !mbar_wait(&qk_full[ps], (uint32_t)((pi / NS) & 1), abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t s_tmem = tmem_base + buf * K::kBufCols;
        const uint32_t qa = smem_u32(qk_s + (size_t)cs * K::kTile);
        const uint32_t pa = smem_u32(qk_s + (size_t)ps * K::kTile) + (kQ - C) * 128;
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (uint32_t)(kk >> 2) * K::kHalf + (uint32_t)(kk & 3) * 32;
          const uint64_t a = sdesc_kmajor_sw128(qa + koff);
          if (has_prev)
            mma_bf16_ss(s_tmem, a, sdesc_kmajor_sw128(pa + koff), idesc_prev, kk > 0);
          mma_bf16_ss(s_tmem + C, a, sdesc_kmajor_sw128(qa + koff), idesc_cur, kk > 0);
        }
        mma_commit(&s_full[buf]);
        if (has_prev) mma_commit(&qk_empty[ps]);
        if (s == U.s1 - 1) mma_commit(&qk_empty[cs]);
        return true;
      };
      // O(s) = P(s) V once the softmax has written P(s).
      auto issue_pv = [&](const Unit& U, long long first, int s, long long ts) -> bool {
        const long long ci = cur_index(U, first, s), pi = ci - 1;
        const bool has_prev = s > 0;
        const int cs = (int)(ci % NS), ps = (int)(((pi % NS) + NS) % NS);
        const int buf = (int)(ts % K::kNbuf);
        const uint32_t bph = (uint32_t)((ts / K::kNbuf) & 1);
        const int pb = (int)(ts % NP);
        if (!mbar_wait(&p_full[pb], (uint32_t)((ts / NP) & 1), abort_flag)) return false;
        if (!mbar_wait(&o_free[buf], bph ^ 1, abort_flag)) return false;
        if (!mbar_wait(&v_full[cs], (uint32_t)((ci / NS) & 1), abort_flag)) return false;
        if (has_prev && s == U.s0 &&
            !mbar_wait(&v_full[ps], (uint32_t)((pi / NS) & 1), abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t o_tmem = tmem_base + buf * K::kBufCols + K::kNk;
        const uint32_t pbase = smem_u32(p_s + (size_t)pb * K::kPBytes);
        const uint32_t vcur = smem_u32(v_s + (size_t)cs * K::kTile);
        const uint32_t vprev = smem_u32(v_s + (size_t)ps * K::kTile) + (kQ - C) * 128;
        bool acc = false;
        for (int kk = has_prev ? 0 : C / 16; kk < K::kNk / 16; ++kk) {
          const uint64_t a = sdesc_kmajor_sw128(pbase + (kk >> 2) * (kQ * 128) + (kk & 3) * 32);
          const int key = kk * 16;  // key column of this k-step
          const uint32_t vb = key < C ? vprev + key * 128 : vcur + (key - C) * 128;
          mma_bf16_ss(o_tmem, a, sdesc_mnmajor_sw128(vb, K::kHalf, 1024), idesc_pv,
                      acc ? 1u : 0u);
          acc = true;
        }
        mma_commit(&o_full[buf]);
        mma_commit(&p_empty[pb]);
        if (has_prev) mma_commit(&v_empty[ps]);
        if (s == U.s1 - 1) mma_commit(&v_empty[cs]);
        return true;
      };
      for (long long u = u_begin; ok && u < p.n_units; u += u_step) {
        const Unit U = unit_of(p, u);
        const long long first = li;
        li += (U.s1 - U.s0) + (U.s0 > 0 ? 1 : 0);
        // S of the next step is computed while the softmax works on this one.
        if (!issue_qk(U, first, U.s0, t)) { ok = false; break; }
        issued = true;
        for (int s = U.s0; s < U.s1; ++s, ++t) {
          if (s + 1 < U.s1 && !issue_qk(U, first, s + 1, t + 1)) { ok = false; break; }
          if (!issue_pv(U, first, s, t)) { ok = false; break; }
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
  } else if (warp == kVWarp) {
    // ================================================================ v producer
    long long li = 0;
    bool ok = true;
    if (lane == 0) tma_prefetch_desc(&vmap);
    for (long long u = u_begin; ok && u < p.n_units; u += u_step) {
      const Unit U = unit_of(p, u);
      const int32_t* perm = p.perm + ((size_t)U.bh * p.n_h + U.r) * p.L;
      const int rowbase = U.bh * p.L;
      for (int b = (U.s0 > 0 ? U.s0 - 1 : U.s0); b < U.s1; ++b, ++li) {
        const int slot = (int)(li % NS);
        const uint32_t ph = (uint32_t)((li / NS) & 1);
        int pos[4];
        load_positions(perm, b * kQ + 4 * lane, p.L, pos);
        if (!mbar_wait(&v_empty[slot], ph ^ 1, abort_flag)) { ok = false; break; }
        if (lane == 0) mbar_expect_tx(&v_full[slot], K::kTile);
        __syncwarp();
        uint8_t* dst = v_s + (size_t)slot * K::kTile + lane * 512;
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_gather4(dst + h * K::kHalf, &vmap, &v_full[slot], h * 64,
                      gather_row(rowbase, pos[0]), gather_row(rowbase, pos[1]),
                      gather_row(rowbase, pos[2]), gather_row(rowbase, pos[3]));
        mbar_arrive(&v_full[slot]);
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kErrWaitProducer);
      *abort_flag = 1;
    }
  } else {
    // ================================================================ softmax
    const int sw = warp - 2;
    const int quad = warp & 3;
    const int half = sw >> 2;        // which alternate 32-key chunks this warp takes
    const int m = quad * 32 + lane;  // query row in the step
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    // window columns of this row: c = 64 -> [0,128) or [64,192); c = 128 -> [0,256)
    const int win_lo = (C == 64 && quad >= 2) ? 64 : 0;
    const int win_hi = (C == 64 && quad < 2) ? 128 : K::kNk;
    long long li = 0, t = 0;
    uint32_t rph = 0;  // phase of this quadrant's redo barrier
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
        // metadata row of key column j0 (a multiple of 32, all in one block)
        auto kbase = [&](int j0) { return j0 < C ? ps * kQ + (kQ - C) + j0 : cs * kQ + (j0 - C); };
        if (!mbar_wait(&p_empty[pb], pbph ^ 1, abort_flag)) { ok = false; break; }
        uint8_t* prow = p_s + (size_t)pb * K::kPBytes;
        float l = 0.f;
        bool any = false;
        for (int j0 = half * 32; j0 < K::kNk; j0 += 64) {
          uint32_t pk[16];
          if (j0 >= lo && j0 < win_hi) {
            uint32_t sv[32];
            __syncwarp();
            tmem_ld_32x32b_x32(s_tmem + j0, sv);
            tmem_ld_wait(sv);
            const int kb = kbase(j0);
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const int4 kp = *reinterpret_cast<const int4*>(pos_s + kb + e);
              const float4 ks = *reinterpret_cast<const float4*>(ksc_s + kb + e);
              const int kpa[4] = {kp.x, kp.y, kp.z, kp.w};
              const float ksa[4] = {ks.x, ks.y, ks.z, ks.w};
              float pr[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const bool valid = kpa[h] <= qlim && kpa[h] != qpos;
                any |= valid;
                const float x = fmaf(__uint_as_float(sv[e + h]), ksa[h], -qref);
                pr[h] = valid ? ex2(x) : 0.f;
                l += pr[h];
              }
              pk[e / 2] = pack_bf16(pr[0], pr[1]);
              pk[e / 2 + 1] = pack_bf16(pr[2], pr[3]);
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
        // The two warps of the quadrant add their partial sums (any key seen is
        // carried as l >= 0, none as -1).
        const int xb = (int)(t & 1);
        xl[(xb * 2 + half) * kQ + m] = any ? l : -1.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xbar[xb]);
        if (!mbar_wait(&xbar[xb], (uint32_t)((t >> 1) & 1), abort_flag)) { ok = false; break; }
        const float lo_part = xl[(xb * 2 + (half ^ 1)) * kQ + m];
        any = any || lo_part >= 0.f;
        float lt = l + fmaxf(lo_part, 0.f);
        float ref = qref;
        // Underflow of every term: redo the row with its exact maximum.
        const bool redo = any && !(lt >= kTinySum);
        if (__any_sync(0xffffffffu, redo)) {
          float mx = -INFINITY;
          for (int j0 = half * 32; j0 < K::kNk; j0 += 64) {
            if (j0 < lo || j0 >= win_hi) continue;
            uint32_t sv[32];
            __syncwarp();
            tmem_ld_32x32b_x32(s_tmem + j0, sv);
            tmem_ld_wait(sv);
            const int kb = kbase(j0);
            for (int e = 0; e < 32; ++e) {
              const int kp = pos_s[kb + e];
              if (kp <= qlim && kp != qpos)
                mx = fmaxf(mx, __uint_as_float(sv[e]) * ksc_s[kb + e]);
            }
          }
          xm[half * kQ + m] = mx;
          __syncwarp();
          if (lane == 0) mbar_arrive(&rbar[quad]);
          if (!mbar_wait(&rbar[quad], rph, abort_flag)) { ok = false; break; }
          rph ^= 1;
          const float gmax = fmaxf(mx, xm[(half ^ 1) * kQ + m]);
          float l2 = 0.f;
          for (int j0 = half * 32; j0 < K::kNk; j0 += 64) {
            if (j0 < lo || j0 >= win_hi) continue;
            uint32_t sv[32];
            __syncwarp();
            tmem_ld_32x32b_x32(s_tmem + j0, sv);
            tmem_ld_wait(sv);
            if (!redo) continue;
            const int kb = kbase(j0);
            uint8_t* base = prow + (j0 / 64) * (kQ * 128);
            for (int e = 0; e < 32; e += 8) {
              uint32_t w[4];
              for (int h = 0; h < 8; h += 2) {
                float pr[2];
                for (int g = 0; g < 2; ++g) {
                  const int kp = pos_s[kb + e + h + g];
                  const bool valid = kp <= qlim && kp != qpos;
                  pr[g] = valid ? ex2(fmaf(__uint_as_float(sv[e + h + g]), ksc_s[kb + e + h + g],
                                           -gmax))
                                : 0.f;
                  l2 += pr[g];
                }
                w[h / 2] = pack_bf16(pr[0], pr[1]);
              }
              *reinterpret_cast<uint4*>(base + sw128_offset(m, (j0 % 64) + e)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
          xl2[half * kQ + m] = l2;
          __syncwarp();
          if (lane == 0) mbar_arrive(&rbar[quad]);
          if (!mbar_wait(&rbar[quad], rph, abort_flag)) { ok = false; break; }
          rph ^= 1;
          if (redo) {
            lt = l2 + xl2[(half ^ 1) * kQ + m];
            ref = gmax;
          }
        }
        tc_fence_before_sync();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s_free[buf]);
          mbar_arrive(&p_full[pb]);
          // the look-back block's metadata is not needed again, nor this
          // block's at the strip's last step (qpos and qref are in registers)
          if (has_prev) mbar_arrive(&qk_empty[ps]);
          if (s == U.s1 - 1) mbar_arrive(&qk_empty[cs]);
        }
        // ---- O / l to the row's original position: this warp's half of the columns
        if (!mbar_wait(&o_full[buf], bph, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        const float inv_l = any ? 1.f / lt : 0.f;
        __nv_bfloat16* orow = o_out + (size_t)(q_valid ? qpos : 0) * D;
#pragma unroll
        for (int d0 = half * (D / 2); d0 < (half + 1) * (D / 2); d0 += 32) {
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
        if (q_valid && half == 0) lse_out[qpos] = any ? ref * kLn2 + logf(lt) : kSelfScore;
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[buf]);
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
  return p.bf16 && (p.d == 64 || p.d == 128) && (p.c == 64 || p.c == 128) &&
         (long long)p.BH() * p.L < (1LL << 31) - 1 && sm100::tensor_map_encoder() != nullptr;
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
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  // [B*H*L, d] views of qk and v: boxes of one row of 64 elements (128 B),
  // 128B swizzle, rows outside the tensor read as zeros.
  CUtensorMap maps[2];
  const void* bases[2] = {qk, v};
  for (int k = 0; k < 2; ++k) {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)pr.BH() * pr.L};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 1};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&maps[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(bases[k]), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<C, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)std::min<long long>(148, p.n_units);
  attn_tc_kernel<C, D><<<grid, kThreads, smem, st>>>(maps[0], maps[1], p);
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
