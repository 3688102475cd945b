// Stage 1 on the 5th-generation tensor cores: the random-rotation hash
// h(x) = argmax([xR; -xR]) of every round ("Reformer: The Efficient
// Transformer", section 2 "LSH attention"; Appendix A, one rotation per
// round) and 1/||x|| (section 5, normalised keys), for bf16 inputs.
//
// The projections x.R are a GEMM (tokens x d) x (d x n_b/2 per round) on
// tcgen05 with fp32 accumulators in TMEM; the argmax is a fused epilogue that
// reads TMEM and never writes the projections anywhere.
//
// Work split: the rounds are cut into groups whose rotations fit in shared
// memory (at most kRBudget bytes); each CTA owns one group, keeps its
// rotations resident (transposed to the K-major operand layout) and walks
// 128-token tiles of every (batch, head).  Per CTA, warp-specialised:
//   warp 0      TMA producer: X tiles (128 x d bf16, 128B swizzle) into a
//               ring of kStages buffers;
//   warp 1      allocates TMEM (2 x 256 fp32 columns) and issues the MMAs
//               (one thread): tile x "piece" of <= 256 rotation columns into
//               one of the two accumulator buffers;
//   warps 2..9  epilogue: two warps per TMEM lane quadrant (32 token rows),
//               splitting each round's 32-column chunks between them; each
//               keeps, per row, the 16-column group that holds its largest
//               |p| (a copy in shared memory, stored only by the lanes whose
//               candidate changes) and resolves the exact index at the end
//               of the round; the two halves' candidates meet through shared
//               memory.
// Argmax order: larger |p| first; among equal |p| the smaller index of
// [xR; -xR] (p_j >= 0 gives index j, else n_b/2 + j), i.e. the lowest index
// among maximal entries.
#include <algorithm>
#include <climits>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lsh {
namespace {

using namespace sm100;

constexpr int kRows = 128;          // tokens per tile = MMA M = TMEM lanes
constexpr int kPieceMax = 256;      // columns per accumulator buffer = MMA N max
constexpr int kChunk = 32;          // columns per tcgen05.ld
// Columns of a chunk saved as a candidate.  Measured on the long-text
// workload: groups of 8 0.520 ms, of 16 0.512 ms, whole 32-column chunks
// 0.551 ms (more shared-memory wavefronts per save).
constexpr int kGroup = 16;
constexpr int kGroups = kChunk / kGroup;  // groups per chunk
constexpr int kSlots = kGroup / 4;        // 16-byte slots of a saved group
static_assert(kGroup == 8 || kGroup == 16, "group of 8 or 16 columns");
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kRBudget = 128 * 1024;
constexpr int kSmemLimit = 227 * 1024;

struct Params {
  const __nv_bfloat16* rot;  // [n_h, d, P]
  int16_t* buckets;          // [BH, n_h, L]
  float* inv_norm;           // [BH, L]
  unsigned int* err;
  unsigned long long first_wait_ns;  // limit of the MMA thread's first wait
  int BH, L, d, n_h, P;
  int gr;                    // rounds per group
  int G;                     // CTAs per group
  int tiles_per_head, n_tiles;
  int n_cols;                // gr * P, columns of the group
  int piece_w;               // nominal piece width (last piece of a tile may be narrower)
  int n_pieces;
  int stages;
};

struct Smem {  // offsets inside the 1024-aligned dynamic shared memory
  uint32_t r, x, save, bars, xch, misc, total;
};

__host__ __device__ inline Smem smem_layout(int n_cols, int d, int stages) {
  Smem s;
  uint32_t off = 0;
  s.r = off;    off += (uint32_t)n_cols * d * 2;
  s.x = off;    off += (uint32_t)stages * kRows * d * 2;
  s.save = off; off += kEpiWarps * 32 * kGroup * 4;   // one saved group per epilogue thread
  s.bars = off; off += (uint32_t)(2 * stages + 4 + 4 + 1) * 8;
  s.xch = off;  off += 2 * kRows * 8;
  s.misc = off; off += 16;
  s.total = off;
  return s;
}

__device__ __forceinline__ bool better(float a, int z, float ba, int bz) {
  return a > ba || (a == ba && z < bz);
}

// max(a, b, c): one three-input instruction on sm_100.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Largest |p| (hash) or p (assignment) of each group of a 32-column chunk:
// a tree of three-input max instructions (four per 8 columns, eight per 16).
template <bool ABS>
__device__ __forceinline__ void group_maxima(const uint32_t* u, float* g) {
#pragma unroll
  for (int k = 0; k < kGroups; ++k) {
    float v[kGroup];
#pragma unroll
    for (int t = 0; t < kGroup; ++t) {
      const float x = __uint_as_float(u[kGroup * k + t]);
      v[t] = ABS ? fabsf(x) : x;
    }
    if constexpr (kGroup == 8) {
      g[k] = max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
    } else {
      const float a = max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]),
                            max3f(v[6], v[7], v[8]));
      const float b = max3f(max3f(v[9], v[10], v[11]), max3f(v[12], v[13], v[14]), v[15]);
      g[k] = fmaxf(a, b);
    }
  }
}

// KM: the routing-style assignment (argmax over the n_b columns of given
// centroids, lowest column on ties) instead of argmax([xR; -xR]).
// NP > 0: every piece is NP pairs of 32-column chunks and a round is a whole
// number of pairs (P % 64 == 0), so each epilogue warp takes one chunk of
// every pair at fixed positions and loads the next chunk while it reduces the
// current one.  NP == 0: any P that is a multiple of 32.
template <int NP, bool KM>
__global__ void __launch_bounds__(kThreads, 1)
hash_tc_kernel(const __grid_constant__ CUtensorMap xmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const Smem L = smem_layout(p.n_cols, p.d, p.stages);
  uint8_t* r_smem = smem + L.r;
  uint8_t* x_smem = smem + L.x;
  uint8_t* save_smem = smem + L.save;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* x_full = bars;
  uint64_t* x_empty = bars + p.stages;
  uint64_t* t_full = bars + 2 * p.stages;      // [2]
  uint64_t* t_empty = t_full + 2;              // [2]
  uint64_t* xc_full = t_empty + 2;             // [2]
  uint64_t* xc_empty = xc_full + 2;            // [2]
  uint64_t* done = xc_empty + 2;               // [1]
  float* xch_a = reinterpret_cast<float*>(smem + L.xch);            // [2][128]
  int* xch_z = reinterpret_cast<int*>(smem + L.xch + 2 * kRows * 4);  // [2][128]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int group = blockIdx.x / p.G, g = blockIdx.x % p.G;
  const int r0 = group * p.gr;
  const bool do_norm = (group == 0);
  const int x_stage_bytes = kRows * p.d * 2;
  const int khalves = p.d / 64;

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1 + (do_norm ? 4 : 0));
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&t_full[b], 1);
      mbar_init(&t_empty[b], kEpiWarps);
      mbar_init(&xc_full[b], 4);
      mbar_init(&xc_empty[b], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  wait_prior_grid();
  // Rotations of this group -> shared memory, K-major with 128B swizzle:
  // operand row n = column (rr * P + j) of the group, k = input dimension.
  for (int idx = tid; idx < p.n_cols * (p.d / 8); idx += kThreads) {
    const int n = idx % p.n_cols, kg = idx / p.n_cols;
    const int rr = n / p.P, j = n % p.P, k0 = kg * 8;
    const __nv_bfloat16* src = p.rot + ((size_t)(r0 + rr) * p.d + k0) * p.P + j;
    alignas(16) __nv_bfloat16 v8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v8[e] = src[(size_t)e * p.P];
    uint8_t* dst = r_smem + (size_t)(k0 / 64) * p.n_cols * 128 + sw128_offset(n, k0 % 64);
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(v8);
  }
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&xmap);
      int it = 0;
      for (int tile = g; tile < p.n_tiles; tile += p.G, ++it) {
        const int s = it % p.stages;
        if (!mbar_wait(&x_empty[s], ((it / p.stages) & 1) ^ 1, abort_flag)) {
          atomicOr(p.err, kErrWaitProducer);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&x_full[s], x_stage_bytes);
        const int bh = tile / p.tiles_per_head, t = tile % p.tiles_per_head;
        for (int h = 0; h < khalves; ++h)
          tma_load_3d(x_smem + (size_t)s * x_stage_bytes + h * (kRows * 128), &xmap, &x_full[s],
                      h * 64, t * kRows, bh);
      }
      // Drain: the last loads must land before the CTA may exit.
      for (int k = (it > p.stages ? it - p.stages : 0); k < it; ++k) {
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(&x_full[k % p.stages], (k / p.stages) & 1)) {
          if (globaltimer() - t0 > kWaitLimitNs) { atomicOr(p.err, kErrWaitDrain); break; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, gp = 0;
      bool ok = true, issued = false;
      for (int tile = g; ok && tile < p.n_tiles; tile += p.G, ++it) {
        const int s = it % p.stages;
        if (!mbar_wait_for(&x_full[s], (it / p.stages) & 1, abort_flag,
                           it == 0 ? p.first_wait_ns : kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t xa = smem_u32(x_smem + (size_t)s * x_stage_bytes);
        for (int pc = 0; pc < p.n_pieces; ++pc, ++gp) {
          const int buf = gp & 1;
          if (!mbar_wait(&t_empty[buf], ((gp >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          const int col0 = pc * p.piece_w;
          const int w = min(p.piece_w, p.n_cols - col0);
          const uint32_t idesc = idesc_bf16_f32(kRows, w);
          const uint32_t rb = smem_u32(r_smem) + (uint32_t)col0 * 128;
          for (int kk = 0; kk < p.d / 16; ++kk) {
            const uint32_t koff = (uint32_t)(kk & 3) * 32;
            const uint64_t a = sdesc_kmajor_sw128(xa + (kk >> 2) * (kRows * 128) + koff);
            const uint64_t b =
                sdesc_kmajor_sw128(rb + (uint32_t)(kk >> 2) * p.n_cols * 128 + koff);
            mma_bf16_ss(tmem_base + buf * kPieceMax, a, b, idesc, kk > 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit(&t_full[buf]);
        }
        if (ok) mma_commit(&x_empty[s]);
      }
      if (!ok) {
        atomicOr(p.err, kErrWaitMma);
        *abort_flag = 1;
      }
      // Every MMA issued must finish before TMEM is released.
      if (issued) {
        mma_commit(done);
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(done, 0)) {
          if (globaltimer() - t0 > kWaitLimitNs) { atomicOr(p.err, kErrWaitDrain); break; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;           // TMEM lanes 32*quad .. 32*quad+31
    const int half = ew >> 2;            // which alternate 32-column chunks
    const int row = quad * 32 + lane;    // token row inside the tile
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    // This thread's copy of the group that holds its row's largest |p| so
    // far: kSlots 16-byte slots, their order permuted per lane so that the
    // eight lanes of a quarter warp hit different banks.
    uint8_t* my_save = save_smem + (size_t)(ew * 32 + lane) * (kGroup * 4);
    const int sx = kGroup == 8 ? ((lane >> 2) & 1) : ((lane >> 1) & 3);
    auto slot_addr = [&](int q) { return smem_u32(my_save) + (uint32_t)((q ^ sx) << 4); };
    // Group k of the chunk u when `take` and k == grp: predicated stores, so
    // that the warp stays converged and each lane writes one group at most.
    auto save_group_if = [&](bool take, int grp, const uint32_t* u) {
#pragma unroll
      for (int k = 0; k < kGroups; ++k) {
        const uint32_t on = (uint32_t)(take && grp == k);
#pragma unroll
        for (int q = 0; q < kSlots; ++q) {
          const uint32_t* w = u + kGroup * k + 4 * q;
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
              "@p st.shared.v4.b32 [%1], {%2, %3, %4, %5};\n\t}" ::"r"(on),
              "r"(slot_addr(q)), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
              : "memory");
        }
      }
    };
    auto load_saved = [&](float* sv) {
#pragma unroll
      for (int q = 0; q < kSlots; ++q) {
        const uint4 w = *reinterpret_cast<const uint4*>(my_save + ((q ^ sx) << 4));
        sv[4 * q] = __uint_as_float(w.x);
        sv[4 * q + 1] = __uint_as_float(w.y);
        sv[4 * q + 2] = __uint_as_float(w.z);
        sv[4 * q + 3] = __uint_as_float(w.w);
      }
    };
    int it = 0, gp = 0, ex = 0;
    bool ok = true;
    // no candidate yet: below every |p| (hash) or every p (assignment)
    constexpr float kNone = KM ? -INFINITY : -1.f;
    float best_a = kNone;
    int best_j0 = 0;

    // One 32-column chunk starting at round column j0: keep its group that
    // holds the largest |p| (hash) or p (assignment) when that beats every
    // earlier chunk of the round.  Equal values keep the earliest entry,
    // except for the hash's rule that a positive entry wins over negative ones
    // (handled on the rare path below, for ties inside the chunk and with the
    // saved group).
    auto take_chunk = [&](const uint32_t* u, int j0) {
      float g[kGroups];
      group_maxima<!KM>(u, g);
      float cm;
      int grp, n_eq;
      if constexpr (kGroups == 4) {
        cm = fmaxf(max3f(g[0], g[1], g[2]), g[3]);
        grp = g[2] == cm ? 2 : 3;
        grp = g[1] == cm ? 1 : grp;
        grp = g[0] == cm ? 0 : grp;
        n_eq = (g[0] == cm) + (g[1] == cm) + (g[2] == cm) + (g[3] == cm);
      } else {
        cm = fmaxf(g[0], g[1]);
        grp = g[0] == cm ? 0 : 1;
        n_eq = g[0] == g[1] ? 2 : 1;
      }
      bool take = cm > best_a;
      if (!KM) {
        if (__any_sync(0xffffffffu, n_eq > 1 || cm == best_a)) {
          // The lowest group holding +cm, if any, carries the chunk's candidate.
          int gpos = -1;
#pragma unroll
          for (int k = kGroups - 1; k >= 0; --k) {
            bool hp = false;
#pragma unroll
            for (int t = 0; t < kGroup; ++t) hp |= (__uint_as_float(u[kGroup * k + t]) == cm);
            if (hp) gpos = k;
          }
          if (gpos >= 0) grp = gpos;
          if (cm == best_a) {
            float sv[kGroup];
            load_saved(sv);
            bool pos_saved = false;
#pragma unroll
            for (int t = 0; t < kGroup; ++t) pos_saved |= (sv[t] == best_a);
            take = !pos_saved && gpos >= 0;
          }
        }
      }
      best_a = take ? cm : best_a;
      best_j0 = take ? j0 + kGroup * grp : best_j0;
      save_group_if(take, grp, u);
    };

    // End of round r0 + rr: this half's candidate, then the two halves meet
    // and half 0 writes the bucket.  Returns false on a wait timeout.
    auto round_end = [&](int bh, int t0, int rr, bool row_valid) -> bool {
      int z = INT_MAX;
      const float a = best_a;
      if (best_a > kNone) {
        float sv[kGroup];
        load_saved(sv);
        int tp = -1, tn = 0;
#pragma unroll
        for (int t = kGroup - 1; t >= 0; --t) {
          if (sv[t] == best_a) tp = t;
          if (!KM && sv[t] == -best_a) tn = t;
        }
        z = tp >= 0 ? best_j0 + tp : p.P + best_j0 + tn;
      }
      best_a = kNone;
      const int xb = ex & 1;
      const uint32_t par = (ex >> 1) & 1;
      ++ex;
      if (half == 1) {
        if (!mbar_wait(&xc_empty[xb], par ^ 1, abort_flag)) return false;
        xch_a[xb * kRows + row] = a;
        xch_z[xb * kRows + row] = z;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xc_full[xb]);
      } else {
        if (!mbar_wait(&xc_full[xb], par, abort_flag)) return false;
        const float oa = xch_a[xb * kRows + row];
        const int oz = xch_z[xb * kRows + row];
        __syncwarp();
        if (lane == 0) mbar_arrive(&xc_empty[xb]);
        if (better(oa, oz, a, z)) z = oz;
        if (row_valid) p.buckets[((size_t)bh * p.n_h + r0 + rr) * p.L + t0 + row] = (int16_t)z;
      }
      return true;
    };

    for (int tile = g; ok && tile < p.n_tiles; tile += p.G, ++it) {
      const int bh = tile / p.tiles_per_head, t0 = (tile % p.tiles_per_head) * kRows;
      const bool row_valid = t0 + row < p.L;
      if (do_norm && half == 0) {
        const int s = it % p.stages;
        if (!mbar_wait(&x_full[s], (it / p.stages) & 1, abort_flag)) { ok = false; break; }
        const uint8_t* xs = x_smem + (size_t)s * x_stage_bytes;
        float ss = 0.f;
        for (int h = 0; h < khalves; ++h) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(
                xs + h * (kRows * 128) + row * 128 + ((c ^ (row & 7)) << 4));
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 f = __bfloat1622float2(b2[q]);
              ss = fmaf(f.x, f.x, ss);
              ss = fmaf(f.y, f.y, ss);
            }
          }
        }
        if (row_valid) p.inv_norm[(size_t)bh * p.L + t0 + row] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&x_empty[s]);
      }
      int rr = 0, j0 = 0;  // round (within the group) and column of the next chunk
      for (int pc = 0; pc < p.n_pieces; ++pc, ++gp) {
        const int buf = gp & 1;
        if (!mbar_wait(&t_full[buf], (gp >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after_sync();
        if constexpr (NP > 0) {
          // My chunk of pair m sits at piece column 64 m + 32 half.
          const uint32_t taddr = lane_addr + (uint32_t)(buf * kPieceMax + kChunk * half);
          uint32_t u[2][kChunk];
          __syncwarp();
          tmem_ld_32x32b_x32(taddr, u[0]);
          tmem_ld_wait(u[0]);
#pragma unroll
          for (int m = 0; m < NP; ++m) {
            if (m + 1 < NP) {
              __syncwarp();
              tmem_ld_32x32b_x32(taddr + (uint32_t)(2 * kChunk * (m + 1)), u[(m + 1) & 1]);
            }
            if (ok) {
              take_chunk(u[m & 1], j0 + kChunk * half);
              j0 += 2 * kChunk;
              if (j0 == p.P) {
                ok = round_end(bh, t0, rr, row_valid);
                j0 = 0;
                ++rr;
              }
            }
            // the load in flight lands before anything else happens
            if (m + 1 < NP) tmem_ld_wait(u[(m + 1) & 1]);
          }
        } else {
          const int col0 = pc * p.piece_w;
          const int w = min(p.piece_w, p.n_cols - col0);
          const uint32_t taddr = lane_addr + (uint32_t)(buf * kPieceMax - col0);
          for (int c = col0; c < col0 + w; c += kChunk) {
            if (((c >> 5) & 1) == half) {
              uint32_t u[kChunk];
              __syncwarp();
              tmem_ld_32x32b_x32(taddr + (uint32_t)c, u);
              tmem_ld_wait(u);
              take_chunk(u, j0);
            }
            j0 += kChunk;
            if (j0 == p.P) {
              if (!round_end(bh, t0, rr, row_valid)) { ok = false; break; }
              j0 = 0;
              ++rr;
            }
          }
        }
        if (!ok) break;
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&t_empty[buf]);
      }
    }
    if (!ok) {
      atomicOr(p.err, kErrWaitEpilogue);
      *abort_flag = 1;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// ---------------------------------------------------------------- host side
// Limit of the MMA thread's first wait (normally the 2 s of every bounded
// wait); lsh_attn_test_hash_first_wait sets it to exercise the timeout path.
std::atomic<unsigned long long> g_first_wait_ns{kWaitLimitNs};

struct Plan {
  int gr, n_groups, G, piece_w, n_pieces, stages;
  int np;  // pairs of chunks per piece for the fixed-position epilogue, 0 = general
  size_t smem;
};

// Projection columns per round: n_b / 2 for the hash, n_b centroids for the
// routing-style assignment.
int round_cols(const Problem& pr) { return pr.kmeans ? pr.n_b : pr.half(); }

bool make_plan(const Problem& pr, Plan* out) {
  const long long n_tiles = (long long)pr.BH() * ((pr.L + kRows - 1) / kRows);
  const int P = round_cols(pr);
  if (P <= 0 || P % kChunk) return false;
  const int d = pr.d;
  // The largest group of rounds (a divisor of n_h) whose rotations, at least
  // two X stages, the save rows and the barriers fit in shared memory.
  for (int gr = pr.n_h; gr >= 1; --gr) {
    if (pr.n_h % gr) continue;
    if ((size_t)gr * P * d * 2 > (size_t)kRBudget) continue;
    const int n_cols = gr * P;
    int piece_w;
    if (P <= kPieceMax) {
      piece_w = std::min(gr, kPieceMax / P) * P;
    } else {
      const int s = (P + kPieceMax - 1) / kPieceMax;
      if (P % s || (P / s) % kChunk) return false;
      piece_w = P / s;
    }
    for (int stages = d == 64 ? 4 : 3; stages >= 2; --stages) {
      const Smem L = smem_layout(n_cols, d, stages);
      if (L.total + 1024 > (uint32_t)kSmemLimit) continue;
      out->gr = gr;
      out->n_groups = pr.n_h / gr;
      out->G = (int)std::max(1LL, std::min<long long>(sm_count() / out->n_groups, n_tiles));
      out->piece_w = piece_w;
      out->n_pieces = (n_cols + piece_w - 1) / piece_w;
      out->stages = stages;
      out->np = (P % (2 * kChunk) == 0 && piece_w % (2 * kChunk) == 0 && n_cols % piece_w == 0)
                    ? piece_w / (2 * kChunk)
                    : 0;
      // At least half the SM's shared memory: one CTA per SM, since each CTA
      // allocates all 512 TMEM columns.
      out->smem = std::max<size_t>(L.total + 1024, 116 * 1024);
      return true;
    }
  }
  return false;
}

}  // namespace

bool hash_tc_supported(const Problem& p) {
  Plan plan;
  return p.bf16 && (p.d == 64 || p.d == 128) && p.n_b >= 2 && make_plan(p, &plan) &&
         tensor_map_encoder() != nullptr;
}

cudaError_t launch_hash_tc(const Problem& pr, const void* qk, const void* rot, int16_t* buckets,
                           float* inv_norm, cudaStream_t st) {
  Plan plan;
  if (!make_plan(pr, &plan)) return cudaErrorNotSupported;
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorUnknown;
  CUtensorMap map;
  const cuuint64_t dims[3] = {(cuuint64_t)pr.d, (cuuint64_t)pr.L, (cuuint64_t)pr.BH()};
  const cuuint64_t strides[2] = {(cuuint64_t)pr.d * 2, (cuuint64_t)pr.L * pr.d * 2};
  const cuuint32_t box[3] = {64, kRows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult cr = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(qk), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  Params p;
  p.first_wait_ns = g_first_wait_ns.load(std::memory_order_relaxed);
  p.rot = static_cast<const __nv_bfloat16*>(rot);
  p.buckets = buckets;
  p.inv_norm = inv_norm;
  p.err = err;
  p.BH = pr.BH(); p.L = pr.L; p.d = pr.d; p.n_h = pr.n_h; p.P = round_cols(pr);
  p.gr = plan.gr;
  p.G = plan.G;
  p.tiles_per_head = (pr.L + kRows - 1) / kRows;
  p.n_tiles = p.BH * p.tiles_per_head;
  p.n_cols = plan.gr * p.P;
  p.piece_w = plan.piece_w;
  p.n_pieces = plan.n_pieces;
  p.stages = plan.stages;
  void (*kernel)(const CUtensorMap, const Params);
  if (pr.kmeans) {
    switch (plan.np) {
      case 1: kernel = hash_tc_kernel<1, true>; break;
      case 2: kernel = hash_tc_kernel<2, true>; break;
      case 3: kernel = hash_tc_kernel<3, true>; break;
      case 4: kernel = hash_tc_kernel<4, true>; break;
      default: kernel = hash_tc_kernel<0, true>; break;
    }
  } else {
    switch (plan.np) {
      case 1: kernel = hash_tc_kernel<1, false>; break;
      case 2: kernel = hash_tc_kernel<2, false>; break;
      case 3: kernel = hash_tc_kernel<3, false>; break;
      case 4: kernel = hash_tc_kernel<4, false>; break;
      default: kernel = hash_tc_kernel<0, false>; break;
    }
  }
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(kernel, dim3(plan.n_groups * plan.G), dim3(kThreads), plan.smem, st, map,
                       p);
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

unsigned long long set_hash_first_wait_ns(unsigned long long ns) {
  return g_first_wait_ns.exchange(ns);
}

}  // namespace lsh
