// Stage 3 on the 5th-generation tensor cores: chunked shared-QK attention of
// every hashing round, stored at original positions ("Reformer: The
// Efficient Transformer", section 2 "LSH attention" and "Causal masking";
// section 5 "Shared query-key space"; Appendix A "Implementation" and
// "Masking"), for bf16 inputs with d_k in {64, 128} and chunks of 64 or 128.
//
// A CTA walks strips of consecutive 128-slot "steps" of (b*h, round)
// segments in sorted order.  Step s has the queries of sorted slots
// [128 s, 128 s + 128) and the keys of slots [128 s - c, 128 s + 128): the
// previous c slots (look-back, none for s = 0) and the queries themselves.
// A query in chunk k sees key chunks k-1 and k; with c = 64 the first 64
// query rows (chunk 2s) see key columns [0, 128) and the last 64 (chunk
// 2s+1) see [64, 192); with c = 128 every row sees all 256 columns.  The
// 128 slots of a step form a "block"; block s is the query block of step s
// and the look-back block of step s+1.
//
// Warp roles (11 warps):
//   warp 0      qk producer: per block, gathers the qk rows named by perm
//               with TMA (tile::gather4, four rows per lane and instruction)
//               into a ring of shared-memory tiles in the 128B-swizzled
//               operand layout, and writes each row's position, key scale
//               (1/||x|| * log2 e / sqrt(d)) and query reference
//               (||x|| * log2 e / sqrt(d)) into a metadata ring.  Positions
//               and norms are loaded two blocks ahead.
//   warp 10     v producer: the same gathers from v into their own ring, so
//               keys never wait for values.
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (two MMAs per
//               k-step: look-back keys and current keys live in different
//               tiles), issued one step ahead; then O = P V with P from
//               shared memory and V as an MN-major operand.
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
//               gives).  The softmax of step s+1 runs before the output of
//               step s, so P V overlaps it.  For the output the two warps of
//               a quadrant split the D columns: each writes its half of O / l
//               for the quadrant's 32 rows straight to their original
//               positions; half 0 writes lse.  Waits spin on the barrier
//               (no suspend), which keeps the hand-offs between roles short.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "step_split.cuh"

namespace lsh {
namespace {

using namespace sm100;

constexpr int kQ = 128;             // queries per step = rows per block = MMA M
constexpr int kSoftWarps = 8;
constexpr int kVWarp = 2 + kSoftWarps;
constexpr int kThreads = (3 + kSoftWarps) * 32;   // qk producer, MMA, softmax, v producer
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMetaSlots = 8;
constexpr int kMaxRounds = 8;  // rounds the duplicate correction carries per row
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
};

struct Params {
  const int32_t* perm;
  const float* inv_norm;
  const __nv_bfloat16* v;
  __nv_bfloat16* o_rounds;
  float* lse_rounds;
  const int16_t* buckets;  // [BH, n_h, L] bucket ids for the bucket-equality mask, else null
  const int32_t* undo;     // [BH, n_h, L] every round's undo for the duplicate correction
  unsigned int* err;
  int L, n_h, causal;
  StepSplit split;    // the CTAs' share of the steps (ceil(L / 128) per segment)
  float ksc;          // log2 e / sqrt(d)
  int o32;            // o_rounds is 32-byte aligned: 32-byte stores
};

struct Layout {
  uint32_t qk, v, p, pos, ksc, qref, bkt, chk, xch, bars, misc, total;
};

// 32 bytes to global memory in one store (the address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* ptr, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(a.x),
               "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

__host__ __device__ constexpr uint32_t n_barriers(int nq, int nv) {
  // rings; S/O/P full/free pairs (2 x 6); exchange (2 x 4); redo (4); done
  return 2 * nq + 2 * nv + 2 * kMetaSlots + 12 + 8 + 4 + 1;
}

template <int C, int D, bool BM = false, bool DD = false>
__host__ __device__ constexpr Layout layout(int nq, int nv, int np) {
  using K = Cfg<C, D>;
  Layout l{};
  uint32_t off = 0;
  l.qk = off;   off += nq * K::kTile;
  l.v = off;    off += nv * K::kTile;
  l.p = off;    off += np * K::kPBytes;
  l.pos = off;  off += kMetaSlots * kQ * 4;
  l.ksc = off;  off += kMetaSlots * kQ * 4;
  l.qref = off; off += kMetaSlots * kQ * 4;
  l.bkt = off;  off += BM ? kMetaSlots * kQ * 4 : 0;  // bucket ids (bucket-equality mask)
  // every round's chunk index per row (duplicate correction)
  l.chk = off;  off += DD ? kMetaSlots * kQ * kMaxRounds * 4 : 0;
  l.xch = off;  off += (2 * 2 + 2 + 2) * kQ * 4;   // partial sums [2][2], maxima [2], redo sums [2]
  l.bars = off; off += n_barriers(nq, nv) * 8;
  l.misc = off; off += 16;
  l.total = off;
  return l;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
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

// The CTA's sequence of blocks to load: for each of its units, the look-back
// block (if s0 > 0) and then blocks s0 .. s1-1.
struct Cursor {
  int k;  // piece index
  Unit U;
  int b;
  bool valid;
};

__device__ __forceinline__ void cursor_start(Cursor& c, const Params& p, int k) {
  int got;
  while ((got = split_piece(p.split, p.n_h, blockIdx.x, gridDim.x, k, c.U)) == kPieceEmpty) ++k;
  c.k = k;
  c.valid = got == kPieceRun;
  if (c.valid) c.b = c.U.s0 > 0 ? c.U.s0 - 1 : c.U.s0;
}

__device__ __forceinline__ void cursor_next(Cursor& c, const Params& p) {
  if (!c.valid) return;
  if (++c.b >= c.U.s1) cursor_start(c, p, c.k + 1);
}

// Positions of sorted slots sl .. sl+3 of a segment (INT_MAX past its end).
__device__ __forceinline__ void load_positions(const int32_t* perm, int sl, int L, int* pos) {
  // one 16-byte load where the four positions are 16-byte aligned (a segment
  // starts on such a boundary only when L is a multiple of 4)
  if (sl + 3 < L && (reinterpret_cast<uintptr_t>(perm + sl) & 15) == 0) {
    const int4 v = *reinterpret_cast<const int4*>(perm + sl);
    pos[0] = v.x; pos[1] = v.y; pos[2] = v.z; pos[3] = v.w;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) pos[k] = sl + k < L ? perm[sl + k] : INT_MAX;
  }
}

// Positions of the 4 rows lane 4l .. 4l+3 owns in the cursor's block.
__device__ __forceinline__ void cursor_positions(const Cursor& c, const Params& p, int lane,
                                                 int* pos) {
  if (!c.valid) {
#pragma unroll
    for (int k = 0; k < 4; ++k) pos[k] = INT_MAX;
    return;
  }
  const int32_t* perm = p.perm + ((size_t)c.U.bh * p.n_h + c.U.r) * p.L;
  load_positions(perm, c.b * kQ + 4 * lane, p.L, pos);
}

// Row of the [B*H*L, d] view that holds position `pos`; a row past the end
// of the tensor for a missing position, which the gather fills with zeros.
__device__ __forceinline__ int gather_row(int rowbase, int pos) {
  return pos == INT_MAX ? INT_MAX : rowbase + pos;
}

// What the softmax keeps of a row between its P pass and its output.
struct RowState {
  int qpos;     // original position (INT_MAX: no such query)
  bool any;     // some key other than itself was visible
  float lt;     // sum of 2^(s' - ref) over the row
  float ref;    // exponent reference, log2 units
};

// Ring depths that fit, preferring (in this order) double-buffered P with at
// least three key tiles, and key tiles before value tiles; at least two of
// each.  Fixed per (chunk, d), so the kernel sees the depths as compile-time
// constants.
struct Plan {
  int nq, nv, np;
  uint32_t smem;
  bool ok;
};

template <int C, int D, bool BM = false, bool DD = false>
__host__ __device__ constexpr Plan make_plan() {
  constexpr uint32_t limit = kSmemLimit - 1024;  // 1024 for aligning the base
  for (int pb = 2; pb >= 1; --pb) {
    const uint32_t fixed = layout<C, D, BM, DD>(0, 0, pb).total + n_barriers(6, 6) * 8;
    if (fixed >= limit) continue;
    const int tiles = (int)((limit - fixed) / Cfg<C, D>::kTile);
    if (tiles < 4 || (pb == 2 && tiles < 6)) continue;
    const int q = (tiles + 1) / 2 < 5 ? (tiles + 1) / 2 : 5;
    const int v = tiles - q < 5 ? tiles - q : 5;
    uint32_t smem = layout<C, D, BM, DD>(q, v, pb).total + 1024;
    if (smem < 116 * 1024) smem = 116 * 1024;
    return Plan{q, v, pb, smem, smem <= (uint32_t)kSmemLimit};
  }
  return Plan{0, 0, 0, 0, false};
}

// log2 of the number of rounds in which a key (its chunk index of every
// round at `ck`) lies in the window of a query (chunk indices `cq`): rounds
// where the query's chunk minus the key's is 0 or 1.
__device__ __forceinline__ float dup_log2(const int* ck, const int (&cq)[kMaxRounds], int n_h) {
  const int4 a = *reinterpret_cast<const int4*>(ck);
  const int4 b = *reinterpret_cast<const int4*>(ck + 4);
  const int k8[kMaxRounds] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  int n = 0;
#pragma unroll
  for (int rr = 0; rr < kMaxRounds; ++rr)
    n += (rr < n_h && (unsigned)(cq[rr] - k8[rr]) <= 1u) ? 1 : 0;
  float l;
  asm("lg2.approx.f32 %0, %1;" : "=f"(l) : "f"((float)max(n, 1)));
  return l;
}

// BMASK: the bucket-equality mask variant (section 2 "LSH attention": a
// query attends only to targets in its own hash bucket): a key whose bucket
// in this round differs from the query's is not visible.
// DEDUP: the duplicate-count correction (Appendix A "Duplicate handling"):
// a visible key's exponent loses log2 N_ij, N_ij = the rounds r' (at most
// kMaxRounds) with chunk_r'(i) - chunk_r'(j) in {0, 1}; each row carries its
// chunk index of every round in the metadata ring.
template <int C, int D, bool CAUSAL, bool BMASK, bool DEDUP>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap vmap,
               const Params p) {
  using K = Cfg<C, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr Plan PL = make_plan<C, D, BMASK, DEDUP>();
  constexpr int NQ = PL.nq, NV = PL.nv, NP = PL.np, NM = kMetaSlots;
  constexpr Layout Ly = layout<C, D, BMASK, DEDUP>(NQ, NV, NP);
  uint8_t* qk_s = smem + Ly.qk;
  uint8_t* v_s = smem + Ly.v;
  uint8_t* p_s = smem + Ly.p;
  int* pos_s = reinterpret_cast<int*>(smem + Ly.pos);
  float* ksc_s = reinterpret_cast<float*>(smem + Ly.ksc);
  float* qref_s = reinterpret_cast<float*>(smem + Ly.qref);
  int* bkt_s = reinterpret_cast<int*>(smem + Ly.bkt);
  int* chk_s = reinterpret_cast<int*>(smem + Ly.chk);  // [NM * kQ][kMaxRounds]
  float* xl = reinterpret_cast<float*>(smem + Ly.xch);  // [2 buf][2 half][kQ]
  float* xm = xl + 4 * kQ;                              // [2 half][kQ]
  float* xl2 = xm + 2 * kQ;                             // [2 half][kQ]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* qk_full = bars;              // [NQ] TMA bytes + 32 producer lanes
  uint64_t* qk_empty = qk_full + NQ;     // [NQ] MMA: keys consumed
  uint64_t* v_full = qk_empty + NQ;      // [NV] TMA bytes + 32 producer lanes
  uint64_t* v_empty = v_full + NV;       // [NV] MMA: values consumed
  uint64_t* m_full = v_empty + NV;       // [NM] metadata written (32 lanes)
  uint64_t* m_empty = m_full + NM;       // [NM] metadata consumed (softmax warps)
  uint64_t* s_full = m_empty + NM;       // [2] S in TMEM
  uint64_t* s_free = s_full + 2;         // [2] S read
  uint64_t* o_full = s_free + 2;         // [2] O in TMEM
  uint64_t* o_free = o_full + 2;         // [2] O read
  uint64_t* p_full = o_free + 2;         // [2] P written
  uint64_t* p_empty = p_full + 2;        // [2] P consumed
  uint64_t* xbar = p_empty + 2;          // [2][4] partial-sum exchange, the two warps of a quadrant
  uint64_t* rbar = xbar + 8;             // [4] redo exchange, the two warps of a quadrant
  uint64_t* done = rbar + 4;             // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly.misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(&qk_full[s], 32);
      mbar_init(&qk_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&v_full[s], 32);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < NM; ++s) {
      mbar_init(&m_full[s], 32);
      mbar_init(&m_empty[s], kSoftWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kSoftWarps);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], kSoftWarps);
      mbar_init(&p_full[b], kSoftWarps);
      mbar_init(&p_empty[b], 1);
      for (int q = 0; q < 4; ++q) mbar_init(&xbar[b * 4 + q], 2);
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
  wait_prior_grid();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ================================================================ qk producer
    // Lane l owns rows 4l .. 4l+3 of every block.  Positions are loaded two
    // blocks ahead and norms one block ahead, so neither waits in line.
    if (lane == 0) tma_prefetch_desc(&qmap);
    Cursor c0, c1, c2;
    cursor_start(c0, p, 0);
    c1 = c0;
    cursor_next(c1, p);
    c2 = c1;
    cursor_next(c2, p);
    int pos0[4], pos1[4];
    float in0[4];
    int bk0[4];
    cursor_positions(c0, p, lane, pos0);
    cursor_positions(c1, p, lane, pos1);
    // bucket id of a row in its round (-1 for a missing row: matches nothing)
    auto bucket_of = [&](const Cursor& c, int pos) -> int {
      if (!BMASK || !c.valid || pos == INT_MAX) return -1;
      return p.buckets[((size_t)c.U.bh * p.n_h + c.U.r) * p.L + pos];
    };
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      in0[k] = pos0[k] != INT_MAX ? p.inv_norm[(size_t)c0.U.bh * p.L + pos0[k]] : 0.f;
      bk0[k] = bucket_of(c0, pos0[k]);
    }
    int li = 0;
    bool ok = true;
    for (; ok && c0.valid; ++li) {
      // prefetch for the next two blocks
      int pos2[4];
      float in1[4];
      int bk1[4];
      cursor_positions(c2, p, lane, pos2);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        in1[k] = (c1.valid && pos1[k] != INT_MAX)
                     ? p.inv_norm[(size_t)c1.U.bh * p.L + pos1[k]] : 0.f;
        bk1[k] = bucket_of(c1, pos1[k]);
      }
      const int qs = (int)(li % NQ), ms = (int)(li % NM);
      if (!mbar_wait_spin(&qk_empty[qs], (uint32_t)(((li / NQ) & 1) ^ 1), abort_flag)) { ok = false; break; }
      if (!mbar_wait_spin(&m_empty[ms], (uint32_t)(((li / NM) & 1) ^ 1), abort_flag)) { ok = false; break; }
      if (lane == 0) mbar_expect_tx(&qk_full[qs], K::kTile);
      __syncwarp();
      const int rowbase = c0.U.bh * p.L;
      uint8_t* dst = qk_s + (size_t)qs * K::kTile + lane * 512;
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_gather4(dst + h * K::kHalf, &qmap, &qk_full[qs], h * 64, gather_row(rowbase, pos0[0]),
                    gather_row(rowbase, pos0[1]), gather_row(rowbase, pos0[2]),
                    gather_row(rowbase, pos0[3]));
      mbar_arrive(&qk_full[qs]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = ms * kQ + 4 * lane + k;
        pos_s[row] = pos0[k];
        ksc_s[row] = in0[k] * p.ksc;
        qref_s[row] = in0[k] > 0.f ? p.ksc / in0[k] : 0.f;
        if (BMASK) bkt_s[row] = bk0[k];
        if (DEDUP) {
          const size_t ub = (size_t)c0.U.bh * p.n_h * p.L;
#pragma unroll
          for (int rr = 0; rr < kMaxRounds; ++rr)
            chk_s[row * kMaxRounds + rr] =
                (rr < p.n_h && pos0[k] != INT_MAX) ? p.undo[ub + (size_t)rr * p.L + pos0[k]] / C
                                                   : -2;
        }
      }
      mbar_arrive(&m_full[ms]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pos0[k] = pos1[k];
        pos1[k] = pos2[k];
        in0[k] = in1[k];
        bk0[k] = bk1[k];
      }
      c0 = c1;
      c1 = c2;
      cursor_next(c2, p);
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kErrWaitProducer);
      *abort_flag = 1;
    }
  } else if (warp == kVWarp) {
    // ================================================================ v producer
    if (lane == 0) tma_prefetch_desc(&vmap);
    Cursor c0, c1;
    cursor_start(c0, p, 0);
    c1 = c0;
    cursor_next(c1, p);
    int pos0[4];
    cursor_positions(c0, p, lane, pos0);
    int li = 0;
    bool ok = true;
    for (; ok && c0.valid; ++li) {
      int pos1[4];
      cursor_positions(c1, p, lane, pos1);
      const int vs = (int)(li % NV);
      if (!mbar_wait_spin(&v_empty[vs], (uint32_t)(((li / NV) & 1) ^ 1), abort_flag)) { ok = false; break; }
      if (lane == 0) mbar_expect_tx(&v_full[vs], K::kTile);
      __syncwarp();
      const int rowbase = c0.U.bh * p.L;
      uint8_t* dst = v_s + (size_t)vs * K::kTile + lane * 512;
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_gather4(dst + h * K::kHalf, &vmap, &v_full[vs], h * 64, gather_row(rowbase, pos0[0]),
                    gather_row(rowbase, pos0[1]), gather_row(rowbase, pos0[2]),
                    gather_row(rowbase, pos0[3]));
      mbar_arrive(&v_full[vs]);
#pragma unroll
      for (int k = 0; k < 4; ++k) pos0[k] = pos1[k];
      c0 = c1;
      cursor_next(c1, p);
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kErrWaitProducer);
      *abort_flag = 1;
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      int li = 0, t = 0;  // blocks consumed, steps issued
      bool ok = true, issued = false;
      const uint32_t idesc_prev = idesc_bf16_f32(kQ, C);
      const uint32_t idesc_cur = idesc_bf16_f32(kQ, kQ);
      const uint32_t idesc_pv = idesc_bf16_f32_bmn(kQ, D);
      // S(s) = Q K^T into the step's TMEM buffer (ts = the step's counter).
      auto issue_qk = [&](const Unit& U, int first, int s, int ts) -> bool {
        const int ci = first + (s - U.s0) + (U.s0 > 0 ? 1 : 0), pi = ci - 1;
        const bool has_prev = s > 0;
        const int cs = (int)(ci % NQ), ps = (int)(((pi % NQ) + NQ) % NQ);
        const int buf = (int)(ts % K::kNbuf);
        // the free S buffer, this block's keys and, at a strip's first
        // step, the look-back block's (tested together)
        {
          const uint32_t pc = (uint32_t)((ci / NQ) & 1);
          const bool back = has_prev && s == U.s0;
          if (!mbar_wait4_spin(&s_free[buf], (uint32_t)(((ts / K::kNbuf) & 1) ^ 1),
                               &qk_full[cs], pc, back ? &qk_full[ps] : &qk_full[cs],
                               back ? (uint32_t)((pi / NQ) & 1) : pc, &qk_full[cs], pc,
                               abort_flag))
            return false;
        }
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
      auto issue_pv = [&](const Unit& U, int first, int s, int ts) -> bool {
        const int ci = first + (s - U.s0) + (U.s0 > 0 ? 1 : 0), pi = ci - 1;
        const bool has_prev = s > 0;
        const int cs = (int)(ci % NV), ps = (int)(((pi % NV) + NV) % NV);
        const int buf = (int)(ts % K::kNbuf);
        const int pb = (int)(ts % NP);
        // P of this step, a free O buffer, this block's values and, at a
        // strip's first step, the look-back block's (tested together)
        {
          const uint32_t vc = (uint32_t)((ci / NV) & 1);
          const bool back = has_prev && s == U.s0;
          if (!mbar_wait4_spin(&p_full[pb], (uint32_t)((ts / NP) & 1), &o_free[buf],
                               (uint32_t)(((ts / K::kNbuf) & 1) ^ 1), &v_full[cs], vc,
                               back ? &v_full[ps] : &v_full[cs],
                               back ? (uint32_t)((pi / NV) & 1) : vc, abort_flag))
            return false;
        }
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
      for (int k = 0; ok; ++k) {
        Unit U;
        const int got = split_piece(p.split, p.n_h, blockIdx.x, gridDim.x, k, U);
        if (got == kPieceEnd) break;
        if (got == kPieceEmpty) continue;
        const int first = li;
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
    uint32_t rph = 0;  // phase of this quadrant's redo barrier
    bool ok = true;

    // P pass of step s (step counter ts): S from TMEM -> P (bf16) in shared
    // memory; returns the row's state for its output.
    auto p_pass = [&](const Unit& U, int first, int s, int ts, RowState& st) -> bool {
      const int ci = first + (s - U.s0) + (U.s0 > 0 ? 1 : 0), pi = ci - 1;
      const bool has_prev = s > 0;
      const int cs = (int)(ci % NM), ps = (int)(((pi % NM) + NM) % NM);
      const int buf = (int)(ts % K::kNbuf);
      const int pb = (int)(ts % NP);
      const uint32_t s_tmem = tmem_base + lane_off + buf * K::kBufCols;
      // S of this step, the step's metadata (and, at a strip's first step,
      // the look-back block's) and a free P buffer, tested together
      {
        const uint32_t mc = (uint32_t)((ci / NM) & 1);
        const bool back = has_prev && s == U.s0;
        if (!mbar_wait4_warp(&s_full[buf], (uint32_t)((ts / K::kNbuf) & 1), &m_full[cs], mc,
                             back ? &m_full[ps] : &m_full[cs],
                             back ? (uint32_t)((pi / NM) & 1) : mc, &p_empty[pb],
                             (uint32_t)(((ts / NP) & 1) ^ 1), abort_flag))
          return false;
      }
      tc_fence_after_sync();
      const int qpos = pos_s[cs * kQ + m];
      const float qref = qref_s[cs * kQ + m];
      const int qb = BMASK ? bkt_s[cs * kQ + m] : 0;
      int cq[kMaxRounds];
#pragma unroll
      for (int rr = 0; rr < kMaxRounds; ++rr)
        cq[rr] = DEDUP ? chk_s[(cs * kQ + m) * kMaxRounds + rr] : 0;
      // log2 N for the key in metadata row kr (0 without the correction)
#define DUP_LOG2(kr) (DEDUP ? dup_log2(chk_s + (kr) * kMaxRounds, cq, p.n_h) : 0.f)
      const int qlim = p.causal ? qpos : INT_MAX - 1;
      const int lo = has_prev ? win_lo : max(win_lo, C);
      // metadata row of key column j0 (a multiple of 32, all in one block)
      auto kbase = [&](int j0) { return j0 < C ? ps * kQ + (kQ - C) + j0 : cs * kQ + (j0 - C); };
      uint8_t* prow = p_s + (size_t)pb * K::kPBytes;
      bool any = false;
      float la[4] = {0.f, 0.f, 0.f, 0.f};
      for (int j0 = half * 32; j0 < K::kNk; j0 += 64) {
        uint32_t pk[16];
        if (j0 >= lo && j0 < win_hi) {
          uint32_t sv[32];
          __syncwarp();
          tmem_ld_32x32b_x32(s_tmem + j0, sv);
          tmem_ld_wait(sv);
          const int kb = kbase(j0);
          // Causal: a key is visible iff its position is below the query's
          // (one comparison, which also leaves the query itself out), and
          // the row sees some key iff the chunk's smallest position does.
          if (CAUSAL && !BMASK) any |= __reduce_min_sync(0xffffffffu, pos_s[kb + lane]) < qpos;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const int4 kp = *reinterpret_cast<const int4*>(pos_s + kb + e);
            const float4 ks = *reinterpret_cast<const float4*>(ksc_s + kb + e);
            const int kpa[4] = {kp.x, kp.y, kp.z, kp.w};
            const float ksa[4] = {ks.x, ks.y, ks.z, ks.w};
            int kba[4] = {0, 0, 0, 0};
            if (BMASK) {
              const int4 kbv = *reinterpret_cast<const int4*>(bkt_s + kb + e);
              kba[0] = kbv.x; kba[1] = kbv.y; kba[2] = kbv.z; kba[3] = kbv.w;
            }
            float pr[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              bool valid;
              if (CAUSAL) {
                valid = kpa[h] < qpos;
              } else {
                valid = kpa[h] <= qlim && kpa[h] != qpos;
              }
              if (BMASK) valid = valid && kba[h] == qb;
              if (!CAUSAL || BMASK) any |= valid;
              float x = fmaf(__uint_as_float(sv[e + h]), ksa[h], -qref);
              if (DEDUP && valid) x -= DUP_LOG2(kb + e + h);
              pr[h] = valid ? ex2(x) : 0.f;
              la[h] += pr[h];
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
      const float l = (la[0] + la[1]) + (la[2] + la[3]);
      // The two warps of the quadrant add their partial sums (a row that saw
      // no key is carried as -1).
      const int xb = (int)(ts & 1);
      xl[(xb * 2 + half) * kQ + m] = any ? l : -1.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xbar[xb * 4 + quad]);
      if (!mbar_wait_spin(&xbar[xb * 4 + quad], (uint32_t)((ts >> 1) & 1), abort_flag)) return false;
      const float other = xl[(xb * 2 + (half ^ 1)) * kQ + m];
      any = any || other >= 0.f;
      float lt = l + fmaxf(other, 0.f);
      float ref = qref;
      // Every term underflowed against the bound: redo the row against its
      // exact maximum.
      const bool need = any && !(lt >= kTinySum);
      if (__any_sync(0xffffffffu, need)) {
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
            if (kp <= qlim && kp != qpos && (!BMASK || bkt_s[kb + e] == qb))
              mx = fmaxf(mx, __uint_as_float(sv[e]) * ksc_s[kb + e] - DUP_LOG2(kb + e));
          }
        }
        xm[half * kQ + m] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(&rbar[quad]);
        if (!mbar_wait_spin(&rbar[quad], rph, abort_flag)) return false;
        rph ^= 1;
        const float gmax = fmaxf(mx, xm[(half ^ 1) * kQ + m]);
        const bool redo = need;
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
                const bool valid =
                    kp <= qlim && kp != qpos && (!BMASK || bkt_s[kb + e + h + g] == qb);
                pr[g] = valid ? ex2(fmaf(__uint_as_float(sv[e + h + g]), ksc_s[kb + e + h + g],
                                         -gmax) - DUP_LOG2(kb + e + h + g))
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
        if (!mbar_wait_spin(&rbar[quad], rph, abort_flag)) return false;
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
        // metadata of the look-back block is not needed again, nor this
        // block's at the strip's last step (the row's state is in registers)
        if (has_prev) mbar_arrive(&m_empty[ps]);
        if (s == U.s1 - 1) mbar_arrive(&m_empty[cs]);
      }
      st.qpos = qpos;
      st.any = any;
      st.lt = lt;
      st.ref = ref;
      return true;
    };

    // Output of step s: the two warps of a quadrant split the D columns; each
    // writes its half of O / l for all 32 rows straight to the rows' original
    // positions (the two halves of a row's line meet in L2), and half 0 the
    // lse.
    auto o_pass = [&](const Unit& U, int ts, int s, const RowState& st) -> bool {
      const int buf = (int)(ts % K::kNbuf);
      const uint32_t o_tmem = tmem_base + lane_off + buf * K::kBufCols + K::kNk;
      if (!mbar_wait_spin(&o_full[buf], (uint32_t)((ts / K::kNbuf) & 1), abort_flag)) return false;
      tc_fence_after_sync();
      const bool q_valid = st.qpos != INT_MAX;
      const size_t seg_row = ((size_t)U.bh * p.n_h + U.r) * p.L;
      const float inv_l = st.any ? 1.f / st.lt : 0.f;
      __nv_bfloat16* orow = p.o_rounds + (seg_row + (q_valid ? st.qpos : 0)) * D;
      const __nv_bfloat16* vrow = p.v + ((size_t)U.bh * p.L + (q_valid ? st.qpos : 0)) * D;
      const bool self_only = q_valid && !st.any;
      const bool any_self_only = __any_sync(0xffffffffu, self_only);
      __syncwarp();
#pragma unroll
      for (int d0 = half * (D / 2); d0 < (half + 1) * (D / 2); d0 += 32) {
        uint32_t ov[32];
        tmem_ld_32x32b_x32(o_tmem + d0, ov);
        tmem_ld_wait(ov);
        uint4 w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          w[q].x = pack_bf16(__uint_as_float(ov[8 * q + 0]) * inv_l,
                             __uint_as_float(ov[8 * q + 1]) * inv_l);
          w[q].y = pack_bf16(__uint_as_float(ov[8 * q + 2]) * inv_l,
                             __uint_as_float(ov[8 * q + 3]) * inv_l);
          w[q].z = pack_bf16(__uint_as_float(ov[8 * q + 4]) * inv_l,
                             __uint_as_float(ov[8 * q + 5]) * inv_l);
          w[q].w = pack_bf16(__uint_as_float(ov[8 * q + 6]) * inv_l,
                             __uint_as_float(ov[8 * q + 7]) * inv_l);
        }
        if (any_self_only) {
          // nothing but itself to attend to: the -1e5 self score makes it v_i
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 vq = self_only ? reinterpret_cast<const uint4*>(vrow + d0)[q] : w[q];
            w[q] = vq;
          }
        }
        if (q_valid) {
          if (p.o32) {
            // two 32-byte stores: each store of the warp touches 32 rows
            st_global_v8(orow + d0, w[0], w[1]);
            st_global_v8(orow + d0 + 16, w[2], w[3]);
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(orow + d0)[q] = w[q];
          }
        }
      }
      if (half == 0 && q_valid)
        p.lse_rounds[seg_row + st.qpos] = st.any ? st.ref * kLn2 + logf(st.lt) : kSelfScore;
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[buf]);
      return true;
    };

    int li = 0, t = 0;
    for (int k = 0; ok; ++k) {
      Unit U;
      const int got = split_piece(p.split, p.n_h, blockIdx.x, gridDim.x, k, U);
      if (got == kPieceEnd) break;
      if (got == kPieceEmpty) continue;
      const int first = li;
      li += (U.s1 - U.s0) + (U.s0 > 0 ? 1 : 0);
      RowState cur, next;
      if (!p_pass(U, first, U.s0, t, cur)) { ok = false; break; }
      for (int s = U.s0; s < U.s1; ++s, ++t) {
        if (s + 1 < U.s1 && !p_pass(U, first, s + 1, t + 1, next)) { ok = false; break; }
        if (!o_pass(U, t, s, cur)) { ok = false; break; }
        cur = next;
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
cudaError_t launch_cd(const Problem& pr, const void* qk, const void* v, const float* inv_norm,
                      const int32_t* perm, const int16_t* buckets, const int32_t* undo,
                      void* o_rounds, float* lse_rounds, cudaStream_t st) {
  constexpr Plan PL = make_plan<C, D, false, false>();
  constexpr Plan PLM = make_plan<C, D, true, false>();
  constexpr Plan PLD = make_plan<C, D, false, true>();
  static_assert(PL.ok && PLM.ok, "no shared-memory plan for this (chunk, d)");
  // the duplicate correction's chunk indices do not fit next to the rings
  // for every (chunk, d): those take the CUDA-core kernel
  if (undo && !PLD.ok) return cudaErrorNotSupported;
  Params p;
  const size_t smem = undo ? PLD.smem : (buckets ? PLM.smem : PL.smem);
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorUnknown;
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.inv_norm = inv_norm;
  p.perm = perm;
  p.o_rounds = static_cast<__nv_bfloat16*>(o_rounds);
  p.lse_rounds = lse_rounds;
  p.buckets = buckets;
  p.undo = undo;
  p.err = err;
  p.L = pr.L;
  p.n_h = pr.n_h;
  p.causal = pr.causal ? 1 : 0;
  int grid = 0;
  p.split = make_step_split((long long)pr.BH() * pr.n_h, (pr.L + kQ - 1) / kQ, sm_count(), grid);
  p.ksc = kLog2e / sqrtf((float)pr.d);
  p.o32 = reinterpret_cast<uintptr_t>(o_rounds) % 32 == 0 ? 1 : 0;
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  // [B*H*L, d] views of qk and v: boxes of one row of 64 elements (128 B),
  // 128B swizzle; gathered rows outside the tensor read as zeros.
  CUtensorMap maps[2];
  const void* bases[2] = {qk, v};
  for (int k = 0; k < 2; ++k) {
    const cuuint64_t rows = (cuuint64_t)pr.BH() * pr.L;
    const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 1};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&maps[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(bases[k]), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const bool bmask = buckets != nullptr, dedup = undo != nullptr;
  // (with no plan for the correction, its instantiations are never launched:
  // they fall back to the plain kernel's symbol and are excluded above)
  constexpr bool kDD = PLD.ok;
  auto kernel =
      pr.causal ? (dedup ? attn_tc_kernel<C, D, true, false, kDD>
                         : (bmask ? attn_tc_kernel<C, D, true, true, false>
                                  : attn_tc_kernel<C, D, true, false, false>))
                : (dedup ? attn_tc_kernel<C, D, false, false, kDD>
                         : (bmask ? attn_tc_kernel<C, D, false, true, false>
                                  : attn_tc_kernel<C, D, false, false, false>));
  cudaError_t e = cudaFuncSetAttribute(kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(kernel, dim3((unsigned)grid), dim3(kThreads), smem, st, maps[0], maps[1], p);
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Problem& p) {
  return p.bf16 && (p.d == 64 || p.d == 128) && (p.c == 64 || p.c == 128) &&
         (long long)p.BH() * p.n_h * p.L < (1LL << 31) - 1 &&
         sm100::tensor_map_encoder() != nullptr;
}

cudaError_t launch_attn_tc(const Problem& p, const void* qk, const void* v, const float* inv_norm,
                           const int32_t* perm, const int16_t* buckets, const int32_t* undo,
                           void* o_rounds, float* lse_rounds, cudaStream_t st) {
  if (!p.bucket_mask) buckets = nullptr;
  if (!p.dedup) undo = nullptr;
  if (buckets && undo) return cudaErrorNotSupported;  // both at once: CUDA-core kernel
  if (undo && p.n_h > kMaxRounds) return cudaErrorNotSupported;
  if (p.c == 64 && p.d == 64)
    return launch_cd<64, 64>(p, qk, v, inv_norm, perm, buckets, undo, o_rounds, lse_rounds, st);
  if (p.c == 64 && p.d == 128)
    return launch_cd<64, 128>(p, qk, v, inv_norm, perm, buckets, undo, o_rounds, lse_rounds, st);
  if (p.c == 128 && p.d == 64)
    return launch_cd<128, 64>(p, qk, v, inv_norm, perm, buckets, undo, o_rounds, lse_rounds, st);
  if (p.c == 128 && p.d == 128)
    return launch_cd<128, 128>(p, qk, v, inv_norm, perm, buckets, undo, o_rounds, lse_rounds,
                               st);
  return cudaErrorNotSupported;
}

}  // namespace lsh
