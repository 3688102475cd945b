// Stage 3 for chunks of 64 and d_k = 64 (bf16), the long-text shape, on the
// 5th-generation tensor cores: chunked shared-QK attention of every hashing
// round, stored at original positions ("Reformer: The Efficient
// Transformer", section 2 "LSH attention" and "Causal masking"; section 5
// "Shared query-key space"; Appendix A "Implementation" and "Masking").
//
// Same step geometry as the general kernel (attn_tc.cu): a CTA walks strips
// of 128-slot steps of (b*h, round) segments in sorted order; step s holds
// the queries of slots [128 s, 128 s + 128) and the keys of slots
// [128 s - 64, 128 s + 128); query rows 0-63 (chunk 2s) see key columns
// [0, 128), rows 64-127 (chunk 2s+1) see [64, 192).  What differs:
//   - the softmax probabilities P never touch shared memory: each softmax
//     warp packs its rows' P (bf16) into the first 16 columns of the 32 S
//     columns it has read, and O = P V runs with A read from tensor memory
//     (no P ring in shared memory, no P stores through the LSU);
//   - the key gathers of a block are issued by two TMA warps (a warp's
//     tile::gather4 operations are serialised: about 66 cycles each);
//   - the MMA issuer is a whole warp (one elected lane issues) working from
//     descriptors computed once per step plus compile-time offsets;
//   - the warps that are not on the critical path (MMA issuer, producers)
//     sleep in try_wait; the softmax warps poll all of a step's barriers in
//     one pass.
//
// Warp roles (12 warps, 168 registers each):
//   warps 0-1   qk producers: rows [64 w, 64 w + 64) of every block: TMA
//               gathers into the key ring, plus each row's position, key
//               scale 1/||x|| * log2 e / sqrt(d) and query reference
//               ||x|| * log2 e / sqrt(d) into the metadata ring;
//   warp 2      v producer: the block's 128 rows of v into the value ring;
//   warp 3      MMA issuer (the warp waits, one elected lane issues):
//               S = Q K^T (look-back keys and the block's own keys are two
//               MMAs per k-step), then O = P V and the row sums of P (P
//               times a block of ones, N = 16);
//   warps 4-11  softmax: two warps per TMEM lane quadrant (32 query rows),
//               each taking alternate 32-key chunks of the row.  Keys are
//               unit vectors, so a score never exceeds ||q|| / sqrt(d):
//               that bound is the exponent's reference (p = 2^(s' - ref)
//               <= 1), and a term is then at least 2^(-2 ref), so the two
//               warps need not exchange anything: each writes its P chunks
//               as it goes and the tensor cores add the row.  Rows whose
//               bound is so large that every term could flush to zero take
//               their exact maximum as the reference instead (the quadrant's
//               two warps exchange their halves' maxima).  Masks: window,
//               causal (key position above the query's), self (the key
//               j == i is left out; a row with no other key, i.e. a zero
//               row sum, outputs v_i with lse -1e5, the value the -1e5 self
//               score gives).  The output: each warp scales its half of the
//               row's O columns by 1/l and stores them at the row's original
//               position as two 32-byte stores (o_rounds 32-byte aligned):
//               a warp's store touches 32 rows, so its number of stores
//               sets the load/store unit's work; the two warps write the
//               row's log-sum-exp on alternate steps.
// TMEM: S in two buffers of 192 columns (P written over the first half of
// each 32-column chunk once read; step t uses buffer t & 1), then one O
// buffer of 64 columns and the row sums.  The softmax of step t+1 runs
// before the output of step t, so P V of step t overlaps it, and P V of step
// t+1 waits only for that output to be read.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "step_split.cuh"

namespace lsh {
namespace {

using namespace sm100;

constexpr int kQ = 128;                 // queries per step = MMA M
constexpr int kC = 64;                  // chunk length
constexpr int kD = 64;                  // d_k
constexpr int kNk = kC + kQ;            // key columns per step = TMEM columns of an S buffer
constexpr int kTile = kQ * kD * 2;      // one 128-row bf16 tile (128B-swizzled)
constexpr int kOCol = 2 * kNk;          // O (one buffer) after the two S buffers
constexpr int kSumCol = kOCol + kD;     // P's row sums (16 equal columns)
constexpr int kOnesBytes = 16 * 128;    // 16 rows of bf16 ones: B of the row-sum MMA
constexpr int kQW = 2;                  // qk producer warps
constexpr int kRowsQW = kQ / kQW;       // rows of a block per qk producer warp
constexpr int kMmaWarp = 3;
constexpr int kVW = 1;                  // v producer warps (warp 2)
constexpr int kSoftBase = 4;
constexpr int kSoftWarps = 8;
constexpr int kThreads = (kSoftBase + kSoftWarps) * 32;  // 3 warps per scheduler: 168 registers

constexpr int kSmemLimit = 227 * 1024;
constexpr int kMetaSlots = 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// A row's terms are 2^(s' - ref) >= 2^(-2 ref) with the bound as reference,
// so below this bound no term can flush to zero; a row above it takes its
// exact maximum instead.
constexpr float kBigRef = 58.f;

static_assert(kRowsQW % 4 == 0, "gather4 moves four rows");

// Rows [vrow0(w), vrow0(w) + vrows(w)) of every block belong to v producer w
// (one producer: the whole block).
__host__ __device__ constexpr int vrow0(int) { return 0; }
__host__ __device__ constexpr int vrows(int) { return kQ; }



struct Params {
  const int32_t* perm;
  const float* inv_norm;
  const __nv_bfloat16* v;
  __nv_bfloat16* o_rounds;
  float* lse_rounds;
  const int16_t* buckets;  // [BH, n_h, L] for the bucket-equality mask, else null
  unsigned int* err;
  int L, n_h, causal;
  StepSplit split;  // the CTAs' share of the steps
  float ksc;  // log2 e / sqrt(d)
};

struct Layout {
  uint32_t qk, v, ones, pos, ksc, qref, bkt, xch, bars, misc, total;
};

__host__ __device__ constexpr uint32_t n_barriers(int nq, int nv) {
  // rings; s_full, p_full, o_full, o_free (2 each); exact-max exchange (4);
  // done
  return 2 * nq + 2 * nv + 2 * kMetaSlots + 8 + 4 + 1;
}

template <bool BM>
__host__ __device__ constexpr Layout layout(int nq, int nv) {
  Layout l{};
  uint32_t off = 0;
  l.qk = off;   off += nq * kTile;
  l.v = off;    off += nv * kTile;
  l.ones = off; off += kOnesBytes;
  l.pos = off;  off += kMetaSlots * kQ * 4;
  l.ksc = off;  off += kMetaSlots * kQ * 4;
  l.qref = off; off += kMetaSlots * kQ * 4;
  l.bkt = off;  off += BM ? kMetaSlots * kQ * 4 : 0;
  l.xch = off;  off += 2 * 2 * kQ * 4;  // exact maxima [2 phases][2 halves]
  l.bars = off; off += n_barriers(nq, nv) * 8;
  l.misc = off; off += 16;
  l.total = off;
  return l;
}

struct Plan {
  int nq, nv;
  uint32_t smem;
  bool ok;
};

// Ring depths that fit: key tiles first (a block is live for two steps as
// queries and look-back keys), at most six of each.
template <bool BM>
__host__ __device__ constexpr Plan make_plan() {
  constexpr uint32_t limit = kSmemLimit - 1024;  // 1024 for aligning the base
  const uint32_t fixed = layout<BM>(0, 0).total + n_barriers(6, 6) * 8;
  if (fixed >= limit) return Plan{0, 0, 0, false};
  const int tiles = (int)((limit - fixed) / kTile);
  if (tiles < 5) return Plan{0, 0, 0, false};
  const int q = (tiles + 1) / 2 < 6 ? (tiles + 1) / 2 : 6;
  const int v = tiles - q < 6 ? tiles - q : 6;
  const uint32_t smem = layout<BM>(q, v).total + 1024;
  return Plan{q, v, smem, smem <= (uint32_t)kSmemLimit};
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Shared-memory descriptor, MN-major, 128B swizzle: 64 contiguous elements
// of N per 128-byte row, K rows 128 B apart, 8-row groups `sbo` apart.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t saddr, uint32_t lbo,
                                                        uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
  return idesc_bf16_f32(M, N) | (1u << 16);
}

// A descriptor's start-address field counts 16-byte units from bit 0; shared
// addresses stay below 2^18, so adding a byte offset / 16 never carries out.
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

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

// Positions of rows r0 .. r0+3 of the cursor's block (INT_MAX past the
// segment's end or for no block).
__device__ __forceinline__ void cursor_positions(const Cursor& c, const Params& p, int r0,
                                                 int* pos) {
  if (!c.valid) {
#pragma unroll
    for (int k = 0; k < 4; ++k) pos[k] = INT_MAX;
    return;
  }
  const int32_t* perm = p.perm + ((size_t)c.U.bh * p.n_h + c.U.r) * p.L;
  const int sl = c.b * kQ + r0;
  // one 16-byte load where the four positions are 16-byte aligned (a
  // segment starts on such a boundary only when L is a multiple of 4)
  if (sl + 3 < p.L && (reinterpret_cast<uintptr_t>(perm + sl) & 15) == 0) {
    const int4 v = *reinterpret_cast<const int4*>(perm + sl);
    pos[0] = v.x; pos[1] = v.y; pos[2] = v.z; pos[3] = v.w;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) pos[k] = sl + k < p.L ? perm[sl + k] : INT_MAX;
  }
}

// Row of the [B*H*L, d] view holding position `pos`; past the end of the
// tensor (read as zeros by the gather) for a missing position.
__device__ __forceinline__ int gather_row(int rowbase, int pos) {
  return pos == INT_MAX ? INT_MAX : rowbase + pos;
}

struct RowState {
  int qpos;   // original position (INT_MAX: no such query)
  float ref;  // exponent reference, log2 units
};

// 32 bytes to global memory in one store (the address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* ptr, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(a.x),
               "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// One column of 32 TMEM lanes: thread t reads lane (base + t).
__device__ __forceinline__ uint32_t tmem_ld_32x32b_x1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  return r;
}

// BMASK: the bucket-equality mask (section 2: a query attends only to
// targets in its own bucket).  The duplicate-count correction runs on the
// general kernel (attn_tc.cu), which measured faster for it.
template <bool CAUSAL, bool BMASK>
__global__ void __launch_bounds__(kThreads, 1)
attn64_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap vmap,
              const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr Plan PL = make_plan<BMASK>();
  constexpr int NQ = PL.nq, NV = PL.nv, NM = kMetaSlots;
  constexpr Layout Ly = layout<BMASK>(NQ, NV);
  uint8_t* qk_s = smem + Ly.qk;
  uint8_t* v_s = smem + Ly.v;
  int* pos_s = reinterpret_cast<int*>(smem + Ly.pos);
  float* ksc_s = reinterpret_cast<float*>(smem + Ly.ksc);
  float* qref_s = reinterpret_cast<float*>(smem + Ly.qref);
  int* bkt_s = reinterpret_cast<int*>(smem + Ly.bkt);
  float* xm = reinterpret_cast<float*>(smem + Ly.xch);  // [2 phases][2 half][kQ]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* qk_full = bars;            // [NQ] TMA bytes + one arrival per qk producer warp
  uint64_t* qk_empty = qk_full + NQ;   // [NQ] MMA: keys consumed
  uint64_t* v_full = qk_empty + NQ;    // [NV] TMA bytes + one arrival per v producer warp
  uint64_t* v_empty = v_full + NV;     // [NV] MMA: values consumed
  uint64_t* m_full = v_empty + NV;     // [NM] metadata written (qk producer warps)
  uint64_t* m_empty = m_full + NM;     // [NM] metadata consumed (softmax warps)
  uint64_t* s_full = m_empty + NM;     // [2] S in TMEM
  uint64_t* p_full = s_full + 2;       // [2] P in TMEM (softmax warps)
  uint64_t* o_full = p_full + 2;       // [2] O in TMEM; P (and with it S's buffer) consumed
  uint64_t* o_free = o_full + 2;       // [2] O read (softmax warps)
  uint64_t* rbar = o_free + 2;         // [4] exact-max exchange, the two warps of a quadrant
  uint64_t* done = rbar + 4;           // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly.misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(&qk_full[s], kQW);
      mbar_init(&qk_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&v_full[s], kVW);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < NM; ++s) {
      mbar_init(&m_full[s], kQW);
      mbar_init(&m_empty[s], kSoftWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kSoftWarps);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], kSoftWarps);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&rbar[q], 2);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  // bf16 ones (every byte pair 0x3F80): the B operand of the row-sum MMA
  for (int i = tid; i < kOnesBytes / 4; i += kThreads)
    reinterpret_cast<uint32_t*>(smem + Ly.ones)[i] = 0x3F803F80u;
  wait_prior_grid();
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kSoftBase) {
  if (warp < kQW) {
    // ============================================================ qk producers
    // Lane l < kRowsQW / 4 owns rows r0 .. r0+3, r0 = kRowsQW * warp + 4 l.
    // Positions are loaded two blocks ahead and norms one block ahead.
    const bool act = lane < kRowsQW / 4;
    const int r0 = kRowsQW * warp + 4 * lane;
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
    cursor_positions(c0, p, r0, pos0);
    cursor_positions(c1, p, r0, pos1);
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
    for (; c0.valid; ++li) {
      int pos2[4];
      float in1[4];
      int bk1[4];
      cursor_positions(c2, p, r0, pos2);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        in1[k] = (c1.valid && pos1[k] != INT_MAX)
                     ? p.inv_norm[(size_t)c1.U.bh * p.L + pos1[k]] : 0.f;
        bk1[k] = bucket_of(c1, pos1[k]);
      }
      const int qs = li % NQ, ms = li % NM;
      if (!mbar_wait(&qk_empty[qs], (uint32_t)(((li / NQ) & 1) ^ 1), abort_flag)) { ok = false; break; }
      if (!mbar_wait(&m_empty[ms], (uint32_t)(((li / NM) & 1) ^ 1), abort_flag)) { ok = false; break; }
      if (lane == 0) mbar_expect_tx(&qk_full[qs], kRowsQW * kD * 2);
      __syncwarp();
      const int rowbase = c0.U.bh * p.L;
      if (act)
        tma_gather4(qk_s + (size_t)qs * kTile + r0 * 128, &qmap, &qk_full[qs], 0,
                    gather_row(rowbase, pos0[0]), gather_row(rowbase, pos0[1]),
                    gather_row(rowbase, pos0[2]), gather_row(rowbase, pos0[3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(&qk_full[qs]);
      if (act) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int row = ms * kQ + r0 + k;
          pos_s[row] = pos0[k];
          ksc_s[row] = in0[k] * p.ksc;
          qref_s[row] = in0[k] > 0.f ? p.ksc / in0[k] : 0.f;
          if (BMASK) bkt_s[row] = bk0[k];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&m_full[ms]);
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
    // The CTA may not exit with copies still landing in its shared memory.
    for (int k = li > NQ ? li - NQ : 0; k < li; ++k) {
      const unsigned long long t0 = globaltimer();
      while (!mbar_test(&qk_full[k % NQ], (uint32_t)((k / NQ) & 1))) {
        if (globaltimer() - t0 > kWaitLimitNs) {
          if (lane == 0) atomicOr(p.err, kErrWaitDrain);
          break;
        }
      }
    }
  } else if (warp >= kQW && warp < kQW + kVW) {
    // ============================================================= v producers
    const int w = warp - kQW;
    const bool act = lane < vrows(w) / 4;
    const int r0 = vrow0(w) + 4 * lane;
    if (lane == 0) tma_prefetch_desc(&vmap);
    Cursor c0, c1, c2;
    cursor_start(c0, p, 0);
    c1 = c0;
    cursor_next(c1, p);
    c2 = c1;
    cursor_next(c2, p);
    int pos0[4], pos1[4];
    cursor_positions(c0, p, r0, pos0);
    cursor_positions(c1, p, r0, pos1);
    int li = 0;
    bool ok = true;
    for (; c0.valid; ++li) {
      int pos2[4];
      cursor_positions(c2, p, r0, pos2);
      const int vs = li % NV;
      if (!mbar_wait(&v_empty[vs], (uint32_t)(((li / NV) & 1) ^ 1), abort_flag)) { ok = false; break; }
      if (lane == 0) mbar_expect_tx(&v_full[vs], vrows(w) * kD * 2);
      __syncwarp();
      const int rowbase = c0.U.bh * p.L;
      if (act)
        tma_gather4(v_s + (size_t)vs * kTile + r0 * 128, &vmap, &v_full[vs], 0,
                    gather_row(rowbase, pos0[0]), gather_row(rowbase, pos0[1]),
                    gather_row(rowbase, pos0[2]), gather_row(rowbase, pos0[3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_full[vs]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pos0[k] = pos1[k];
        pos1[k] = pos2[k];
      }
      c0 = c1;
      c1 = c2;
      cursor_next(c2, p);
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kErrWaitProducer);
      *abort_flag = 1;
    }
    for (int k = li > NV ? li - NV : 0; k < li; ++k) {
      const unsigned long long t0 = globaltimer();
      while (!mbar_test(&v_full[k % NV], (uint32_t)((k / NV) & 1))) {
        if (globaltimer() - t0 > kWaitLimitNs) {
          if (lane == 0) atomicOr(p.err, kErrWaitDrain);
          break;
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ============================================================== MMA issuer
    // The whole warp runs the loop and one elected lane issues (on the
    // long-text workload 0.47 ms a launch against 0.50 with the loop in lane
    // 0 alone; the general kernel and the hash measured slower that way and
    // keep the lone lane).  Its waits sleep in try_wait instead of polling,
    // as the producers' do: a polling warp takes issue slots and shared-
    // memory round trips from the two softmax warps of its scheduler, which
    // then finish their P pass last (0.441 against 0.469 ms).
    {
      int li = 0, t = 0;  // blocks consumed, steps issued
      bool ok = true, issued = false;
      constexpr uint32_t idesc_prev = idesc_bf16_f32(kQ, kC);
      constexpr uint32_t idesc_cur = idesc_bf16_f32(kQ, kQ);
      constexpr uint32_t idesc_pv = idesc_bf16_f32_bmn(kQ, kD);
      constexpr uint32_t idesc_sum = idesc_bf16_f32(kQ, 16);
      const uint32_t qk_base = smem_u32(qk_s), v_base = smem_u32(v_s);
      // every byte pair of the tile is bf16 1.0, so one K-major descriptor
      // (16 rows of N) serves every K step of the row-sum MMA
      const uint64_t ones_desc = sdesc_kmajor_sw128(smem_u32(smem + Ly.ones));
      // S(s) = Q K^T into buffer ts & 1, once P V of step ts - 2 (which read
      // P from that buffer) is done.
      auto issue_qk = [&](const Unit& U, int first, int s, int ts) -> bool {
        const int ci = first + (s - U.s0) + (U.s0 > 0 ? 1 : 0), pi = ci - 1;
        const bool has_prev = s > 0;
        const int cs = ci % NQ, ps = (pi + NQ) % NQ;
        const int b = ts & 1;
        // the buffer's last P V (step ts - 2), this block's keys and, at a
        // strip's first step, the look-back block's
        const uint32_t pc = (uint32_t)((ci / NQ) & 1);
        const bool old = ts >= 2, back = has_prev && s == U.s0;
        if (!mbar_wait4_sleep(&qk_full[cs], pc,
                             old ? &o_full[b] : &qk_full[cs],
                             old ? (uint32_t)(((ts >> 1) - 1) & 1) : pc,
                             back ? &qk_full[ps] : &qk_full[cs],
                             back ? (uint32_t)((pi / NQ) & 1) : pc, &qk_full[cs], pc, abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t s_tmem = tmem_base + b * kNk;
        const uint64_t a0 = sdesc_kmajor_sw128(qk_base + cs * kTile);
        const uint64_t bp0 = sdesc_kmajor_sw128(qk_base + ps * kTile + (kQ - kC) * 128);
        if (elect_one_sync()) {
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t a = desc_add(a0, kk * 32);
            if (has_prev) mma_bf16_ss(s_tmem, a, desc_add(bp0, kk * 32), idesc_prev, kk > 0);
            mma_bf16_ss(s_tmem + kC, a, a, idesc_cur, kk > 0);
          }
          mma_commit(&s_full[b]);
          if (has_prev) mma_commit(&qk_empty[ps]);
          if (s == U.s1 - 1) mma_commit(&qk_empty[cs]);
        }
        __syncwarp();
        return true;
      };
      // O(s) = P(s) V, P read from tensor memory: keys [16 kk, 16 kk + 16)
      // sit in columns 32 (kk / 2) + 8 (kk % 2) of the buffer.
      auto issue_pv = [&](const Unit& U, int first, int s, int ts) -> bool {
        const int ci = first + (s - U.s0) + (U.s0 > 0 ? 1 : 0), pi = ci - 1;
        const bool has_prev = s > 0;
        const int cs = ci % NV, ps = (pi + NV) % NV;
        const int b = ts & 1;
        // P of this step, the one O buffer read by the output pass of step
        // ts - 1, this block's values and, at a strip's first step, the
        // look-back block's
        const uint32_t pp = (uint32_t)((ts >> 1) & 1), vc = (uint32_t)((ci / NV) & 1);
        const bool back = has_prev && s == U.s0;
        if (!mbar_wait4_sleep(&p_full[b], pp,
                             ts >= 1 ? &o_free[(ts - 1) & 1] : &p_full[b],
                             ts >= 1 ? (uint32_t)(((ts - 1) >> 1) & 1) : pp, &v_full[cs], vc,
                             back ? &v_full[ps] : &v_full[cs],
                             back ? (uint32_t)((pi / NV) & 1) : vc, abort_flag))
          return false;
        tc_fence_after_sync();
        const uint32_t p_tmem = tmem_base + b * kNk;
        const uint32_t o_tmem = tmem_base + kOCol;
        const uint32_t sum_tmem = tmem_base + kSumCol;
        const uint64_t dprev =
            sdesc_mnmajor_sw128(v_base + ps * kTile + (kQ - kC) * 128, kTile, 1024);
        const uint64_t dcur = sdesc_mnmajor_sw128(v_base + cs * kTile, kTile, 1024);
        if (elect_one_sync()) {
          if (has_prev) {
#pragma unroll
            for (int kk = 0; kk < kC / 16; ++kk)
              mma_bf16_ts(o_tmem, p_tmem + 32 * (kk >> 1) + 8 * (kk & 1),
                          desc_add(dprev, kk * 16 * 128), idesc_pv, kk > 0);
          }
#pragma unroll
          for (int kk = kC / 16; kk < kNk / 16; ++kk)
            mma_bf16_ts(o_tmem, p_tmem + 32 * (kk >> 1) + 8 * (kk & 1),
                        desc_add(dcur, (kk - kC / 16) * 16 * 128), idesc_pv,
                        (has_prev || kk > kC / 16) ? 1u : 0u);
          // the row sums of P: P times a column block of ones (N = 16)
          for (int kk = has_prev ? 0 : kC / 16; kk < kNk / 16; ++kk)
            mma_bf16_ts(sum_tmem, p_tmem + 32 * (kk >> 1) + 8 * (kk & 1),
                        desc_add(ones_desc, (kk & 3) * 32), idesc_sum,
                        kk > (has_prev ? 0 : kC / 16) ? 1u : 0u);
          mma_commit(&o_full[b]);
          if (has_prev) mma_commit(&v_empty[ps]);
          if (s == U.s1 - 1) mma_commit(&v_empty[cs]);
        }
        __syncwarp();
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
      if (!ok && lane == 0) {
        atomicOr(p.err, kErrWaitMma);
        *abort_flag = 1;
      }
      if (issued && elect_one_sync()) {
        mma_commit(done);
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(done, 0)) {
          if (globaltimer() - t0 > kWaitLimitNs) { atomicOr(p.err, kErrWaitDrain); break; }
        }
      }
    }
  }
  } else {
    // ================================================================= softmax
    const int sw = warp - kSoftBase;
    const int quad = warp & 3;           // TMEM lanes 32 quad .. 32 quad + 31
    const int half = sw >> 2;            // which alternate 32-key chunks this warp takes
    const int m = quad * 32 + lane;      // query row in the step
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    // window columns of this row: [0, 128) for chunk 2s, [64, 192) for 2s+1
    const int win_lo = quad >= 2 ? kC : 0;
    // the warp's chunks j0 = 32 half + 64 k: k = kv0, kv0 + 1 may be in the
    // window, k = kz never is
    const int kv0 = quad >= 2 ? 1 : 0;
    const int kz = quad >= 2 ? 0 : 2;
    const uint32_t zeros[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    uint32_t rph = 0;  // phase of this quadrant's redo barrier
    bool ok = true;

    // P pass of step s (step counter ts): S from TMEM -> P (bf16) back into
    // TMEM; returns the row's state for its output.
    auto p_pass = [&](const Unit& U, int first, int s, int ts, RowState& st) -> bool {
      const int ci = first + (s - U.s0) + (U.s0 > 0 ? 1 : 0), pi = ci - 1;
      const bool has_prev = s > 0;
      const int cs = ci % NM, ps = (pi + NM) % NM;
      const int b = ts & 1;
      const uint32_t s_tmem = tmem_base + lane_off + b * kNk;
      {
        const uint32_t mc = (uint32_t)((ci / NM) & 1), sp = (uint32_t)((ts >> 1) & 1);
        const bool back = has_prev && s == U.s0;
        if (!mbar_wait4_warp(&s_full[b], sp, &m_full[cs], mc,
                             back ? &m_full[ps] : &m_full[cs],
                             back ? (uint32_t)((pi / NM) & 1) : mc, &s_full[b], sp, abort_flag))
          return false;
      }
      tc_fence_after_sync();
      const int qpos = pos_s[cs * kQ + m];
      const float qref = qref_s[cs * kQ + m];
      const int qb = BMASK ? bkt_s[cs * kQ + m] : 0;
      const int qlim = p.causal ? qpos : INT_MAX - 1;
      const int lo = has_prev ? win_lo : max(win_lo, kC);
      // metadata row of key column j0 (a multiple of 32, all in one block)
      auto kbase = [&](int j0) { return j0 < kC ? ps * kQ + (kQ - kC) + j0 : cs * kQ + (j0 - kC); };
      // The exponent reference is the row's bound ||q|| log2 e / sqrt(d)
      // (every term <= 1), except in rows whose bound is so large that all
      // their terms could flush to zero: those take their exact maximum over
      // the visible keys (the two warps of the quadrant exchange halves).
      float ref = qref;
      if (__any_sync(0xffffffffu, qref > kBigRef)) {
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int j0 = 32 * half + 64 * (kv0 + i);
          if (j0 < lo) continue;
          uint32_t sv[32];
          __syncwarp();
          tmem_ld_32x32b_x32(s_tmem + j0, sv);
          tmem_ld_wait(sv);
          const int kb = kbase(j0);
          for (int e = 0; e < 32; ++e) {
            const int kp = pos_s[kb + e];
            if (kp <= qlim && kp != qpos && (!BMASK || bkt_s[kb + e] == qb))
              mx = fmaxf(mx, __uint_as_float(sv[e]) * ksc_s[kb + e]);
          }
        }
        float* xmp = xm + rph * 2 * kQ;  // two phases: the other warp may still read the last
        xmp[half * kQ + m] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(&rbar[quad]);
        if (!mbar_wait_spin(&rbar[quad], rph, abort_flag)) return false;
        rph ^= 1;
        const float gmax = fmaxf(mx, xmp[(half ^ 1) * kQ + m]);
        if (qref > kBigRef && gmax > -INFINITY) ref = gmax;
      }
      // P (bf16) over the first 16 columns of each of this warp's 32-key
      // chunks of S, zeros where the row's window does not reach; the row
      // sums come from the tensor cores (P times ones) with P V.
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int j0 = 32 * half + 64 * (kv0 + i);
        uint32_t pk[16];
        if (j0 >= lo) {
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
            int kba[4] = {0, 0, 0, 0};
            if (BMASK) {
              const int4 kbv = *reinterpret_cast<const int4*>(bkt_s + kb + e);
              kba[0] = kbv.x; kba[1] = kbv.y; kba[2] = kbv.z; kba[3] = kbv.w;
            }
            float pr[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              // Causal: a key is visible iff its position is below the
              // query's (one comparison, which also leaves the query out).
              bool valid;
              if (CAUSAL) {
                valid = kpa[h] < qpos;
              } else {
                valid = kpa[h] <= qlim && kpa[h] != qpos;
              }
              if (BMASK) valid = valid && kba[h] == qb;
              const float x = fmaf(__uint_as_float(sv[e + h]), ksa[h], -ref);
              pr[h] = valid ? ex2(x) : 0.f;
            }
            pk[e / 2] = pack_bf16(pr[0], pr[1]);
            pk[e / 2 + 1] = pack_bf16(pr[2], pr[3]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        __syncwarp();
        tmem_st_32x32b_x16(s_tmem + j0, pk);
      }
      tmem_st_32x32b_x16(s_tmem + 32 * half + 64 * kz, zeros);
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&p_full[b]);
        // metadata of the look-back block is not needed again, nor this
        // block's at the strip's last step (the row's state is in registers)
        if (has_prev) mbar_arrive(&m_empty[ps]);
        if (s == U.s1 - 1) mbar_arrive(&m_empty[cs]);
      }
      st.qpos = qpos;
      st.ref = ref;
      return true;
    };

    // Output of step s: the two warps of a quadrant each take half of the D
    // columns of its 32 rows, scale them by 1/l, and each lane writes its
    // row's half (64 bytes) to the row's original position as two 32-byte
    // stores; the half-0 warp also writes the row's log-sum-exp.
    auto o_pass = [&](const Unit& U, int ts, int s, const RowState& st) -> bool {
      const int b = ts & 1;
      if (!mbar_wait_spin(&o_full[b], (uint32_t)((ts >> 1) & 1), abort_flag)) return false;
      tc_fence_after_sync();
      uint32_t ov[32];
      __syncwarp();
      tmem_ld_32x32b_x32(tmem_base + lane_off + kOCol + 32 * half, ov);
      uint32_t lsum = tmem_ld_32x32b_x1(tmem_base + lane_off + kSumCol);
      tmem_ld_wait(ov);
      asm volatile("" : "+r"(lsum));  // not read before the wait above
      const float lt = __uint_as_float(lsum);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[b]);
      const bool q_valid = st.qpos != INT_MAX;
      // every visible key adds a positive term (no term flushes to zero, see
      // kBigRef), so the row saw a key other than itself iff its sum is > 0
      const bool any = lt > 0.f;
      const float inv_l = any ? 1.f / lt : 0.f;
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
      const bool self_only = q_valid && !any;
      if (__any_sync(0xffffffffu, self_only)) {
        // nothing but itself to attend to: the -1e5 self score makes it v_i
        const __nv_bfloat16* vrow = p.v + ((size_t)U.bh * p.L + (q_valid ? st.qpos : 0)) * kD;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (self_only) w[q] = reinterpret_cast<const uint4*>(vrow + 32 * half)[q];
      }
      if (q_valid) {
        // the half row (64 bytes, 32-byte aligned) as two 32-byte stores
        __nv_bfloat16* orow =
            p.o_rounds + (((size_t)U.bh * p.n_h + U.r) * p.L + st.qpos) * kD + 32 * half;
        st_global_v8(orow, w[0], w[1]);
        st_global_v8(orow + 16, w[2], w[3]);
      }
      const size_t seg_row = ((size_t)U.bh * p.n_h + U.r) * p.L;
      // the two warps of the quadrant take turns (a step each)
      if (half == (ts & 1) && q_valid)
        p.lse_rounds[seg_row + st.qpos] = any ? (st.ref + lg2(lt)) * kLn2 : kSelfScore;
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
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, 512);
}

}  // namespace

bool attn_tc64_supported(const Problem& p) {
  return p.bf16 && p.d == kD && p.c == kC && !p.dedup &&
         (long long)p.BH() * p.n_h * p.L < (1LL << 31) - 1 &&
         sm100::tensor_map_encoder() != nullptr;
}

cudaError_t launch_attn_tc64(const Problem& pr, const void* qk, const void* v,
                             const float* inv_norm, const int32_t* perm, const int16_t* buckets,
                             const int32_t* undo, void* o_rounds, float* lse_rounds,
                             cudaStream_t st) {
  if (!pr.bucket_mask) buckets = nullptr;
  (void)undo;  // the duplicate correction runs on the general kernel
  if (pr.dedup) return cudaErrorNotSupported;
  constexpr Plan PL = make_plan<false>();
  constexpr Plan PLM = make_plan<true>();
  static_assert(PL.ok && PLM.ok, "no shared-memory plan");
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorUnknown;
  Params p;
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.inv_norm = inv_norm;
  p.perm = perm;
  p.o_rounds = static_cast<__nv_bfloat16*>(o_rounds);
  p.lse_rounds = lse_rounds;
  p.buckets = buckets;
  p.err = err;
  p.L = pr.L;
  p.n_h = pr.n_h;
  p.causal = pr.causal ? 1 : 0;
  const int sms = sm_count();
  int grid = 0;
  p.split = make_step_split((long long)pr.BH() * pr.n_h, (pr.L + kQ - 1) / kQ, sms, grid);
  p.ksc = kLog2e / sqrtf((float)pr.d);
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  // [B*H*L, d] views of qk and v: boxes of one row of 64 elements (128 B),
  // 128B swizzle; gathered rows outside the tensor read as zeros.
  CUtensorMap maps[2];
  const void* bases[2] = {qk, v};
  for (int k = 0; k < 2; ++k) {
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)pr.BH() * pr.L};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, 1};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&maps[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(bases[k]), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const bool bmask = buckets != nullptr;
  const size_t smem = bmask ? PLM.smem : PL.smem;
  auto kernel = pr.causal ? (bmask ? attn64_kernel<true, true> : attn64_kernel<true, false>)
                          : (bmask ? attn64_kernel<false, true> : attn64_kernel<false, false>);
  cudaError_t e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(kernel, dim3((unsigned)grid), dim3(kThreads), smem, st, maps[0], maps[1], p);
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
