// Backward of the forward pass with the hash and the sort held fixed (the
// hash is piecewise constant, so no gradient flows through bucket ids).
// "Reformer: The Efficient Transformer", section 2
// "LSH attention" and Appendix A define the forward; its gradient follows
// from the multiset form of the combined output,
//   out_i = sum_r sum_{j in W_r(i)} exp(s_ij - LSE_i) v_j,
// where W_r(i) is i's window in round r and LSE_i the combined log-sum-exp:
//   dv_j     += exp(s_ij - LSE_i) dout_i                       (every pair)
//   ds_ij     = exp(s_ij - LSE_i) (dout_i . v_j - dout_i . out_i)
//   dq_i     += ds_ij k_hat_j / sqrt(d),  dk_hat_j += ds_ij q_i / sqrt(d)
//                                          (pairs j != i, not masked)
//   dqk_i     = dq_i + (dk_hat_i - k_hat_i (k_hat_i . dk_hat_i)) / ||qk_i||.
// The self pair's score is the constant -1e5 (no gradient to qk), and a key
// of zero norm has k_hat = 0 and passes no gradient through the key.
//
// CUDA cores, float32, one CTA per (b*h, round, chunk); dv, dq and dk_hat
// are accumulated across CTAs with float32 atomics, so the summation order
// (and the last bits) can change from run to run.  For c = 64 and d = 64 the
// chunk's pairs run as register tiles (bwd_pairs_tiled_kernel).  Other shapes
// take one warp per query (the forward's CUDA-core layout): when the window's
// keys, values and sums fit in shared memory the CTA stages them there
// (bwd_pairs_staged_kernel), else it keeps only the sums there (SACC) or
// adds every pair's terms to global memory.
#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxD = 256;
constexpr int kThreads = 256;
constexpr size_t kSaccLimit = 200 * 1024;  // shared memory for the window sums

// delta_i = dout_i . out_i; zero the accumulators.
template <typename T>
__global__ void __launch_bounds__(kThreads)
bwd_prep_kernel(const T* __restrict__ out, const T* __restrict__ dout, float* __restrict__ delta,
                float* __restrict__ dqk, float* __restrict__ dv, float* __restrict__ dkh,
                long long rows, int d) {
  const int lane = threadIdx.x & 31;
  const long long row = ((long long)blockIdx.x * kThreads + threadIdx.x) / 32;
  if (row >= rows) return;
  float acc = 0.f;
  for (int e = lane; e < d; e += 32) {
    const size_t k = (size_t)row * d + e;
    acc = fmaf(to_f32(dout[k]), to_f32(out[k]), acc);
    dqk[k] = 0.f;
    dv[k] = 0.f;
    dkh[k] = 0.f;
  }
  acc = warp_sum(acc);
  if (lane == 0) delta[row] = acc;
}

template <typename T, bool SACC>
__global__ void __launch_bounds__(kWarps * 32)
bwd_pairs_kernel(const T* __restrict__ qk, const T* __restrict__ v,
                 const float* __restrict__ inv_norm, const int32_t* __restrict__ perm,
                 const float* __restrict__ lse, const T* __restrict__ dout,
                 const float* __restrict__ delta, float* __restrict__ dq, float* __restrict__ dv,
                 float* __restrict__ dkh, int L, int d, int n_h, int c, int causal, float scale) {
  // [kWarps][2][d]: the query row and its dout; with SACC then dv and dk_hat
  // of the window's rows, [2c][d] each
  extern __shared__ float sh[];
  const int n_c = (L + c - 1) / c;
  const int k = (int)(blockIdx.x % n_c);
  const int r = (int)((blockIdx.x / n_c) % n_h);
  const size_t bh = blockIdx.x / ((size_t)n_c * n_h);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* P = perm + (bh * n_h + r) * (size_t)L;
  const T* X = qk + bh * (size_t)L * d;
  const T* V = v + bh * (size_t)L * d;
  const T* G = dout + bh * (size_t)L * d;
  const float* IN = inv_norm + bh * (size_t)L;
  float* DQ = dq + bh * (size_t)L * d;
  float* DV = dv + bh * (size_t)L * d;
  float* DK = dkh + bh * (size_t)L * d;
  float* qs = sh + warp * 2 * d;
  float* gs = qs + d;
  const int k0 = k > 0 ? (k - 1) * c : 0, k1 = min((k + 1) * c, L);
  constexpr int kPer = kMaxD / 32;
  float* dv_s = sh + kWarps * 2 * d;       // SACC only
  float* dk_s = dv_s + (size_t)2 * c * d;
  if (SACC) {
    for (int t = threadIdx.x; t < (k1 - k0) * d; t += blockDim.x) {
      dv_s[t] = 0.f;
      dk_s[t] = 0.f;
    }
    __syncthreads();
  }

  for (int qslot = k * c + warp; qslot < k1; qslot += kWarps) {
    const int i = P[qslot];
    for (int e = lane; e < d; e += 32) {
      qs[e] = to_f32(X[(size_t)i * d + e]);
      gs[e] = to_f32(G[(size_t)i * d + e]);
    }
    __syncwarp();
    const float LSE = lse[bh * (size_t)L + i];
    const float dl = delta[bh * (size_t)L + i];
    float acc[kPer];  // dq_i, dimensions lane, lane + 32, ...
#pragma unroll
    for (int t = 0; t < kPer; ++t) acc[t] = 0.f;

    for (int t0 = k0; t0 < k1; t0 += 32) {
      const int js = t0 + lane;
      const bool in_window = js < k1;
      const int j = in_window ? P[js] : 0;
      const bool visible = in_window && !(causal && j > i);
      float e_ij = 0.f, ds = 0.f, inj = 0.f;
      if (visible) {
        const T* xj = X + (size_t)j * d;
        const T* vj = V + (size_t)j * d;
        float dot = 0.f, gv = 0.f;
        for (int e = 0; e < d; ++e) {
          dot = fmaf(qs[e], to_f32(xj[e]), dot);
          gv = fmaf(gs[e], to_f32(vj[e]), gv);
        }
        inj = IN[j];
        const float s = (j == i) ? kSelfScore : dot * inj * scale;
        e_ij = expf(s - LSE);
        if (j != i) ds = e_ij * (gv - dl);
        // dv_j += e_ij dout_i;  dk_hat_j += ds q_i / sqrt(d)
        float* dvj = SACC ? dv_s + (size_t)(js - k0) * d : DV + (size_t)j * d;
        float* dkj = SACC ? dk_s + (size_t)(js - k0) * d : DK + (size_t)j * d;
        for (int e = 0; e < d; ++e) {
          atomicAdd(&dvj[e], e_ij * gs[e]);
          if (ds != 0.f && inj != 0.f) atomicAdd(&dkj[e], ds * scale * qs[e]);
        }
      }
      // dq_i += ds k_hat_j / sqrt(d): broadcast each lane's pair
      for (int src = 0; src < 32; ++src) {
        const float dss = __shfl_sync(0xffffffffu, ds * inj * scale, src);
        const int jj = __shfl_sync(0xffffffffu, j, src);
        if (dss == 0.f) continue;
        const T* xj = X + (size_t)jj * d;
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
          const int e = lane + 32 * t;
          if (e < d) acc[t] = fmaf(dss, to_f32(xj[e]), acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int e = lane + 32 * t;
      if (e < d) atomicAdd(&DQ[(size_t)i * d + e], acc[t]);
    }
    __syncwarp();
  }
  if (SACC) {
    __syncthreads();
    for (int t = threadIdx.x; t < (k1 - k0) * d; t += blockDim.x) {
      const int j = P[k0 + t / d], e = t % d;
      atomicAdd(&DV[(size_t)j * d + e], dv_s[t]);
      if (dk_s[t] != 0.f) atomicAdd(&DK[(size_t)j * d + e], dk_s[t]);
    }
  }
}

// The same pairs with the window staged: the chunk's window keys (already
// normalised) and values are copied once into padded shared-memory rows
// (d + 1 floats, so lanes reading different rows hit different banks) and
// every query warp of the chunk reads them there; the window's dv and dk_hat
// sums stay in shared memory as in SACC.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_pairs_staged_kernel(const T* __restrict__ qk, const T* __restrict__ v,
                        const float* __restrict__ inv_norm, const int32_t* __restrict__ perm,
                        const float* __restrict__ lse, const T* __restrict__ dout,
                        const float* __restrict__ delta, float* __restrict__ dq,
                        float* __restrict__ dv, float* __restrict__ dkh, int L, int d, int n_h,
                        int c, int causal, float scale) {
  extern __shared__ float sh[];
  const int n_c = (L + c - 1) / c;
  const int k = (int)(blockIdx.x % n_c);
  const int r = (int)((blockIdx.x / n_c) % n_h);
  const size_t bh = blockIdx.x / ((size_t)n_c * n_h);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* P = perm + (bh * n_h + r) * (size_t)L;
  const T* X = qk + bh * (size_t)L * d;
  const T* V = v + bh * (size_t)L * d;
  const T* G = dout + bh * (size_t)L * d;
  const float* IN = inv_norm + bh * (size_t)L;
  float* DQ = dq + bh * (size_t)L * d;
  float* DV = dv + bh * (size_t)L * d;
  float* DK = dkh + bh * (size_t)L * d;
  const int k0 = k > 0 ? (k - 1) * c : 0, k1 = min((k + 1) * c, L), nw = k1 - k0;
  const int dp = d + 1;                      // padded row
  float* qs = sh + warp * 2 * d;
  float* gs = qs + d;
  float* ks = sh + kWarps * 2 * d;           // [2c][dp] normalised keys
  float* vs = ks + (size_t)2 * c * dp;       // [2c][dp] values
  float* dv_s = vs + (size_t)2 * c * dp;     // [2c][dp]
  float* dk_s = dv_s + (size_t)2 * c * dp;   // [2c][dp]
  int* pos_w = reinterpret_cast<int*>(dk_s + (size_t)2 * c * dp);  // [2c]
  for (int t = threadIdx.x; t < nw * d; t += blockDim.x) {
    const int w = t / d, e = t % d;
    const int j = P[k0 + w];
    ks[w * dp + e] = to_f32(X[(size_t)j * d + e]) * IN[j];
    vs[w * dp + e] = to_f32(V[(size_t)j * d + e]);
    dv_s[w * dp + e] = 0.f;
    dk_s[w * dp + e] = 0.f;
    if (e == 0) pos_w[w] = j;
  }
  __syncthreads();
  constexpr int kPer = kMaxD / 32;

  for (int qslot = k * c + warp; qslot < k1; qslot += kWarps) {
    const int i = P[qslot];
    for (int e = lane; e < d; e += 32) {
      qs[e] = to_f32(X[(size_t)i * d + e]);
      gs[e] = to_f32(G[(size_t)i * d + e]);
    }
    __syncwarp();
    const float LSE = lse[bh * (size_t)L + i];
    const float dl = delta[bh * (size_t)L + i];
    float acc[kPer];
#pragma unroll
    for (int t = 0; t < kPer; ++t) acc[t] = 0.f;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      const bool in_window = w < nw;
      const int j = in_window ? pos_w[w] : 0;
      const bool visible = in_window && !(causal && j > i);
      float e_ij = 0.f, ds = 0.f;
      if (visible) {
        const float* kr = ks + w * dp;
        const float* vr = vs + w * dp;
        float dot = 0.f, gv = 0.f;
        for (int e = 0; e < d; ++e) {
          dot = fmaf(qs[e], kr[e], dot);
          gv = fmaf(gs[e], vr[e], gv);
        }
        const float s = (j == i) ? kSelfScore : dot * scale;
        e_ij = expf(s - LSE);
        if (j != i) ds = e_ij * (gv - dl);
        float* dvr = dv_s + w * dp;
        float* dkr = dk_s + w * dp;
        for (int e = 0; e < d; ++e) {
          atomicAdd(&dvr[e], e_ij * gs[e]);
          if (ds != 0.f) atomicAdd(&dkr[e], ds * scale * qs[e]);
        }
      }
      for (int src = 0; src < 32; ++src) {
        const float dss = __shfl_sync(0xffffffffu, ds * scale, src);
        if (dss == 0.f) continue;
        const float* kr = ks + (w0 + src) * dp;
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
          const int e = lane + 32 * t;
          if (e < d) acc[t] = fmaf(dss, kr[e], acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int e = lane + 32 * t;
      if (e < d) atomicAdd(&DQ[(size_t)i * d + e], acc[t]);
    }
    __syncwarp();
  }
  __syncthreads();
  for (int t = threadIdx.x; t < nw * d; t += blockDim.x) {
    const int w = t / d, e = t % d;
    const int j = pos_w[w];
    atomicAdd(&DV[(size_t)j * d + e], dv_s[w * dp + e]);
    const float x = dk_s[w * dp + e];
    if (x != 0.f && IN[j] != 0.f) atomicAdd(&DK[(size_t)j * d + e], x);
  }
}

// The pairs of one chunk for c = 64 and d = 64 as register tiles.  The
// chunk's queries (qk and dout rows) and its window's keys (normalised) and
// values are staged once in shared memory; the chunk's products then run on
// CUDA cores with each thread holding a tile of the result in registers:
//   S = Q K_hat^T and dP = dout V^T        64 x 128, 4 x 8 per thread
//   P = exp(S/sqrt(d) - LSE), dS = P (dP - delta)/sqrt(d), masks applied
//   dV = P^T dout and dK_hat = dS^T Q      128 x 64, 8 x 4 per thread
//   dQ = dS K_hat                          64 x 64, 4 x 4 per thread
// and the CTA adds each row of dV, dK_hat and dQ to global memory once, in
// 16-byte vector atomics.  Missing rows (a short last chunk, the first
// chunk's absent look-back) are zeros with position -1: never visible.
namespace tiled {
constexpr int C = 64, D = 64, NW = 2 * C, kTileThreads = 256;
constexpr int kKt = NW + 1;   // row of the transposed keys and values [D][NW + 1]
constexpr int kPs = NW + 16;  // row of P and dS [C][NW + 16]
constexpr int oQ = 0, oG = oQ + C * D, oKt = oG + C * D, oVt = oKt + D * kKt,
              oP = oVt + D * kKt, oDS = oP + C * kPs, oLse = oDS + C * kPs, oDl = oLse + C,
              oPq = oDl + C, oPk = oPq + C, kFloats = oPk + NW;
constexpr size_t kSmem = (size_t)kFloats * sizeof(float);
static_assert(NW * D <= D * kKt, "the row-major keys reuse the values' buffer");
static_assert(oG % 4 == 0 && oVt % 4 == 0, "float4 rows");
static_assert(kTileThreads == 16 * 16 && C == 4 * 16 && NW == 8 * 16 && D == 4 * 16, "tiling");
}  // namespace tiled

template <typename T>
__global__ void __launch_bounds__(tiled::kTileThreads, 1)
bwd_pairs_tiled_kernel(const T* __restrict__ qk, const T* __restrict__ v,
                       const float* __restrict__ inv_norm, const int32_t* __restrict__ perm,
                       const float* __restrict__ lse, const T* __restrict__ dout,
                       const float* __restrict__ delta, float* __restrict__ dq,
                       float* __restrict__ dv, float* __restrict__ dkh, int L, int n_h,
                       int causal, float scale) {
  using namespace tiled;
  extern __shared__ float4 sh4[];
  float* sh = reinterpret_cast<float*>(sh4);
  float* Qs = sh + oQ;    // [C][D] query rows of qk
  float* Gs = sh + oG;    // [C][D] query rows of dout
  float* Kt = sh + oKt;   // [D][kKt] normalised keys, transposed
  float* Vt = sh + oVt;   // [D][kKt] values, transposed; later the keys row-major
  float* Ps = sh + oP;    // [C][kPs]
  float* DSs = sh + oDS;  // [C][kPs], already divided by sqrt(d)
  float* lse_q = sh + oLse;
  float* dl_q = sh + oDl;
  int* pos_q = reinterpret_cast<int*>(sh + oPq);
  int* pos_k = reinterpret_cast<int*>(sh + oPk);
  const int n_c = (L + C - 1) / C;
  const int k = (int)(blockIdx.x % n_c);
  const int r = (int)((blockIdx.x / n_c) % n_h);
  const size_t bh = blockIdx.x / ((size_t)n_c * n_h);
  const int tid = threadIdx.x;
  const int32_t* P = perm + (bh * n_h + r) * (size_t)L;
  const T* X = qk + bh * (size_t)L * D;
  const T* V = v + bh * (size_t)L * D;
  const T* G = dout + bh * (size_t)L * D;
  const float* IN = inv_norm + bh * (size_t)L;
  float* DQ = dq + bh * (size_t)L * D;
  float* DV = dv + bh * (size_t)L * D;
  float* DK = dkh + bh * (size_t)L * D;
  const int q0 = k * C, nq = min(C, L - q0);
  const int k0 = k > 0 ? q0 - C : 0, nw = min(q0 + C, L) - k0;

  if (tid < C) {
    const int i = tid < nq ? P[q0 + tid] : -1;
    pos_q[tid] = i;
    lse_q[tid] = i >= 0 ? lse[bh * (size_t)L + i] : 0.f;
    dl_q[tid] = i >= 0 ? delta[bh * (size_t)L + i] : 0.f;
  }
  if (tid < NW) pos_k[tid] = tid < nw ? P[k0 + tid] : -1;
  __syncthreads();
  for (int idx = tid; idx < C * D; idx += kTileThreads) {
    const int i = pos_q[idx / D], e = idx % D;
    Qs[idx] = i >= 0 ? to_f32(X[(size_t)i * D + e]) : 0.f;
    Gs[idx] = i >= 0 ? to_f32(G[(size_t)i * D + e]) : 0.f;
  }
  for (int idx = tid; idx < NW * D; idx += kTileThreads) {
    const int w = idx / D, e = idx % D, j = pos_k[w];
    Kt[e * kKt + w] = j >= 0 ? to_f32(X[(size_t)j * D + e]) * IN[j] : 0.f;
    Vt[e * kKt + w] = j >= 0 ? to_f32(V[(size_t)j * D + e]) : 0.f;
  }
  __syncthreads();

  {  // S, dP -> P, dS: rows m = mq + 16a, columns w = kw + 16b
    const int mq = tid >> 4, kw = tid & 15;
    float s[4][8], gp[4][8];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) s[a][b] = gp[a][b] = 0.f;
#pragma unroll 2
    for (int e = 0; e < D; ++e) {
      float qv[4], gv[4], kv[8], vv[8];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        qv[a] = Qs[(mq + 16 * a) * D + e];
        gv[a] = Gs[(mq + 16 * a) * D + e];
      }
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        kv[b] = Kt[e * kKt + kw + 16 * b];
        vv[b] = Vt[e * kKt + kw + 16 * b];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          s[a][b] = fmaf(qv[a], kv[b], s[a][b]);
          gp[a][b] = fmaf(gv[a], vv[b], gp[a][b]);
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int m = mq + 16 * a, i = pos_q[m];
      const float LSE = lse_q[m], dl = dl_q[m];
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const int w = kw + 16 * b, j = pos_k[w];
        float pv = 0.f, ds = 0.f;
        if (i >= 0 && j >= 0 && !(causal && j > i)) {
          pv = expf((j == i ? kSelfScore : s[a][b] * scale) - LSE);
          if (j != i) ds = pv * (gp[a][b] - dl) * scale;
        }
        Ps[m * kPs + w] = pv;
        DSs[m * kPs + w] = ds;
      }
    }
  }
  __syncthreads();
  float* Kr = Vt;  // [NW][D] normalised keys, row-major (the values are done)
  for (int idx = tid; idx < NW * D; idx += kTileThreads) Kr[idx] = Kt[(idx % D) * kKt + idx / D];
  __syncthreads();

  {  // dV = P^T dout, dK_hat = dS^T Q: rows w = kw + 16b, columns 4 eq .. 4 eq + 3
    const int kw = tid & 15, eq = tid >> 4;
    float av[8][4], ak[8][4];
#pragma unroll
    for (int b = 0; b < 8; ++b)
#pragma unroll
      for (int t = 0; t < 4; ++t) av[b][t] = ak[b][t] = 0.f;
#pragma unroll 2
    for (int m = 0; m < C; ++m) {
      const float4 g4 = *reinterpret_cast<const float4*>(Gs + m * D + 4 * eq);
      const float4 x4 = *reinterpret_cast<const float4*>(Qs + m * D + 4 * eq);
      const float gq[4] = {g4.x, g4.y, g4.z, g4.w}, xq[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const float pb = Ps[m * kPs + kw + 16 * b], db = DSs[m * kPs + kw + 16 * b];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          av[b][t] = fmaf(pb, gq[t], av[b][t]);
          ak[b][t] = fmaf(db, xq[t], ak[b][t]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int j = pos_k[kw + 16 * b];
      if (j < 0) continue;
      atomicAdd(reinterpret_cast<float4*>(DV + (size_t)j * D + 4 * eq),
                make_float4(av[b][0], av[b][1], av[b][2], av[b][3]));
      atomicAdd(reinterpret_cast<float4*>(DK + (size_t)j * D + 4 * eq),
                make_float4(ak[b][0], ak[b][1], ak[b][2], ak[b][3]));
    }
  }
  {  // dQ = dS K_hat: rows m = mq + 16a, columns 4 eq .. 4 eq + 3
    const int eq = tid & 15, mq = tid >> 4;
    float aq[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int t = 0; t < 4; ++t) aq[a][t] = 0.f;
#pragma unroll 4
    for (int w = 0; w < NW; ++w) {
      const float4 k4 = *reinterpret_cast<const float4*>(Kr + w * D + 4 * eq);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float d_ = DSs[(mq + 16 * a) * kPs + w];
        aq[a][0] = fmaf(d_, k4.x, aq[a][0]);
        aq[a][1] = fmaf(d_, k4.y, aq[a][1]);
        aq[a][2] = fmaf(d_, k4.z, aq[a][2]);
        aq[a][3] = fmaf(d_, k4.w, aq[a][3]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = pos_q[mq + 16 * a];
      if (i < 0) continue;
      atomicAdd(reinterpret_cast<float4*>(DQ + (size_t)i * D + 4 * eq),
                make_float4(aq[a][0], aq[a][1], aq[a][2], aq[a][3]));
    }
  }
}

// dqk_i += (dk_hat_i - k_hat_i (k_hat_i . dk_hat_i)) / ||qk_i||
template <typename T>
__global__ void __launch_bounds__(kThreads)
bwd_finish_kernel(const T* __restrict__ qk, const float* __restrict__ inv_norm,
                  const float* __restrict__ dkh, float* __restrict__ dqk, long long rows, int d) {
  const int lane = threadIdx.x & 31;
  const long long row = ((long long)blockIdx.x * kThreads + threadIdx.x) / 32;
  if (row >= rows) return;
  const float in = inv_norm[row];
  if (in == 0.f) return;  // zero key: k_hat is the constant 0
  float kd = 0.f;
  for (int e = lane; e < d; e += 32) {
    const size_t k = (size_t)row * d + e;
    kd = fmaf(to_f32(qk[k]) * in, dkh[k], kd);
  }
  kd = warp_sum(kd);
  for (int e = lane; e < d; e += 32) {
    const size_t k = (size_t)row * d + e;
    dqk[k] += (dkh[k] - to_f32(qk[k]) * in * kd) * in;
  }
}

template <typename T>
cudaError_t launch_t(const Problem& p, const void* qk, const void* v, const float* inv_norm,
                     const int32_t* perm, const void* out, const float* lse, const void* dout,
                     float* dqk, float* dv, float* delta, float* dkh, cudaStream_t st) {
  const long long rows = (long long)p.BH() * p.L;
  const unsigned row_blocks = (unsigned)((rows * 32 + kThreads - 1) / kThreads);
  bwd_prep_kernel<T><<<row_blocks, kThreads, 0, st>>>(
      static_cast<const T*>(out), static_cast<const T*>(dout), delta, dqk, dv, dkh, rows, p.d); note_launch();
  const unsigned grid = (unsigned)((long long)p.n_chunks() * p.n_h * p.BH());
  if (p.c == tiled::C && p.d == tiled::D) {
    cudaError_t e = cudaFuncSetAttribute(bwd_pairs_tiled_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tiled::kSmem);
    if (e != cudaSuccess) return e;
    bwd_pairs_tiled_kernel<T><<<grid, tiled::kTileThreads, tiled::kSmem, st>>>(
        static_cast<const T*>(qk), static_cast<const T*>(v), inv_norm, perm, lse,
        static_cast<const T*>(dout), delta, dqk, dv, dkh, p.L, p.n_h, p.causal ? 1 : 0,
        1.0f / sqrtf((float)p.d)); note_launch();
    bwd_finish_kernel<T><<<row_blocks, kThreads, 0, st>>>(static_cast<const T*>(qk), inv_norm,
                                                          dkh, dqk, rows, p.d); note_launch();
    return cudaGetLastError();
  }
  const size_t base = (size_t)kWarps * 2 * p.d * sizeof(float);
  const size_t staged = base + (size_t)4 * 2 * p.c * (p.d + 1) * sizeof(float) +
                        (size_t)2 * p.c * sizeof(int);
  if (staged <= kSaccLimit) {
    cudaError_t e = cudaFuncSetAttribute(bwd_pairs_staged_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)staged);
    if (e != cudaSuccess) return e;
    bwd_pairs_staged_kernel<T><<<grid, kWarps * 32, staged, st>>>(
        static_cast<const T*>(qk), static_cast<const T*>(v), inv_norm, perm, lse,
        static_cast<const T*>(dout), delta, dqk, dv, dkh, p.L, p.d, p.n_h, p.c,
        p.causal ? 1 : 0, 1.0f / sqrtf((float)p.d)); note_launch();
    bwd_finish_kernel<T><<<row_blocks, kThreads, 0, st>>>(static_cast<const T*>(qk), inv_norm,
                                                          dkh, dqk, rows, p.d); note_launch();
    return cudaGetLastError();
  }
  const size_t acc = (size_t)2 * (2 * (size_t)p.c) * p.d * sizeof(float);
  const bool sacc = base + acc <= kSaccLimit;
  const size_t smem = sacc ? base + acc : base;
  auto kernel = sacc ? bwd_pairs_kernel<T, true> : bwd_pairs_kernel<T, false>;
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kernel<<<grid, kWarps * 32, smem, st>>>(
      static_cast<const T*>(qk), static_cast<const T*>(v), inv_norm, perm, lse,
      static_cast<const T*>(dout), delta, dqk, dv, dkh, p.L, p.d, p.n_h, p.c, p.causal ? 1 : 0,
      1.0f / sqrtf((float)p.d)); note_launch();
  bwd_finish_kernel<T><<<row_blocks, kThreads, 0, st>>>(static_cast<const T*>(qk), inv_norm, dkh,
                                                        dqk, rows, p.d); note_launch();
  return cudaGetLastError();
}

}  // namespace

size_t backward_workspace_bytes(const Problem& p) {
  const size_t rows = (size_t)p.BH() * p.L;
  return ((rows * sizeof(float) + 255) & ~(size_t)255) + rows * p.d * sizeof(float);
}

cudaError_t launch_backward(const Problem& p, const void* qk, const void* v,
                            const float* inv_norm, const int32_t* perm, const void* out,
                            const float* lse, const void* dout, float* dqk, float* dv,
                            void* workspace, cudaStream_t st) {
  if (p.d > kMaxD) return cudaErrorInvalidValue;
  const size_t rows = (size_t)p.BH() * p.L;
  float* delta = static_cast<float*>(workspace);
  float* dkh = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                        ((rows * sizeof(float) + 255) & ~(size_t)255));
  return p.bf16 ? launch_t<__nv_bfloat16>(p, qk, v, inv_norm, perm, out, lse, dout, dqk, dv,
                                          delta, dkh, st)
                : launch_t<float>(p, qk, v, inv_norm, perm, out, lse, dout, dqk, dv, delta, dkh,
                                  st);
}

}  // namespace lsh
