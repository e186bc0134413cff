// Gated DeltaNet-2 (burn-gdn2 config.rs): the delta rule with a per-key-channel decay and
// channel-wise erase (b, key channels) and write (w, value channels) gates, state S [K, V]
// per (batch, head) in fp32:
//
//   S' = Diag(e^{g_t}) S,  r = S'^T k_t,  S = S' - (b_t o k_t) r^T + k_t (w_t o v_t)^T,  o_t = S^T q_t
//
// gdn2_recurrent_kernel  Gdn2Mode::FusedRecurrent.  One warp owns C value columns of one head
//   for the whole sequence; lane l holds key rows l, l+32, ... of those columns in registers,
//   so the two reductions over K per token (r and o) are warp shuffles (the eight columns
//   reduced together in 9 shuffles, r broadcast back in 8) and the state never
//   leaves the chip between tokens.  With T = 1 and the state in place this is the decode step
//   (one HBM read and write of S); gdn2_step_kernel below lays the state out for that case.
// gdn2_chunk_prep_kernel + gdn2_chunk_scan_kernel  Gdn2Mode::Chunk.  Per chunk, with G the
//   cumulative log decay inside the chunk (every exponent below <= 0):
//     LA[t,s] = sum_i k_ti k_si e^{G_ti-G_si} (s<t),  LE[t,s] = sum_i k_ti bk_si e^{..} (s<t),
//     QA, QE the same with q_t (s<=t);
//     R = (I + LE)^{-1} (k e^{G} S + LA U)            (U = w o v; one triangular solve)
//     o = (q e^{G}) S + QA U - QE R
//     S <- e^{G_L} o S + (k e^{G_L-G})^T U - (bk e^{G_L-G})^T R
//   i.e. the WY-style block form of the recurrence: dense products inside the chunk, the state
//   carried between chunks.  The prep kernel builds every chunk's L x L matrices, the inverse
//   of I + LE and the decayed rows at once (one CTA per chunk) into the workspace; the scan
//   kernel (one CTA per head and value tile, chunks in order) is left with dense products.
//   fp32 SIMT, the state tile in shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace mlstm {
namespace {

__device__ __forceinline__ float ld_in(const float* p) { return *p; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// ------------------------------------------------------------------ fused recurrent
constexpr int REC_WARPS = 4;
constexpr int REC_C = 8;  // value columns per warp

// Sums of 8 values over the 32 lanes of a warp in 9 shuffles: at each of the offsets 16, 8, 4
// a lane keeps half of its values and adds its partner's copy of them, then offsets 2 and 1
// finish the sum.  Lane l returns the total of value (l >> 2) & 7.
__device__ __forceinline__ float warp_sum8(const float (&v)[8], int lane) {
  const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4;
  float a[4], b[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = h4 ? v[i] : v[i + 4];
    a[i] = (h4 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = h3 ? a[i] : a[i + 2];
    b[i] = (h3 ? a[i + 2] : a[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float c = (h2 ? b[1] : b[0]) + __shfl_xor_sync(0xffffffffu, h2 ? b[0] : b[1], 4);
  c += __shfl_xor_sync(0xffffffffu, c, 2);
  c += __shfl_xor_sync(0xffffffffu, c, 1);
  return c;
}

template <typename T, int KPL>
__global__ void __launch_bounds__(32 * REC_WARPS) gdn2_recurrent_kernel(Gdn2Args a) {
  static_assert(REC_C == 8, "warp_sum8 reduces eight columns");
  constexpr int K = 32 * KPL;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long bh = blockIdx.y;
  const int j0 = (blockIdx.x * REC_WARPS + warp) * REC_C;
  if (j0 >= a.V) return;  // whole warp
  const int nc = min(REC_C, a.V - j0);
  const T* q = static_cast<const T*>(a.q) + bh * a.T * K;
  const T* k = static_cast<const T*>(a.k) + bh * a.T * K;
  const T* v = static_cast<const T*>(a.v) + bh * a.T * a.V + j0;
  const float* g = a.g + bh * a.T * K;
  const float* b = a.b + bh * a.T * K;
  const float* w = a.w + bh * a.T * a.V + j0;
  T* o = static_cast<T*>(a.o) + bh * a.T * a.V + j0;
  float S[KPL][REC_C];
  const float* S0 = a.S0 ? a.S0 + bh * K * a.V : nullptr;
#pragma unroll
  for (int m = 0; m < KPL; ++m)
#pragma unroll
    for (int c = 0; c < REC_C; ++c) S[m][c] = (S0 && c < nc) ? S0[(size_t)(lane + 32 * m) * a.V + j0 + c] : 0.f;
  // inputs of token t, loaded one token ahead
  float qn[KPL], kn[KPL], gn[KPL], bn[KPL], un[REC_C];
  auto load = [&](int t) {
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
      const size_t i = (size_t)t * K + lane + 32 * m;
      qn[m] = ld_in(q + i);
      kn[m] = ld_in(k + i);
      gn[m] = g[i];
      bn[m] = b[i];
    }
#pragma unroll
    for (int c = 0; c < REC_C; ++c)
      un[c] = c < nc ? w[(size_t)t * a.V + c] * ld_in(v + (size_t)t * a.V + c) : 0.f;
  };
  if (a.T > 0) load(0);
  for (int t = 0; t < a.T; ++t) {
    float qv[KPL], kv[KPL], ev[KPL], bk[KPL], u[REC_C];
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
      qv[m] = qn[m];
      kv[m] = kn[m];
      ev[m] = expf(gn[m]);
      bk[m] = bn[m] * kn[m];
    }
#pragma unroll
    for (int c = 0; c < REC_C; ++c) u[c] = un[c];
    if (t + 1 < a.T) load(t + 1);
    float r[REC_C];
#pragma unroll
    for (int c = 0; c < REC_C; ++c) {
      float s = 0.f;
#pragma unroll
      for (int m = 0; m < KPL; ++m) {
        S[m][c] *= ev[m];
        s = fmaf(kv[m], S[m][c], s);
      }
      r[c] = s;
    }
    {  // r of column c sits in lanes 4c..4c+3; every lane needs all eight
      const float rs = warp_sum8(r, lane);
#pragma unroll
      for (int c = 0; c < REC_C; ++c) r[c] = __shfl_sync(0xffffffffu, rs, 4 * c);
    }
    float y[REC_C];
#pragma unroll
    for (int c = 0; c < REC_C; ++c) {
      float s = 0.f;
#pragma unroll
      for (int m = 0; m < KPL; ++m) {
        S[m][c] = fmaf(kv[m], u[c], fmaf(-bk[m], r[c], S[m][c]));
        s = fmaf(qv[m], S[m][c], s);
      }
      y[c] = s;
    }
    const float ys = warp_sum8(y, lane);
    if ((lane & 3) == 0 && (lane >> 2) < nc) st_out(o + (size_t)t * a.V + (lane >> 2), ys);
  }
  if (a.S_out) {
    float* So = a.S_out + bh * K * a.V;
#pragma unroll
    for (int m = 0; m < KPL; ++m)
#pragma unroll
      for (int c = 0; c < REC_C; ++c)
        if (c < nc) So[(size_t)(lane + 32 * m) * a.V + j0 + c] = S[m][c];
  }
}

// ------------------------------------------------------------------ decode step (T = 1)
// One token per sequence: the state is read and written once, so the layout is chosen for
// HBM: lane = value column (a warp reads 128 contiguous bytes of a state row), the 8 warps
// split the key rows, and the two reductions over K go through shared memory.
constexpr int STEP_WARPS = 8;

template <typename T, int RPW>
__global__ void __launch_bounds__(32 * STEP_WARPS) gdn2_step_kernel(Gdn2Args a) {
  constexpr int K = RPW * STEP_WARPS;
  __shared__ float qs[K], ks[K], es[K], bks[K], red[2][STEP_WARPS][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long bh = blockIdx.y;
  const int j = blockIdx.x * 32 + lane;
  const bool col = j < a.V;
  const int i0 = warp * RPW;
  const float* S0 = a.S0 ? a.S0 + bh * K * a.V : nullptr;
  float S[RPW];
#pragma unroll
  for (int m = 0; m < RPW; ++m) S[m] = (S0 && col) ? S0[(size_t)(i0 + m) * a.V + j] : 0.f;
  for (int i = threadIdx.x; i < K; i += 32 * STEP_WARPS) {
    const size_t x = bh * K + i;
    const float kk = ld_in(static_cast<const T*>(a.k) + x);
    qs[i] = ld_in(static_cast<const T*>(a.q) + x);
    ks[i] = kk;
    es[i] = expf(a.g[x]);
    bks[i] = a.b[x] * kk;
  }
  const float u = col ? a.w[bh * a.V + j] * ld_in(static_cast<const T*>(a.v) + bh * a.V + j) : 0.f;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int m = 0; m < RPW; ++m) {
    S[m] *= es[i0 + m];
    r = fmaf(ks[i0 + m], S[m], r);
  }
  red[0][warp][lane] = r;
  __syncthreads();
  r = 0.f;
#pragma unroll
  for (int x = 0; x < STEP_WARPS; ++x) r += red[0][x][lane];
  float y = 0.f;
#pragma unroll
  for (int m = 0; m < RPW; ++m) {
    S[m] = fmaf(ks[i0 + m], u, fmaf(-bks[i0 + m], r, S[m]));
    y = fmaf(qs[i0 + m], S[m], y);
  }
  if (a.S_out && col) {
    float* So = a.S_out + bh * K * a.V;
#pragma unroll
    for (int m = 0; m < RPW; ++m) So[(size_t)(i0 + m) * a.V + j] = S[m];
  }
  red[1][warp][lane] = y;
  __syncthreads();
  if (warp == 0 && col) {
    y = 0.f;
#pragma unroll
    for (int x = 0; x < STEP_WARPS; ++x) y += red[1][x][lane];
    st_out(static_cast<T*>(a.o) + bh * a.V + j, y);
  }
}

// The same step with 16-byte state accesses, for V a multiple of 128: a CTA takes 128 value
// columns of one head, lane = four adjacent columns (a warp covers a 512-byte stretch of a
// state row), the 8 warps split the key rows; every state load of a thread is issued before
// the first use.
template <typename T, int RPW>
__global__ void __launch_bounds__(32 * STEP_WARPS, 2) gdn2_step_v4_kernel(Gdn2Args a) {
  constexpr int K = RPW * STEP_WARPS;
  __shared__ float qs[K], ks[K], es[K], bks[K];
  __shared__ float4 red[2][STEP_WARPS][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long bh = blockIdx.y;
  const int j = blockIdx.x * 128 + 4 * lane;  // first of this lane's four columns
  const int i0 = warp * RPW;
  const float* S0 = a.S0 ? a.S0 + bh * K * a.V : nullptr;
  float4 S[RPW];
#pragma unroll
  for (int m = 0; m < RPW; ++m)
    S[m] = S0 ? *reinterpret_cast<const float4*>(S0 + (size_t)(i0 + m) * a.V + j) : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = threadIdx.x; i < K; i += 32 * STEP_WARPS) {
    const size_t x = bh * K + i;
    const float kk = ld_in(static_cast<const T*>(a.k) + x);
    qs[i] = ld_in(static_cast<const T*>(a.q) + x);
    ks[i] = kk;
    es[i] = expf(a.g[x]);
    bks[i] = a.b[x] * kk;
  }
  float4 u;
  {
    const float4 wv = *reinterpret_cast<const float4*>(a.w + bh * a.V + j);
    const T* vp = static_cast<const T*>(a.v) + bh * a.V + j;
    u = make_float4(wv.x * ld_in(vp), wv.y * ld_in(vp + 1), wv.z * ld_in(vp + 2), wv.w * ld_in(vp + 3));
  }
  __syncthreads();
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int m = 0; m < RPW; ++m) {
    const float e = es[i0 + m], kk = ks[i0 + m];
    S[m].x *= e, S[m].y *= e, S[m].z *= e, S[m].w *= e;
    r.x = fmaf(kk, S[m].x, r.x), r.y = fmaf(kk, S[m].y, r.y), r.z = fmaf(kk, S[m].z, r.z), r.w = fmaf(kk, S[m].w, r.w);
  }
  red[0][warp][lane] = r;
  __syncthreads();
  r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int x = 0; x < STEP_WARPS; ++x) {
    const float4 p = red[0][x][lane];
    r.x += p.x, r.y += p.y, r.z += p.z, r.w += p.w;
  }
  float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
  float* So = a.S_out ? a.S_out + bh * K * a.V : nullptr;
#pragma unroll
  for (int m = 0; m < RPW; ++m) {
    const float kk = ks[i0 + m], bk = bks[i0 + m], qq = qs[i0 + m];
    S[m].x = fmaf(kk, u.x, fmaf(-bk, r.x, S[m].x));
    S[m].y = fmaf(kk, u.y, fmaf(-bk, r.y, S[m].y));
    S[m].z = fmaf(kk, u.z, fmaf(-bk, r.z, S[m].z));
    S[m].w = fmaf(kk, u.w, fmaf(-bk, r.w, S[m].w));
    y.x = fmaf(qq, S[m].x, y.x), y.y = fmaf(qq, S[m].y, y.y), y.z = fmaf(qq, S[m].z, y.z), y.w = fmaf(qq, S[m].w, y.w);
    if (So) *reinterpret_cast<float4*>(So + (size_t)(i0 + m) * a.V + j) = S[m];
  }
  red[1][warp][lane] = y;
  __syncthreads();
  if (warp == 0) {
    y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int x = 0; x < STEP_WARPS; ++x) {
      const float4 p = red[1][x][lane];
      y.x += p.x, y.y += p.y, y.z += p.z, y.w += p.w;
    }
    T* op = static_cast<T*>(a.o) + bh * a.V + j;
    st_out(op, y.x);
    st_out(op + 1, y.y);
    st_out(op + 2, y.z);
    st_out(op + 3, y.w);
  }
}

// ------------------------------------------------------------------ chunk (WY block form)
constexpr int CH_THREADS = 256;

// Per-chunk slot of the workspace written by the prep kernel (floats, unpadded rows):
//   Qd = q e^{G}, Kd = k e^{G}, Kt = k e^{G_L-G}, Bt = bk e^{G_L-G}   [L][K] each
//   LA, Tinv = (I + LE)^{-1}, QA, QE                                   [L][L] each
//   eGL = e^{G_L}                                                      [K]
__host__ __device__ inline size_t chunk_slot_floats(int L, int K) { return (size_t)4 * L * K + (size_t)4 * L * L + K; }

// shared-memory plans (floats; rows padded by one against bank conflicts)
__host__ __device__ inline size_t prep_smem_floats(int L, int K) {
  return (size_t)4 * L * (K + 1) + (size_t)5 * L * (L + 1) + K;
}
__host__ __device__ inline size_t scan_smem_floats(int L, int K, int VT) {
  return (size_t)4 * L * (K + 1) + (size_t)4 * L * (L + 1) + K + (size_t)K * VT + (size_t)3 * L * VT;
}

// Prep: one CTA per (chunk, head), every chunk at once.  Builds the chunk's weight matrices
// (the exponential-heavy part, e^{G_t - G_s} per pair and key channel, every exponent <= 0),
// the inverse of the unit lower-triangular I + LE, and the decayed row forms.
template <typename T>
__global__ void __launch_bounds__(CH_THREADS) gdn2_chunk_prep_kernel(Gdn2Args a, int L, float* ws) {
  extern __shared__ float sm[];
  const int K = a.K, tid = threadIdx.x, lk = K + 1, ll = L + 1;
  float *G = sm, *Kc = G + L * lk, *Bk = Kc + L * lk, *Qc = Bk + L * lk, *LA = Qc + L * lk, *LE = LA + L * ll,
        *QA = LE + L * ll, *QE = QA + L * ll, *TI = QE + L * ll, *gL = TI + L * ll;
  const long long bh = blockIdx.y;
  const int c = blockIdx.x, t0 = c * L, Lc = min(L, a.T - t0);
  const int nch = (a.T + L - 1) / L;
  const T* q = static_cast<const T*>(a.q) + bh * a.T * K;
  const T* k = static_cast<const T*>(a.k) + bh * a.T * K;
  const float* g = a.g + bh * a.T * K;
  const float* b = a.b + bh * a.T * K;
  for (int e = tid; e < L * K; e += CH_THREADS) {
    const int t = e / K, i = e % K;
    float qq = 0.f, kk = 0.f, gg = 0.f, bb = 0.f;
    if (t < Lc) {
      const size_t x = (size_t)(t0 + t) * K + i;
      qq = ld_in(q + x), kk = ld_in(k + x), gg = g[x], bb = b[x];
    }
    Qc[t * lk + i] = qq, Kc[t * lk + i] = kk, G[t * lk + i] = gg, Bk[t * lk + i] = bb * kk;
  }
  __syncthreads();
  for (int i = tid; i < K; i += CH_THREADS) {  // cumulative log decay per key channel
    float s = 0.f;
    for (int t = 0; t < L; ++t) {
      s += G[t * lk + i];
      G[t * lk + i] = s;
    }
    gL[i] = s;
  }
  __syncthreads();
  // the four L x L weight matrices, 4 x 4 (t, s) blocks per thread, lower triangle only
  const int nb4 = L / 4;
  for (int blk = tid; blk < nb4 * nb4; blk += CH_THREADS) {
    const int tb = blk / nb4, sb = blk % nb4;
    float la[4][4] = {}, le[4][4] = {}, qa[4][4] = {}, qe[4][4] = {};
    if (sb <= tb) {
      for (int i = 0; i < K; ++i) {
        float gt[4], kt[4], qt[4], gs[4], ks[4], bs[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int t = 4 * tb + x, s2 = 4 * sb + x;
          gt[x] = G[t * lk + i], kt[x] = Kc[t * lk + i], qt[x] = Qc[t * lk + i];
          gs[x] = G[s2 * lk + i], ks[x] = Kc[s2 * lk + i], bs[x] = Bk[s2 * lk + i];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const float e = expf(fminf(gt[x] - gs[y], 0.f));
            const float ek = e * ks[y], eb = e * bs[y];
            la[x][y] = fmaf(kt[x], ek, la[x][y]);
            le[x][y] = fmaf(kt[x], eb, le[x][y]);
            qa[x][y] = fmaf(qt[x], ek, qa[x][y]);
            qe[x][y] = fmaf(qt[x], eb, qe[x][y]);
          }
      }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const int t = 4 * tb + x, s2 = 4 * sb + y;
        LA[t * ll + s2] = s2 < t ? la[x][y] : 0.f;
        LE[t * ll + s2] = s2 < t ? le[x][y] : 0.f;
        QA[t * ll + s2] = s2 <= t ? qa[x][y] : 0.f;
        QE[t * ll + s2] = s2 <= t ? qe[x][y] : 0.f;
      }
  }
  __syncthreads();
  // inverse of I + LE, one column per thread: TI[t][col] = -sum_{col<=s<t} LE[t][s] TI[s][col]
  for (int col = tid; col < L; col += CH_THREADS) {
    for (int t = 0; t < L; ++t) {
      if (t < col) {
        TI[t * ll + col] = 0.f;
        continue;
      }
      if (t == col) {
        TI[t * ll + col] = 1.f;
        continue;
      }
      float a0 = 0.f, a1 = 0.f;
      int s2 = col;
      for (; s2 + 1 < t; s2 += 2) {
        a0 = fmaf(LE[t * ll + s2], TI[s2 * ll + col], a0);
        a1 = fmaf(LE[t * ll + s2 + 1], TI[(s2 + 1) * ll + col], a1);
      }
      if (s2 < t) a0 = fmaf(LE[t * ll + s2], TI[s2 * ll + col], a0);
      TI[t * ll + col] = -(a0 + a1);
    }
  }
  // the slot: decayed rows, then the L x L matrices and e^{G_L}
  float* slot = ws + ((size_t)bh * nch + c) * chunk_slot_floats(L, K);
  float *oQd = slot, *oKd = oQd + L * K, *oKt = oKd + L * K, *oBt = oKt + L * K, *oLA = oBt + L * K,
        *oTI = oLA + L * L, *oQA = oTI + L * L, *oQE = oQA + L * L, *oGL = oQE + L * L;
  for (int e = tid; e < L * K; e += CH_THREADS) {
    const int t = e / K, i = e % K, x = t * lk + i;
    const float gg = G[x], up = expf(gg), tail = expf(gL[i] - gg);
    oQd[e] = Qc[x] * up;
    oKd[e] = Kc[x] * up;
    oKt[e] = Kc[x] * tail;
    oBt[e] = Bk[x] * tail;
  }
  for (int i = tid; i < K; i += CH_THREADS) oGL[i] = expf(gL[i]);
  __syncthreads();  // TI complete
  for (int e = tid; e < L * L; e += CH_THREADS) {
    const int t = e / L, s2 = e % L;
    oLA[e] = LA[t * ll + s2];
    oTI[e] = TI[t * ll + s2];
    oQA[e] = QA[t * ll + s2];
    oQE[e] = QE[t * ll + s2];
  }
}

// Scan: one CTA per (value tile, head) walks the chunks in order; per chunk only dense
// products on the prepared slot:
//   R = Tinv (Kd S + LA U),  o = Qd S + QA U - QE R,  S <- e^{G_L} o S + Kt^T U - Bt^T R
template <typename T>
__global__ void __launch_bounds__(CH_THREADS) gdn2_chunk_scan_kernel(Gdn2Args a, int L, int VT, const float* ws) {
  extern __shared__ float sm[];
  const int K = a.K, tid = threadIdx.x, lk = K + 1, ll = L + 1;
  float *Qd = sm, *Kd = Qd + L * lk, *Kt = Kd + L * lk, *Bt = Kt + L * lk, *LA = Bt + L * lk, *TI = LA + L * ll,
        *QA = TI + L * ll, *QE = QA + L * ll, *eGL = QE + L * ll, *S = eGL + K, *U = S + K * VT, *X = U + L * VT,
        *R = X + L * VT;
  const long long bh = blockIdx.y;
  const int j0 = blockIdx.x * VT, nch = (a.T + L - 1) / L;
  const T* v = static_cast<const T*>(a.v) + bh * a.T * a.V + j0;
  const float* w = a.w + bh * a.T * a.V + j0;
  T* o = static_cast<T*>(a.o) + bh * a.T * a.V + j0;
  for (int e = tid; e < K * VT; e += CH_THREADS) {
    const int i = e / VT, j = e % VT;
    S[e] = a.S0 ? a.S0[(bh * K + i) * a.V + j0 + j] : 0.f;
  }
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * L, Lc = min(L, a.T - t0);
    const float* slot = ws + ((size_t)bh * nch + c) * chunk_slot_floats(L, K);
    __syncthreads();  // the previous chunk is done with every buffer
    for (int e = tid; e < L * K; e += CH_THREADS) {
      const int t = e / K, i = e % K, x = t * lk + i;
      Qd[x] = slot[e];
      Kd[x] = slot[L * K + e];
      Kt[x] = slot[2 * L * K + e];
      Bt[x] = slot[3 * L * K + e];
    }
    const float* sl2 = slot + 4 * L * K;
    for (int e = tid; e < L * L; e += CH_THREADS) {
      const int t = e / L, s2 = e % L, x = t * ll + s2;
      LA[x] = sl2[e];
      TI[x] = sl2[L * L + e];
      QA[x] = sl2[2 * L * L + e];
      QE[x] = sl2[3 * L * L + e];
    }
    for (int i = tid; i < K; i += CH_THREADS) eGL[i] = sl2[4 * L * L + i];
    for (int e = tid; e < L * VT; e += CH_THREADS) {
      const int t = e / VT, j = e % VT;
      U[e] = t < Lc ? w[(size_t)(t0 + t) * a.V + j] * ld_in(v + (size_t)(t0 + t) * a.V + j) : 0.f;
    }
    __syncthreads();
    // Each thread computes four rows t, t + L/4, t + L/2, t + 3L/4 of one column j with
    // independent accumulators, so the column operand is loaded once per four FMAs and the
    // four dependency chains overlap.
    const int L4 = L / 4, K4 = K / 4;
    for (int e = tid; e < L4 * VT; e += CH_THREADS) {  // X = Kd S + LA U
      const int t = e / VT, j = e % VT;
      float acc[4] = {};
      for (int i = 0; i < K; ++i) {
        const float sv = S[i * VT + j];
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[x] = fmaf(Kd[(t + x * L4) * lk + i], sv, acc[x]);
      }
      for (int s2 = 0; s2 < t + 3 * L4; ++s2) {
        const float uv = U[s2 * VT + j];
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[x] = fmaf(LA[(t + x * L4) * ll + s2], uv, acc[x]);  // LA = 0 for s >= t
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) X[(t + x * L4) * VT + j] = acc[x];
    }
    __syncthreads();
    for (int e = tid; e < L4 * VT; e += CH_THREADS) {  // R = Tinv X
      const int t = e / VT, j = e % VT;
      float acc[4] = {};
      for (int s2 = 0; s2 <= t + 3 * L4; ++s2) {
        const float xv = X[s2 * VT + j];
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[x] = fmaf(TI[(t + x * L4) * ll + s2], xv, acc[x]);  // TI = 0 above the diagonal
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) R[(t + x * L4) * VT + j] = acc[x];
    }
    __syncthreads();
    for (int e = tid; e < L4 * VT; e += CH_THREADS) {  // o = Qd S + QA U - QE R
      const int t = e / VT, j = e % VT;
      float acc[4] = {};
      for (int i = 0; i < K; ++i) {
        const float sv = S[i * VT + j];
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[x] = fmaf(Qd[(t + x * L4) * lk + i], sv, acc[x]);
      }
      for (int s2 = 0; s2 <= t + 3 * L4; ++s2) {
        const float uv = U[s2 * VT + j], rv = R[s2 * VT + j];
#pragma unroll
        for (int x = 0; x < 4; ++x)  // QA, QE = 0 above the diagonal
          acc[x] = fmaf(QA[(t + x * L4) * ll + s2], uv, fmaf(-QE[(t + x * L4) * ll + s2], rv, acc[x]));
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
        if (t + x * L4 < Lc) st_out(o + (size_t)(t0 + t + x * L4) * a.V + j, acc[x]);
    }
    __syncthreads();  // every read of S for o is done
    for (int e = tid; e < K4 * VT; e += CH_THREADS) {  // S <- e^{G_L} S + Kt^T U - Bt^T R
      const int i = e / VT, j = e % VT;
      float acc[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[x] = eGL[i + x * K4] * S[(i + x * K4) * VT + j];
      for (int s2 = 0; s2 < L; ++s2) {
        const float uv = U[s2 * VT + j], rv = R[s2 * VT + j];
#pragma unroll
        for (int x = 0; x < 4; ++x)
          acc[x] = fmaf(Kt[s2 * lk + i + x * K4], uv, fmaf(-Bt[s2 * lk + i + x * K4], rv, acc[x]));
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) S[(i + x * K4) * VT + j] = acc[x];
    }
  }
  __syncthreads();
  if (a.S_out)
    for (int e = tid; e < K * VT; e += CH_THREADS) {
      const int i = e / VT, j = e % VT;
      a.S_out[(bh * K + i) * a.V + j0 + j] = S[e];
    }
}

}  // namespace

bool gdn2_recurrent_supported(int K) { return K == 32 || K == 64 || K == 128 || K == 256; }

int gdn2_chunk_vtile(int L, int K, int V) {
  if (L < 4 || L > 64 || L % 4 || K < 4 || K % 4 || V < 1) return 0;
  if (prep_smem_floats(L, K) * sizeof(float) > 227 * 1024) return 0;
  for (int vt = 64; vt >= 1; vt /= 2)
    if (V % vt == 0 && scan_smem_floats(L, K, vt) * sizeof(float) <= 227 * 1024) return vt;
  return 0;
}

size_t gdn2_chunk_workspace_bytes(long long BH, int T, int L, int K) {
  const long long nch = (T + L - 1) / L;
  return (size_t)BH * nch * chunk_slot_floats(L, K) * sizeof(float);
}

cudaError_t launch_gdn2(const Gdn2Args& a, int mode, int chunk, void* ws, cudaStream_t stream) {
  const long long BH = (long long)a.B * a.H;
  if (BH == 0 || (a.T == 0 && !a.S_out)) return cudaSuccess;
  if (BH > 65535) return cudaErrorInvalidValue;
  if (mode == 0 && a.T == 1 && a.V % 128 == 0 && a.K <= 128) {  // (K 256 would not fit the registers)
    const dim3 grid(a.V / 128, (unsigned)BH);
#define STEP4(RPW)                                                                        \
  if (a.dtype == 0)                                                                       \
    gdn2_step_v4_kernel<float, RPW><<<grid, 32 * STEP_WARPS, 0, stream>>>(a);             \
  else                                                                                    \
    gdn2_step_v4_kernel<__nv_bfloat16, RPW><<<grid, 32 * STEP_WARPS, 0, stream>>>(a);
    switch (a.K) {
      case 32: STEP4(4) break;
      case 64: STEP4(8) break;
      case 128: STEP4(16) break;
      default: return cudaErrorInvalidValue;
    }
#undef STEP4
    return cudaGetLastError();
  }
  if (mode == 0 && a.T == 1) {
    const dim3 grid((a.V + 31) / 32, (unsigned)BH);
#define STEP(RPW)                                                                         \
  if (a.dtype == 0)                                                                       \
    gdn2_step_kernel<float, RPW><<<grid, 32 * STEP_WARPS, 0, stream>>>(a);                \
  else                                                                                    \
    gdn2_step_kernel<__nv_bfloat16, RPW><<<grid, 32 * STEP_WARPS, 0, stream>>>(a);
    switch (a.K) {
      case 32: STEP(4) break;
      case 64: STEP(8) break;
      case 128: STEP(16) break;
      case 256: STEP(32) break;
      default: return cudaErrorInvalidValue;
    }
#undef STEP
    return cudaGetLastError();
  }
  if (mode == 0) {
    const dim3 grid((a.V + REC_WARPS * REC_C - 1) / (REC_WARPS * REC_C), (unsigned)BH);
    const dim3 block(32 * REC_WARPS);
#define REC(KPL)                                                                         \
  if (a.dtype == 0)                                                                      \
    gdn2_recurrent_kernel<float, KPL><<<grid, block, 0, stream>>>(a);                    \
  else                                                                                   \
    gdn2_recurrent_kernel<__nv_bfloat16, KPL><<<grid, block, 0, stream>>>(a);
    switch (a.K) {
      case 32: REC(1) break;
      case 64: REC(2) break;
      case 128: REC(4) break;
      case 256: REC(8) break;
      default: return cudaErrorInvalidValue;
    }
#undef REC
    return cudaGetLastError();
  }
  const int VT = gdn2_chunk_vtile(chunk, a.K, a.V);
  if (VT == 0 || !ws) return cudaErrorInvalidValue;
  const long long nch = (a.T + chunk - 1) / chunk;
  if (nch > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int smem_p = (int)(prep_smem_floats(chunk, a.K) * sizeof(float));
  const int smem_s = (int)(scan_smem_floats(chunk, a.K, VT) * sizeof(float));
  float* wsf = static_cast<float*>(ws);
  const dim3 grid_p((unsigned)nch, (unsigned)BH), grid_s(a.V / VT, (unsigned)BH);
  cudaError_t e;
  if (a.dtype == 0) {
    e = cudaFuncSetAttribute(gdn2_chunk_prep_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_p);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn2_chunk_scan_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_s);
    if (e != cudaSuccess) return e;
    gdn2_chunk_prep_kernel<float><<<grid_p, CH_THREADS, smem_p, stream>>>(a, chunk, wsf);
    gdn2_chunk_scan_kernel<float><<<grid_s, CH_THREADS, smem_s, stream>>>(a, chunk, VT, wsf);
  } else {
    e = cudaFuncSetAttribute(gdn2_chunk_prep_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_p);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn2_chunk_scan_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem_s);
    if (e != cudaSuccess) return e;
    gdn2_chunk_prep_kernel<__nv_bfloat16><<<grid_p, CH_THREADS, smem_p, stream>>>(a, chunk, wsf);
    gdn2_chunk_scan_kernel<__nv_bfloat16><<<grid_s, CH_THREADS, smem_s, stream>>>(a, chunk, VT, wsf);
  }
  return cudaGetLastError();
}

}  // namespace mlstm
