// Gated DeltaNet-2 (burn-gdn2 config.rs): the delta rule with a per-key-channel decay and
// channel-wise erase (b, key channels) and write (w, value channels) gates, state S [K, V]
// per (batch, head) in fp32:
//
//   S' = Diag(e^{g_t}) S,  r = S'^T k_t,  S = S' - (b_t o k_t) r^T + k_t (w_t o v_t)^T,  o_t = S^T q_t
//
// gdn2_recurrent_kernel  Gdn2Mode::FusedRecurrent.  One warp owns C value columns of one head
//   for the whole sequence; lane l holds key rows l, l+32, ... of those columns in registers,
//   so the two reductions over K per token (r and o) are warp shuffles and the state never
//   leaves the chip between tokens.  With T = 1 and the state in place this is the decode step
//   (one HBM read and write of S); gdn2_step_kernel below lays the state out for that case.
// gdn2_chunk_kernel  Gdn2Mode::Chunk.  One CTA owns a (head, value tile) and walks the chunks;
//   per chunk, with G the cumulative log decay inside the chunk (every exponent below <= 0):
//     LA[t,s] = sum_i k_ti k_si e^{G_ti-G_si} (s<t),  LE[t,s] = sum_i k_ti bk_si e^{..} (s<t),
//     QA, QE the same with q_t (s<=t);
//     R = (I + LE)^{-1} (k e^{G} S + LA U)            (U = w o v; one triangular solve)
//     o = (q e^{G}) S + QA U - QE R
//     S <- e^{G_L} o S + (k e^{G_L-G})^T U - (bk e^{G_L-G})^T R
//   i.e. the WY-style block form of the recurrence: dense products inside the chunk, the state
//   carried between chunks.  fp32 SIMT, state tile in shared memory.
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

template <typename T, int KPL>
__global__ void __launch_bounds__(32 * REC_WARPS) gdn2_recurrent_kernel(Gdn2Args a) {
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
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int c = 0; c < REC_C; ++c) r[c] += __shfl_xor_sync(0xffffffffu, r[c], off);
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
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int c = 0; c < REC_C; ++c) y[c] += __shfl_xor_sync(0xffffffffu, y[c], off);
#pragma unroll
    for (int c = 0; c < REC_C; ++c)
      if (lane == c && c < nc) st_out(o + (size_t)t * a.V + c, y[c]);
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

// ------------------------------------------------------------------ chunk (WY block form)
constexpr int CH_THREADS = 256;

struct ChunkSmem {
  int L, K, VT, lk, ll;
  // offsets in floats
  size_t G, Kc, Bk, Qc, S, U, R, LA, LE, QA, QE, gL, total;
};
__host__ __device__ inline ChunkSmem chunk_smem(int L, int K, int VT) {
  ChunkSmem m;
  m.L = L;
  m.K = K;
  m.VT = VT;
  m.lk = K + 1;  // padded rows: threads on different tokens read different banks
  m.ll = L + 1;
  size_t o = 0;
  m.G = o, o += (size_t)L * m.lk;
  m.Kc = o, o += (size_t)L * m.lk;
  m.Bk = o, o += (size_t)L * m.lk;
  m.Qc = o, o += (size_t)L * m.lk;
  m.S = o, o += (size_t)K * VT;
  m.U = o, o += (size_t)L * VT;
  m.R = o, o += (size_t)L * VT;
  m.LA = o, o += (size_t)L * m.ll;
  m.LE = o, o += (size_t)L * m.ll;
  m.QA = o, o += (size_t)L * m.ll;
  m.QE = o, o += (size_t)L * m.ll;
  m.gL = o, o += (size_t)K;
  m.total = o;
  return m;
}

template <typename T>
__global__ void __launch_bounds__(CH_THREADS) gdn2_chunk_kernel(Gdn2Args a, int L, int VT) {
  extern __shared__ float sm[];
  const int K = a.K, tid = threadIdx.x;
  const ChunkSmem M = chunk_smem(L, K, VT);
  const int lk = M.lk, ll = M.ll;
  float *G = sm + M.G, *Kc = sm + M.Kc, *Bk = sm + M.Bk, *Qc = sm + M.Qc, *S = sm + M.S, *U = sm + M.U,
        *R = sm + M.R, *LA = sm + M.LA, *LE = sm + M.LE, *QA = sm + M.QA, *QE = sm + M.QE, *gL = sm + M.gL;
  const long long bh = blockIdx.y;
  const int j0 = blockIdx.x * VT;
  const T* q = static_cast<const T*>(a.q) + bh * a.T * K;
  const T* k = static_cast<const T*>(a.k) + bh * a.T * K;
  const T* v = static_cast<const T*>(a.v) + bh * a.T * a.V + j0;
  const float* g = a.g + bh * a.T * K;
  const float* b = a.b + bh * a.T * K;
  const float* w = a.w + bh * a.T * a.V + j0;
  T* o = static_cast<T*>(a.o) + bh * a.T * a.V + j0;
  for (int e = tid; e < K * VT; e += CH_THREADS) {
    const int i = e / VT, j = e % VT;
    S[e] = a.S0 ? a.S0[(bh * K + i) * a.V + j0 + j] : 0.f;
  }
  for (int t0 = 0; t0 < a.T; t0 += L) {
    const int Lc = min(L, a.T - t0);
    __syncthreads();  // the previous chunk is done with every buffer
    // 1. inputs of the chunk (rows past the end: zeros, which add nothing below)
    for (int e = tid; e < L * K; e += CH_THREADS) {
      const int t = e / K, i = e % K;
      float qq = 0.f, kk = 0.f, gg = 0.f, bb = 0.f;
      if (t < Lc) {
        const size_t x = (size_t)(t0 + t) * K + i;
        qq = ld_in(q + x), kk = ld_in(k + x), gg = g[x], bb = b[x];
      }
      Qc[t * lk + i] = qq, Kc[t * lk + i] = kk, G[t * lk + i] = gg, Bk[t * lk + i] = bb * kk;
    }
    for (int e = tid; e < L * VT; e += CH_THREADS) {
      const int t = e / VT, j = e % VT;
      U[e] = t < Lc ? w[(size_t)(t0 + t) * a.V + j] * ld_in(v + (size_t)(t0 + t) * a.V + j) : 0.f;
    }
    __syncthreads();
    // 2. cumulative log decay per key channel
    for (int i = tid; i < K; i += CH_THREADS) {
      float s = 0.f;
      for (int t = 0; t < L; ++t) {
        s += G[t * lk + i];
        G[t * lk + i] = s;
      }
      gL[i] = s;
    }
    __syncthreads();
    // 3. the four L x L weight matrices, 4 x 4 (t, s) blocks per thread, lower triangle only
    {
      const int nb4 = L / 4;
      for (int blk = tid; blk < nb4 * nb4; blk += CH_THREADS) {
        const int tb = blk / nb4, sb = blk % nb4;
        if (sb > tb) continue;
        float la[4][4] = {}, le[4][4] = {}, qa[4][4] = {}, qe[4][4] = {};
        for (int i = 0; i < K; ++i) {
          float gt[4], kt[4], qt[4], gs[4], ks[4], bs[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int t = 4 * tb + x, s = 4 * sb + x;
            gt[x] = G[t * lk + i], kt[x] = Kc[t * lk + i], qt[x] = Qc[t * lk + i];
            gs[x] = G[s * lk + i], ks[x] = Kc[s * lk + i], bs[x] = Bk[s * lk + i];
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
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const int t = 4 * tb + x, s = 4 * sb + y;
            LA[t * ll + s] = s < t ? la[x][y] : 0.f;
            LE[t * ll + s] = s < t ? le[x][y] : 0.f;
            QA[t * ll + s] = s <= t ? qa[x][y] : 0.f;
            QE[t * ll + s] = s <= t ? qe[x][y] : 0.f;
          }
      }
    }
    __syncthreads();
    // 4. decayed forms of the rows: Qc <- q e^{G}, G <- k e^{G} (read-out and right-hand side),
    //    Kc <- k e^{G_L - G}, Bk <- bk e^{G_L - G} (state update)
    for (int e = tid; e < L * K; e += CH_THREADS) {
      const int t = e / K, i = e % K, x = t * lk + i;
      const float gg = G[x], up = expf(gg), tail = expf(gL[i] - gg);
      Qc[x] *= up;
      G[x] = Kc[x] * up;
      Kc[x] *= tail;
      Bk[x] *= tail;
    }
    __syncthreads();
    // 5. right-hand side of the solve: R = (k e^G) S + LA U
    for (int e = tid; e < L * VT; e += CH_THREADS) {
      const int t = e / VT, j = e % VT;
      float acc = 0.f;
      for (int i = 0; i < K; ++i) acc = fmaf(G[t * lk + i], S[i * VT + j], acc);
      for (int s = 0; s < t; ++s) acc = fmaf(LA[t * ll + s], U[s * VT + j], acc);
      R[e] = acc;
    }
    __syncthreads();
    // 6. unit lower-triangular solve (I + LE) R = rhs, column by column
    for (int j = tid; j < VT; j += CH_THREADS) {
      for (int t = 1; t < L; ++t) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int s = 0;
        for (; s + 3 < t; s += 4) {
          a0 = fmaf(LE[t * ll + s], R[s * VT + j], a0);
          a1 = fmaf(LE[t * ll + s + 1], R[(s + 1) * VT + j], a1);
          a2 = fmaf(LE[t * ll + s + 2], R[(s + 2) * VT + j], a2);
          a3 = fmaf(LE[t * ll + s + 3], R[(s + 3) * VT + j], a3);
        }
        for (; s < t; ++s) a0 = fmaf(LE[t * ll + s], R[s * VT + j], a0);
        R[t * VT + j] -= (a0 + a1) + (a2 + a3);
      }
    }
    __syncthreads();
    // 7. outputs: o = (q e^G) S + QA U - QE R
    for (int e = tid; e < L * VT; e += CH_THREADS) {
      const int t = e / VT, j = e % VT;
      if (t >= Lc) continue;
      float acc = 0.f;
      for (int i = 0; i < K; ++i) acc = fmaf(Qc[t * lk + i], S[i * VT + j], acc);
      for (int s = 0; s <= t; ++s) acc = fmaf(QA[t * ll + s], U[s * VT + j], fmaf(-QE[t * ll + s], R[s * VT + j], acc));
      st_out(o + (size_t)(t0 + t) * a.V + j, acc);
    }
    // 8. state: S <- e^{G_L} S + (k e^{G_L-G})^T U - (bk e^{G_L-G})^T R  (reads S, R, U only
    //    after step 7 read them: each thread updates the elements no other thread reads here)
    __syncthreads();
    for (int e = tid; e < K * VT; e += CH_THREADS) {
      const int i = e / VT, j = e % VT;
      float acc = expf(gL[i]) * S[e];
      for (int s = 0; s < L; ++s) acc = fmaf(Kc[s * lk + i], U[s * VT + j], fmaf(-Bk[s * lk + i], R[s * VT + j], acc));
      S[e] = acc;
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
  if (L < 4 || L > 64 || L % 4 || K < 1 || V < 1) return 0;
  for (int vt = 64; vt >= 1; vt /= 2)
    if (V % vt == 0 && chunk_smem(L, K, vt).total * sizeof(float) <= 227 * 1024) return vt;
  return 0;
}

size_t gdn2_chunk_smem_bytes(int L, int K, int VT) { return chunk_smem(L, K, VT).total * sizeof(float); }

cudaError_t launch_gdn2(const Gdn2Args& a, int mode, int chunk, cudaStream_t stream) {
  const long long BH = (long long)a.B * a.H;
  if (BH == 0 || (a.T == 0 && !a.S_out)) return cudaSuccess;
  if (BH > 65535) return cudaErrorInvalidValue;
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
  if (VT == 0) return cudaErrorInvalidValue;
  const size_t smem = gdn2_chunk_smem_bytes(chunk, a.K, VT);
  const dim3 grid(a.V / VT, (unsigned)BH);
  cudaError_t e;
  if (a.dtype == 0) {
    e = cudaFuncSetAttribute(gdn2_chunk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gdn2_chunk_kernel<float><<<grid, CH_THREADS, smem, stream>>>(a, chunk, VT);
  } else {
    e = cudaFuncSetAttribute(gdn2_chunk_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    gdn2_chunk_kernel<__nv_bfloat16><<<grid, CH_THREADS, smem, stream>>>(a, chunk, VT);
  }
  return cudaGetLastError();
}

}  // namespace mlstm
