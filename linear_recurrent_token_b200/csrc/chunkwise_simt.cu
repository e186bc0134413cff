// Chunkwise prefill, SIMT fp32 variant (sm_100a).  Used for fp32 inputs (where a
// bf16/tf32 tensor-core product would not meet fp32 accuracy) and for shapes the
// tensor-core kernels do not cover.  One CTA owns a (batch, head, block, value-row
// tile) and walks the chunks of the sequence in order, keeping its tile of the state
// C [dv_tile x dk] and the normaliser n [dk] in shared memory.
//
// Per chunk of L tokens (local index t, s), with b the inclusive cumulative sum of
// log f inside the chunk, g its total, m_c the stabiliser at the end of the previous
// chunk and m_t the per-token stabiliser from the gate-prep scan:
//   P[t,s] = (q_t . k_s) exp(b_t - b_s + itilde_s - m_t)          for s <= t
//   h_t    = o_t [sum_s P[t,s] v_s + e^{b_t+m_c-m_t} C q_t]
//            / max(|sum_s P[t,s] + e^{b_t+m_c-m_t} n . q_t|, e^{-m_t})
//   C     <- e^{g+m_c-m_next} C + sum_s e^{g-b_s+itilde_s-m_next} v_s k_s^T   (same for n)
// Retention replaces the gate weights by powers of gamma_h and drops the normaliser
// (RetNet "Key Innovation": D[n,m] = gamma^(n-m)).
// With a.nbias set, the normaliser is the scalar n_t = f n_{t-1} + i of Edifice.Recurrent.
// XLSTMv2 ("Key Improvements" #2) and the denominator max(|n_t + bias|, 1), i.e. in these units
//   max(|sum_s exp(b_t - b_s + itilde_s - m_t) + e^{b_t+m_c-m_t} n + bias e^{-m_t}|, e^{-m_t}).
#include "common.cuh"
#include "kernels.h"

namespace mlstm {

static __host__ __device__ inline size_t simt_floats(int L, int dk, int TV) {
  const size_t ldk = dk + 1;
  return 2 * L * ldk + TV * ldk + (size_t)L * TV + (size_t)L * (L + 1) + dk + 6 * (size_t)L + 4;
}

size_t simt_walk_smem_bytes(int chunk, int dk, int dv_tile) {
  return simt_floats(chunk, dk, dv_tile) * sizeof(float);
}

int simt_walk_pick_tile(int chunk, int dk, int dv) {
  // value-row tile: 32 rows, or 16 for narrow blocks so that more CTAs share the work
  int tv = dv <= 32 ? (dv < 16 ? dv : 16) : 32;
  while (tv > 1 && simt_walk_smem_bytes(chunk, dk, tv) > 227 * 1024) tv /= 2;
  return simt_walk_smem_bytes(chunk, dk, tv) <= 227 * 1024 ? tv : 0;
}

// Shared-memory dot products with four independent partial sums (the loops are latency-bound
// with one accumulator).
__device__ __forceinline__ float dot_smem(const float* x, const float* y, int n) {
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  int i = 0;
  for (; i + 4 <= n; i += 4)
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] = fmaf(x[i + u], y[i + u], a[u]);
  for (; i < n; ++i) a[0] = fmaf(x[i], y[i], a[0]);
  return (a[0] + a[1]) + (a[2] + a[3]);
}
// sum_i x[i] y[i * ystride]
__device__ __forceinline__ float dot_smem_strided(const float* x, const float* y, int ystride, int n) {
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  int i = 0;
  for (; i + 4 <= n; i += 4)
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] = fmaf(x[i + u], y[(i + u) * ystride], a[u]);
  for (; i < n; ++i) a[0] = fmaf(x[i], y[i * ystride], a[0]);
  return (a[0] + a[1]) + (a[2] + a[3]);
}
__device__ __forceinline__ float sum_smem(const float* x, int n) {
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  int i = 0;
  for (; i + 4 <= n; i += 4)
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] += x[i + u];
  for (; i < n; ++i) a[0] += x[i];
  return (a[0] + a[1]) + (a[2] + a[3]);
}

template <typename T>
__global__ void __launch_bounds__(256) simt_walk_kernel(WalkArgs a) {
  extern __shared__ float smem[];
  const int L = a.chunk, dk = a.dk, TV = a.dv_tile, ldk = dk + 1;
  float* Qs = smem;
  float* Ks = Qs + (size_t)L * ldk;
  float* Cs = Ks + (size_t)L * ldk;
  float* Vs = Cs + (size_t)TV * ldk;
  float* Ps = Vs + (size_t)L * TV;
  float* ns = Ps + (size_t)L * (L + 1);
  float* bl = ns + dk;
  float* li = bl + L;
  float* mt = li + L;
  float* sint = mt + L;
  float* wv = sint + L;
  float* den = wv + L;
  float* scal = den + L;

  const int tid = threadIdx.x, nt = blockDim.x;
  const int slice = blockIdx.y;
  const int blk = slice % a.nb, bh = slice / a.nb, head = bh % a.NH;
  const int v0 = blockIdx.x * TV;
  const int tv = min(TV, a.dv - v0);
  const int S = a.S, DHQK = a.DHQK, DHV = a.DHV, dv = a.dv;
  const bool ret = a.retention != 0;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* og = static_cast<const T*>(a.og);
  T* h = static_cast<T*>(a.h);
  const float lg = ret ? retention_log_gamma(head) : 0.f;

  for (int i = tid; i < tv * dk; i += nt) {
    const int r = i / dk, c = i % dk;
    Cs[r * ldk + c] = a.C0 ? a.C0[((size_t)slice * dv + v0 + r) * dk + c] : 0.f;
  }
  const bool scalar_n = a.nbias != nullptr && !ret;
  const float nbias = scalar_n ? a.nbias[head] : 0.f;
  if (scalar_n) {
    if (tid == 0) ns[0] = a.n_init[bh];
  } else {
    for (int c = tid; c < dk; c += nt) ns[c] = ret ? 0.f : a.n_init[(size_t)slice * dk + c];
  }
  float m_c = ret ? 0.f : a.m_init[bh];

  for (int c0 = 0; c0 < S; c0 += L) {
    const int Lc = min(L, S - c0);
    const size_t tok0 = (size_t)bh * S + c0;
    for (int i = tid; i < L * dk; i += nt) {
      const int t = i / dk, c = i % dk;
      const bool ok = t < Lc;
      Qs[t * ldk + c] = ok ? io<T>::load(q, (tok0 + t) * DHQK + (size_t)blk * dk + c) : 0.f;
      Ks[t * ldk + c] = ok ? io<T>::load(k, (tok0 + t) * DHQK + (size_t)blk * dk + c) : 0.f;
    }
    for (int i = tid; i < L * TV; i += nt) {
      const int t = i / TV, r = i % TV;
      Vs[i] = (t < Lc && r < tv) ? io<T>::load(v, (tok0 + t) * DHV + (size_t)blk * dv + v0 + r) : 0.f;
    }
    if (tid < L) {
      const int t = tid;
      if (ret) {
        bl[t] = (float)(t + 1) * lg;
        li[t] = 0.f;
        mt[t] = 0.f;
      } else {
        bl[t] = t < Lc ? log_sigmoid(a.fg[tok0 + t]) : 0.f;
        li[t] = t < Lc ? a.ig[tok0 + t] : 0.f;
        mt[t] = t < Lc ? a.m_tok[tok0 + t] : 0.f;
      }
    }
    __syncthreads();
    if (tid < 32 && !ret) {  // inclusive cumulative sum of log f over the chunk: a warp scan, each
                             // lane over a run of ceil(Lc / 32) consecutive entries
      const int per = (Lc + 31) / 32, t0 = tid * per, t1 = min(t0 + per, Lc);
      float part = 0.f;
      for (int t = t0; t < t1; ++t) part += bl[t];
      float run = part;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, run, o);
        if (tid >= o) run += u;
      }
      float acc = run - part;
      for (int t = t0; t < t1; ++t) {
        acc += bl[t];
        bl[t] = acc;
      }
    }
    __syncthreads();
    const float g = bl[Lc - 1];
    const float m_next = ret ? 0.f : mt[Lc - 1];
    if (tid < Lc) {
      sint[tid] = expf(bl[tid] + m_c - mt[tid]);
      wv[tid] = expf(g - bl[tid] + li[tid] - m_next);
    }
    const float decay = expf(g + m_c - m_next);
    for (int i = tid; i < L * L; i += nt) {
      const int t = i / L, s = i % L;
      float p = 0.f;
      if (s <= t && t < Lc) {
        p = dot_smem(Qs + t * ldk, Ks + s * ldk, dk) * expf(bl[t] - bl[s] + li[s] - mt[t]);
      }
      Ps[t * (L + 1) + s] = p;
    }
    __syncthreads();
    if (scalar_n) {
      for (int t = tid; t < Lc; t += nt) {
        float rs = 0.f;
        for (int s = 0; s <= t; ++s) rs += expf(bl[t] - bl[s] + li[s] - mt[t]);
        const float emt = expf(-mt[t]);
        den[t] = fmaxf(fabsf(rs + sint[t] * ns[0] + nbias * emt), emt);
      }
    } else if (!ret) {
      for (int t = tid; t < Lc; t += nt) {
        const float rs = sum_smem(Ps + t * (L + 1), t + 1), qn = dot_smem(Qs + t * ldk, ns, dk);
        den[t] = fmaxf(fabsf(rs + sint[t] * qn), expf(-mt[t]));
      }
    }
    __syncthreads();
    for (int i = tid; i < Lc * tv; i += nt) {
      const int t = i / tv, r = i % tv;
      const float acc_i = dot_smem_strided(Ps + t * (L + 1), Vs + r, TV, t + 1);
      const float acc_c = dot_smem(Qs + t * ldk, Cs + r * ldk, dk);
      float hv = acc_i + sint[t] * acc_c;
      const size_t hi = (tok0 + t) * DHV + (size_t)blk * dv + v0 + r;
      if (!ret) {
        hv = hv / den[t];
        if (og) hv *= io<T>::load(og, hi);
      }
      io<T>::store(h, hi, hv);
    }
    __syncthreads();
    for (int i = tid; i < tv * dk; i += nt) {
      const int r = i / dk, c = i % dk;
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
      int s = 0;
      for (; s + 4 <= Lc; s += 4)
#pragma unroll
        for (int u = 0; u < 4; ++u) a4[u] = fmaf(wv[s + u] * Vs[(s + u) * TV + r], Ks[(s + u) * ldk + c], a4[u]);
      for (; s < Lc; ++s) a4[0] = fmaf(wv[s] * Vs[s * TV + r], Ks[s * ldk + c], a4[0]);
      Cs[r * ldk + c] = decay * Cs[r * ldk + c] + ((a4[0] + a4[1]) + (a4[2] + a4[3]));
    }
    if (scalar_n) {
      if (tid == 0) {
        float acc = 0.f;
        for (int s = 0; s < Lc; ++s) acc += wv[s];
        ns[0] = decay * ns[0] + acc;
      }
    } else if (!ret) {
      for (int c = tid; c < dk; c += nt) {
        float acc = 0.f;
        for (int s = 0; s < Lc; ++s) acc += wv[s] * Ks[s * ldk + c];
        ns[c] = decay * ns[c] + acc;
      }
    }
    m_c = m_next;
    __syncthreads();
  }
  (void)scal;
  if (a.C_out)
    for (int i = tid; i < tv * dk; i += nt) {
      const int r = i / dk, c = i % dk;
      a.C_out[((size_t)slice * dv + v0 + r) * dk + c] = Cs[r * ldk + c];
    }
  if (!ret && blockIdx.x == 0) {
    if (a.n_out && scalar_n) {
      if (blk == 0 && tid == 0) a.n_out[bh] = ns[0];
    } else if (a.n_out) {
      for (int c = tid; c < dk; c += nt) a.n_out[(size_t)slice * dk + c] = ns[c];
    }
    if (a.m_out && blk == 0 && tid == 0) a.m_out[bh] = m_c;
  }
}

cudaError_t launch_simt_walk(const WalkArgs& a, cudaStream_t stream) {
  const int slices = a.B * a.NH * a.nb;
  if (slices == 0) return cudaSuccess;
  const size_t smem = simt_walk_smem_bytes(a.chunk, a.dk, a.dv_tile);
  if (a.dv_tile <= 0 || smem > 227 * 1024) return cudaErrorInvalidValue;
  dim3 grid((a.dv + a.dv_tile - 1) / a.dv_tile, slices);
  if (grid.y > 65535) return cudaErrorInvalidValue;
  cudaError_t e;
  if (a.dtype == 0) {
    e = cudaFuncSetAttribute(simt_walk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    simt_walk_kernel<float><<<grid, 256, smem, stream>>>(a);
  } else {
    e = cudaFuncSetAttribute(simt_walk_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    simt_walk_kernel<__nv_bfloat16><<<grid, 256, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mlstm
