// Backward of the mLSTM / retention recurrence (gradients of h and of the final state with
// respect to q, k, v, the gate pre-activations, the output gate and the initial state).
//
// One CTA per (batch, head); the head's blocks are taken in turn.  The stabiliser m is a
// function of the gates that h does not depend on (C' = exp(-m) C for any sequence m, and
// the division by max(|n'.q|, exp(-m)) removes the factor), so the steps are differentiated
// with m held at the values this kernel computes: any sequence works as long as f', i' and
// the floor use the same one.  In stabilised units (D = dL/dC'_t, G = dL/dn'_t accumulated
// from the end):
//   dnum_t = o_t dh_t / den_t,   P_t = sum_r o dh num / den,   dd_t = -P_t / den_t * sign(d_t)
//   when |d_t| > exp(-m_t) (0 on the floor),  d_t = n'_t . q_t
//   dq_t = C'_t^T dnum_t + dd_t n'_t
//   D += dnum_t q_t^T, G += dd_t q_t;  dv_t = i'_t D k_t;  dk_t = i'_t (D^T v_t + G)
//   ditilde_t = v_t . dv_t + i'_t G . k_t;  then D, G *= f'_t
// The forget gate's gradient uses the identity (from C'_t = f' C'_{t-1} + i' v k^T and the
// recursion of <D_t, C'_t>)
//   dlf_t = sum_{tau >= t} (dnum_tau . num_tau + dd_tau d_tau - ditilde_tau)
//           + <dC_S, C'_S> + dn_S . n'_S,
// so no pass needs C'_{t-1} and D_t together; dftilde = dlf * sigmoid(-ftilde).
// Retention: f' = gamma_h, i' = 1, no n, no floor, no output gate.
//
// Phase 1 walks t forward (C', n', the read-out and the denominators, dq); phase 2 walks t
// backward (D, G: dv, dk, ditilde); a last pass forms the gate gradients.  The state of one
// block lives in shared memory (value rows padded by one column against bank conflicts):
// a thread per value row for row products, a thread per key column for column products.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace mlstm {
namespace {

constexpr int NTB = 256;

// block-wide sum of one value per thread (every thread gets the total)
__device__ __forceinline__ float block_sum(float x, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();  // red is free
  if (lane == 0) red[warp] = x;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < NTB / 32; ++w) s += red[w];
  return s;
}

// Products over the block state St [dv][dk + 1] with all threads.  Thread t owns key column
// c = t % dk and the value rows r = t / dk (mod NTB / dk) (column map), or value row
// r = t % dv and the key columns c = t / dv (mod NTB / dv) (row map); partial sums meet in
// `part` [NTB] and one thread per output adds them.  Each call ends with a barrier.
//   col_prod: out[c] = sum_r St[r][c] x[r]      row_prod: out[r] = sum_c St[r][c] x[c]
__device__ __forceinline__ void col_prod(const float* St, int ld, int dk, int dv, const float* x, float* part,
                                         float* out) {
  const int t = threadIdx.x, rg = NTB / dk;
  if (t < rg * dk) {
    const int c = t % dk;
    float s = 0.f;
    for (int r = t / dk; r < dv; r += rg) s += St[r * ld + c] * x[r];
    part[t] = s;
  }
  __syncthreads();
  if (t < dk) {
    float s = 0.f;
    for (int j = 0; j < rg; ++j) s += part[j * dk + t];
    out[t] = s;
  }
  __syncthreads();
}
__device__ __forceinline__ void row_prod(const float* St, int ld, int dk, int dv, const float* x, float* part,
                                         float* out) {
  const int t = threadIdx.x, sl = NTB / dv;
  if (t < sl * dv) {
    const int r = t % dv;
    float s = 0.f;
    for (int c = t / dv; c < dk; c += sl) s += St[r * ld + c] * x[c];
    part[t] = s;
  }
  __syncthreads();
  if (t < dv) {
    float s = 0.f;
    for (int j = 0; j < sl; ++j) s += part[j * dv + t];
    out[t] = s;
  }
  __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(NTB, 1) bwd_kernel(BwdArgs a) {
  extern __shared__ float smf[];
  const int dk = a.dk, dv = a.dv, S = a.S, ld = dk + 1;
  float* St = smf;               // [dv][dk + 1]: C' in phase 1, D in phase 2
  float* nv = St + dv * ld;      // [dk]: n' in phase 1, G in phase 2
  float* qs = nv + dk;           // [dk]
  float* ks = qs + dk;           // [dk]
  float* vs = ks + dk;           // [dv]
  float* dhs = vs + dv;          // [dv]
  float* os = dhs + dv;          // [dv]
  float* dnum = os + dv;         // [dv]
  float* red = dnum + dv;        // [NTB / 32]
  float* part = red + NTB / 32;  // [NTB] partial sums of the state products
  float* rowv = part + NTB;      // [dv] row products
  float* colv = rowv + dv;       // [dk] column products
  __shared__ float sc[4];

  const int tid = threadIdx.x;
  const int bh = blockIdx.x, head = bh % a.NH;
  // column map of the state loops: column tid % dk, rows tid / dk + j * cstep
  const int cstep = NTB / dk, ccol = tid % dk, crow0 = tid / dk;
  const bool ret = a.retention != 0;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* dh = static_cast<const T*>(a.dh);
  const T* og = ret ? nullptr : static_cast<const T*>(a.og);
  // per-head workspace: m, f', i', the per-token sums over blocks (r_t for the forget
  // gradient, ditilde_t) and per-block den_t, d_t, dd_t
  float* wm = a.ws + (size_t)bh * 8 * S;
  float* wf = wm + S;
  float* wi = wf + S;
  float* wr = wi + S;
  float* wdi = wr + S;
  float* wden = wdi + S;
  float* wd = wden + S;
  float* wdd = wd + S;

  // ---- gates: m_t = max(lf_t + m_{t-1}, itilde_t), f'_t, i'_t (one thread; cheap)
  if (tid == 0) {
    if (ret) {
      const float g = expf(retention_log_gamma(head));
      for (int t = 0; t < S; ++t) {
        wm[t] = 0.f;
        wf[t] = g;
        wi[t] = 1.f;
      }
    } else {
      float m = a.m0 ? a.m0[bh] : 0.f;
      for (int t = 0; t < S; ++t) {
        const float lf = log_sigmoid(a.fg[(size_t)bh * S + t]);
        const float li = a.ig[(size_t)bh * S + t];
        const float mn = fmaxf(lf + m, li);
        wf[t] = expf(lf + m - mn);
        wi[t] = expf(li - mn);
        wm[t] = mn;
        m = mn;
      }
    }
  }
  for (int t = tid; t < S; t += NTB) {
    wr[t] = 0.f;
    wdi[t] = 0.f;
  }
  if (tid == 0) {
    sc[2] = 0.f;  // final-state term of the forget gradient, summed over blocks
    sc[3] = 0.f;  // dm0, summed over blocks
  }
  __syncthreads();

  for (int blk = 0; blk < a.nb; ++blk) {
    const size_t slice = (size_t)bh * a.nb + blk;
    const size_t qoff = (size_t)bh * S * a.DHQK + (size_t)blk * dk;
    const size_t voff = (size_t)bh * S * a.DHV + (size_t)blk * dv;
    // ---------------------------------------------------------------- phase 1 (forward)
    for (int e = tid; e < dv * dk; e += NTB) {
      const int r = e / dk, c = e % dk;
      St[r * ld + c] = a.C0 ? a.C0[slice * dv * dk + e] : 0.f;
    }
    for (int c = tid; c < dk; c += NTB) nv[c] = (!ret && a.n0) ? a.n0[slice * dk + c] : 0.f;
    __syncthreads();
    // the next token's inputs are loaded into registers while this token is worked on
    // (dk, dv <= NTB: one element of each vector per thread)
    float pq = 0.f, pk = 0.f, pv = 0.f, pdh = 0.f, po = 1.f, pfp = 0.f, pip = 0.f, pmt = 0.f;
    auto fetch1 = [&](int t) {
      if (tid < dk) {
        pq = io<T>::load(q, qoff + (size_t)t * a.DHQK + tid);
        pk = io<T>::load(k, qoff + (size_t)t * a.DHQK + tid);
      }
      if (tid < dv) {
        pv = io<T>::load(v, voff + (size_t)t * a.DHV + tid);
        pdh = io<T>::load(dh, voff + (size_t)t * a.DHV + tid);
        po = og ? io<T>::load(og, voff + (size_t)t * a.DHV + tid) : 1.f;
      }
      pfp = wf[t];
      pip = wi[t];
      pmt = wm[t];
    };
    if (S > 0) fetch1(0);
    for (int t = 0; t < S; ++t) {
      const float fp = pfp, ip = pip, mt = pmt;
      if (tid < dk) {
        qs[tid] = pq;
        ks[tid] = pk;
      }
      if (tid < dv) {
        vs[tid] = pv;
        dhs[tid] = pdh;
        os[tid] = po;
      }
      __syncthreads();
      if (t + 1 < S) fetch1(t + 1);
      if (tid < cstep * dk) {
        const float kc = ip * ks[ccol];
        for (int r = crow0; r < dv; r += cstep) St[r * ld + ccol] = fp * St[r * ld + ccol] + vs[r] * kc;
      }
      if (!ret)
        for (int c = tid; c < dk; c += NTB) nv[c] = fp * nv[c] + ip * ks[c];
      __syncthreads();
      // d_t = n'_t . q_t and the floor
      float dpart = 0.f;
      if (!ret)
        for (int c = tid; c < dk; c += NTB) dpart += nv[c] * qs[c];
      const float d = ret ? 0.f : block_sum(dpart, red);
      const float den = ret ? 1.f : fmaxf(fabsf(d), expf(-mt));
      // read-out rows: num_r = C'_t[r,:] . q_t
      row_prod(St, ld, dk, dv, qs, part, rowv);
      float ppart = 0.f;
      for (int r = tid; r < dv; r += NTB) {
        const float hn = rowv[r] / den;
        dnum[r] = os[r] * dhs[r] / den;
        ppart += os[r] * dhs[r] * hn;
        if (a.dog) a.dog[voff + (size_t)t * a.DHV + r] = dhs[r] * hn;
      }
      const float P = ret ? 0.f : block_sum(ppart, red);  // also orders the dnum stores
      if (ret) __syncthreads();
      const float dd = (!ret && fabsf(d) > expf(-mt)) ? -P / den * copysignf(1.f, d) : 0.f;
      col_prod(St, ld, dk, dv, dnum, part, colv);
      for (int c = tid; c < dk; c += NTB) a.dq[qoff + (size_t)t * a.DHQK + c] = colv[c] + dd * nv[c];
      if (tid == 0) {
        wden[t] = den;
        wd[t] = d;
        wdd[t] = dd;
        wr[t] += P + dd * d;
      }
      __syncthreads();
    }
    // final-state term <dC_S, C'_S> + dn_S . n'_S of the forget gradient
    if (!ret && (a.dC || a.dn)) {
      float part = 0.f;
      if (a.dC)
        for (int e = tid; e < dv * dk; e += NTB) part += a.dC[slice * dv * dk + e] * St[(e / dk) * ld + e % dk];
      if (a.dn)
        for (int c = tid; c < dk; c += NTB) part += a.dn[slice * dk + c] * nv[c];
      const float s = block_sum(part, red);
      if (tid == 0) sc[2] += s;
    }
    __syncthreads();
    // ---------------------------------------------------------------- phase 2 (backward)
    for (int e = tid; e < dv * dk; e += NTB) {
      const int r = e / dk, c = e % dk;
      St[r * ld + c] = a.dC ? a.dC[slice * dv * dk + e] : 0.f;
    }
    for (int c = tid; c < dk; c += NTB) nv[c] = (!ret && a.dn) ? a.dn[slice * dk + c] : 0.f;
    __syncthreads();
    float pden = 1.f, pdd = 0.f;
    auto fetch2 = [&](int t) {
      fetch1(t);
      pden = wden[t];
      pdd = wdd[t];
    };
    if (S > 0) fetch2(S - 1);
    for (int t = S - 1; t >= 0; --t) {
      const float fp = pfp, ip = pip, den = pden, dd = pdd;
      if (tid < dk) {
        qs[tid] = pq;
        ks[tid] = pk;
      }
      if (tid < dv) {
        vs[tid] = pv;
        dnum[tid] = po * pdh / den;
      }
      __syncthreads();
      if (t > 0) fetch2(t - 1);
      if (tid < cstep * dk) {
        const float qc = qs[ccol];
        for (int r = crow0; r < dv; r += cstep) St[r * ld + ccol] += dnum[r] * qc;
      }
      if (!ret)
        for (int c = tid; c < dk; c += NTB) nv[c] += dd * qs[c];
      __syncthreads();
      row_prod(St, ld, dk, dv, ks, part, rowv);
      col_prod(St, ld, dk, dv, vs, part, colv);
      float bpart = 0.f;
      for (int r = tid; r < dv; r += NTB) {
        const float g = ip * rowv[r];
        a.dv_out[voff + (size_t)t * a.DHV + r] = g;
        bpart += vs[r] * g;
      }
      for (int c = tid; c < dk; c += NTB) {
        const float gn = ret ? 0.f : ip * nv[c];
        a.dk_out[qoff + (size_t)t * a.DHQK + c] = ip * colv[c] + gn;
        bpart += gn * ks[c];
      }
      if (!ret) {
        const float di = block_sum(bpart, red);
        if (tid == 0) {
          wdi[t] += di;
          wr[t] -= di;
        }
      }
      __syncthreads();
      if (tid < cstep * dk)
        for (int r = crow0; r < dv; r += cstep) St[r * ld + ccol] *= fp;
      if (!ret)
        for (int c = tid; c < dk; c += NTB) nv[c] *= fp;
      __syncthreads();
    }
    // initial-state gradients: dC0 = D, dn0 = G; dm0 = <dC0, C0> + dn0 . n0
    float part = 0.f;
    for (int e = tid; e < dv * dk; e += NTB) {
      const float g = St[(e / dk) * ld + e % dk];
      if (a.dC0) a.dC0[slice * dv * dk + e] = g;
      if (a.C0) part += g * a.C0[slice * dv * dk + e];
    }
    if (!ret)
      for (int c = tid; c < dk; c += NTB) {
        if (a.dn0) a.dn0[slice * dk + c] = nv[c];
        if (a.n0) part += nv[c] * a.n0[slice * dk + c];
      }
    if (!ret) {
      const float s = block_sum(part, red);
      if (tid == 0) sc[3] += s;
    }
    __syncthreads();
  }
  // ---- gate gradients: dlf_t = sum_{tau >= t} r_tau + final-state term (one thread)
  if (!ret && tid == 0) {
    float acc = sc[2];
    for (int t = S - 1; t >= 0; --t) {
      acc += wr[t];
      const float ft = a.fg[(size_t)bh * S + t];
      if (a.dfg) a.dfg[(size_t)bh * S + t] = acc / (1.f + expf(ft));  // d logsigmoid = sigmoid(-x)
      if (a.dig) a.dig[(size_t)bh * S + t] = wdi[t];
    }
    if (a.dm0) a.dm0[bh] = sc[3];
  }
}

}  // namespace

size_t bwd_smem_bytes(int dk, int dv) {
  return ((size_t)dv * (dk + 1) + 4 * (size_t)dk + 5 * (size_t)dv + NTB / 32 + NTB) * sizeof(float);
}

size_t bwd_workspace_bytes(long long BH, int S) { return (size_t)BH * 8 * (size_t)S * sizeof(float); }

bool bwd_supported(int dk, int dv) {
  return dk >= 1 && dv >= 1 && dk <= NTB && dv <= NTB && bwd_smem_bytes(dk, dv) <= 200 * 1024;
}

cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  const long long BH = (long long)a.B * a.NH;
  if (BH == 0) return cudaSuccess;
  const size_t smem = bwd_smem_bytes(a.dk, a.dv);
  cudaError_t e;
  if (a.dtype == 1) {
    e = cudaFuncSetAttribute(bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_kernel<__nv_bfloat16><<<(unsigned)BH, NTB, smem, stream>>>(a);
  } else {
    e = cudaFuncSetAttribute(bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_kernel<float><<<(unsigned)BH, NTB, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mlstm
