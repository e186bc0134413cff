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
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

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

// ---------------------------------------------------------------------------------------
// Chunked form of the same backward: the sequence is taken L tokens at a time and every
// product inside a chunk is a small dense one over all threads (barriers per chunk, not per
// token).  With A_t = prod_{u=t0..t} f'_u (the chunk's cumulative decay), W[t][s] =
// A_t / A_s i'_s (s <= t; the stable form exp(lA_t - lA_s + log i'_s)) and P = W o (Q K^T):
//   phase 1 (chunks forward; C', n' at the chunk start):
//     num = diag(A) Q C'^T + P V,  d = diag(A) Q n' + rowsum(P),  den, dnum, dd as before
//     dq  = diag(A) dNum C' + (W o (dNum V^T)) K + diag(dd) (diag(A) 1 n'^T + W K)
//     C' <- A_L C' + V^T diag(w) K,  n' <- A_L n' + K^T w    (w = the last row of W)
//   phase 2 (chunks backward; D, G entering from the later chunks):
//     dv  = P^T dNum + diag(w) K D^T
//     dk  = (W o (dNum V^T))^T Q + diag(w) V D + W^T diag(dd) Q + w G^T
//     D   <- A_L D + dNum^T diag(A) Q,  G <- A_L G + Q^T (A o dd)
// A numpy evaluation of these formulas equals the step-by-step oracle to rounding.
template <typename T, int L>
__global__ void __launch_bounds__(NTB, 1) bwd_chunk_kernel(BwdArgs a) {
  extern __shared__ float smf[];
  // chunk tiles have rows padded by one element, so that reading one column across the rows
  // of a warp's tokens hits distinct banks
  const int dk = a.dk, dv = a.dv, S = a.S, ld = dk + 1, lq = dk + 1, lv = dv + 1;
  float* St = smf;             // [dv][dk + 1]: C' in phase 1, D in phase 2
  float* nv = St + dv * ld;    // [dk]: n' / G
  float* Qc = nv + dk;         // [L][dk + 1]
  float* Kc = Qc + L * lq;     // [L][dk + 1]
  float* Vc = Kc + L * lq;     // [L][dv + 1]
  float* dHc = Vc + L * lv;    // [L][dv + 1]
  float* Oc = dHc + L * lv;    // [L][dv + 1] output gate, then scratch
  float* dN = Oc + L * lv;     // [L][dv + 1] dnum
  float* Pm = dN + L * lv;     // [L][L]  W o (Q K^T)
  float* Wm = Pm + L * L;      // [L][L]  W
  float* Xm = Wm + L * L;      // [L][L]  W o (dNum V^T)
  float* lA = Xm + L * L;      // [L] log A_t
  float* li = lA + L;          // [L] log i'_t (-inf past the end)
  float* tden = li + L;        // [L]
  float* tdd = tden + L;       // [L]
  float* td = tdd + L;         // [L]
  float* tP = td + L;          // [L]
  float* tmt = tP + L;         // [L] m_t
  float* eA = tmt + L;         // [L] A_t = exp(lA_t)
  float* red = eA + L;         // [NTB / 32]
  __shared__ float sc[4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, head = bh % a.NH;
  const bool ret = a.retention != 0;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* dh = static_cast<const T*>(a.dh);
  const T* og = ret ? nullptr : static_cast<const T*>(a.og);
  // per-head workspace: log f'_t, log i'_t, m_t, r_t (forget-gradient terms), ditilde_t,
  // and per block den_t, d_t, dd_t
  float* wlf = a.ws + (size_t)bh * 8 * S;
  float* wli = wlf + S;
  float* wm = wli + S;
  float* wr = wm + S;
  float* wdi = wr + S;
  float* wden = wdi + S;
  float* wd = wden + S;
  float* wdd = wd + S;

  // ---- gates by warp 0: the stabiliser recurrence m_t = max(lf_t + m_{t-1}, itilde_t) as
  // a scan of max-plus maps over the lanes' contiguous segments, then each lane walks its own
  if (warp == 0) {
    if (ret) {
      const float lg = retention_log_gamma(head);
      for (int t = lane; t < S; t += 32) {
        wlf[t] = lg;
        wli[t] = 0.f;
        wm[t] = 0.f;
      }
    } else {
      const int seg = (S + 31) / 32, t_lo = lane * seg, t_hi = min(S, t_lo + seg);
      MaxPlus mp{0.f, -INFINITY};
      for (int t = t_lo; t < t_hi; ++t)
        mp = mp_then(mp, MaxPlus{log_sigmoid(a.fg[(size_t)bh * S + t]), a.ig[(size_t)bh * S + t]});
      for (int o = 1; o < 32; o <<= 1) {
        const float A = __shfl_up_sync(0xffffffffu, mp.A, o), Bm = __shfl_up_sync(0xffffffffu, mp.Bm, o);
        if (lane >= o) mp = mp_then(MaxPlus{A, Bm}, mp);
      }
      float ex_A = __shfl_up_sync(0xffffffffu, mp.A, 1), ex_B = __shfl_up_sync(0xffffffffu, mp.Bm, 1);
      if (lane == 0) {
        ex_A = 0.f;
        ex_B = -INFINITY;
      }
      const float m0 = a.m0 ? a.m0[bh] : 0.f;
      float m = mp_apply(MaxPlus{ex_A, ex_B}, m0);
      for (int t = t_lo; t < t_hi; ++t) {
        const float lf = log_sigmoid(a.fg[(size_t)bh * S + t]), it = a.ig[(size_t)bh * S + t];
        const float mn = fmaxf(lf + m, it);
        wlf[t] = lf + m - mn;
        wli[t] = it - mn;
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
    sc[2] = 0.f;
    sc[3] = 0.f;
  }
  __syncthreads();

  const int nck = (S + L - 1) / L;
  for (int blk = 0; blk < a.nb; ++blk) {
    const size_t slice = (size_t)bh * a.nb + blk;
    const size_t qoff = (size_t)bh * S * a.DHQK + (size_t)blk * dk;
    const size_t voff = (size_t)bh * S * a.DHV + (size_t)blk * dv;
    // chunk inputs into shared memory, tokens past the end as zeros; gate logs; W and P
    auto load_chunk = [&](int t0, int Lc, bool with_o) {
#pragma unroll 4
      for (int e = tid; e < L * dk; e += NTB) {
        const int t = e / dk, c = e % dk;
        const bool in = t < Lc;
        Qc[t * lq + c] = in ? io<T>::load(q, qoff + (size_t)(t0 + t) * a.DHQK + c) : 0.f;
        Kc[t * lq + c] = in ? io<T>::load(k, qoff + (size_t)(t0 + t) * a.DHQK + c) : 0.f;
      }
#pragma unroll 4
      for (int e = tid; e < L * dv; e += NTB) {
        const int t = e / dv, r = e % dv;
        const bool in = t < Lc;
        Vc[t * lv + r] = in ? io<T>::load(v, voff + (size_t)(t0 + t) * a.DHV + r) : 0.f;
        dHc[t * lv + r] = in ? io<T>::load(dh, voff + (size_t)(t0 + t) * a.DHV + r) : 0.f;
        Oc[t * lv + r] = (in && with_o && og) ? io<T>::load(og, voff + (size_t)(t0 + t) * a.DHV + r) : 1.f;
      }
      if (warp == 0) {
        // inclusive prefix sum of log f' over the chunk (L <= 32: one warp)
        float x = lane < Lc ? wlf[t0 + lane] : 0.f;
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane < L) {
          lA[lane] = x;
          eA[lane] = expf(x);
          li[lane] = lane < Lc ? wli[t0 + lane] : -INFINITY;
          tmt[lane] = lane < Lc ? wm[t0 + lane] : 0.f;
        }
      }
      __syncthreads();
      for (int e = tid; e < L * L; e += NTB) {
        const int t = e / L, s2 = e % L;
        float w = 0.f, p = 0.f;
        if (s2 <= t && t < Lc) {
          w = expf(lA[t] - lA[s2] + li[s2]);
          float x = 0.f;
          for (int c = 0; c < dk; ++c) x += Qc[t * lq + c] * Kc[s2 * lq + c];
          p = w * x;
        }
        Wm[e] = w;
        Pm[e] = p;
      }
      __syncthreads();
    };
    // Xm = W o (dNum V^T)
    auto make_x = [&](int Lc) {
      for (int e = tid; e < L * L; e += NTB) {
        const int t = e / L, s2 = e % L;
        float x = 0.f;
        if (s2 <= t && t < Lc)
          for (int r = 0; r < dv; ++r) x += dN[t * lv + r] * Vc[s2 * lv + r];
        Xm[e] = Wm[e] * x;
      }
      __syncthreads();
    };

    // ---------------------------------------------------------------- phase 1 (forward)
    for (int e = tid; e < dv * dk; e += NTB) {
      const int r = e / dk, c = e % dk;
      St[r * ld + c] = a.C0 ? a.C0[slice * dv * dk + e] : 0.f;
    }
    for (int c = tid; c < dk; c += NTB) nv[c] = (!ret && a.n0) ? a.n0[slice * dk + c] : 0.f;
    __syncthreads();
    for (int ch = 0; ch < nck; ++ch) {
      const int t0 = ch * L, Lc = min(L, S - t0);
      load_chunk(t0, Lc, true);
      // d_t and den_t (a warp per token)
      for (int t = warp; t < L; t += NTB / 32) {
        float x = 0.f;
        if (!ret && t < Lc) {
          for (int c = lane; c < dk; c += 32) x += Qc[t * lq + c] * nv[c];
          x *= eA[t];
          for (int s2 = lane; s2 < L; s2 += 32) x += Pm[t * L + s2];
        }
        for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) {
          td[t] = x;
          tden[t] = ret ? 1.f : fmaxf(fabsf(x), expf(-tmt[t]));
        }
      }
      __syncthreads();
      // read-out, h / den, dnum, the output-gate gradient; products o dh h/den into Oc
      for (int e = tid; e < L * dv; e += NTB) {
        const int t = e / dv, r = e % dv;
        float num = 0.f;
        if (t < Lc) {
          for (int c = 0; c < dk; ++c) num += St[r * ld + c] * Qc[t * lq + c];
          num *= eA[t];
          for (int s2 = 0; s2 <= t; ++s2) num += Pm[t * L + s2] * Vc[s2 * lv + r];
        }
        const int ev = t * lv + r;
        const float den = tden[t], hn = num / den, o = Oc[ev];
        dN[ev] = t < Lc ? o * dHc[ev] / den : 0.f;
        if (a.dog && t < Lc) a.dog[voff + (size_t)(t0 + t) * a.DHV + r] = dHc[ev] * hn;
        Oc[ev] = o * dHc[ev] * hn;
      }
      __syncthreads();
      for (int t = warp; t < L; t += NTB / 32) {
        float x = 0.f;
        if (!ret && t < Lc)
          for (int r = lane; r < dv; r += 32) x += Oc[t * lv + r];
        for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) {
          tP[t] = x;
          const float d = td[t], den = tden[t];
          tdd[t] = (!ret && t < Lc && fabsf(d) > expf(-tmt[t])) ? -x / den * copysignf(1.f, d) : 0.f;
        }
      }
      __syncthreads();
      make_x(Lc);
      // dq
      for (int e = tid; e < L * dk; e += NTB) {
        const int t = e / dk, c = e % dk;
        if (t >= Lc) continue;
        float x = 0.f;
        for (int r = 0; r < dv; ++r) x += St[r * ld + c] * dN[t * lv + r];
        const float At = eA[t];
        x *= At;
        float wk = 0.f;
        for (int s2 = 0; s2 <= t; ++s2) {
          x += Xm[t * L + s2] * Kc[s2 * lq + c];
          wk += Wm[t * L + s2] * Kc[s2 * lq + c];
        }
        const float dd = tdd[t];
        a.dq[qoff + (size_t)(t0 + t) * a.DHQK + c] = x + (ret ? 0.f : dd * (At * nv[c] + wk));
      }
      for (int t = tid; t < Lc; t += NTB) {
        wden[t0 + t] = tden[t];
        wd[t0 + t] = td[t];
        wdd[t0 + t] = tdd[t];
        if (!ret) wr[t0 + t] += tP[t] + tdd[t] * td[t];
      }
      __syncthreads();
      // state to the chunk end
      {
        const float AL = eA[Lc - 1];
        const float* wend = Wm + (Lc - 1) * L;
        for (int e = tid; e < dv * dk; e += NTB) {
          const int r = e / dk, c = e % dk;
          float x = AL * St[r * ld + c];
          for (int s2 = 0; s2 < Lc; ++s2) x += wend[s2] * Vc[s2 * lv + r] * Kc[s2 * lq + c];
          St[r * ld + c] = x;
        }
        if (!ret)
          for (int c = tid; c < dk; c += NTB) {
            float x = AL * nv[c];
            for (int s2 = 0; s2 < Lc; ++s2) x += wend[s2] * Kc[s2 * lq + c];
            nv[c] = x;
          }
      }
      __syncthreads();
    }
    // final-state term of the forget gradient
    if (!ret && (a.dC || a.dn)) {
      float part = 0.f;
      if (a.dC)
        for (int e = tid; e < dv * dk; e += NTB) part += a.dC[slice * dv * dk + e] * St[(e / dk) * ld + e % dk];
      if (a.dn)
        for (int c = tid; c < dk; c += NTB) part += a.dn[slice * dk + c] * nv[c];
      const float s2 = block_sum(part, red);
      if (tid == 0) sc[2] += s2;
    }
    __syncthreads();
    // ---------------------------------------------------------------- phase 2 (backward)
    for (int e = tid; e < dv * dk; e += NTB) {
      const int r = e / dk, c = e % dk;
      St[r * ld + c] = a.dC ? a.dC[slice * dv * dk + e] : 0.f;
    }
    for (int c = tid; c < dk; c += NTB) nv[c] = (!ret && a.dn) ? a.dn[slice * dk + c] : 0.f;
    __syncthreads();
    for (int ch = nck - 1; ch >= 0; --ch) {
      const int t0 = ch * L, Lc = min(L, S - t0);
      load_chunk(t0, Lc, true);
      for (int t = tid; t < L; t += NTB) {
        tden[t] = t < Lc ? wden[t0 + t] : 1.f;
        tdd[t] = t < Lc ? wdd[t0 + t] : 0.f;
      }
      __syncthreads();
      for (int e = tid; e < L * dv; e += NTB) {
        const int t = e / dv, ev = t * lv + e % dv;
        dN[ev] = t < Lc ? Oc[ev] * dHc[ev] / tden[t] : 0.f;
      }
      __syncthreads();
      make_x(Lc);
      const float* wend = Wm + (Lc - 1) * L;
      for (int t = tid; t < L; t += NTB) td[t] = 0.f;  // ditilde_t = v . dv + k . dk_n
      __syncthreads();
      // dv
      for (int e = tid; e < L * dv; e += NTB) {
        const int t = e / dv, r = e % dv;
        float x = 0.f;
        if (t < Lc) {
          for (int tau = t; tau < Lc; ++tau) x += Pm[tau * L + t] * dN[tau * lv + r];
          float y = 0.f;
          for (int c = 0; c < dk; ++c) y += St[r * ld + c] * Kc[t * lq + c];
          x += wend[t] * y;
          a.dv_out[voff + (size_t)(t0 + t) * a.DHV + r] = x;
          if (!ret) atomicAdd(&td[t], Vc[t * lv + r] * x);
        }
      }
      // dk (C part and n part)
      for (int e = tid; e < L * dk; e += NTB) {
        const int t = e / dk, c = e % dk;
        if (t >= Lc) continue;
        float x = 0.f, xn = 0.f;
        for (int tau = t; tau < Lc; ++tau) {
          x += Xm[tau * L + t] * Qc[tau * lq + c];
          xn += Wm[tau * L + t] * tdd[tau] * Qc[tau * lq + c];
        }
        float y = 0.f;
        for (int r = 0; r < dv; ++r) y += Vc[t * lv + r] * St[r * ld + c];
        x += wend[t] * y;
        xn = ret ? 0.f : xn + wend[t] * nv[c];
        a.dk_out[qoff + (size_t)(t0 + t) * a.DHQK + c] = x + xn;
        if (!ret) atomicAdd(&td[t], xn * Kc[t * lq + c]);
      }
      __syncthreads();
      if (!ret)
        for (int t = tid; t < Lc; t += NTB) {
          wdi[t0 + t] += td[t];
          wr[t0 + t] -= td[t];
        }
      {
        const float AL = eA[Lc - 1];
        for (int e = tid; e < dv * dk; e += NTB) {
          const int r = e / dk, c = e % dk;
          float x = AL * St[r * ld + c];
          for (int tau = 0; tau < Lc; ++tau) x += eA[tau] * dN[tau * lv + r] * Qc[tau * lq + c];
          St[r * ld + c] = x;
        }
        if (!ret)
          for (int c = tid; c < dk; c += NTB) {
            float x = AL * nv[c];
            for (int tau = 0; tau < Lc; ++tau) x += eA[tau] * tdd[tau] * Qc[tau * lq + c];
            nv[c] = x;
          }
      }
      __syncthreads();
    }
    // initial-state gradients
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
      const float s2 = block_sum(part, red);
      if (tid == 0) sc[3] += s2;
    }
    __syncthreads();
  }
  // ---- gate gradients: dlf_t = sum_{tau >= t} r_tau + final-state term (warp 0: scan of
  // the lanes' segment sums from the end)
  if (!ret && warp == 0) {
    const int seg = (S + 31) / 32, t_lo = lane * seg, t_hi = min(S, t_lo + seg);
    float sum = 0.f;
    for (int t = t_lo; t < t_hi; ++t) sum += wr[t];
    // sum of the later lanes' segments
    float later = sum;
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_down_sync(0xffffffffu, later, o);
      if (lane + o < 32) later += y;
    }
    float acc = later - sum + sc[2];
    for (int t = t_hi - 1; t >= t_lo; --t) {
      acc += wr[t];
      const float ft = a.fg[(size_t)bh * S + t];
      if (a.dfg) a.dfg[(size_t)bh * S + t] = acc / (1.f + expf(ft));
      if (a.dig) a.dig[(size_t)bh * S + t] = wdi[t];
    }
    if (lane == 0 && a.dm0) a.dm0[bh] = sc[3];
  }
}

}  // namespace

// =======================================================================================
// Cluster form of the chunked backward, for blocks whose state does not fit one CTA (the
// 256 x 512 head): a thread-block cluster per (batch, head), CTA `rank` owning value rows
// [64 rank, 64 rank + 64) of each block's state (C' in phase 1, D in phase 2) in registers
// as warp-MMA accumulators, bf16 inputs.  The chunk algebra is the one of bwd_chunk_kernel
// (32-token chunks); every product over the chunk is an m16n8k16 bf16 MMA with fp32
// accumulation (operands from shared memory by ldmatrix), and the sums over value rows that
// span the cluster meet in distributed shared memory:
//   phase 1: P_t = sum_r o dh num / den (every CTA reads every CTA's partial, so each has
//            dd_t), dq (each CTA adds the partials of its 1/NC of the key columns, plus the
//            dd term);
//   phase 2: dk (the same column split, plus the dd and G terms), ditilde_t by atomics on the
//            per-head workspace.
// n' / G (one key vector per block) is kept by every CTA.  Two cluster barriers per chunk:
// after the partials are written, and before they are overwritten.
namespace {

namespace cg = cooperative_groups;
using namespace sm100;
typedef __nv_bfloat16 bf16_t;

constexpr int BCL = 32;          // chunk length
constexpr int BCV = 64;          // value rows per CTA
constexpr int BCT = 256;         // threads per CTA
constexpr int LDV = BCV + 8;     // bf16 row stride of [BCL][BCV] tiles (16-byte rows, odd 16-byte count)
constexpr int LDL = BCL + 8;     // bf16 row stride of [BCL][BCL] tiles
constexpr int LDF = BCV + 1;     // fp32 row stride of [BCL][BCV] tiles
constexpr int LDW = BCL + 1;     // fp32 row stride of [BCL][BCL] tiles

template <int DK>
struct BcSmem {
  static constexpr int LDK = DK + 8;  // bf16 row stride of [.][DK] tiles
  static constexpr int Q = 0;                        // bf16 [BCL][LDK]
  static constexpr int K = Q + BCL * LDK * 2;        // bf16 [BCL][LDK]
  static constexpr int CB = K + BCL * LDK * 2;       // bf16 [BCV][LDK]: copy of the state (C' or D)
  static constexpr int VB = CB + BCV * LDK * 2;      // bf16 [BCL][LDV]
  static constexpr int AB = VB + BCL * LDV * 2;      // bf16 [BCL][LDV]: V o w (phase 1), dN o A (phase 2)
  static constexpr int DNB = AB + BCL * LDV * 2;     // bf16 [BCL][LDV]: dN
  static constexpr int PB = DNB + BCL * LDV * 2;     // bf16 [BCL][LDL]: P
  static constexpr int XB = PB + BCL * LDL * 2;      // bf16 [BCL][LDL]: X = W o (dN V^T), this CTA's rows
  static constexpr int DH = XB + BCL * LDL * 2;      // f32 [BCL][LDF]
  static constexpr int O = DH + BCL * LDF * 4;       // f32 [BCL][LDF]
  static constexpr int W = O + BCL * LDF * 4;        // f32 [BCL][LDW]
  static constexpr int P = W + BCL * LDW * 4;        // f32 [BCL][LDW]
  static constexpr int R = P + BCL * LDW * 4;        // f32 [BCL][DK]: this CTA's partial dq / dk
  static constexpr int NV = R + BCL * DK * 4;        // f32 [DK]: n' (phase 1) / G (phase 2)
  static constexpr int TOK = NV + DK * 4;            // f32 [12][BCL] per-token values
  static constexpr int BYTES = TOK + 12 * BCL * 4;
};

// acc[NT] (16 x 8 tiles at rows m0.., columns n0 + 8 nt) += A[m0 : m0 + 16, 0 : K] B[0 : K, n0 : ..].
// A bf16 in shared memory stored [m][k] (ATR false) or [k][m] (ATR true), row stride lda;
// B stored [n][k] (BTR false) or [k][n] (BTR true), row stride ldb.  One warp.
template <bool ATR, bool BTR, int NT>
__device__ __forceinline__ void warp_mma(float (&acc)[NT][4], const bf16_t* A, int lda, const bf16_t* B, int ldb,
                                         int m0, int n0, int K) {
  const int lane = threadIdx.x & 31;
  for (int k0 = 0; k0 < K; k0 += 16) {
    uint32_t a0, a1, a2, a3;
    if (!ATR)
      ldmatrix_x4(smem_u32(A + (m0 + (lane & 15)) * lda + k0 + ((lane >> 4) << 3)), a0, a1, a2, a3);
    else
      ldmatrix_x4_trans(smem_u32(A + (k0 + (lane & 7) + ((lane >> 4) << 3)) * lda + m0 + (((lane >> 3) & 1) << 3)), a0,
                        a1, a2, a3);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      uint32_t b0, b1;
      if (!BTR)
        ldmatrix_x2(smem_u32(B + (n0 + 8 * nt + (lane & 7)) * ldb + k0 + (((lane >> 3) & 1) << 3)), b0, b1);
      else
        ldmatrix_x2_trans(smem_u32(B + (k0 + (lane & 15)) * ldb + n0 + 8 * nt), b0, b1);
      mma_m16n8k16_bf16(acc[nt], a0, a1, a2, a3, b0, b1);
    }
  }
}

// sum over the cluster's CTAs (nc <= 8) of four floats at the same shared-memory offset; the
// remote loads are all issued before the first add
__device__ __forceinline__ float4 sum_remote4(cg::cluster_group& cl, float* local, int nc) {
  float4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    v[i] = i < nc ? *reinterpret_cast<const float4*>(cl.map_shared_rank(local, i)) : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 s = v[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    s.x += v[i].x;
    s.y += v[i].y;
    s.z += v[i].z;
    s.w += v[i].w;
  }
  return s;
}

template <int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NT][4]) {
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
}

__device__ __forceinline__ uint32_t bf2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float cl_block_sum(float x, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();
  if (lane == 0) red[warp] = x;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < BCT / 32; ++w) s += red[w];
  __syncthreads();
  return s;
}

template <int DK>
__global__ void __launch_bounds__(BCT, 1) bwd_cluster_kernel(BwdArgs a) {
  using SM = BcSmem<DK>;
  constexpr int LDK = SM::LDK;
  constexpr int NS = DK / 16;   // n8 tiles of a warp's share of the state (16 rows x DK/2 columns)
  constexpr int NQ = DK / 32;   // n8 tiles of a warp's share of a [BCL][DK] product
  extern __shared__ __align__(16) uint8_t smb[];
  bf16_t* Qb = reinterpret_cast<bf16_t*>(smb + SM::Q);
  bf16_t* Kb = reinterpret_cast<bf16_t*>(smb + SM::K);
  bf16_t* Cb = reinterpret_cast<bf16_t*>(smb + SM::CB);
  bf16_t* Vb = reinterpret_cast<bf16_t*>(smb + SM::VB);
  bf16_t* Ab = reinterpret_cast<bf16_t*>(smb + SM::AB);
  bf16_t* dNb = reinterpret_cast<bf16_t*>(smb + SM::DNB);
  bf16_t* Pb = reinterpret_cast<bf16_t*>(smb + SM::PB);
  bf16_t* Xb = reinterpret_cast<bf16_t*>(smb + SM::XB);
  float* dHf = reinterpret_cast<float*>(smb + SM::DH);
  float* Of = reinterpret_cast<float*>(smb + SM::O);
  float* Wm = reinterpret_cast<float*>(smb + SM::W);
  float* Pm = reinterpret_cast<float*>(smb + SM::P);
  float* Rp = reinterpret_cast<float*>(smb + SM::R);
  float* nv = reinterpret_cast<float*>(smb + SM::NV);
  float* tok = reinterpret_cast<float*>(smb + SM::TOK);
  float* lA = tok;              // log A_t (cumulative log f' inside the chunk)
  float* eA = tok + BCL;        // A_t
  float* li = tok + 2 * BCL;    // log i'_t (-inf past the end)
  float* tmt = tok + 3 * BCL;   // m_t
  float* td = tok + 4 * BCL;    // d_t = n'_t . q_t
  float* tden = tok + 5 * BCL;  // den_t
  float* tdd = tok + 6 * BCL;   // dd_t
  float* tpp = tok + 7 * BCL;   // this CTA's partial of P_t; ditilde partials in phase 2
  float* wv = tok + 8 * BCL;    // w_s = W[Lc-1][s]
  float* tdn = tok + 9 * BCL;   // ditilde partial of the n part (phase 2)
  float* red = tok + 10 * BCL;  // [8] block sums
  float* scal = red + 8;        // [0] final-state term, [1] dm0 (partials of this CTA)

  cg::cluster_group cl = cg::this_cluster();
  const int NC = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  // one cluster per (batch x head, block): the blocks of a head run side by side
  const int bh = blockIdx.y, blk = blockIdx.z, head = bh % a.NH;
  const int dv = a.dv, S = a.S, r0 = rank * BCV;
  const bool ret = a.retention != 0;
  const bf16_t* q = static_cast<const bf16_t*>(a.q);
  const bf16_t* k = static_cast<const bf16_t*>(a.k);
  const bf16_t* v = static_cast<const bf16_t*>(a.v);
  const bf16_t* dh = static_cast<const bf16_t*>(a.dh);
  const bf16_t* og = ret ? nullptr : static_cast<const bf16_t*>(a.og);
  // workspace (bwd_workspace_bytes): per (batch x head, block) the gate logs and the per-token
  // values of phase 1; per batch x head the forget / input gate gradient sums (zeroed before the
  // launch, added to by every block); per (batch x head, block) the block's final-state terms
  const size_t nbh = (size_t)a.B * a.NH;
  float* wlf = a.ws + ((size_t)bh * a.nb + blk) * 6 * S;
  float* wli = wlf + S;
  float* wm = wli + S;
  float* wden = wm + S;
  float* wd = wden + S;
  float* wdd = wd + S;
  float* wr = a.ws + nbh * a.nb * 6 * S + (size_t)bh * 2 * S;
  float* wdi = wr + S;
  float* wsc = a.ws + nbh * a.nb * 6 * S + nbh * 2 * S + ((size_t)bh * a.nb + blk) * 2;
  // this warp's share of the state: rows 16 rt .. +16, key columns hc DK/2 .. +DK/2
  const int rt = warp & 3, hc = warp >> 2;
  float st[NS][4];

  // ---- gates (rank 0, warp 0: the stabiliser recurrence as a max-plus scan), workspace sums zeroed
  if (rank == 0) {
    if (warp == 0) {
      if (ret) {
        const float lg = retention_log_gamma(head);
        for (int t = lane; t < S; t += 32) {
          wlf[t] = lg;
          wli[t] = 0.f;
          wm[t] = 0.f;
        }
      } else {
        const int seg = (S + 31) / 32, t_lo = lane * seg, t_hi = min(S, t_lo + seg);
        MaxPlus mp{0.f, -INFINITY};
        for (int t = t_lo; t < t_hi; ++t)
          mp = mp_then(mp, MaxPlus{log_sigmoid(a.fg[(size_t)bh * S + t]), a.ig[(size_t)bh * S + t]});
        for (int o = 1; o < 32; o <<= 1) {
          const float A = __shfl_up_sync(0xffffffffu, mp.A, o), Bm = __shfl_up_sync(0xffffffffu, mp.Bm, o);
          if (lane >= o) mp = mp_then(MaxPlus{A, Bm}, mp);
        }
        float ex_A = __shfl_up_sync(0xffffffffu, mp.A, 1), ex_B = __shfl_up_sync(0xffffffffu, mp.Bm, 1);
        if (lane == 0) {
          ex_A = 0.f;
          ex_B = -INFINITY;
        }
        float m = mp_apply(MaxPlus{ex_A, ex_B}, a.m0 ? a.m0[bh] : 0.f);
        for (int t = t_lo; t < t_hi; ++t) {
          const float lf = log_sigmoid(a.fg[(size_t)bh * S + t]), it = a.ig[(size_t)bh * S + t];
          const float mn = fmaxf(lf + m, it);
          wlf[t] = lf + m - mn;
          wli[t] = it - mn;
          wm[t] = mn;
          m = mn;
        }
      }
    }
  }
  if (tid == 0) {
    scal[0] = 0.f;
    scal[1] = 0.f;
  }
  cl.sync();

  const int nck = (S + BCL - 1) / BCL;
  {
    const size_t slice = (size_t)bh * a.nb + blk;
    // (blocks narrower than DK key columns or BCV value rows run zero-padded: every global
    // access below is masked to the block's dk x dv)
    const int dkr = a.dk;
    const size_t qoff = (size_t)bh * S * a.DHQK + (size_t)blk * dkr;
    const size_t voff = (size_t)bh * S * a.DHV + (size_t)blk * dv + r0;
    const size_t soff = slice * (size_t)dv * dkr + (size_t)r0 * dkr;  // this CTA's rows of a state

    // chunk inputs, gate logs, W and P (every CTA: the key-side products are redundant)
    auto load_chunk = [&](int t0, int Lc) {
      // every load of this thread is issued before the first store, so they are in flight together
      constexpr int NQL = BCL * (DK / 8) / BCT;  // 16-byte pieces of Q (and of K) per thread
      static_assert(NQL * BCT == BCL * (DK / 8) && BCL * (BCV / 8) == BCT, "chunk tiles map onto the threads");
      uint4 uq[NQL], uk[NQL];
#pragma unroll
      for (int i = 0; i < NQL; ++i) {
        const int e = tid + i * BCT, t = e / (DK / 8), c = (e % (DK / 8)) * 8;
        uq[i] = uk[i] = make_uint4(0, 0, 0, 0);
        if (t < Lc && c < dkr) {
          uq[i] = *reinterpret_cast<const uint4*>(q + qoff + (size_t)(t0 + t) * a.DHQK + c);
          uk[i] = *reinterpret_cast<const uint4*>(k + qoff + (size_t)(t0 + t) * a.DHQK + c);
        }
      }
      {
        const int t = tid / (BCV / 8), c = (tid % (BCV / 8)) * 8;
        uint4 uv = make_uint4(0, 0, 0, 0), uh = uv, uo = uv;
        if (t < Lc && r0 + c < dv) {
          const size_t off = voff + (size_t)(t0 + t) * a.DHV + c;
          uv = *reinterpret_cast<const uint4*>(v + off);
          uh = *reinterpret_cast<const uint4*>(dh + off);
          if (og) uo = *reinterpret_cast<const uint4*>(og + off);
        }
#pragma unroll
        for (int i = 0; i < NQL; ++i) {
          const int e = tid + i * BCT, tt = e / (DK / 8), cc = (e % (DK / 8)) * 8;
          *reinterpret_cast<uint4*>(Qb + tt * LDK + cc) = uq[i];
          *reinterpret_cast<uint4*>(Kb + tt * LDK + cc) = uk[i];
        }
        *reinterpret_cast<uint4*>(Vb + t * LDV + c) = uv;
        const bf16_t* hb = reinterpret_cast<const bf16_t*>(&uh);
        const bf16_t* ob = reinterpret_cast<const bf16_t*>(&uo);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          dHf[t * LDF + c + j] = __bfloat162float(hb[j]);
          Of[t * LDF + c + j] = og ? __bfloat162float(ob[j]) : 1.f;
        }
      }
      if (warp == 0) {
        float x = lane < Lc ? wlf[t0 + lane] : 0.f;
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        lA[lane] = x;
        eA[lane] = expf(x);
        li[lane] = lane < Lc ? wli[t0 + lane] : -INFINITY;
        tmt[lane] = lane < Lc ? wm[t0 + lane] : 0.f;
      }
      __syncthreads();
      {  // S = Q K^T: warp -> rows 16 (w >> 2), columns 8 (w & 3)
        float acc[1][4];
        zero_acc(acc);
        const int m0 = 16 * (warp >> 2), n0 = 8 * (warp & 3);
        warp_mma<false, false, 1>(acc, Qb, LDK, Kb, LDK, m0, n0, DK);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int t = m0 + g + 8 * h2, s0 = n0 + 2 * tq;
          float wv2[2], pv2[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int s2 = s0 + j;
            const float w = (s2 <= t && t < Lc) ? expf(lA[t] - lA[s2] + li[s2]) : 0.f;
            wv2[j] = w;
            pv2[j] = w * acc[0][2 * h2 + j];
            Wm[t * LDW + s2] = w;
            Pm[t * LDW + s2] = pv2[j];
          }
          *reinterpret_cast<uint32_t*>(Pb + t * LDL + s0) = bf2(pv2[0], pv2[1]);
        }
      }
      __syncthreads();
      if (tid < BCL) wv[tid] = Wm[(Lc - 1) * LDW + tid];
    };
    // X = W o (dN V^T) over this CTA's value rows, into Xb: warp -> rows 16 (w >> 2), cols 8 (w & 3)
    auto make_x = [&]() {
      float acc[1][4];
      zero_acc(acc);
      const int m0 = 16 * (warp >> 2), n0 = 8 * (warp & 3);
      warp_mma<false, false, 1>(acc, dNb, LDV, Vb, LDV, m0, n0, BCV);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int t = m0 + g + 8 * h2, s0 = n0 + 2 * tq;
        *reinterpret_cast<uint32_t*>(Xb + t * LDL + s0) =
            bf2(Wm[t * LDW + s0] * acc[0][2 * h2], Wm[t * LDW + s0 + 1] * acc[0][2 * h2 + 1]);
      }
    };
    // the bf16 copy of this CTA's state rows (the warps' accumulators) for the products
    auto state_to_cb = [&]() {
#pragma unroll
      for (int nt = 0; nt < NS; ++nt) {
        const int c = hc * (DK / 2) + 8 * nt + 2 * tq, r = 16 * rt + g;
        *reinterpret_cast<uint32_t*>(Cb + r * LDK + c) = bf2(st[nt][0], st[nt][1]);
        *reinterpret_cast<uint32_t*>(Cb + (r + 8) * LDK + c) = bf2(st[nt][2], st[nt][3]);
      }
    };
    // a state (C0 or dC, [dv][DK] per slice) into the accumulators; NULL = zeros
    auto load_state = [&](const float* src) {
#pragma unroll
      for (int nt = 0; nt < NS; ++nt) {
        const int c = hc * (DK / 2) + 8 * nt + 2 * tq, r = 16 * rt + g;
        float2 x = make_float2(0.f, 0.f), y = x;
        if (src && c < dkr) {
          if (r0 + r < dv) x = *reinterpret_cast<const float2*>(src + soff + (size_t)r * dkr + c);
          if (r0 + r + 8 < dv) y = *reinterpret_cast<const float2*>(src + soff + (size_t)(r + 8) * dkr + c);
        }
        st[nt][0] = x.x;
        st[nt][1] = x.y;
        st[nt][2] = y.x;
        st[nt][3] = y.y;
      }
    };
    // <state, src> over this CTA's rows (src [dv][DK] per slice)
    auto state_dot = [&](const float* src) {
      float part = 0.f;
#pragma unroll
      for (int nt = 0; nt < NS; ++nt) {
        const int c = hc * (DK / 2) + 8 * nt + 2 * tq, r = 16 * rt + g;
        if (c >= dkr) continue;
        const float2 x = r0 + r < dv ? *reinterpret_cast<const float2*>(src + soff + (size_t)r * dkr + c)
                                     : make_float2(0.f, 0.f);
        const float2 y = r0 + r + 8 < dv ? *reinterpret_cast<const float2*>(src + soff + (size_t)(r + 8) * dkr + c)
                                         : make_float2(0.f, 0.f);
        part += st[nt][0] * x.x + st[nt][1] * x.y + st[nt][2] * y.x + st[nt][3] * y.y;
      }
      return part;
    };
    // key columns this CTA reduces, in groups of four (the last rank may have fewer)
    const int CW4 = (DK / 4 + NC - 1) / NC;

    // ------------------------------------------------------------------ phase 1 (forward)
    load_state(a.C0);
    for (int c = tid; c < DK; c += BCT) nv[c] = (!ret && a.n0 && c < dkr) ? a.n0[slice * dkr + c] : 0.f;
    for (int ch = 0; ch < nck; ++ch) {
      const int t0 = ch * BCL, Lc = min(BCL, S - t0);
      state_to_cb();
      if (tid < BCL) tpp[tid] = 0.f;
      load_chunk(t0, Lc);  // ends with a barrier after W, P
      // d_t and den_t (every CTA; a warp per token)
      for (int t = warp; t < BCL; t += BCT / 32) {
        float x = 0.f;
        if (!ret && t < Lc)
          for (int c = lane; c < DK; c += 32) x += __bfloat162float(Qb[t * LDK + c]) * nv[c];
        x *= eA[t];
        if (!ret && t < Lc) x += Pm[t * LDW + lane];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) {
          td[t] = ret ? 0.f : x;
          tden[t] = ret ? 1.f : fmaxf(fabsf(x), expf(-tmt[t]));
        }
      }
      __syncthreads();
      {  // num = diag(A) Q C'^T + P V (this CTA's rows): warp -> tokens 16 (w & 1), rows 16 (w >> 1)
        float acc[2][4];
        zero_acc(acc);
        const int m0 = 16 * (warp & 1), n0 = 16 * (warp >> 1);
        warp_mma<false, false, 2>(acc, Qb, LDK, Cb, LDK, m0, n0, DK);
        const float e_lo = eA[m0 + g], e_hi = eA[m0 + g + 8];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          acc[nt][0] *= e_lo;
          acc[nt][1] *= e_lo;
          acc[nt][2] *= e_hi;
          acc[nt][3] *= e_hi;
        }
        warp_mma<false, true, 2>(acc, Pb, LDL, Vb, LDV, m0, n0, BCL);
        float pp[2] = {0.f, 0.f};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int t = m0 + g + 8 * h2;
          const float den = tden[t];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int r = n0 + 8 * nt + 2 * tq;
            float dn2[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float hn = acc[nt][2 * h2 + j] / den;
              const float o = Of[t * LDF + r + j], dhv = dHf[t * LDF + r + j];
              dn2[j] = t < Lc ? o * dhv / den : 0.f;
              pp[h2] += o * dhv * hn;
              if (a.dog && t < Lc && r0 + r + j < dv) a.dog[voff + (size_t)(t0 + t) * a.DHV + r + j] = dhv * hn;
            }
            *reinterpret_cast<uint32_t*>(dNb + t * LDV + r) = bf2(dn2[0], dn2[1]);
          }
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          pp[h2] += __shfl_xor_sync(0xffffffffu, pp[h2], 1);
          pp[h2] += __shfl_xor_sync(0xffffffffu, pp[h2], 2);
          if (tq == 0 && !ret) atomicAdd(&tpp[m0 + g + 8 * h2], pp[h2]);
        }
      }
      cl.sync();  // every CTA's P partials (and this CTA's dN) are written
      if (tid < BCL) {
        const int t = tid;
        float part[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) part[i] = i < NC ? cl.map_shared_rank(tpp, i)[t] : 0.f;
        float P = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) P += part[i];
        const float d = td[t], den = tden[t];
        const float dd = (!ret && t < Lc && fabsf(d) > expf(-tmt[t])) ? -P / den * copysignf(1.f, d) : 0.f;
        tdd[t] = dd;
        if (rank == 0 && t < Lc) {
          wden[t0 + t] = den;
          wd[t0 + t] = d;
          wdd[t0 + t] = dd;
          if (!ret) atomicAdd(&wr[t0 + t], P + dd * d);
        }
      }
      make_x();
      // V o w for the state update
      for (int e = tid; e < BCL * BCV / 2; e += BCT) {
        const int s2 = e / (BCV / 2), r = 2 * (e % (BCV / 2));
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Vb + s2 * LDV + r));
        *reinterpret_cast<uint32_t*>(Ab + s2 * LDV + r) = bf2(x.x * wv[s2], x.y * wv[s2]);
      }
      __syncthreads();
      {  // partial dq = diag(A) dN C' + X K: warp -> tokens 16 (w & 1), key columns (w >> 1) DK/4
        float acc[NQ][4];
        zero_acc(acc);
        const int m0 = 16 * (warp & 1), n0 = (warp >> 1) * (DK / 4);
        warp_mma<false, true, NQ>(acc, dNb, LDV, Cb, LDK, m0, n0, BCV);
        const float e_lo = eA[m0 + g], e_hi = eA[m0 + g + 8];
#pragma unroll
        for (int nt = 0; nt < NQ; ++nt) {
          acc[nt][0] *= e_lo;
          acc[nt][1] *= e_lo;
          acc[nt][2] *= e_hi;
          acc[nt][3] *= e_hi;
        }
        warp_mma<false, true, NQ>(acc, Xb, LDL, Kb, LDK, m0, n0, BCL);
#pragma unroll
        for (int nt = 0; nt < NQ; ++nt) {
          const int c = n0 + 8 * nt + 2 * tq;
          *reinterpret_cast<float2*>(Rp + (m0 + g) * DK + c) = make_float2(acc[nt][0], acc[nt][1]);
          *reinterpret_cast<float2*>(Rp + (m0 + g + 8) * DK + c) = make_float2(acc[nt][2], acc[nt][3]);
        }
      }
      cl.sync();  // every CTA's partial dq is written
      for (int e = tid; e < BCL * CW4; e += BCT) {
        const int t = e / CW4, c = rank * CW4 * 4 + (e % CW4) * 4;
        if (t >= Lc || c >= DK) continue;
        const float4 x = sum_remote4(cl, Rp + t * DK + c, NC);
        float4 y = x;
        const float dd = tdd[t];
        if (!ret && dd != 0.f) {
          float4 wk = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int s2 = 0; s2 <= t; ++s2) {
            const float w = Wm[t * LDW + s2];
            const uint2 kk = *reinterpret_cast<const uint2*>(Kb + s2 * LDK + c);
            const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kk.x));
            const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kk.y));
            wk.x += w * k01.x;
            wk.y += w * k01.y;
            wk.z += w * k23.x;
            wk.w += w * k23.y;
          }
          const float At = eA[t];
          y.x += dd * (At * nv[c] + wk.x);
          y.y += dd * (At * nv[c + 1] + wk.y);
          y.z += dd * (At * nv[c + 2] + wk.z);
          y.w += dd * (At * nv[c + 3] + wk.w);
        }
        if (c < dkr) *reinterpret_cast<float4*>(a.dq + qoff + (size_t)(t0 + t) * a.DHQK + c) = y;
      }
      {  // state to the chunk end: C' <- A_L C' + (V o w)^T K
        const float AL = eA[Lc - 1];
#pragma unroll
        for (int nt = 0; nt < NS; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) st[nt][j] *= AL;
        warp_mma<true, true, NS>(st, Ab, LDV, Kb, LDK, 16 * rt, hc * (DK / 2), BCL);
      }
      __syncthreads();  // n' is read above (dd term)
      if (!ret) {
        const float AL = eA[Lc - 1];
        for (int c = tid; c < DK; c += BCT) {
          float x = AL * nv[c];
          for (int s2 = 0; s2 < Lc; ++s2) x += wv[s2] * __bfloat162float(Kb[s2 * LDK + c]);
          nv[c] = x;
        }
      }
      __syncthreads();
    }
    // final-state term <dC_S, C'_S> + dn_S . n'_S of the forget gradient
    if (!ret && (a.dC || a.dn)) {
      float part = a.dC ? state_dot(a.dC) : 0.f;
      if (a.dn && rank == 0)
        for (int c = tid; c < dkr; c += BCT) part += a.dn[slice * dkr + c] * nv[c];
      const float s2 = cl_block_sum(part, red);
      if (tid == 0) scal[0] += s2;
    }
    cl.sync();  // the per-token workspace of phase 1 is complete

    // ------------------------------------------------------------------ phase 2 (backward)
    load_state(a.dC);
    for (int c = tid; c < DK; c += BCT) nv[c] = (!ret && a.dn && c < dkr) ? a.dn[slice * dkr + c] : 0.f;
    for (int ch = nck - 1; ch >= 0; --ch) {
      const int t0 = ch * BCL, Lc = min(BCL, S - t0);
      state_to_cb();  // D entering from the later chunks
      if (tid < BCL) {
        tpp[tid] = 0.f;
        tdn[tid] = 0.f;
      }
      load_chunk(t0, Lc);
      if (tid < BCL) {
        tden[tid] = tid < Lc ? wden[t0 + tid] : 1.f;
        tdd[tid] = tid < Lc ? wdd[t0 + tid] : 0.f;
      }
      __syncthreads();
      for (int e = tid; e < BCL * BCV / 2; e += BCT) {
        const int t = e / (BCV / 2), r = 2 * (e % (BCV / 2));
        float d0 = 0.f, d1 = 0.f;
        if (t < Lc) {
          d0 = Of[t * LDF + r] * dHf[t * LDF + r] / tden[t];
          d1 = Of[t * LDF + r + 1] * dHf[t * LDF + r + 1] / tden[t];
        }
        *reinterpret_cast<uint32_t*>(dNb + t * LDV + r) = bf2(d0, d1);
        *reinterpret_cast<uint32_t*>(Ab + t * LDV + r) = bf2(d0 * eA[t], d1 * eA[t]);
      }
      __syncthreads();
      make_x();
      __syncthreads();
      {  // dv = P^T dN + diag(w) K D^T (this CTA's rows): warp -> tokens 16 (w & 1), rows 16 (w >> 1)
        float acc[2][4], acc2[2][4];
        zero_acc(acc);
        zero_acc(acc2);
        const int m0 = 16 * (warp & 1), n0 = 16 * (warp >> 1);
        warp_mma<false, false, 2>(acc2, Kb, LDK, Cb, LDK, m0, n0, DK);
        warp_mma<true, true, 2>(acc, Pb, LDL, dNb, LDV, m0, n0, BCL);
        float dip[2] = {0.f, 0.f};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int s2 = m0 + g + 8 * h2;
          const float w = wv[s2];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int r = n0 + 8 * nt + 2 * tq;
            const float x0 = acc[nt][2 * h2] + w * acc2[nt][2 * h2];
            const float x1 = acc[nt][2 * h2 + 1] + w * acc2[nt][2 * h2 + 1];
            if (s2 < Lc) {
              if (r0 + r < dv)
                *reinterpret_cast<float2*>(a.dv_out + voff + (size_t)(t0 + s2) * a.DHV + r) = make_float2(x0, x1);
              const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Vb + s2 * LDV + r));
              dip[h2] += vv.x * x0 + vv.y * x1;
            }
          }
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          dip[h2] += __shfl_xor_sync(0xffffffffu, dip[h2], 1);
          dip[h2] += __shfl_xor_sync(0xffffffffu, dip[h2], 2);
          if (tq == 0 && !ret) atomicAdd(&tpp[m0 + g + 8 * h2], dip[h2]);
        }
      }
      {  // partial dk = diag(w) V D + X^T Q: warp -> tokens 16 (w & 1), key columns (w >> 1) DK/4
        float acc[NQ][4];
        zero_acc(acc);
        const int m0 = 16 * (warp & 1), n0 = (warp >> 1) * (DK / 4);
        warp_mma<false, true, NQ>(acc, Vb, LDV, Cb, LDK, m0, n0, BCV);
        const float w_lo = wv[m0 + g], w_hi = wv[m0 + g + 8];
#pragma unroll
        for (int nt = 0; nt < NQ; ++nt) {
          acc[nt][0] *= w_lo;
          acc[nt][1] *= w_lo;
          acc[nt][2] *= w_hi;
          acc[nt][3] *= w_hi;
        }
        warp_mma<true, true, NQ>(acc, Xb, LDL, Qb, LDK, m0, n0, BCL);
#pragma unroll
        for (int nt = 0; nt < NQ; ++nt) {
          const int c = n0 + 8 * nt + 2 * tq;
          *reinterpret_cast<float2*>(Rp + (m0 + g) * DK + c) = make_float2(acc[nt][0], acc[nt][1]);
          *reinterpret_cast<float2*>(Rp + (m0 + g + 8) * DK + c) = make_float2(acc[nt][2], acc[nt][3]);
        }
      }
      cl.sync();  // every CTA's partial dk is written
      for (int e = tid; e < BCL * CW4; e += BCT) {
        const int s2 = e / CW4, c = rank * CW4 * 4 + (e % CW4) * 4;
        if (s2 >= Lc || c >= DK) continue;
        float4 x = sum_remote4(cl, Rp + s2 * DK + c, NC);
        if (!ret) {
          const float w = wv[s2];
          float4 xn = make_float4(w * nv[c], w * nv[c + 1], w * nv[c + 2], w * nv[c + 3]);
          for (int tau = s2; tau < Lc; ++tau) {
            const float f = Wm[tau * LDW + s2] * tdd[tau];
            const uint2 qq = *reinterpret_cast<const uint2*>(Qb + tau * LDK + c);
            const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qq.x));
            const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qq.y));
            xn.x += f * q01.x;
            xn.y += f * q01.y;
            xn.z += f * q23.x;
            xn.w += f * q23.y;
          }
          x.x += xn.x;
          x.y += xn.y;
          x.z += xn.z;
          x.w += xn.w;
          const uint2 kk = *reinterpret_cast<const uint2*>(Kb + s2 * LDK + c);
          const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kk.x));
          const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kk.y));
          atomicAdd(&tdn[s2], xn.x * k01.x + xn.y * k01.y + xn.z * k23.x + xn.w * k23.y);
        }
        if (c < dkr) *reinterpret_cast<float4*>(a.dk_out + qoff + (size_t)(t0 + s2) * a.DHQK + c) = x;
      }
      {  // D <- A_L D + (dN o A)^T Q
        const float AL = eA[Lc - 1];
#pragma unroll
        for (int nt = 0; nt < NS; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) st[nt][j] *= AL;
        warp_mma<true, true, NS>(st, Ab, LDV, Qb, LDK, 16 * rt, hc * (DK / 2), BCL);
      }
      __syncthreads();  // G is read above; the ditilde partials are complete
      if (!ret) {
        const float AL = eA[Lc - 1];
        for (int c = tid; c < DK; c += BCT) {
          float x = AL * nv[c];
          for (int tau = 0; tau < Lc; ++tau) x += eA[tau] * tdd[tau] * __bfloat162float(Qb[tau * LDK + c]);
          nv[c] = x;
        }
        if (tid < Lc) {
          const float di = tpp[tid] + tdn[tid];
          atomicAdd(&wdi[t0 + tid], di);
          atomicAdd(&wr[t0 + tid], -di);
        }
      }
      cl.sync();  // the partials have been read before the next chunk overwrites them
    }
    // initial-state gradients: dC0 = D, dn0 = G; dm0 = <dC0, C0> + dn0 . n0
    if (a.dC0) {
#pragma unroll
      for (int nt = 0; nt < NS; ++nt) {
        const int c = hc * (DK / 2) + 8 * nt + 2 * tq, r = 16 * rt + g;
        if (c >= dkr) continue;
        if (r0 + r < dv)
          *reinterpret_cast<float2*>(a.dC0 + soff + (size_t)r * dkr + c) = make_float2(st[nt][0], st[nt][1]);
        if (r0 + r + 8 < dv)
          *reinterpret_cast<float2*>(a.dC0 + soff + (size_t)(r + 8) * dkr + c) = make_float2(st[nt][2], st[nt][3]);
      }
    }
    if (!ret) {
      float part = a.C0 ? state_dot(a.C0) : 0.f;
      if (rank == 0)
        for (int c = tid; c < dkr; c += BCT) {
          if (a.dn0) a.dn0[slice * dkr + c] = nv[c];
          if (a.n0) part += nv[c] * a.n0[slice * dkr + c];
        }
      const float s2 = cl_block_sum(part, red);
      if (tid == 0) scal[1] += s2;
    }
    cl.sync();
  }
  // ---- this block's final-state terms (summed over the cluster) for the gate gradients, which
  // bwd_gate_grad_kernel forms once every block of the head is done
  if (rank == 0 && tid == 0) {
    float sc2 = 0.f, sc3 = 0.f;
    for (int i = 0; i < NC; ++i) {
      sc2 += cl.map_shared_rank(scal, i)[0];
      sc3 += cl.map_shared_rank(scal, i)[1];
    }
    wsc[0] = sc2;
    wsc[1] = sc3;
  }
  cl.sync();  // no CTA leaves while rank 0 may still read its shared memory
}

// Gate gradients of the cluster kernel, one warp per batch x head, after every block of the head:
// dlf_t = sum_{tau >= t} r_tau + the final-state terms (summed over the blocks), the forget-gate
// pre-activation gradient dlf_t sigmoid(-f_t), the input-gate gradient and dm0.
__global__ void __launch_bounds__(32) bwd_gate_grad_kernel(BwdArgs a) {
  const int bh = blockIdx.x, lane = threadIdx.x, S = a.S;
  const size_t nbh = (size_t)a.B * a.NH;
  const float* wr = a.ws + nbh * a.nb * 6 * S + (size_t)bh * 2 * S;
  const float* wdi = wr + S;
  const float* wsc = a.ws + nbh * a.nb * 6 * S + nbh * 2 * S + (size_t)bh * a.nb * 2;
  float sc2 = 0.f, sc3 = 0.f;
  for (int b = 0; b < a.nb; ++b) {
    sc2 += wsc[2 * b];
    sc3 += wsc[2 * b + 1];
  }
  const int seg = (S + 31) / 32, t_lo = lane * seg, t_hi = min(S, t_lo + seg);
  float sum = 0.f;
  for (int t = t_lo; t < t_hi; ++t) sum += wr[t];
  float later = sum;
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_down_sync(0xffffffffu, later, o);
    if (lane + o < 32) later += y;
  }
  float acc = later - sum + sc2;
  for (int t = t_hi - 1; t >= t_lo; --t) {
    acc += wr[t];
    const float ft = a.fg[(size_t)bh * S + t];
    if (a.dfg) a.dfg[(size_t)bh * S + t] = acc / (1.f + expf(ft));
    if (a.dig) a.dig[(size_t)bh * S + t] = wdi[t];
  }
  if (lane == 0 && a.dm0) a.dm0[bh] = sc3;
}

// value rows per CTA of the cluster kernel, and its cluster size for these widths (0: not
// supported): bf16, block key width 64 / 128 / 256, value width a multiple of 64 up to 512
int bwd_cluster_size(int dtype, int dk, int dv) {
  if (dtype != 1) return 0;
  // key widths 64 / 128 / 256, or narrower (a multiple of 8) run as 64 with zero padding;
  // value widths a multiple of 64 up to 512, or narrower (a multiple of 8) as one padded CTA
  if (dk != 64 && dk != 128 && dk != 256 && !(dk < 64 && dk % 8 == 0)) return 0;
  if (dv < BCV) return dv % 8 == 0 && dk <= 64 ? 1 : 0;
  if (dv % BCV != 0 || dv / BCV > 8) return 0;
  return dv / BCV;
}

template <int DK>
cudaError_t launch_cluster_dk(const BwdArgs& a, long long BH, int nc, cudaStream_t stream) {
  const int smem = BcSmem<DK>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(bwd_cluster_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nc, (unsigned)BH, (unsigned)a.nb);
  cfg.blockDim = dim3(BCT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)nc;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  // the gate-gradient sums that every block adds to start at zero
  const size_t nbh = (size_t)BH;
  e = cudaMemsetAsync(a.ws + nbh * a.nb * 6 * a.S, 0, nbh * 2 * a.S * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&cfg, bwd_cluster_kernel<DK>, a);
  if (e != cudaSuccess || a.retention) return e;
  bwd_gate_grad_kernel<<<(unsigned)BH, 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_smem_bytes(int dk, int dv) {
  return ((size_t)dv * (dk + 1) + 4 * (size_t)dk + 5 * (size_t)dv + NTB / 32 + NTB) * sizeof(float);
}

// the SIMT kernels: 8 floats per token of each batch x head; the cluster kernel: 6 per token of each
// (batch x head, block), 2 per token of each batch x head and 2 per (batch x head, block)
size_t bwd_workspace_bytes(long long BH, int S, int nb) {
  const size_t simt = (size_t)BH * 8 * (size_t)S;
  const size_t cluster = (size_t)BH * ((size_t)nb * 6 * S + 2 * (size_t)S + 2 * (size_t)nb);
  return (simt > cluster ? simt : cluster) * sizeof(float);
}

namespace {
size_t bwd_chunk_smem_bytes(int dk, int dv, int L) {
  return ((size_t)dv * (dk + 1) + dk + 2 * (size_t)L * (dk + 1) + 4 * (size_t)L * (dv + 1) + 3 * (size_t)L * L +
          8 * (size_t)L + NTB / 32) *
         sizeof(float);
}
constexpr size_t SMEM_LIMIT = 200 * 1024;
// chunk length of the chunked kernel for these widths (0: use the per-token kernel)
int bwd_chunk_len(int dk, int dv) {
  if (dk > 128 || dv > 128) return 0;
  if (bwd_chunk_smem_bytes(dk, dv, 32) <= SMEM_LIMIT) return 32;
  if (bwd_chunk_smem_bytes(dk, dv, 16) <= SMEM_LIMIT) return 16;
  return 0;
}
template <typename T, int L>
cudaError_t launch_chunked(const BwdArgs& a, long long BH, cudaStream_t stream) {
  const size_t smem = bwd_chunk_smem_bytes(a.dk, a.dv, L);
  cudaError_t e = cudaFuncSetAttribute(bwd_chunk_kernel<T, L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  bwd_chunk_kernel<T, L><<<(unsigned)BH, NTB, smem, stream>>>(a);
  return cudaGetLastError();
}
}  // namespace

bool bwd_supported(int dk, int dv, int dtype) {
  if (dk >= 1 && dv >= 1 && dk <= NTB && dv <= NTB && bwd_smem_bytes(dk, dv) <= 200 * 1024) return true;
  return bwd_cluster_size(dtype, dk, dv) > 0;
}

cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  const long long BH = (long long)a.B * a.NH;
  if (BH == 0) return cudaSuccess;
  // bf16 blocks of key width 64 / 128 / 256 and value width a multiple of 64 (up to 512): the
  // cluster kernel (warp-level MMAs; one CTA per 64 value rows); everything else (fp32 inputs,
  // narrower blocks): the SIMT kernels with the whole block state in one CTA
  const int nc = bwd_cluster_size(a.dtype, a.dk, a.dv);
  if (nc > 0) {
    if (a.dk == 256) return launch_cluster_dk<256>(a, BH, nc, stream);
    if (a.dk == 128) return launch_cluster_dk<128>(a, BH, nc, stream);
    if (a.dk <= 64) return launch_cluster_dk<64>(a, BH, nc, stream);
    return cudaErrorInvalidValue;
  }
  const int L = bwd_chunk_len(a.dk, a.dv);
  if (L == 32) return a.dtype == 1 ? launch_chunked<__nv_bfloat16, 32>(a, BH, stream) : launch_chunked<float, 32>(a, BH, stream);
  if (L == 16) return a.dtype == 1 ? launch_chunked<__nv_bfloat16, 16>(a, BH, stream) : launch_chunked<float, 16>(a, BH, stream);
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
