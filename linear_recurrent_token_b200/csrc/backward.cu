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

size_t bwd_smem_bytes(int dk, int dv) {
  return ((size_t)dv * (dk + 1) + 4 * (size_t)dk + 5 * (size_t)dv + NTB / 32 + NTB) * sizeof(float);
}

size_t bwd_workspace_bytes(long long BH, int S) { return (size_t)BH * 8 * (size_t)S * sizeof(float); }

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

bool bwd_supported(int dk, int dv) {
  return dk >= 1 && dv >= 1 && dk <= NTB && dv <= NTB && bwd_smem_bytes(dk, dv) <= 200 * 1024;
}

cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  const long long BH = (long long)a.B * a.NH;
  if (BH == 0) return cudaSuccess;
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
