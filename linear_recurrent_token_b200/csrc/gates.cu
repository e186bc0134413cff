// Gate / stabiliser preparation for the chunkwise prefill (sm_100a, SIMT fp32).
//
// For every (batch, head) it evaluates the stabiliser recurrence of the mLSTM
// (gates "stabilized in log space", DeepChrInteract-v2 "mLSTM Model", "Core idea"):
//     m_t = max(log f_t + m_{t-1}, itilde_t),   log f_t = logsigmoid(ftilde_t),
// for all t in parallel as a max-plus scan: each step is the map x -> max(a + x, b),
// maps compose associatively, so one CTA scans a whole sequence.  It also snapshots
// the initial normaliser n0 and stabiliser m0 into the workspace, so that the later
// kernels may overwrite the caller's n / m in place without a read-after-write race.
#include "common.cuh"
#include "kernels.h"

namespace mlstm {

__global__ void __launch_bounds__(1024) gate_prep_kernel(int S, int n_per_head, const float* __restrict__ ig,
                                                         const float* __restrict__ fg,
                                                         const float* __restrict__ m0,
                                                         const float* __restrict__ n0,
                                                         float* __restrict__ m_tok,
                                                         float* __restrict__ m_init,
                                                         float* __restrict__ n_init) {
  __shared__ MaxPlus warp_tot[32];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const float mstart = m0 ? m0[bh] : 0.f;
  for (int i = tid; i < n_per_head; i += blockDim.x)
    n_init[(size_t)bh * n_per_head + i] = n0 ? n0[(size_t)bh * n_per_head + i] : 0.f;
  if (tid == 0) m_init[bh] = mstart;

  const int per = (S + blockDim.x - 1) / blockDim.x;
  const int t0 = min(S, tid * per), t1 = min(S, t0 + per);
  const float* igh = ig + (size_t)bh * S;
  const float* fgh = fg + (size_t)bh * S;

  MaxPlus loc{0.f, -INFINITY};
  for (int t = t0; t < t1; ++t) loc = mp_then(loc, MaxPlus{log_sigmoid(fgh[t]), igh[t]});

  // exclusive block scan of the per-thread maps
  MaxPlus inc = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    MaxPlus u{__shfl_up_sync(0xffffffffu, inc.A, o), __shfl_up_sync(0xffffffffu, inc.Bm, o)};
    if (lane >= o) inc = mp_then(u, inc);
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    MaxPlus w = lane < nwarps ? warp_tot[lane] : MaxPlus{0.f, -INFINITY};
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      MaxPlus u{__shfl_up_sync(0xffffffffu, w.A, o), __shfl_up_sync(0xffffffffu, w.Bm, o)};
      if (lane >= o) w = mp_then(u, w);
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  MaxPlus excl_lane{__shfl_up_sync(0xffffffffu, inc.A, 1), __shfl_up_sync(0xffffffffu, inc.Bm, 1)};
  if (lane == 0) excl_lane = MaxPlus{0.f, -INFINITY};
  MaxPlus prefix = warp > 0 ? mp_then(warp_tot[warp - 1], excl_lane) : excl_lane;

  float x = mp_apply(prefix, mstart);
  float* mh = m_tok + (size_t)bh * S;
  for (int t = t0; t < t1; ++t) {
    x = fmaxf(log_sigmoid(fgh[t]) + x, igh[t]);
    mh[t] = x;
  }
}

cudaError_t launch_gate_prep(int BH, int S, int n_per_head, const float* ig, const float* fg,
                             const float* m0, const float* n0, float* m_tok, float* m_init,
                             float* n_init, cudaStream_t stream) {
  if (BH == 0) return cudaSuccess;
  int threads = 1024;
  while (threads > 32 && threads / 2 >= S) threads /= 2;
  gate_prep_kernel<<<BH, threads, 0, stream>>>(S, n_per_head, ig, fg, m0, n0, m_tok, m_init, n_init);
  return cudaGetLastError();
}

}  // namespace mlstm
