// Chunkwise prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA), bf16 inputs,
// fp32 state.  Chunk length 64; per-block key width DK in {64, 128, 256}; the value
// rows of a block's state are split into tiles of DVT in {64, 128} rows (the MMA M).
//
// Parallel structure.  One (batch, head, block) has a single chain of chunks, and a
// B200 has 148 SMs, so the sequence is cut into G segments of whole chunks:
//   phase A  (tc_segment_kernel)  for every segment but the last, its own contribution
//            to the state, as if it started from zero:  dC_g = sum_s w_s v_s k_s^T,
//            dn_g = sum_s w_s k_s, with w_s = exp(Gtot_g - G_s + itilde_s - M_g),
//            G the inclusive cumulative log forget gate inside the segment and
//            M_g = max_s(Gtot_g - G_s + itilde_s).  One long-K tensor-core GEMM per
//            (segment, value tile): D[dv, dk] += (V o w)^T K over the segment's tokens.
//   phase C  (tc_walk_kernel)  per (segment, value tile): combine the initial state and
//            the summaries of all earlier segments into the segment's start state
//            (max-plus composition of (Gtot, M) gives the stabiliser), load it into TMEM
//            as fp32, and walk the segment's chunks:
//              S = Q K^T                       (tcgen05, M=64 N=64, K=DK)
//              P = S o D',  D'[t,s] = exp(b_t - b_s + itilde_s - m_t)  (s <= t)
//              H^T = C_bf16 Q^T  (read-out)    (tcgen05, M=DVT N=64 K=DK)
//              H^T += ... V^T P^T (intra)      (tcgen05, M=DVT N=64 K=64, own accumulator)
//              C <- a C + (V o w)^T K          (TMEM round trip for a, then tcgen05 M=DVT N=DK)
//              h_t = o_t (e^{b_t+m_c-m_t} H_inter + H_intra) / max(|r_t + e^{..} n.q_t|, e^{-m_t})
//            The last segment writes the final (C, n, m).
// Retention (RetNet "Key Innovation"): log f = log gamma_h, itilde = 0, m = 0, no
// normaliser; the same kernels with those gate values.
//
// Every mbarrier wait is bounded (~2 s); on expiry the kernel records a bit in the
// workspace error word, stops issuing work, frees its TMEM and returns.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mlstm {

using namespace sm100;

namespace {

constexpr int L = 64;            // chunk length of the tensor-core path
constexpr int NT = 128;          // threads per CTA (4 warps = the 4 TMEM lane quarters)
constexpr long long WAIT = 4000000000LL;

struct TcParams {
  int S, NH, nb, dk, dv, DHQK, DHV, retention, dtype;
  int G, seg_chunks, n_tiles;
  const float *ig, *fg;
  const float *C0, *n0, *m0;  // initial state (snapshots where needed), may be NULL
  const __nv_bfloat16* og;
  __nv_bfloat16* h;
  float *C_out, *n_out, *m_out;
  float *dC, *dn, *segA, *segB;  // workspace: summaries of segments 0..G-2
  unsigned int* err;
};

// Lane / row mapping of an M-row accumulator: thread (warp w, lane l) owns row
// 32w+l for M=128; row 16w+l for M=64 (lanes 16..31 hold no row).
template <int M>
__device__ __forceinline__ int acc_row(int warp, int lane) {
  return M == 128 ? 32 * warp + lane : (lane < 16 ? 16 * warp + lane : -1);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ float bf16_at(const uint8_t* tile, int row, int col) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + sw128_offset(row, col)));
}

// Gate values of token t (global index) for head `head`: (log f, itilde).
__device__ __forceinline__ void gate_vals(const TcParams& p, size_t tok, int head, float& lf, float& li) {
  if (p.retention) {
    lf = retention_log_gamma(head);
    li = 0.f;
  } else {
    lf = log_sigmoid(p.fg[tok]);
    li = p.ig[tok];
  }
}

}  // namespace

// ===================================================================== phase A
template <int DK, int DVT>
__global__ void __launch_bounds__(NT, 1)
    tc_segment_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV, TcParams p) {
  constexpr int KB = DK * 128;   // bytes of one K chunk tile (DK/64 boxes of 8 KiB)
  constexpr int VB = DVT * 128;  // bytes of one V chunk tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Ks[2] = {sm, sm + KB};
  uint8_t* Vs[2] = {sm + 2 * KB, sm + 2 * KB + VB};
  float* omega = reinterpret_cast<float*>(sm + 2 * KB + 2 * VB);  // [seg_chunks * L]
  __shared__ uint64_t bar_load[2], bar_mma[2];
  __shared__ uint32_t tmem_base;
  __shared__ float red[NT / 32];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, g = blockIdx.y, slice = blockIdx.z;
  const int blk = slice % p.nb, bh = slice / p.nb, head = bh % p.NH;
  const int seg_len = p.seg_chunks * L;
  const int T0 = g * seg_len;  // phase A covers full segments only
  const int v0 = tile * DVT;

  if (tid == 0) {
    mbar_init(&bar_load[0], 1);
    mbar_init(&bar_load[1], 1);
    mbar_init(&bar_mma[0], 1);
    mbar_init(&bar_mma[1], 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mapK);
    prefetch_tensormap(&mapV);
  }
  if (warp == 0) tmem_alloc(&tmem_base, DK);
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;

  // first chunk in flight while the gates are prepared
  const int nck = p.seg_chunks;
  auto issue = [&](int c) {
    const int st = c & 1;
    mbar_arrive_expect_tx(&bar_load[st], KB + VB);
    for (int j = 0; j < DK / 64; ++j) tma_load_3d(Ks[st] + j * 8192, &mapK, blk * p.dk + 64 * j, T0 + c * L, bh, &bar_load[st]);
    for (int j = 0; j < DVT / 64; ++j)
      tma_load_3d(Vs[st] + j * 8192, &mapV, blk * p.dv + v0 + 64 * j, T0 + c * L, bh, &bar_load[st]);
  };
  if (tid == 0) issue(0);

  // ---- gates: G_s (inclusive cumulative log f), Gtot, M, omega_s
  const size_t tok0 = (size_t)bh * p.S + T0;
  const int per = (seg_len + NT - 1) / NT;
  const int r0 = min(seg_len, tid * per), r1 = min(seg_len, r0 + per);
  float run = 0.f;
  for (int t = r0; t < r1; ++t) {
    float lf, li;
    gate_vals(p, tok0 + t, head, lf, li);
    run += lf;
  }
  // exclusive scan of run sums over the block
  float inc = run;
  for (int o = 1; o < 32; o <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  float wexcl = 0.f, total = 0.f;
  for (int w = 0; w < NT / 32; ++w) {
    if (w < warp) wexcl += red[w];
    total += red[w];
  }
  float Gs = wexcl + inc - run;  // exclusive prefix of this thread's run
  float lmax = -INFINITY;
  for (int t = r0; t < r1; ++t) {
    float lf, li;
    gate_vals(p, tok0 + t, head, lf, li);
    Gs += lf;
    const float x = li - Gs;  // log weight minus Gtot
    omega[t] = x;
    lmax = fmaxf(lmax, total + x);
  }
  for (int o = 16; o >= 1; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  __syncthreads();
  if (lane == 0) red[warp] = lmax;
  __syncthreads();
  float Mg = -INFINITY;
  for (int w = 0; w < NT / 32; ++w) Mg = fmaxf(Mg, red[w]);
  if (p.retention) Mg = 0.f;
  for (int t = r0; t < r1; ++t) omega[t] = expf(total + omega[t] - Mg);
  if (tile == 0 && blk == 0 && tid == 0) {
    p.segA[(size_t)bh * (p.G - 1) + g] = total;
    p.segB[(size_t)bh * (p.G - 1) + g] = Mg;
  }
  __syncthreads();

  // ---- main loop: D[dv, dk] += (V o omega)^T K over the segment
  const uint32_t idesc = idesc_bf16(DVT, DK, 1, 1);
  float dn_acc[2] = {0.f, 0.f};  // columns tid and tid + 128 of dn (value tile 0 only)
  for (int c = 0; c < nck; ++c) {
    const int st = c & 1;
    if (c + 1 < nck) {
      if (c >= 1 && !abort_flag) {  // the MMAs of chunk c-1 read stage st^1
        if (!mbar_wait(&bar_mma[st ^ 1], ((c - 1) >> 1) & 1, WAIT)) atomicOr(&abort_flag, 1);
      }
      __syncthreads();
      if (tid == 0 && !abort_flag) issue(c + 1);
    }
    if (!abort_flag && !mbar_wait(&bar_load[st], (c >> 1) & 1, WAIT)) atomicOr(&abort_flag, 1);
    __syncthreads();
    if (abort_flag) break;
    // V rows scaled in place by omega (a row is 128 contiguous bytes whatever the swizzle)
    const float* om = omega + c * L;
    for (int i = tid; i < L * (DVT / 8); i += NT) {
      const int row = i / (DVT / 8), ch = i % (DVT / 8);
      uint8_t* ptr = Vs[st] + (ch >> 3) * 8192 + row * 128 + ((ch & 7) << 4);
      uint4 u = *reinterpret_cast<uint4*>(ptr);
      __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
      const float w = om[row];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = __bfloat1622float2(b2[j]);
        b2[j] = __floats2bfloat162_rn(f.x * w, f.y * w);
      }
      *reinterpret_cast<uint4*>(ptr) = u;
    }
    if (tile == 0) {
      for (int j = 0; j < 2; ++j) {
        const int col = tid + 128 * j;
        if (col < DK) {
          float a = 0.f;
          for (int s = 0; s < L; ++s) a += om[s] * bf16_at(Ks[st] + (col >> 6) * 8192, s, col & 63);
          dn_acc[j] += a;
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < L / 16; ++ks) {
        const uint64_t ad = smem_desc_sw128(smem_u32(Vs[st]) + ks * 2048, 8192, 1024);
        const uint64_t bd = smem_desc_sw128(smem_u32(Ks[st]) + ks * 2048, 8192, 1024);
        mma_bf16_ss(tm, ad, bd, idesc, (c > 0 || ks > 0) ? 1u : 0u);
      }
      mma_commit(&bar_mma[st]);
    }
  }
  if (!abort_flag && !mbar_wait(&bar_mma[(nck - 1) & 1], ((nck - 1) >> 1) & 1, WAIT)) atomicOr(&abort_flag, 1);
  __syncthreads();
  tc_fence_after();
  if (!abort_flag) {
    const int row = acc_row<DVT>(warp, lane);
    float* dst = row >= 0 ? p.dC + (((size_t)slice * (p.G - 1) + g) * p.dv + v0 + row) * p.dk : nullptr;
    for (int c0 = 0; c0 < DK; c0 += 16) {
      float r[16];
      tmem_ld16(tm + ((uint32_t)(32 * warp) << 16) + c0, r);
      tmem_wait_ld();
      if (dst)
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4*>(dst + c0 + j) = make_float4(r[j], r[j + 1], r[j + 2], r[j + 3]);
    }
    if (tile == 0)
      for (int j = 0; j < 2; ++j) {
        const int col = tid + 128 * j;
        if (col < DK) p.dn[((size_t)slice * (p.G - 1) + g) * p.dk + col] = dn_acc[j];
      }
  } else if (tid == 0) {
    atomicOr(p.err, 1u);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, DK);
}

// ===================================================================== phase C
template <int DK, int DVT>
struct WalkSmem {
  static constexpr int QB = DK * 128, KB = DK * 128, VB = DVT * 128, PB = 64 * 128, CB = DVT * DK * 2;
  static constexpr int OQ = 0, OK = OQ + QB, OV = OK + KB, OVW = OV + VB, OP = OVW + VB, OC = OP + PB;
  static constexpr int OF = OC + CB;                   // floats start here
  static constexpr int NF = DK + 8 * L + 16;           // n, per-token arrays, scalars
  static constexpr int BYTES = OF + NF * 4 + 1024;     // + alignment slack
};

template <int DK, int DVT>
__global__ void __launch_bounds__(NT, 1)
    tc_walk_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, TcParams p) {
  using SM = WalkSmem<DK, DVT>;
  constexpr uint32_t TM_C = 0, TM_S = DK, TM_I = DK + 64, TM_J = DK + 128;  // TMEM columns
  constexpr uint32_t TM_COLS = (DK + 192 <= 256) ? 256 : 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *Qs = sm + SM::OQ, *Ks = sm + SM::OK, *Vs = sm + SM::OV, *Vw = sm + SM::OVW, *Ps = sm + SM::OP,
          *Cb = sm + SM::OC;
  float* nvec = reinterpret_cast<float*>(sm + SM::OF);
  float* bl = nvec + DK;
  float* li = bl + L;
  float* mt = li + L;
  float* sint = mt + L;
  float* wv = sint + L;
  float* den = wv + L;
  float* nq = den + L;
  float* scal = nq + L;  // [0] decay a, [1] m_c, [2] m_next
  __shared__ uint64_t bar_load, bar_s, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, g = blockIdx.y, slice = blockIdx.z;
  const int blk = slice % p.nb, bh = slice / p.nb, head = bh % p.NH;
  const int v0 = tile * DVT;
  const int seg_len = p.seg_chunks * L;
  const int T0 = g * seg_len, T1 = min(p.S, T0 + seg_len);
  const bool ret = p.retention != 0;
  const bool last_seg = g == p.G - 1;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

  if (tid == 0) {
    mbar_init(&bar_load, 1);
    mbar_init(&bar_s, 1);
    mbar_init(&bar_mma, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mapQ);
    prefetch_tensormap(&mapK);
    prefetch_tensormap(&mapV);
  }
  if (warp == 0) tmem_alloc(&tmem_base, TM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;

  auto issue = [&](int t0) {
    mbar_arrive_expect_tx(&bar_load, SM::QB + SM::KB + SM::VB);
    for (int j = 0; j < DK / 64; ++j) {
      tma_load_3d(Qs + j * 8192, &mapQ, blk * p.dk + 64 * j, t0, bh, &bar_load);
      tma_load_3d(Ks + j * 8192, &mapK, blk * p.dk + 64 * j, t0, bh, &bar_load);
    }
    for (int j = 0; j < DVT / 64; ++j) tma_load_3d(Vs + j * 8192, &mapV, blk * p.dv + v0 + 64 * j, t0, bh, &bar_load);
  };
  if (tid == 0) issue(T0);

  // ---- start state of the segment: stabiliser by max-plus composition of the earlier
  // segments' (Gtot, M); C and n as the matching weighted sum of C0 and the summaries.
  float m_start = ret ? 0.f : (p.m0 ? p.m0[bh] : 0.f);
  const float m_init = m_start;
  float gsum = 0.f;  // sum of Gtot over segments 0..g-1
  for (int j = 0; j < g; ++j) {
    const float A = p.segA[(size_t)bh * (p.G - 1) + j], Bm = p.segB[(size_t)bh * (p.G - 1) + j];
    if (!ret) m_start = fmaxf(A + m_start, Bm);
    gsum += A;
  }
  // weight of C0: exp(gsum + m_init - m_start); of summary j: exp(M_j + sum_{j<i<g} Gtot_i - m_start)
  {
    const int row = acc_row<DVT>(warp, lane);
    const float wc0 = expf(gsum + m_init - m_start);
    for (int c0 = 0; c0 < DK; c0 += 16) {
      float r[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) r[j] = 0.f;
      if (row >= 0) {
        if (p.C0) {
          const float* src = p.C0 + ((size_t)slice * p.dv + v0 + row) * p.dk + c0;
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] = wc0 * src[j];
        }
        float after = gsum;
        for (int jg = 0; jg < g; ++jg) {
          after -= p.segA[(size_t)bh * (p.G - 1) + jg];
          const float wj = expf(p.segB[(size_t)bh * (p.G - 1) + jg] + after - m_start);
          const float* src = p.dC + (((size_t)slice * (p.G - 1) + jg) * p.dv + v0 + row) * p.dk + c0;
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] += wj * src[j];
        }
      }
      tmem_st16(tm + lane_off + TM_C + c0, r);
    }
    tmem_wait_st();
    if (!ret)
      for (int col = tid; col < DK; col += NT) {
        float x = p.n0 ? wc0 * p.n0[(size_t)slice * p.dk + col] : 0.f;
        float after = gsum;
        for (int jg = 0; jg < g; ++jg) {
          after -= p.segA[(size_t)bh * (p.G - 1) + jg];
          x += expf(p.segB[(size_t)bh * (p.G - 1) + jg] + after - m_start) *
               p.dn[((size_t)slice * (p.G - 1) + jg) * p.dk + col];
        }
        nvec[col] = x;
      }
  }
  if (tid == 0) scal[1] = m_start;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t id_s = idesc_bf16(64, 64, 0, 0);
  const uint32_t id_ro = idesc_bf16(DVT, 64, 0, 0);
  const uint32_t id_pv = idesc_bf16(DVT, 64, 1, 0);
  const uint32_t id_up = idesc_bf16(DVT, DK, 1, 1);
  const float lg = ret ? retention_log_gamma(head) : 0.f;

  int it = 0;
  for (int t0 = T0; t0 < T1; t0 += L, ++it) {
    const int Lc = min(L, T1 - t0);
    const size_t tok0 = (size_t)bh * p.S + t0;
    // ---- per-token gate quantities (warp 0): b (cumulative log f), m_t, scales
    if (warp == 0) {
      const float mc = scal[1];
      float lfa, lia, lfb, lib;
      const int ta = 2 * lane, tb = 2 * lane + 1;
      if (ta < Lc) gate_vals(p, tok0 + ta, head, lfa, lia); else { lfa = 0.f; lia = -INFINITY; }
      if (tb < Lc) gate_vals(p, tok0 + tb, head, lfb, lib); else { lfb = 0.f; lib = -INFINITY; }
      float sum = lfa + lfb;
      float isum = sum;
      MaxPlus mp = mp_then(MaxPlus{lfa, lia}, MaxPlus{lfb, lib});
      MaxPlus imp = mp;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float us = __shfl_up_sync(0xffffffffu, isum, o);
        const MaxPlus um{__shfl_up_sync(0xffffffffu, imp.A, o), __shfl_up_sync(0xffffffffu, imp.Bm, o)};
        if (lane >= o) {
          isum += us;
          imp = mp_then(um, imp);
        }
      }
      float esum = __shfl_up_sync(0xffffffffu, isum, 1);
      MaxPlus emp{__shfl_up_sync(0xffffffffu, imp.A, 1), __shfl_up_sync(0xffffffffu, imp.Bm, 1)};
      if (lane == 0) {
        esum = 0.f;
        emp = MaxPlus{0.f, -INFINITY};
      }
      const float ba = esum + lfa, bb = esum + lfa + lfb;
      float ma, mb;
      if (ret) {
        ma = mb = 0.f;
      } else {
        const MaxPlus pa = mp_then(emp, MaxPlus{lfa, lia});
        ma = mp_apply(pa, mc);
        mb = mp_apply(mp_then(pa, MaxPlus{lfb, lib}), mc);
      }
      if (ret) {
        bl[ta] = (float)(ta + 1) * lg;
        bl[tb] = (float)(tb + 1) * lg;
      } else {
        bl[ta] = ba;
        bl[tb] = bb;
      }
      li[ta] = ret ? 0.f : lia;
      li[tb] = ret ? 0.f : lib;
      mt[ta] = ma;
      mt[tb] = mb;
      __syncwarp();
      const float gtot = bl[Lc - 1];
      const float mn = mt[Lc - 1];
      sint[ta] = expf(bl[ta] + mc - ma);
      sint[tb] = expf(bl[tb] + mc - mb);
      wv[ta] = ta < Lc ? expf(gtot - bl[ta] + li[ta] - mn) : 0.f;
      wv[tb] = tb < Lc ? expf(gtot - bl[tb] + li[tb] - mn) : 0.f;
      if (lane == 0) {
        scal[0] = expf(gtot + mc - mn);
        scal[2] = mn;
      }
    }
    if (!abort_flag && !mbar_wait(&bar_load, it & 1, WAIT)) atomicOr(&abort_flag, 1);
    __syncthreads();
    if (abort_flag) break;
    // ---- S = Q K^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < DK; k += 16) {
        const uint32_t off = (k >> 6) * 8192 + (k & 63) * 2;
        mma_bf16_ss(tm + TM_S, smem_desc_sw128(smem_u32(Qs) + off, 16, 1024),
                    smem_desc_sw128(smem_u32(Ks) + off, 16, 1024), id_s, k > 0 ? 1u : 0u);
      }
      mma_commit(&bar_s);
    }
    // ---- n . q_t (two threads per token) and V o w
    if (!ret) {
      const int t = tid >> 1, half = tid & 1;
      float a = 0.f;
      for (int col = half * (DK / 2); col < (half + 1) * (DK / 2); col += 8) {
        const uint8_t* ptr = Qs + (col >> 6) * 8192 + sw128_offset(t, col & 63);
        const uint4 u = *reinterpret_cast<const uint4*>(ptr);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(b2[j]);
          a += f.x * nvec[col + 2 * j] + f.y * nvec[col + 2 * j + 1];
        }
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      if (half == 0) nq[t] = a;
    }
    for (int i = tid; i < L * (DVT / 8); i += NT) {
      const int row = i / (DVT / 8), ch = i % (DVT / 8);
      const int off = (ch >> 3) * 8192 + row * 128 + ((ch & 7) << 4);
      uint4 u = *reinterpret_cast<const uint4*>(Vs + off);
      __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
      const float w = wv[row];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(b2[j]);
        b2[j] = __floats2bfloat162_rn(f.x * w, f.y * w);
      }
      *reinterpret_cast<uint4*>(Vw + off) = u;
    }
    if (!mbar_wait(&bar_s, it & 1, WAIT)) atomicOr(&abort_flag, 1);
    __syncthreads();
    if (abort_flag) break;
    tc_fence_after();
    // ---- P = S o D' (bf16, K-major rows t), row sums, denominators
    {
      const int t = acc_row<64>(warp, lane);
      float rs = 0.f;
      for (int s0 = 0; s0 < L; s0 += 16) {
        float r[16];
        tmem_ld16(tm + lane_off + TM_S + s0, r);
        tmem_wait_ld();
        if (t >= 0) {
          float pv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int s = s0 + j;
            float v = 0.f;
            if (s <= t && t < Lc) v = r[j] * expf(bl[t] - bl[s] + li[s] - mt[t]);
            pv[j] = v;
            rs += v;
          }
          const uint32_t base = smem_u32(Ps);
          st_shared_v4(base + sw128_offset(t, s0), pack_bf16(pv[0], pv[1]), pack_bf16(pv[2], pv[3]),
                       pack_bf16(pv[4], pv[5]), pack_bf16(pv[6], pv[7]));
          st_shared_v4(base + sw128_offset(t, s0 + 8), pack_bf16(pv[8], pv[9]), pack_bf16(pv[10], pv[11]),
                       pack_bf16(pv[12], pv[13]), pack_bf16(pv[14], pv[15]));
        }
      }
      if (t >= 0 && !ret) den[t] = fmaxf(fabsf(rs + sint[t] * nq[t]), expf(-mt[t]));
    }
    // ---- C round trip: bf16 copy of C_c for the read-out, C <- a C in TMEM
    {
      const int row = acc_row<DVT>(warp, lane);
      const float a = scal[0];
      const uint32_t cb = smem_u32(Cb);
      for (int c0 = 0; c0 < DK; c0 += 16) {
        float r[16];
        tmem_ld16(tm + lane_off + TM_C + c0, r);
        tmem_wait_ld();
        if (row >= 0) {
          const uint32_t base = cb + (c0 >> 6) * (DVT * 128);
          st_shared_v4(base + sw128_offset(row, c0 & 63), pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]),
                       pack_bf16(r[4], r[5]), pack_bf16(r[6], r[7]));
          st_shared_v4(base + sw128_offset(row, (c0 & 63) + 8), pack_bf16(r[8], r[9]), pack_bf16(r[10], r[11]),
                       pack_bf16(r[12], r[13]), pack_bf16(r[14], r[15]));
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) r[j] *= a;
        tmem_st16(tm + lane_off + TM_C + c0, r);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- read-out, intra-chunk and state-update MMAs
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < DK; k += 16) {
        const uint32_t aoff = (k >> 6) * (DVT * 128) + (k & 63) * 2;
        const uint32_t boff = (k >> 6) * 8192 + (k & 63) * 2;
        mma_bf16_ss(tm + TM_I, smem_desc_sw128(smem_u32(Cb) + aoff, 16, 1024),
                    smem_desc_sw128(smem_u32(Qs) + boff, 16, 1024), id_ro, k > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int ks = 0; ks < L / 16; ++ks)
        mma_bf16_ss(tm + TM_J, smem_desc_sw128(smem_u32(Vs) + ks * 2048, 8192, 1024),
                    smem_desc_sw128(smem_u32(Ps) + ks * 32, 16, 1024), id_pv, ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < L / 16; ++ks)
        mma_bf16_ss(tm + TM_C, smem_desc_sw128(smem_u32(Vw) + ks * 2048, 8192, 1024),
                    smem_desc_sw128(smem_u32(Ks) + ks * 2048, 8192, 1024), id_up, 1u);
      mma_commit(&bar_mma);
    }
    // ---- normaliser update n <- a n + sum_s w_s k_s (reads K while the MMAs run)
    if (!ret) {
      const float a = scal[0];
      for (int col = tid; col < DK; col += NT) {
        float acc = 0.f;
        const uint8_t* kt = Ks + (col >> 6) * 8192;
        for (int s = 0; s < Lc; ++s) acc += wv[s] * bf16_at(kt, s, col & 63);
        nvec[col] = a * nvec[col] + acc;
      }
    }
    if (!mbar_wait(&bar_mma, it & 1, WAIT)) atomicOr(&abort_flag, 1);
    __syncthreads();
    if (abort_flag) break;
    tc_fence_after();
    // ---- outputs h_t for this value tile
    {
      const int row = acc_row<DVT>(warp, lane);
      const size_t hcol = (size_t)blk * p.dv + v0 + (row >= 0 ? row : 0);
      for (int tt = 0; tt < L; tt += 16) {
        float ri[16], rj[16];
        tmem_ld16(tm + lane_off + TM_I + tt, ri);
        tmem_ld16(tm + lane_off + TM_J + tt, rj);
        tmem_wait_ld();
        if (row >= 0) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = tt + j;
            if (t < Lc) {
              float hv = sint[t] * ri[j] + rj[j];
              const size_t idx = (tok0 + t) * p.DHV + hcol;
              if (!ret) {
                hv = hv / den[t];
                if (p.og) hv *= __bfloat162float(p.og[idx]);
              }
              p.h[idx] = __float2bfloat16_rn(hv);
            }
          }
        }
      }
    }
    if (tid == 0) scal[1] = scal[2];
    tc_fence_before();
    __syncthreads();
    // next chunk's operands
    if (tid == 0 && t0 + L < T1) issue(t0 + L);
  }

  // ---- final state (last segment)
  tc_fence_after();
  if (!abort_flag && last_seg) {
    const int row = acc_row<DVT>(warp, lane);
    if (p.C_out)
      for (int c0 = 0; c0 < DK; c0 += 16) {
        float r[16];
        tmem_ld16(tm + lane_off + TM_C + c0, r);
        tmem_wait_ld();
        if (row >= 0) {
          float* dst = p.C_out + ((size_t)slice * p.dv + v0 + row) * p.dk + c0;
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(r[j], r[j + 1], r[j + 2], r[j + 3]);
        }
      }
    if (!ret && tile == 0) {
      if (p.n_out)
        for (int col = tid; col < DK; col += NT) p.n_out[(size_t)slice * p.dk + col] = nvec[col];
      if (p.m_out && blk == 0 && tid == 0) p.m_out[bh] = scal[1];
    }
  }
  if (abort_flag && tid == 0) atomicOr(p.err, 2u);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, TM_COLS);
}

// ===================================================================== host side
bool tc_supported(int dtype, int chunk, int dk, int dv, int DHQK, int DHV) {
  if (dtype != 1 || chunk != L) return false;
  if (dk != 64 && dk != 128 && dk != 256) return false;
  if (dv % 64 != 0) return false;
  if (DHQK % 8 != 0 || DHV % 8 != 0) return false;
  return true;
}

int tc_num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

TcPlan tc_plan(int B, int NH, int S, int nb, int dk, int dv, int num_sms) {
  TcPlan pl;
  pl.dvt = (dv % 128 == 0) ? 128 : 64;
  pl.n_tiles = dv / pl.dvt;
  const int chunks = (S + L - 1) / L;
  const long long base = (long long)B * NH * nb * pl.n_tiles;
  int G = base > 0 ? (int)(num_sms / base) : 1;
  if (G < 1) G = 1;
  // at least 4 chunks per segment, segments no longer than 8192 tokens (phase A keeps
  // one fp32 weight per token in shared memory)
  if (G > chunks / 4) G = chunks / 4 > 0 ? chunks / 4 : 1;
  while ((chunks + G - 1) / G * L > 8192) ++G;
  pl.seg_chunks = chunks > 0 ? (chunks + G - 1) / G : 1;
  pl.G = chunks > 0 ? (chunks + pl.seg_chunks - 1) / pl.seg_chunks : 1;
  return pl;
}

size_t tc_workspace_bytes(const TcPlan& pl, long long BH, int nb, int dk, int dv) {
  const long long slices = BH * nb;
  const size_t G1 = pl.G > 1 ? pl.G - 1 : 0;
  size_t off = 256;  // error word
  off += ((size_t)slices * G1 * dv * dk * 4 + 255) / 256 * 256;
  off += ((size_t)slices * G1 * dk * 4 + 255) / 256 * 256;
  off += 2 * (((size_t)BH * G1 * 4 + 255) / 256 * 256);
  return off;
}

template <int DK, int DVT>
static cudaError_t launch_tc_dk(const TcPlan& pl, const TcParams& prm, const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, long long slices, cudaStream_t stream, cudaEvent_t ev0,
                                cudaEvent_t ev1) {
  cudaError_t e;
  if (pl.G > 1) {
    const int smemA = 2 * DK * 128 + 2 * DVT * 128 + pl.seg_chunks * L * 4 + 1024;
    e = cudaFuncSetAttribute(tc_segment_kernel<DK, DVT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smemA);
    if (e != cudaSuccess) return e;
    dim3 gridA(pl.n_tiles, pl.G - 1, (unsigned)slices);
    tc_segment_kernel<DK, DVT><<<gridA, NT, smemA, stream>>>(mk, mv, prm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int smemC = WalkSmem<DK, DVT>::BYTES;
  e = cudaFuncSetAttribute(tc_walk_kernel<DK, DVT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smemC);
  if (e != cudaSuccess) return e;
  if (ev0) cudaEventRecord(ev0, stream);
  dim3 gridC(pl.n_tiles, pl.G, (unsigned)slices);
  tc_walk_kernel<DK, DVT><<<gridC, NT, smemC, stream>>>(mq, mk, mv, prm);
  e = cudaGetLastError();
  if (ev1) cudaEventRecord(ev1, stream);
  return e;
}

cudaError_t launch_tc(const WalkArgs& a, const TcPlan& pl, void* ws, cudaStream_t stream, cudaEvent_t ev0,
                      cudaEvent_t ev1) {
  const long long BH = (long long)a.B * a.NH, slices = BH * a.nb;
  if (slices == 0 || a.S == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16_3d(&mq, a.q, a.DHQK, a.S, BH, L) || !make_map_bf16_3d(&mk, a.k, a.DHQK, a.S, BH, L) ||
      !make_map_bf16_3d(&mv, a.v, a.DHV, a.S, BH, L))
    return cudaErrorInvalidValue;
  TcParams prm;
  prm.S = a.S;
  prm.NH = a.NH;
  prm.nb = a.nb;
  prm.dk = a.dk;
  prm.dv = a.dv;
  prm.DHQK = a.DHQK;
  prm.DHV = a.DHV;
  prm.retention = a.retention;
  prm.dtype = a.dtype;
  prm.G = pl.G;
  prm.seg_chunks = pl.seg_chunks;
  prm.n_tiles = pl.n_tiles;
  prm.ig = a.ig;
  prm.fg = a.fg;
  prm.C0 = a.C0;
  prm.n0 = a.n_init;
  prm.m0 = a.m_init;
  prm.og = static_cast<const __nv_bfloat16*>(a.og);
  prm.h = static_cast<__nv_bfloat16*>(a.h);
  prm.C_out = a.C_out;
  prm.n_out = a.n_out;
  prm.m_out = a.m_out;
  char* w = static_cast<char*>(ws);
  const size_t G1 = pl.G > 1 ? pl.G - 1 : 0;
  prm.err = reinterpret_cast<unsigned int*>(w);
  size_t off = 256;
  prm.dC = reinterpret_cast<float*>(w + off);
  off += ((size_t)slices * G1 * a.dv * a.dk * 4 + 255) / 256 * 256;
  prm.dn = reinterpret_cast<float*>(w + off);
  off += ((size_t)slices * G1 * a.dk * 4 + 255) / 256 * 256;
  prm.segA = reinterpret_cast<float*>(w + off);
  off += ((size_t)BH * G1 * 4 + 255) / 256 * 256;
  prm.segB = reinterpret_cast<float*>(w + off);
  cudaError_t e = cudaMemsetAsync(w, 0, 4, stream);
  if (e != cudaSuccess) return e;
  if (a.dk == 256 && pl.dvt == 128) return launch_tc_dk<256, 128>(pl, prm, mq, mk, mv, slices, stream, ev0, ev1);
  if (a.dk == 256 && pl.dvt == 64) return launch_tc_dk<256, 64>(pl, prm, mq, mk, mv, slices, stream, ev0, ev1);
  if (a.dk == 128 && pl.dvt == 128) return launch_tc_dk<128, 128>(pl, prm, mq, mk, mv, slices, stream, ev0, ev1);
  if (a.dk == 128 && pl.dvt == 64) return launch_tc_dk<128, 64>(pl, prm, mq, mk, mv, slices, stream, ev0, ev1);
  if (a.dk == 64 && pl.dvt == 128) return launch_tc_dk<64, 128>(pl, prm, mq, mk, mv, slices, stream, ev0, ev1);
  if (a.dk == 64 && pl.dvt == 64) return launch_tc_dk<64, 64>(pl, prm, mq, mk, mv, slices, stream, ev0, ev1);
  return cudaErrorInvalidValue;
}

}  // namespace mlstm
