// Recurrent decode step (sm_100a): one token per sequence, state updated in place.
//
//   m' = max(log f + m, itilde);  f' = e^{log f + m - m'};  i' = e^{itilde - m'}
//   C' = f' C + i' v k^T;  n' = f' n + i' k;  h = o * (C' q) / max(|n' . q|, e^{-m'})
// Retention: C' = gamma_h C + v k^T, h = C' q.
// (RetNet recurrent_retention_step; burn-gdn2 FusedRecurrent: state carried across
// tokens and updated in place.)
//
// The step is a pure stream over C: every fp32 element is read once and written once
// (99.5 % of the bytes of a step at DHQK 256 / DHV 512).  Each (batch, head)
// is handled by one thread-block cluster: nb x CS CTAs, CS per block, splitting
// the value rows of each block's C.  A warp covers whole rows with 128-bit loads; the
// dot product C'q of a row is reduced with warp shuffles.  Every CTA needs the old n
// and m to form the denominator, and CTA 0 of each block rewrites them in place: the
// hardware cluster barrier (arrive after reading, wait before writing) orders the two
// without any spin loop.  The blocks of a head share m, hence one cluster per head.
#include "common.cuh"
#include "kernels.h"

namespace mlstm {

template <typename T> struct io4;
template <> struct io4<float> {
  static __device__ __forceinline__ float4 load(const float* p) { return *reinterpret_cast<const float4*>(p); }
};
template <> struct io4<__nv_bfloat16> {
  static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
};

__device__ __forceinline__ float4 ld_stream(const float* p) {
  float4 r;
  asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// DK: key width of one block (power of two, 4..512).  U: row-steps of a warp in flight.
template <int DK, int U, typename T>
__global__ void __launch_bounds__(256) step_kernel(StepArgs a, int CS, int rows_per_cta) {
  // cluster of CPH = nb * CS CTAs per head; rank -> (block, row part)
  constexpr int VPR = DK / 4;                 // float4 per row
  constexpr int LPR = VPR < 32 ? VPR : 32;    // lanes per row
  constexpr int RPW = 32 / LPR;               // rows per warp-step
  constexpr int F4 = VPR / LPR;               // float4 per lane per row

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int CPH = a.nb * CS;
  const int bh = blockIdx.x / CPH;
  const int blk = (blockIdx.x % CPH) / CS;
  const int rank = blockIdx.x % CS;
  const int slice = bh * a.nb + blk;
  const int head = bh % a.NH;
  const int cg = lane % LPR, ro = lane / LPR;
  const int dv = a.dv;
  const bool ret = a.retention != 0;

  const T* qh = static_cast<const T*>(a.q) + (size_t)bh * a.DHQK + (size_t)blk * DK;
  const T* kh = static_cast<const T*>(a.k) + (size_t)bh * a.DHQK + (size_t)blk * DK;
  const T* vh = static_cast<const T*>(a.v) + (size_t)bh * a.DHV + (size_t)blk * dv;
  const T* oh = a.og ? static_cast<const T*>(a.og) + (size_t)bh * a.DHV + (size_t)blk * dv : nullptr;
  T* hh = static_cast<T*>(a.h) + (size_t)bh * a.DHV + (size_t)blk * dv;
  float* Ch = a.C + (size_t)slice * dv * DK;

  float fp, ip, m_new = 0.f;
  if (ret) {
    fp = 1.f - exp2f(-5.f - (float)head);
    ip = 1.f;
  } else {
    const float lf = log_sigmoid(a.fg[bh]);
    const float li = a.ig[bh];
    const float mp = a.m[bh];
    m_new = fmaxf(lf + mp, li);
    fp = expf(lf + mp - m_new);
    ip = expf(li - m_new);
  }

  float4 qr[F4], kr[F4];
#pragma unroll
  for (int i = 0; i < F4; ++i) {
    const int col = (cg + LPR * i) * 4;
    qr[i] = io4<T>::load(qh + col);
    kr[i] = io4<T>::load(kh + col);
  }

  float den = 1.f;
  float4 nn[F4];
  if (!ret) {
    const float* nh = a.n + (size_t)slice * DK;
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < F4; ++i) {
      const int col = (cg + LPR * i) * 4;
      const float4 n4 = *reinterpret_cast<const float4*>(nh + col);
      nn[i] = make_float4(fp * n4.x + ip * kr[i].x, fp * n4.y + ip * kr[i].y, fp * n4.z + ip * kr[i].z,
                          fp * n4.w + ip * kr[i].w);
      part += dot4(nn[i], qr[i]);
    }
#pragma unroll
    for (int o = LPR / 2; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    den = fmaxf(fabsf(part), expf(-m_new));
  }
  if (CPH > 1) cluster_arrive();  // this CTA has read n and m

  const int r_begin = rank * rows_per_cta;
  const int r_end = min(dv, r_begin + rows_per_cta);
  const int step_rows = nwarps * RPW;
  for (int base = r_begin + warp * RPW; base < r_end; base += step_rows * U) {
    float4 c[U][F4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * step_rows + ro;
#pragma unroll
      for (int i = 0; i < F4; ++i)
        c[u][i] = row < r_end ? ld_stream(Ch + (size_t)row * DK + (cg + LPR * i) * 4) : make_float4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * step_rows + ro;
      const bool ok = row < r_end;
      const float vr = ok ? io<T>::load(vh, row) * ip : 0.f;
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < F4; ++i) {
        float4 cn;
        cn.x = fp * c[u][i].x + vr * kr[i].x;
        cn.y = fp * c[u][i].y + vr * kr[i].y;
        cn.z = fp * c[u][i].z + vr * kr[i].z;
        cn.w = fp * c[u][i].w + vr * kr[i].w;
        dot += dot4(cn, qr[i]);
        if (ok) st_stream(Ch + (size_t)row * DK + (cg + LPR * i) * 4, cn);
      }
#pragma unroll
      for (int o = LPR / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (ok && cg == 0) {
        float hv = dot;
        if (!ret) {
          hv = hv / den;
          if (oh) hv *= io<T>::load(oh, row);
        }
        io<T>::store(hh, row, hv);
      }
    }
  }

  if (CPH > 1)
    cluster_wait();  // every CTA of the head's cluster has read n and m
  else
    __syncthreads();  // every warp of the only CTA has read n and m
  if (!ret && rank == 0) {
    if (warp == 0 && ro == 0) {
      float* nh = a.n + (size_t)slice * DK;
#pragma unroll
      for (int i = 0; i < F4; ++i) *reinterpret_cast<float4*>(nh + (cg + LPR * i) * 4) = nn[i];
    }
    if (threadIdx.x == 0 && blk == 0) a.m[bh] = m_new;
  }
}

bool step_supported_dk(int dk) {
  return dk == 4 || dk == 8 || dk == 16 || dk == 32 || dk == 64 || dk == 128 || dk == 256 || dk == 512;
}

template <int DK, typename T>
static cudaError_t launch_dk(const StepArgs& a, cudaStream_t stream) {
  constexpr int U = DK >= 256 ? 4 : 8;
  const int heads = a.B * a.NH;
  // CTAs per block: at least 128 KiB of C each (fewer, longer CTAs stream C faster than
  // many short ones: 98 % against 92 % of the copy bandwidth at 256 x 512); nb * CS <= 8
  // (portable cluster size)
  long long bytes = (long long)a.dv * DK * 4;
  int CS = 1;
  while (a.nb * CS * 2 <= 8 && bytes / (CS * 2) >= 128 * 1024 && (a.dv + CS * 2 - 1) / (CS * 2) >= 8) CS *= 2;
  const int CPH = a.nb * CS;
  const int rows_per_cta = (a.dv + CS - 1) / CS;
  constexpr int RPW = 32 / ((DK / 4) < 32 ? (DK / 4) : 32);
  int warps = (rows_per_cta + RPW - 1) / RPW;
  warps = warps < 1 ? 1 : (warps > 8 ? 8 : warps);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(CPH * heads));
  cfg.blockDim = dim3(32 * warps);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CPH;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, step_kernel<DK, U, T>, a, CS, rows_per_cta);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_t(const StepArgs& a, cudaStream_t stream) {
  switch (a.dk) {
    case 4: return launch_dk<4, T>(a, stream);
    case 8: return launch_dk<8, T>(a, stream);
    case 16: return launch_dk<16, T>(a, stream);
    case 32: return launch_dk<32, T>(a, stream);
    case 64: return launch_dk<64, T>(a, stream);
    case 128: return launch_dk<128, T>(a, stream);
    case 256: return launch_dk<256, T>(a, stream);
    case 512: return launch_dk<512, T>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_step(const StepArgs& a, cudaStream_t stream) {
  if (a.B * a.NH == 0) return cudaSuccess;
  if (a.nb > 8) return cudaErrorInvalidValue;
  return a.dtype == 0 ? launch_t<float>(a, stream) : launch_t<__nv_bfloat16>(a, stream);
}

}  // namespace mlstm
