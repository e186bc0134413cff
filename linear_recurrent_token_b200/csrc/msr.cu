// The steps either side of retention in RetNet's multi-scale retention block
// (Edifice.Attention.RetNet, "Key Innovation": Y = (Q Theta) D (K Theta)^T V; "Multi-Scale
// Retention (MSR)": per-head GroupNorm, then Y = SiLU(X W_G) * GroupNorm(Retention(X))).
//
// theta_rotate_kernel   q, k -> q Theta, k Theta.  Entries (2j, 2j+1) of a head vector form
//                       one complex number, multiplied by e^{i p theta_j} at position p,
//                       theta_j = base^{-2j/D}.  The angles depend on (token, pair) only, so a
//                       thread computes its cos/sin once (in double, so that positions in the
//                       thousands keep fp32-exact angles) and applies them to every head and
//                       to both q and k.  HBM-bound: one read and one write of q and k.
// gn_gate_kernel        y = (h - mean) / sqrt(var + eps) * w + b, times silu(g), one group =
//                       one (batch, head, token) row of DHV values, two passes over values
//                       held in registers; narrow rows take four rows per thread with every
//                       load issued up front.  HBM-bound: read h and g, write y.
//
// Both take tensors laid out [B, NH, S, D] with D contiguous, fp32 or bf16, 16-byte vectors.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace mlstm {
namespace {

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& u, float* x) {
    x[0] = __uint_as_float(u.x);
    x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z);
    x[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 pack(const float* x) {
    return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& u, float* x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static uint4 pack(const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

constexpr int ROT_THREADS = 256;
constexpr int ROT_HEADS = 2;  // heads whose vectors are loaded before any is stored

// grid (ceil(S / tokens per CTA), B); thread = (token, 16-byte vector of the head dimension)
template <typename T>
// (four CTAs per SM: the 512 CTAs of the retention workload run in one wave)
__global__ void __launch_bounds__(ROT_THREADS, 4)
    theta_rotate_kernel(const T* q, const T* k, T* qo, T* ko, int NH, int S, int D, const long long* pos0, float base) {
  using V = Vec<T>;
  constexpr int PP = V::N / 2;  // pairs per vector
  const int cpr = D / V::N, tpc = ROT_THREADS / cpr;
  const int tl = threadIdx.x / cpr, c = threadIdx.x % cpr;
  const int b = blockIdx.y;
  const long long t = (long long)blockIdx.x * tpc + tl;
  if (tl >= tpc || t >= S) return;
  float cs[PP], sn[PP];
  const size_t head_stride = (size_t)S * D;
  const size_t base_off = ((size_t)b * NH * S + t) * D + (size_t)c * V::N;
  for (int h0 = 0; h0 < NH; h0 += ROT_HEADS) {
    // the loads of this round are issued first; the first round's angles are computed while
    // they are in flight
    uint4 xq[ROT_HEADS], xk[ROT_HEADS];
#pragma unroll
    for (int u = 0; u < ROT_HEADS; ++u) {
      if (h0 + u < NH) {
        const size_t off = base_off + (size_t)(h0 + u) * head_stride;
        xq[u] = *reinterpret_cast<const uint4*>(q + off);
        xk[u] = *reinterpret_cast<const uint4*>(k + off);
      }
    }
    if (h0 == 0) {
      // angle p theta_j in double (positions in the millions keep it exact to far below fp32
      // resolution), reduced to [-pi, pi] by the nearest multiple of 2 pi in double, then
      // cos / sin in fp32 on the reduced angle; theta_{j+1} = theta_j base^{-2/D}
      const double pos = (double)((pos0 ? pos0[b] : 0LL) + t);
      const double l2b = log2((double)base);
      double theta = exp2(-(2.0 * (c * PP) / D) * l2b);
      const double ratio = exp2(-(2.0 / D) * l2b);
#pragma unroll
      for (int u = 0; u < PP; ++u) {
        const double x = pos * theta;
        const double turns = rint(x * 0.15915494309189535);  // x / (2 pi)
        sincosf((float)fma(-turns, 6.283185307179586, x), &sn[u], &cs[u]);
        theta *= ratio;
      }
    }
#pragma unroll
    for (int u = 0; u < ROT_HEADS; ++u) {
      if (h0 + u < NH) {
        const size_t off = base_off + (size_t)(h0 + u) * head_stride;
        float a[V::N], r[V::N];
        V::unpack(xq[u], a);
#pragma unroll
        for (int e = 0; e < PP; ++e) {
          r[2 * e] = a[2 * e] * cs[e] - a[2 * e + 1] * sn[e];
          r[2 * e + 1] = a[2 * e] * sn[e] + a[2 * e + 1] * cs[e];
        }
        *reinterpret_cast<uint4*>(qo + off) = V::pack(r);
        V::unpack(xk[u], a);
#pragma unroll
        for (int e = 0; e < PP; ++e) {
          r[2 * e] = a[2 * e] * cs[e] - a[2 * e + 1] * sn[e];
          r[2 * e + 1] = a[2 * e] * sn[e] + a[2 * e + 1] * cs[e];
        }
        *reinterpret_cast<uint4*>(ko + off) = V::pack(r);
      }
    }
  }
}

constexpr int GN_THREADS = 256;

// Sum of v over the R threads of a row (R a power of two; R > 32 spans R/32 whole warps).
template <int R>
__device__ __forceinline__ float row_sum(float v, float* red) {
  if (R <= 32) {
#pragma unroll
    for (int o = R / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    constexpr int WPR = R > 32 ? R / 32 : 1;  // warps per row
    const int warp = threadIdx.x >> 5, first = warp / WPR * WPR;
    __syncthreads();  // red free (an earlier call's readers are done)
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < WPR; ++i) s += red[first + i];
    return s;
  }
}

// CTA = a block of token rows of one (batch, head); a row of DHV = R * NV * Vec::N values is
// spread over R threads with NV 16-byte vectors each, and a thread takes RT rows GN_THREADS / R
// apart.  The thread's channels are the same for all its rows, so their weight and bias are
// loaded once; every h and g load of the thread is issued before the first reduction.
template <typename T, int R, int NV, int RT>
__global__ void __launch_bounds__(GN_THREADS, 3) gn_gate_kernel(const T* h, const T* g, const float* w, const float* bb,
                                                            float eps, T* y, int NH, int S, int nblk) {
  using V = Vec<T>;
  constexpr int RPC = GN_THREADS / R, E = NV * V::N, DHV = R * E;
  __shared__ float red[GN_THREADS / 32];
  const int rl = threadIdx.x / R, c = threadIdx.x % R;
  const int bh = blockIdx.x / nblk, tb = blockIdx.x - bh * nblk;
  const int ch = (bh % NH) * DHV + c * E;  // this thread's first channel
  float wv[E], bv[E];
#pragma unroll
  for (int e = 0; e < E; e += 4) {
    const float4 w4 = w ? *reinterpret_cast<const float4*>(w + ch + e) : make_float4(1.f, 1.f, 1.f, 1.f);
    const float4 b4 = bb ? *reinterpret_cast<const float4*>(bb + ch + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    wv[e] = w4.x, wv[e + 1] = w4.y, wv[e + 2] = w4.z, wv[e + 3] = w4.w;
    bv[e] = b4.x, bv[e + 1] = b4.y, bv[e + 2] = b4.z, bv[e + 3] = b4.w;
  }
  uint4 hraw[RT][NV], graw[RT][NV];
  size_t off[RT];
  bool act[RT];
#pragma unroll
  for (int i = 0; i < RT; ++i) {
    const int t = (tb * RT + i) * RPC + rl;  // token of the row
    act[i] = t < S;
    off[i] = ((size_t)bh * S + t) * DHV + (size_t)c * E;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      hraw[i][v] = graw[i][v] = make_uint4(0, 0, 0, 0);
      if (act[i]) {
        hraw[i][v] = *reinterpret_cast<const uint4*>(h + off[i] + v * V::N);
        if (g) graw[i][v] = *reinterpret_cast<const uint4*>(g + off[i] + v * V::N);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RT; ++i) {
    float x[E];
#pragma unroll
    for (int v = 0; v < NV; ++v) V::unpack(hraw[i][v], x + v * V::N);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) s += x[e];
    const float mean = row_sum<R>(s, red) * (1.f / DHV);
    float d2 = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) d2 = fmaf(x[e] - mean, x[e] - mean, d2);
    const float var = row_sum<R>(d2, red) * (1.f / DHV);
    if (act[i]) {
      const float rstd = rsqrtf(var + eps);
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float gv[V::N];
        V::unpack(graw[i][v], gv);
#pragma unroll
        for (int e = 0; e < V::N; ++e) {
          const int k = v * V::N + e;
          float o = fmaf((x[k] - mean) * rstd, wv[k], bv[k]);
          // silu(g) = g / (1 + e^{-g}); the fast exponential and divide are accurate to a few
          // fp32 ulps, far inside the bf16 rounding of the output (fp32 outputs keep expf)
          if (g) o *= V::N == 8 ? __fdividef(gv[e], 1.f + __expf(-gv[e])) : gv[e] / (1.f + expf(-gv[e]));
          x[k] = o;
        }
        *reinterpret_cast<uint4*>(y + off[i] + v * V::N) = V::pack(x + v * V::N);
      }
    }
  }
}

template <typename T>
cudaError_t launch_gn_t(long long rows, int NH, int S, int DHV, const void* h, const void* g, const float* w,
                        const float* b, float eps, void* y, cudaStream_t stream) {
  const int n = DHV / Vec<T>::N;           // 16-byte vectors per row
  const int nv = n >= 2 ? 2 : 1, R = n / nv;  // two vectors per thread where the row has them
  const int rt = R <= 32 ? 2 : 1;          // rows per thread while a row's reduction stays in a warp
  const long long rpc = (long long)rt * (GN_THREADS / R);
  const long long nblk = ((long long)S + rpc - 1) / rpc, BH = rows / S;
  if (nblk * BH > 0x7fffffffLL) return cudaErrorInvalidValue;
  const unsigned blocks = (unsigned)(nblk * BH);
  const T* hp = static_cast<const T*>(h);
  const T* gp = static_cast<const T*>(g);
  T* yp = static_cast<T*>(y);
#define GN_CASE(RR, NVV)                                                                                  \
  if (R == RR && nv == NVV) {                                                                             \
    gn_gate_kernel<T, RR, NVV, (RR <= 32 ? 2 : 1)><<<blocks, GN_THREADS, 0, stream>>>(hp, gp, w, b, eps, yp, NH, S, \
                                                                                      (int)nblk);         \
    return cudaGetLastError();                                                                            \
  }
  GN_CASE(1, 1)
  GN_CASE(1, 2)
  GN_CASE(2, 2)
  GN_CASE(4, 2)
  GN_CASE(8, 2)
  GN_CASE(16, 2)
  GN_CASE(32, 2)
  GN_CASE(64, 2)
  GN_CASE(128, 2)
#undef GN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

bool theta_rotate_supported(int D, int dtype) {
  const int n = dtype == 0 ? 4 : 8;
  return D > 0 && D % n == 0 && D / n <= ROT_THREADS;
}

bool gn_gate_supported(int DHV, int dtype) {
  const int n = dtype == 0 ? 4 : 8;
  if (DHV <= 0 || DHV % n) return false;
  const int v = DHV / n;  // 16-byte vectors per row: 1 .. 256, a power of two
  return v <= GN_THREADS && (v & (v - 1)) == 0;
}

cudaError_t launch_theta_rotate(int B, int NH, int S, int D, int dtype, const void* q, const void* k, void* qo,
                                void* ko, const long long* pos0, float base, cudaStream_t stream) {
  if (B == 0 || NH == 0 || S == 0) return cudaSuccess;
  if (!theta_rotate_supported(D, dtype)) return cudaErrorInvalidValue;
  const int cpr = D / (dtype == 0 ? 4 : 8), tpc = ROT_THREADS / cpr;
  const long long gx = ((long long)S + tpc - 1) / tpc;
  if (gx > 0x7fffffffLL || B > 65535) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)gx, (unsigned)B);
  if (dtype == 0)
    theta_rotate_kernel<float><<<grid, ROT_THREADS, 0, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<float*>(qo), static_cast<float*>(ko),
        NH, S, D, pos0, base);
  else
    theta_rotate_kernel<__nv_bfloat16><<<grid, ROT_THREADS, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(qo),
        static_cast<__nv_bfloat16*>(ko), NH, S, D, pos0, base);
  return cudaGetLastError();
}

cudaError_t launch_gn_gate(long long rows, int NH, int S, int DHV, int dtype, const void* h, const void* g,
                           const float* w, const float* b, float eps, void* y, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  if (!gn_gate_supported(DHV, dtype)) return cudaErrorInvalidValue;
  return dtype == 0 ? launch_gn_t<float>(rows, NH, S, DHV, h, g, w, b, eps, y, stream)
                    : launch_gn_t<__nv_bfloat16>(rows, NH, S, DHV, h, g, w, b, eps, y, stream);
}

}  // namespace mlstm
