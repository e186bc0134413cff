// Gated DeltaNet-2, chunk mode (burn-gdn2 Gdn2Mode::Chunk) on the tensor cores: bf16 inputs,
// key width K = 128, value width V = 64 or 128, chunks of L = 64 tokens.
//
// The chunk form of gdn2.cu, with everything that does not depend on the carried state moved
// out of the sequential part.  Per chunk (G = cumulative log decay inside the chunk, U = w o v,
// bk = b o k, LA / LE / QA / QE and (I + LE)^{-1} as in gdn2.cu):
//     R = (I + LE)^{-1} (Kd S + LA U) = Wk S + Ur      Wk = (I + LE)^{-1} Kd,  Ur = (I + LE)^{-1} LA U
//     o = Qd S + QA U - QE R          = Qw S + Ou      Qw = Qd - QE Wk,        Ou = QA U - QE Ur
//     S <- e^{G_L} o S + Kt^T U + nBt^T R              Kt = k e^{G_L-G},       nBt = -bk e^{G_L-G}
// (Kd = k e^{G}, Qd = q e^{G}).  gdn2_tc_prep_kernel builds Wk, Qw, Ur, Ou, Kt, nBt, U and
// e^{G_L} for every chunk at once (one CTA per chunk, warp-level bf16 MMAs) into a workspace
// slot laid out as the scan's shared-memory stage; gdn2_tc_scan_kernel walks a head's chunks
// in order with the state in tensor memory and three tcgen05 products per chunk: R and o from
// a bf16 snapshot of S (A operand in tensor memory), then the update of S.
//
// The L x L matrices: for blocks of 16 tokens, an off-diagonal block (rows in block a, columns
// in block b < a) is (X o e^{G - G_r}) (Y o e^{G_r - G})^T with r the last row of block b, where
// both exponents are <= 0 (g <= 0); a diagonal block uses its middle row as r, where the two
// factors stay within e^{+-40} unless the block's decay spans more than that, in which case
// that block is summed exactly in fp32 (every exponent G_t - G_s <= 0 per pair).  The inverse
// of the unit lower-triangular I + LE is taken by 16 x 16 blocks in fp32.  Operands of the
// products are bf16, accumulation fp32; a numpy emulation of exactly these roundings on the
// prefill inputs gave 5e-3 relative error against the token-by-token recurrence.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bounds.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mlstm {
namespace {
using namespace sm100;

constexpr int TL = 64;    // tokens per chunk
constexpr int TK = 128;   // key width
constexpr int KP = TK + 8;  // bf16 pitch of [64][K] tiles: 272-byte rows put ldmatrix rows in distinct banks
constexpr int GP = TK + 1;  // fp32 pitch of G
constexpr int LP = TL + 8;  // bf16 pitch of [64][64] tiles
constexpr int EP = TL + 1;  // fp32 pitch of LE and of the inverse
constexpr int PREP_THREADS = 512;

// Workspace slot of one (batch x head, chunk), byte offsets; the scan copies it whole into a
// shared-memory stage of the same layout.  Wk, Qw: K-major B operands (rows t, 64-wide 128-byte
// swizzled column blocks of 8 KiB); Kt an MN-major B operand and U an MN-major A operand in the
// same tile layout; nBt transposed (rows = key channels, the 64 tokens of a row one 128-byte
// swizzled block): a K-major B operand; Ur, Ou plain [t][v] bf16; e^{G_L} [K] fp32.
template <int V>
struct Slot {
  static constexpr int WK = 0, QW = 16384, KT = 32768, NBT = 49152, U = 65536, UR = U + V * 128,
                       OU = UR + V * 128, EGL = OU + V * 128, BYTES = EGL + TK * 4;
};

// `bytes` (a multiple of 16) of global memory from `src` (16-byte aligned) into L2, no completion
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
// byte offset of the 16-byte chunk holding columns [col, col + 8) of row t in a tile of 64-wide
// 128-byte swizzled column blocks of 64 rows
__device__ __forceinline__ uint32_t tile_chunk(int t, int col) {
  return (uint32_t)((col >> 6) * 8192 + t * 128 + ((((col & 63) >> 3) ^ (t & 7)) << 4));
}

// C[64 x N] (+)= A[64 x 64] B[64 x N]: bf16 operands in shared memory (A pitch LP, B row-major
// [k][n] pitch bp), fp32 accumulators, on eight warps: warp w (0..7) takes rows 16 (w % 4) ..
// and columns [(w / 4) N / 2, +N / 2): NT = N / 16 tiles of 8 columns.  neg_a flips the sign of A.
template <int NT>
__device__ __forceinline__ void warp_gemm64(const __nv_bfloat16* A, const __nv_bfloat16* B, int bp, float (&acc)[NT][4],
                                            int warp, int lane, bool neg_a = false) {
  const int m0 = 16 * (warp & 3), n0 = (warp >> 2) * NT * 8;
  const uint32_t sgn = neg_a ? 0x80008000u : 0u;
#pragma unroll
  for (int k0 = 0; k0 < TL; k0 += 16) {
    uint32_t a0, a1, a2, a3;
    ldmatrix_x4(smem_u32(A + (m0 + (lane & 15)) * LP + k0 + (lane >> 4) * 8), a0, a1, a2, a3);
    a0 ^= sgn, a1 ^= sgn, a2 ^= sgn, a3 ^= sgn;
#pragma unroll
    for (int j = 0; j < NT; j += 2) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(smem_u32(B + (k0 + (lane & 15)) * bp + n0 + 8 * j + (lane >> 4) * 8), b0, b1, b2, b3);
      mma_m16n8k16_bf16(acc[j], a0, a1, a2, a3, b0, b1);
      mma_m16n8k16_bf16(acc[j + 1], a0, a1, a2, a3, b2, b3);
    }
  }
}
// Rows and first column of the accumulator values of warp_gemm64: acc[j][0..1] are row
// m0 + lane/4, columns n0 + 8 j + 2 (lane % 4) + {0, 1}; acc[j][2..3] the same 8 rows below.
template <int NT, typename F>
__device__ __forceinline__ void warp_gemm64_each(const float (&acc)[NT][4], int warp, int lane, F f) {
  const int m0 = 16 * (warp & 3), n0 = (warp >> 2) * NT * 8;
  const int r = m0 + (lane >> 2), c = n0 + 2 * (lane & 3);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    f(r, c + 8 * j, acc[j][0], acc[j][1]);
    f(r + 8, c + 8 * j, acc[j][2], acc[j][3]);
  }
}

template <int V>
struct PrepSmem {
  static constexpr int VP = V + 8;
  static constexpr int G = 0;                          // fp32 [64][GP]: G (cumulative log decay)
  static constexpr int KB = G + TL * GP * 4;           // bf16 [64][KP]: k; later the inverse in bf16
  static constexpr int QB = KB + TL * KP * 2;          // bf16 [64][KP]: q
  static constexpr int BKB = QB + TL * KP * 2;         // bf16 [64][KP]: b o k; later the inverse (fp32)
  static constexpr int UB = BKB + TL * KP * 2;         // bf16 [64][VP]: U = w o v
  static constexpr int KD = UB + TL * VP * 2;          // bf16 [64][KP]: k e^{G}; later Qw staged
  static constexpr int LE = KD + TL * KP * 2;          // fp32 [64][EP]
  static constexpr int LA = LE + TL * EP * 4;          // bf16 [64][LP] x 3: LA, QA, QE
  static constexpr int QA = LA + TL * LP * 2;
  static constexpr int QE = QA + TL * LP * 2;
  static constexpr int WKB = QE + TL * LP * 2;         // bf16 [64][KP]: Wk
  static constexpr int Y1 = WKB + TL * KP * 2;         // bf16 [64][VP]: LA U; later Ou staged
  static constexpr int URB = Y1 + TL * VP * 2;         // bf16 [64][VP]: Ur
  static constexpr int MB = URB + TL * VP * 2;         // fp32 [3][16][16]: inverse scratch
  static constexpr int BYTES = MB + 3 * 256 * 4;
  static_assert(TL * EP * 4 <= TL * KP * 2, "the inverse fits the b o k tile");
  static_assert(TL * LP * 2 <= TL * KP * 2, "the bf16 inverse fits the k tile");
};

// One CTA per (chunk, batch x head): the chunk's slot (see Slot).
template <int V>
__global__ void __launch_bounds__(PREP_THREADS, 1) gdn2_tc_prep_kernel(Gdn2Args a, uint8_t* ws, unsigned int* err) {
  using SM = PrepSmem<V>;
  using SL = Slot<V>;
  constexpr int VP = SM::VP;
  extern __shared__ __align__(16) uint8_t smp[];
  float* Gs = reinterpret_cast<float*>(smp + SM::G);
  __nv_bfloat16* kb = reinterpret_cast<__nv_bfloat16*>(smp + SM::KB);
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(smp + SM::QB);
  __nv_bfloat16* bkb = reinterpret_cast<__nv_bfloat16*>(smp + SM::BKB);
  __nv_bfloat16* Ub = reinterpret_cast<__nv_bfloat16*>(smp + SM::UB);
  __nv_bfloat16* Kd = reinterpret_cast<__nv_bfloat16*>(smp + SM::KD);
  float* LEs = reinterpret_cast<float*>(smp + SM::LE);
  __nv_bfloat16* LAb = reinterpret_cast<__nv_bfloat16*>(smp + SM::LA);
  __nv_bfloat16* QAb = reinterpret_cast<__nv_bfloat16*>(smp + SM::QA);
  __nv_bfloat16* QEb = reinterpret_cast<__nv_bfloat16*>(smp + SM::QE);
  __nv_bfloat16* Wkb = reinterpret_cast<__nv_bfloat16*>(smp + SM::WKB);
  __nv_bfloat16* Y1b = reinterpret_cast<__nv_bfloat16*>(smp + SM::Y1);
  __nv_bfloat16* Urb = reinterpret_cast<__nv_bfloat16*>(smp + SM::URB);
  float* Mb = reinterpret_cast<float*>(smp + SM::MB);
  float* TI = reinterpret_cast<float*>(smp + SM::BKB);                  // after the L x L matrices
  __nv_bfloat16* TIb = reinterpret_cast<__nv_bfloat16*>(smp + SM::KB);  // after the L x L matrices

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int t0 = c * TL, Lc = min(TL, a.T - t0);
  const size_t tok0 = (size_t)bh * a.T + t0;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) + tok0 * TK;
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(a.k) + tok0 * TK;
  const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(a.v) + tok0 * V;
  const float* g = a.g + tok0 * TK;
  const float* b = a.b + tok0 * TK;
  const float* w = a.w + tok0 * V;
  uint8_t* slot = ws + ((size_t)bh * gridDim.x + c) * SL::BYTES;

  // ---- A: inputs of the chunk into shared memory (rows past the sequence: zeros, g = 0).  Every
  // global load of a thread is issued before the first store, so the chunk arrives in about one
  // memory latency.
  for (int e = tid; e < TL * EP; e += PREP_THREADS) LEs[e] = 0.f;
  for (int e = tid; e < 3 * TL * LP / 2; e += PREP_THREADS) reinterpret_cast<uint32_t*>(LAb)[e] = 0u;
  {
    constexpr int NA = TL * TK / 4 / PREP_THREADS, NW = TL * V / 4 / PREP_THREADS;
    float4 gv[NA], bv[NA], wv[NW];
    uint2 kr[NA], qr[NA], vr[NW];
#pragma unroll
    for (int x = 0; x < NA; ++x) {
      const int e = tid + x * PREP_THREADS, t = e / (TK / 4), i = 4 * (e % (TK / 4));
      gv[x] = bv[x] = make_float4(0.f, 0.f, 0.f, 0.f);
      kr[x] = qr[x] = make_uint2(0u, 0u);
      if (t < Lc && in_bounds(err, BS_GDN_INPUT, (long long)(tok0 + t) * TK + i + 3, (long long)a.B * a.H * a.T * TK)) {
        gv[x] = *reinterpret_cast<const float4*>(g + (size_t)t * TK + i);
        bv[x] = *reinterpret_cast<const float4*>(b + (size_t)t * TK + i);
        kr[x] = *reinterpret_cast<const uint2*>(k + (size_t)t * TK + i);
        qr[x] = *reinterpret_cast<const uint2*>(q + (size_t)t * TK + i);
      }
    }
#pragma unroll
    for (int x = 0; x < NW; ++x) {
      const int e = tid + x * PREP_THREADS, t = e / (V / 4), j = 4 * (e % (V / 4));
      wv[x] = make_float4(0.f, 0.f, 0.f, 0.f);
      vr[x] = make_uint2(0u, 0u);
      if (t < Lc && in_bounds(err, BS_GDN_INPUT, (long long)(tok0 + t) * V + j + 3, (long long)a.B * a.H * a.T * V)) {
        wv[x] = *reinterpret_cast<const float4*>(w + (size_t)t * V + j);
        vr[x] = *reinterpret_cast<const uint2*>(v + (size_t)t * V + j);
      }
    }
#pragma unroll
    for (int x = 0; x < NA; ++x) {
      const int e = tid + x * PREP_THREADS, t = e / (TK / 4), i = 4 * (e % (TK / 4));
      float* gr = Gs + t * GP + i;
      gr[0] = gv[x].x, gr[1] = gv[x].y, gr[2] = gv[x].z, gr[3] = gv[x].w;
      *reinterpret_cast<uint2*>(kb + t * KP + i) = kr[x];
      *reinterpret_cast<uint2*>(qb + t * KP + i) = qr[x];
      const float2 k01 = unpack2(kr[x].x), k23 = unpack2(kr[x].y);
      *reinterpret_cast<uint2*>(bkb + t * KP + i) =
          make_uint2(pack2(bv[x].x * k01.x, bv[x].y * k01.y), pack2(bv[x].z * k23.x, bv[x].w * k23.y));
    }
#pragma unroll
    for (int x = 0; x < NW; ++x) {
      const int e = tid + x * PREP_THREADS, t = e / (V / 4), j = 4 * (e % (V / 4));
      const float2 v01 = unpack2(vr[x].x), v23 = unpack2(vr[x].y);
      *reinterpret_cast<uint2*>(Ub + t * VP + j) =
          make_uint2(pack2(wv[x].x * v01.x, wv[x].y * v01.y), pack2(wv[x].z * v23.x, wv[x].w * v23.y));
    }
  }
  __syncthreads();
  // The CTAs run one per SM, in waves: the inputs of the chunk of the CTA one wave later (block
  // index + the SM count) are prefetched into L2 while this chunk is computed, so that CTA's
  // loads above find them there instead of all CTAs of a wave fetching from HBM at once.
  if (warp == 0 && lane < 6 && a.nsm > 0) {
    const long long nid = (long long)blockIdx.y * gridDim.x + blockIdx.x + a.nsm;
    if (nid < (long long)gridDim.x * gridDim.y) {
      const int t2 = (int)(nid % gridDim.x) * TL;
      const size_t tok2 = (size_t)(nid / gridDim.x) * a.T + t2;
      const uint32_t rows = (uint32_t)min(TL, a.T - t2);
      const void* src = lane == 0 ? (const void*)(static_cast<const __nv_bfloat16*>(a.q) + tok2 * TK)
                        : lane == 1 ? (const void*)(static_cast<const __nv_bfloat16*>(a.k) + tok2 * TK)
                        : lane == 2 ? (const void*)(static_cast<const __nv_bfloat16*>(a.v) + tok2 * V)
                        : lane == 3 ? (const void*)(a.g + tok2 * TK)
                        : lane == 4 ? (const void*)(a.b + tok2 * TK)
                                    : (const void*)(a.w + tok2 * V);
      const uint32_t row_bytes = lane < 2 ? TK * 2 : lane == 2 ? V * 2 : lane < 5 ? TK * 4 : V * 4;
      prefetch_l2_bulk(src, rows * row_bytes);
    }
  }
  {  // G: cumulative sums down each key channel, four threads per channel (16 rows each)
    const int i = tid & (TK - 1), part = tid >> 7;
    float run = 0.f;
#pragma unroll
    for (int t = 16 * part; t < 16 * part + 16; ++t) {
      run += Gs[t * GP + i];
      Gs[t * GP + i] = run;
    }
    Mb[part * TK + i] = run;  // the part's total
    __syncthreads();
    float off = 0.f;
    for (int pp = 0; pp < part; ++pp) off += Mb[pp * TK + i];
    if (part > 0)
#pragma unroll
      for (int t = 16 * part; t < 16 * part + 16; ++t) Gs[t * GP + i] += off;
  }
  __syncthreads();

  // ---- B (warps 10-15, while warps 0-9 run C): the decayed rows.  Kd = k e^{G} (shared memory);
  // Kt = k e^{G_L-G}, nBt = -bk e^{G_L-G}, U and e^{G_L} into the slot.  (The fast exponential: a
  // few fp32 ulps, far inside the bf16 rounding of every value it makes.)
  constexpr int CW = 10, BT = PREP_THREADS - 32 * CW;  // warps of C, threads of B
  if (warp >= CW) {
  const int bt = tid - 32 * CW;
  const float* GLr = Gs + (TL - 1) * GP;
  for (int e = bt; e < TL * TK / 8; e += BT) {
    // the lanes of a warp take 32 consecutive rows of one 8-column chunk: G reads and the
    // transposed nBt writes below then fall in distinct banks
    const int t = e & (TL - 1), col = 8 * (e >> 6);
    const uint4 kr = *reinterpret_cast<const uint4*>(kb + t * KP + col);
    const uint4 br = *reinterpret_cast<const uint4*>(bkb + t * KP + col);
    const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w}, bw[4] = {br.x, br.y, br.z, br.w};
    uint32_t kd[4], kt[4], nb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 kk = unpack2(kw[j]), bk = unpack2(bw[j]);
      const float g0 = Gs[t * GP + col + 2 * j], g1 = Gs[t * GP + col + 2 * j + 1];
      const float e0 = __expf(g0), e1 = __expf(g1);
      const float f0 = __expf(GLr[col + 2 * j] - g0), f1 = __expf(GLr[col + 2 * j + 1] - g1);
      kd[j] = pack2(kk.x * e0, kk.y * e1);
      kt[j] = pack2(kk.x * f0, kk.y * f1);
      nb[j] = pack2(-bk.x * f0, -bk.y * f1);
    }
    *reinterpret_cast<uint4*>(Kd + t * KP + col) = make_uint4(kd[0], kd[1], kd[2], kd[3]);
    if (in_bounds(err, BS_GDN_SLOT, SL::KT + tile_chunk(t, col) + 15, SL::NBT))
      *reinterpret_cast<uint4*>(slot + SL::KT + tile_chunk(t, col)) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
    // nBt transposed (rows = key channels, 64 tokens wide: a K-major operand) staged where Wk
    // will be, in the slot's swizzled layout
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = col + j;
      const uint32_t w2 = nb[j >> 1];
      reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(Wkb) + i * 128 + (((t >> 3) ^ (i & 7)) << 4))[t & 7] =
          (uint16_t)((j & 1) ? (w2 >> 16) : (w2 & 0xffffu));
    }
  }
  for (int e = bt; e < TL * V / 8; e += BT) {
    const int t = e / (V / 8), col = 8 * (e % (V / 8));
    if (in_bounds(err, BS_GDN_SLOT, SL::U + tile_chunk(t, col) + 15, SL::UR))
      *reinterpret_cast<uint4*>(slot + SL::U + tile_chunk(t, col)) = *reinterpret_cast<const uint4*>(Ub + t * VP + col);
  }
  for (int i = bt; i < TK; i += BT) reinterpret_cast<float*>(slot + SL::EGL)[i] = __expf(GLr[i]);
  }

  // ---- C: LA, LE (s < t), QA, QE (s <= t) by blocks of 16 x 16: ten blocks on the lower
  // triangle, one warp each.  Fragments of the scaled operands are formed in registers straight
  // from G, k, q and bk.
  for (int u = warp; u < CW; u += PREP_THREADS / 32) {
    int ba, bb;  // row block, column block
    if (u < 4) {
      ba = bb = u;
    } else {
      const int pa[6] = {1, 2, 3, 2, 3, 3}, pb[6] = {0, 0, 0, 1, 1, 2};
      ba = pa[u - 4];
      bb = pb[u - 4];
    }
    const bool diag = ba == bb;
    const int ref = diag ? 16 * ba + 8 : 16 * bb + 15;
    const float* Gr = Gs + ref * GP;
    bool exact = false;
    if (diag) {  // the factors e^{+-(G_t - G_ref)} inside the block stay below e^{40}?
      float sp = 0.f;
      for (int e = lane; e < 16 * TK; e += 32) {
        const int t = 16 * ba + e / TK, i = e % TK;
        sp = fmaxf(sp, fabsf(Gs[t * GP + i] - Gr[i]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sp = fmaxf(sp, __shfl_xor_sync(0xffffffffu, sp, o));
      exact = !(sp <= 40.f);
    }
    const int gq = lane >> 2, t4 = lane & 3;
    if (!exact) {
      float acc[4][2][4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int x = 0; x < 4; ++x) acc[m][j][x] = 0.f;
      const int ta = 16 * ba + gq, tb = ta + 8;
#pragma unroll 4
      for (int kk = 0; kk < TK / 16; ++kk) {
        const int c0 = 16 * kk + 2 * t4;
        const float r0 = Gr[c0], r1 = Gr[c0 + 1], r8 = Gr[c0 + 8], r9 = Gr[c0 + 9];
        // A fragments (rows ta, tb; channels c0, c0+1 and c0+8, c0+9) of k and q scaled by e^{G - G_ref}
        uint32_t ak[4], aq[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // h: 0 (ta, c0), 1 (tb, c0), 2 (ta, c0+8), 3 (tb, c0+8)
          const int t = (h & 1) ? tb : ta, ch = c0 + (h >> 1) * 8;
          const float f0 = __expf(Gs[t * GP + ch] - ((h >> 1) ? r8 : r0));
          const float f1 = __expf(Gs[t * GP + ch + 1] - ((h >> 1) ? r9 : r1));
          const float2 kv = unpack2(*reinterpret_cast<const uint32_t*>(kb + t * KP + ch));
          const float2 qv = unpack2(*reinterpret_cast<const uint32_t*>(qb + t * KP + ch));
          ak[h] = pack2(kv.x * f0, kv.y * f1);
          aq[h] = pack2(qv.x * f0, qv.y * f1);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          // B fragments: column s = 16 bb + 8 j + gq, channels c0, c0+1 (b0) and c0+8, c0+9 (b1)
          // of k and bk scaled by e^{G_ref - G}
          const int s = 16 * bb + 8 * j + gq;
          uint32_t bk_[2], bb_[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ch = c0 + 8 * h;
            const float f0 = __expf((h ? r8 : r0) - Gs[s * GP + ch]);
            const float f1 = __expf((h ? r9 : r1) - Gs[s * GP + ch + 1]);
            const float2 kv = unpack2(*reinterpret_cast<const uint32_t*>(kb + s * KP + ch));
            const float2 bv = unpack2(*reinterpret_cast<const uint32_t*>(bkb + s * KP + ch));
            bk_[h] = pack2(kv.x * f0, kv.y * f1);
            bb_[h] = pack2(bv.x * f0, bv.y * f1);
          }
          mma_m16n8k16_bf16(acc[0][j], ak[0], ak[1], ak[2], ak[3], bk_[0], bk_[1]);  // LA
          mma_m16n8k16_bf16(acc[1][j], ak[0], ak[1], ak[2], ak[3], bb_[0], bb_[1]);  // LE
          mma_m16n8k16_bf16(acc[2][j], aq[0], aq[1], aq[2], aq[3], bk_[0], bk_[1]);  // QA
          mma_m16n8k16_bf16(acc[3][j], aq[0], aq[1], aq[2], aq[3], bb_[0], bb_[1]);  // QE
        }
      }
      // a diagonal block keeps s < t (LA, LE) or s <= t (QA, QE); the rest is left at zero
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int t = (x < 2 ? ta : tb), s = 16 * bb + 8 * j + 2 * t4 + (x & 1);
          const bool strict = !diag || s < t, incl = !diag || s <= t;
          if (strict) {
            LEs[t * EP + s] = acc[1][j][x];
            LAb[t * LP + s] = __float2bfloat16_rn(acc[0][j][x]);
          }
          if (incl) {
            QAb[t * LP + s] = __float2bfloat16_rn(acc[2][j][x]);
            QEb[t * LP + s] = __float2bfloat16_rn(acc[3][j][x]);
          }
        }
    } else {
      // exact per pair: e^{G_t - G_s} <= 1 for s <= t, lanes over the key channels
      for (int tt = 0; tt < 16; ++tt)
        for (int ss = 0; ss <= tt; ++ss) {
          const int t = 16 * ba + tt, s = 16 * ba + ss;
          float la = 0.f, le = 0.f, qa = 0.f, qe = 0.f;
          for (int i = lane; i < TK; i += 32) {
            const float e = __expf(Gs[t * GP + i] - Gs[s * GP + i]);
            const float kt = __bfloat162float(kb[t * KP + i]), qt = __bfloat162float(qb[t * KP + i]);
            const float ks = __bfloat162float(kb[s * KP + i]) * e, bs = __bfloat162float(bkb[s * KP + i]) * e;
            la = fmaf(kt, ks, la);
            le = fmaf(kt, bs, le);
            qa = fmaf(qt, ks, qa);
            qe = fmaf(qt, bs, qe);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            la += __shfl_xor_sync(0xffffffffu, la, o);
            le += __shfl_xor_sync(0xffffffffu, le, o);
            qa += __shfl_xor_sync(0xffffffffu, qa, o);
            qe += __shfl_xor_sync(0xffffffffu, qe, o);
          }
          if (lane == 0) {
            if (ss < tt) {
              LEs[t * EP + s] = le;
              LAb[t * LP + s] = __float2bfloat16_rn(la);
            }
            QAb[t * LP + s] = __float2bfloat16_rn(qa);
            QEb[t * LP + s] = __float2bfloat16_rn(qe);
          }
        }
    }
  }
  __syncthreads();

  // ---- D (warps 0-7): TI = (I + LE)^{-1}, unit lower triangular, by 16 x 16 blocks in fp32:
  // the diagonal blocks by forward substitution (a thread per column), then block rows below
  // them, T_ab = -T_aa sum_{b <= c < a} LE_ac T_cb, one block diagonal at a time.  TI takes the
  // place of the b o k tile, its bf16 copy that of the k tile.  Meanwhile warps 8-15 form
  // Y1 = LA U and move the staged nBt to the slot.
  constexpr int NK = TK / 16, NV = V / 16;
  const int hw = warp & 7;  // warp within its half of the CTA
  if (warp < 8) {
    for (int e = tid; e < TL * EP; e += 256) TI[e] = 0.f;
    named_bar(1, 256);
    if (tid < 64) {
      const int base = 16 * (tid >> 4), j = tid & 15;
      float col[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float s = 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m)
          if (m >= j) s = fmaf(LEs[(base + i) * EP + base + m], col[m], s);
        col[i] = i < j ? 0.f : (i == j ? 1.f : -s);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) TI[(base + i) * EP + base + j] = col[i];
    }
    named_bar(1, 256);
    for (int d = 1; d < 4; ++d) {
      const int nblk = 4 - d;
      for (int e = tid; e < nblk * 256; e += 256) {
        const int be = e >> 8, al = be + d, i = (e >> 4) & 15, j = e & 15;
        float s = 0.f;
        for (int cb = be; cb < al; ++cb)
#pragma unroll
          for (int m = 0; m < 16; ++m)
            s = fmaf(LEs[(16 * al + i) * EP + 16 * cb + m], TI[(16 * cb + m) * EP + 16 * be + j], s);
        Mb[e] = s;
      }
      named_bar(1, 256);
      for (int e = tid; e < nblk * 256; e += 256) {
        const int be = e >> 8, al = be + d, i = (e >> 4) & 15, j = e & 15;
        float s = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) s = fmaf(TI[(16 * al + i) * EP + 16 * al + m], Mb[(be << 8) + m * 16 + j], s);
        TI[(16 * al + i) * EP + 16 * be + j] = -s;
      }
      named_bar(1, 256);
    }
    for (int e = tid; e < TL * TL / 2; e += 256) {
      const int t = e >> 5, s = 2 * (e & 31);
      *reinterpret_cast<uint32_t*>(TIb + t * LP + s) = pack2(TI[t * EP + s], TI[t * EP + s + 1]);
    }
  } else {
    float acc[NV][4] = {};
    warp_gemm64<NV>(LAb, Ub, VP, acc, hw, lane);
    warp_gemm64_each<NV>(acc, hw, lane, [&](int r, int col, float x0, float x1) {
      *reinterpret_cast<uint32_t*>(Y1b + r * VP + col) = pack2(x0, x1);
    });
    for (int e = tid - 256; e < TK * TL * 2 / 16; e += 256)
      reinterpret_cast<uint4*>(slot + SL::NBT)[e] = reinterpret_cast<const uint4*>(Wkb)[e];
  }
  __syncthreads();

  // ---- E: the remaining products (warp-level bf16 MMAs, fp32 accumulation), two at a time on
  // the two halves of the CTA
  if (warp < 8) {  // Wk = TI Kd -> shared memory (bf16)
    float acc[NK][4] = {};
    warp_gemm64<NK>(TIb, Kd, KP, acc, hw, lane);
    warp_gemm64_each<NK>(acc, hw, lane, [&](int r, int col, float x0, float x1) {
      *reinterpret_cast<uint32_t*>(Wkb + r * KP + col) = pack2(x0, x1);
    });
  } else {  // Ur = TI Y1 -> shared memory
    float acc[NV][4] = {};
    warp_gemm64<NV>(TIb, Y1b, VP, acc, hw, lane);
    warp_gemm64_each<NV>(acc, hw, lane, [&](int r, int col, float x0, float x1) {
      *reinterpret_cast<uint32_t*>(Urb + r * VP + col) = pack2(x0, x1);
    });
  }
  __syncthreads();
  if (warp < 8) {  // Qw = q e^{G} - QE Wk -> staged where Kd was
    float acc[NK][4] = {};
    warp_gemm64<NK>(QEb, Wkb, KP, acc, hw, lane);
    __nv_bfloat16* Qst = Kd;
    warp_gemm64_each<NK>(acc, hw, lane, [&](int r, int col, float x0, float x1) {
      const float2 qv = unpack2(*reinterpret_cast<const uint32_t*>(qb + r * KP + col));
      const float q0 = qv.x * __expf(Gs[r * GP + col]), q1 = qv.y * __expf(Gs[r * GP + col + 1]);
      *reinterpret_cast<uint32_t*>(Qst + r * KP + col) = pack2(q0 - x0, q1 - x1);
    });
  } else {  // Ou = QA U - QE Ur -> staged where Y1 was
    float acc[NV][4] = {};
    warp_gemm64<NV>(QAb, Ub, VP, acc, hw, lane);
    warp_gemm64<NV>(QEb, Urb, VP, acc, hw, lane, true);
    warp_gemm64_each<NV>(acc, hw, lane, [&](int r, int col, float x0, float x1) {
      *reinterpret_cast<uint32_t*>(Y1b + r * VP + col) = pack2(x0, x1);
    });
  }
  __syncthreads();
  // Wk, Qw (swizzled tiles), Ur and Ou into the slot
  for (int e = tid; e < TL * TK / 8; e += PREP_THREADS) {
    const int t = e >> 4, col = 8 * (e & 15);
    if (!in_bounds(err, BS_GDN_SLOT, SL::QW + tile_chunk(t, col) + 15, SL::KT)) continue;
    *reinterpret_cast<uint4*>(slot + SL::WK + tile_chunk(t, col)) = *reinterpret_cast<const uint4*>(Wkb + t * KP + col);
    *reinterpret_cast<uint4*>(slot + SL::QW + tile_chunk(t, col)) = *reinterpret_cast<const uint4*>(Kd + t * KP + col);
  }
  for (int e = tid; e < TL * V / 8; e += PREP_THREADS) {
    const int t = e / (V / 8), col = 8 * (e % (V / 8));
    if (!in_bounds(err, BS_GDN_SLOT, SL::OU + (t * V + col) * 2 + 15, SL::EGL)) continue;
    *reinterpret_cast<uint4*>(slot + SL::UR + (t * V + col) * 2) = *reinterpret_cast<const uint4*>(Urb + t * VP + col);
    *reinterpret_cast<uint4*>(slot + SL::OU + (t * V + col) * 2) = *reinterpret_cast<const uint4*>(Y1b + t * VP + col);
  }
}

// ===================================================================== scan
// CTA = one (batch x head); the state S^T [V rows (tensor-memory lanes)][K] fp32 stays in
// tensor memory for the whole sequence.  320 threads:
//   warp 0     producer: the chunk's slot into one of two shared-memory stages (one bulk copy)
//   warp 1     MMA warp: R^T = Sb^T Wk^T and o^T = Sb^T Qw^T (A = the bf16 snapshot in tensor
//              memory), S^T += U^T Kt, then S^T += Rb^T nBt once Rb is in tensor memory
//   warps 2-5  state group: the bf16 snapshot Sb of S and the decay S <- e^{G_L} o S in one
//              pass, then Rb = R + Ur (bf16) for the update
//   warps 6-9  output group: o = o^T + Ou to global memory (bf16), two accumulator buffers
// Waits are bounded: when one runs out the CTA sets bit 0 of the workspace error word, every
// later wait returns at once, and the CTA drains its own copies and MMAs before it frees
// tensor memory.
constexpr int SCAN_THREADS = 320;
constexpr long long SCAN_WAIT = 4000000000LL;  // SM cycles (~2 s)
constexpr uint32_t TM_S = 0, TM_SB = 128, TM_R = 192, TM_RB = 256, TM_O = 288, TM_COLS = 512;

struct ScanBars {
  uint64_t full[2], empty[2], sb_ready, r_full, rb_ready, upd_done, o_full[2], o_empty[2], drain;
};

// shared memory of the scan: stage 0 (rounded up to the 1 KiB swizzle-atom alignment), stage 1,
// the barriers, and the slack of aligning the base to 1 KiB
template <int V>
struct ScanSmem {
  static constexpr int STAGE = (Slot<V>::BYTES + 1023) / 1024 * 1024;
  static constexpr int BYTES = STAGE + Slot<V>::BYTES + (int)sizeof(ScanBars) + 1024;
};

// (a wait that took longer than the limit counts as run out even when the phase completed during
// a hardware suspension: the limit is the caller's bound on the time spent waiting)
__device__ __noinline__ bool scan_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                            long long limit) {
  const long long t0 = clock64();
  const bool ok = !*abort_flag && mbar_wait(bar, parity, limit) && clock64() - t0 <= limit;
  if (!ok) *abort_flag = 1;
  return __all_sync(0xffffffffu, ok);
}

template <int V>
__global__ void __launch_bounds__(SCAN_THREADS, 1) gdn2_tc_scan_kernel(Gdn2Args a, const uint8_t* ws,
                                                                      unsigned int* err, int nch) {
  using SL = Slot<V>;
  constexpr int STAGE = ScanSmem<V>::STAGE;
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  ScanBars& bars = *reinterpret_cast<ScanBars*>(sm + STAGE + SL::BYTES);
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const uint32_t sm_u = smem_u32(sm);
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.full[b], 1);
      mbar_init(&bars.empty[b], 9);  // the update's commit, four state warps, four output warps
      mbar_init(&bars.o_full[b], 1);
      mbar_init(&bars.o_empty[b], 4);
    }
    mbar_init(&bars.sb_ready, 4);
    mbar_init(&bars.r_full, 1);
    mbar_init(&bars.rb_ready, 4);
    mbar_init(&bars.upd_done, 1);
    mbar_init(&bars.drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, TM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;
  const long long wlim = a.wait > 0 ? a.wait : SCAN_WAIT;  // (the drain below keeps the default)
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_test_wait(bar, parity)) || scan_wait_slow(bar, parity, &abort_flag, wlim);
  };
  const uint8_t* slots = ws + (size_t)bh * nch * SL::BYTES;
  int n_issued = 0;

  if (warp == 0) {
    // =============================================================== producer
    for (int c = 0; c < nch; ++c) {
      const int b = c & 1;
      if (!wait(&bars.empty[b], ((c >> 1) & 1) ^ 1)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars.full[b], SL::BYTES);
        if (in_bounds(err, BS_GDN_COPY, c, nch))
          bulk_load(sm + b * STAGE, slots + (size_t)c * SL::BYTES, SL::BYTES, &bars.full[b]);
      }
      n_issued = c + 1;
      __syncwarp();
    }
  } else if (warp == 1) {
    // =============================================================== MMA warp
    constexpr uint32_t id_ro = idesc_bf16(V, 64, 0, 0);   // A in tensor memory, B K-major
    constexpr uint32_t id_u1 = idesc_bf16(V, TK, 1, 1);   // A, B MN-major
    constexpr uint32_t id_u2 = idesc_bf16(V, TK, 0, 0);   // A in tensor memory, B K-major
    for (int c = 0; c < nch; ++c) {
      const int b = c & 1, ob = c & 1;
      const uint32_t st = sm_u + b * STAGE;
      const uint64_t wk = smem_desc_sw128(st + SL::WK, 16, 1024), qw = smem_desc_sw128(st + SL::QW, 16, 1024);
      const uint64_t u_mn = smem_desc_sw128(st + SL::U, 8192, 1024), kt_mn = smem_desc_sw128(st + SL::KT, 8192, 1024);
      const uint64_t nb_k = smem_desc_sw128(st + SL::NBT, 16, 1024);
      if (!wait(&bars.full[b], (c >> 1) & 1) || !wait(&bars.sb_ready, c & 1) ||
          !wait(&bars.o_empty[ob], ((c >> 1) & 1) ^ 1))
        break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < TK; k += 16)
          mma_bf16_ts(tm + TM_R, tm + TM_SB + k / 2, wk + (uint64_t)(((k >> 6) * 8192 + (k & 63) * 2) >> 4), id_ro,
                      k > 0 ? 1u : 0u);
        mma_commit(&bars.r_full);
#pragma unroll
        for (int k = 0; k < TK; k += 16)
          mma_bf16_ts(tm + TM_O + 64 * ob, tm + TM_SB + k / 2, qw + (uint64_t)(((k >> 6) * 8192 + (k & 63) * 2) >> 4),
                      id_ro, k > 0 ? 1u : 0u);
        mma_commit(&bars.o_full[ob]);
#pragma unroll
        for (int ks = 0; ks < TL / 16; ++ks)
          mma_bf16_ss(tm + TM_S, u_mn + (uint64_t)(ks * 128), kt_mn + (uint64_t)(ks * 128), id_u1, 1u);
      }
      __syncwarp();
      if (!wait(&bars.rb_ready, c & 1)) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < TL / 16; ++ks)
          mma_bf16_ts(tm + TM_S, tm + TM_RB + 8 * ks, nb_k + (uint64_t)(ks * 2), id_u2, 1u);
        mma_commit(&bars.upd_done);
        mma_commit(&bars.empty[b]);
      }
      __syncwarp();
    }
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
  } else if (warp < 6) {
    // =============================================================== state group
    const int q4 = warp & 3;
    const uint32_t lo = (uint32_t)(32 * q4) << 16;
    const int row = V == 128 ? 32 * q4 + lane : (lane < 16 ? 16 * q4 + lane : -1);  // value row of this lane
    // S0^T into tensor memory
    for (int i0 = 0; i0 < TK; i0 += 16) {
      float r[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        r[j] = (row >= 0 && a.S0 &&
                in_bounds(err, BS_GDN_STATE, ((long long)bh * TK + i0 + j) * V + row, (long long)a.B * a.H * TK * V))
                   ? a.S0[((size_t)bh * TK + i0 + j) * V + row]
                   : 0.f;
      tmem_st16(tm + lo + TM_S + i0, r);
    }
    tmem_wait_st();
    for (int c = 0; c < nch; ++c) {
      const int b = c & 1;
      const uint8_t* st = sm + b * STAGE;
      if (!wait(&bars.full[b], (c >> 1) & 1) || (c > 0 && !wait(&bars.upd_done, (c - 1) & 1))) break;
      tc_fence_after();
      // snapshot Sb = bf16(S) and decay S <- e^{G_L} o S (per key column), one pass
      const float* egl = reinterpret_cast<const float*>(st + SL::EGL);
#pragma unroll 1
      for (int i0 = 0; i0 < TK; i0 += 32) {
        float r[32], pk[16];
        tmem_ld32(tm + lo + TM_S + i0, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = __uint_as_float(pack2(r[2 * j], r[2 * j + 1]));
        tmem_st16(tm + lo + TM_SB + i0 / 2, pk);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] *= egl[i0 + j];
        tmem_st16(tm + lo + TM_S + i0, *reinterpret_cast<float(*)[16]>(r));
        tmem_st16(tm + lo + TM_S + i0 + 16, *reinterpret_cast<float(*)[16]>(r + 16));
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.sb_ready);
      // Rb = bf16(R + Ur) into tensor memory for the update
      if (!wait(&bars.r_full, c & 1)) break;
      tc_fence_after();
      {
        float r[32], pk[16];
        const __nv_bfloat16* ur = reinterpret_cast<const __nv_bfloat16*>(st + SL::UR);
#pragma unroll 1
        for (int t0 = 0; t0 < TL; t0 += 32) {
          tmem_ld32(tm + lo + TM_R + t0, r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float u0 = row >= 0 ? __bfloat162float(ur[(t0 + 2 * j) * V + row]) : 0.f;
            const float u1 = row >= 0 ? __bfloat162float(ur[(t0 + 2 * j + 1) * V + row]) : 0.f;
            pk[j] = __uint_as_float(pack2(r[2 * j] + u0, r[2 * j + 1] + u1));
          }
          tmem_st16(tm + lo + TM_RB + t0 / 2, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.rb_ready);
        mbar_arrive(&bars.empty[b]);
      }
    }
    // the final state once the last update is done
    if (a.S_out && nch > 0 && wait(&bars.upd_done, (nch - 1) & 1)) {
      tc_fence_after();
      for (int i0 = 0; i0 < TK; i0 += 32) {
        float r[32];
        tmem_ld32(tm + lo + TM_S + i0, r);
        tmem_wait_ld();
        if (row >= 0 && !abort_flag)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (in_bounds(err, BS_GDN_STATE, ((long long)bh * TK + i0 + j) * V + row, (long long)a.B * a.H * TK * V))
              a.S_out[((size_t)bh * TK + i0 + j) * V + row] = r[j];
      }
    }
  } else {
    // =============================================================== output group
    const int q4 = warp & 3;
    const uint32_t lo = (uint32_t)(32 * q4) << 16;
    const int row = V == 128 ? 32 * q4 + lane : (lane < 16 ? 16 * q4 + lane : -1);
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o) + (size_t)bh * a.T * V;
    for (int c = 0; c < nch; ++c) {
      const int b = c & 1, ob = c & 1;
      const int t0 = c * TL, Lc = min(TL, a.T - t0);
      if (!wait(&bars.full[b], (c >> 1) & 1) || !wait(&bars.o_full[ob], (c >> 1) & 1)) break;
      tc_fence_after();
      float r[64];
      tmem_ld32(tm + lo + TM_O + 64 * ob, *reinterpret_cast<float(*)[32]>(r));
      tmem_ld32(tm + lo + TM_O + 64 * ob + 32, *reinterpret_cast<float(*)[32]>(r + 32));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.o_empty[ob]);
      const __nv_bfloat16* ou = reinterpret_cast<const __nv_bfloat16*>(sm + b * STAGE + SL::OU);
      if (row >= 0 && !abort_flag)
#pragma unroll
        for (int t = 0; t < TL; ++t)
          if (t < Lc && in_bounds(err, BS_GDN_OUT, ((long long)bh * a.T + t0 + t) * V + row, (long long)a.B * a.H * a.T * V))
            o[(size_t)(t0 + t) * V + row] = __float2bfloat16_rn(r[t] + __bfloat162float(ou[t * V + row]));
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.empty[b]);
    }
  }

  // drain before tensor memory is freed: every MMA issued has completed and every copy issued
  // has landed (the loops above may have stopped early after an expired wait)
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    bool ok = mbar_wait(&bars.drain, 0, SCAN_WAIT);
    for (int b = 0; b < 2; ++b)
      if (n_issued > b) {
        const int c_last = b + 2 * ((n_issued - 1 - b) / 2);
        ok = mbar_wait(&bars.full[b], (c_last >> 1) & 1, SCAN_WAIT) && ok;
      }
    if (!ok) abort_flag = 1;
    if (abort_flag) atomicOr(err, 1u);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, TM_COLS);
}

template <int V>
cudaError_t launch_tc_v(const Gdn2Args& a, void* ws, cudaStream_t stream) {
  const long long BH = (long long)a.B * a.H;
  const int nch = (a.T + TL - 1) / TL;
  unsigned int* err = static_cast<unsigned int*>(ws);
  uint8_t* slots = static_cast<uint8_t*>(ws) + GDN2_TC_HEADER;
  // the error word and, for the bounds-checked build, its record (bytes 16..39)
  cudaError_t e = cudaMemsetAsync(err, 0, 64, stream);
  if (e != cudaSuccess) return e;
  const int smem_p = PrepSmem<V>::BYTES, smem_s = ScanSmem<V>::BYTES;
  e = cudaFuncSetAttribute(gdn2_tc_prep_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_p);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gdn2_tc_scan_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_s);
  if (e != cudaSuccess) return e;
  Gdn2Args pa = a;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&pa.nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    pa.nsm = 0;  // no prefetch
  gdn2_tc_prep_kernel<V><<<dim3((unsigned)nch, (unsigned)BH), PREP_THREADS, smem_p, stream>>>(pa, slots, err);
  gdn2_tc_scan_kernel<V><<<(unsigned)BH, SCAN_THREADS, smem_s, stream>>>(a, slots, err, nch);
  return cudaGetLastError();
}

}  // namespace

bool gdn2_tc_supported(int chunk, int K, int V, int dtype, int T) {
  return dtype == 1 && chunk == TL && K == TK && (V == 64 || V == 128) && T > 0;
}

size_t gdn2_tc_workspace_bytes(long long BH, int T, int V) {
  const long long nch = (T + TL - 1) / TL;
  const size_t slot = V == 64 ? Slot<64>::BYTES : Slot<128>::BYTES;
  return GDN2_TC_HEADER + (size_t)BH * nch * slot;
}

cudaError_t launch_gdn2_tc(const Gdn2Args& a, void* ws, cudaStream_t stream) {
  if ((long long)a.B * a.H > 65535 || a.T <= 0) return cudaErrorInvalidValue;
  return a.V == 64 ? launch_tc_v<64>(a, ws, stream) : launch_tc_v<128>(a, ws, stream);
}

}  // namespace mlstm
