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
//            as fp32, and walk the segment's chunks (Q, K, V double-buffered by TMA):
//              S   = Q K^T                          tcgen05 M=64 N=64 K=DK
//              P   = S o D',  D'[t,s] = exp(b_t - b_s + itilde_s - m_t), s <= t
//              Cb  = bf16(C) written into TMEM; C <- a C   (TMEM round trip)
//              H^T = Cb (e^{b_t+m_c-m_t} Q)^T       tcgen05, A from TMEM, M=DVT N=64
//              H^T += V^T P^T                      tcgen05 M=DVT N=64 K=64 (same accumulator)
//              C   += (V o w)^T K                  tcgen05 M=DVT N=DK K=64
//              h_t = o_t H_t / max(|sum_s P[t,s] + e^{b_t+m_c-m_t} n.q_t|, e^{-m_t})
//            with n <- a n + sum_s w_s k_s kept in fp32 shared memory.  The last segment
//            writes the final (C, n, m).
// Retention (RetNet "Key Innovation"): log f = log gamma_h, itilde = 0, m = 0, no
// normaliser; the same kernels with those gate values.
//
// Every mbarrier wait is bounded (~2 s); on expiry the kernel records a bit in the
// workspace error word, stops issuing work, frees its TMEM and returns.
#include <cuda_bf16.h>

#include <string.h>

#include <utility>

#include "common.cuh"
#include "kernels.h"
#include "bounds.cuh"
#include "sm100.cuh"
#include "tma_host.h"

namespace mlstm {

using namespace sm100;

namespace {

constexpr int L = 64;            // chunk length of the tensor-core path
constexpr int NTA = 192;         // phase A threads per CTA (producer, MMA warp, 4 SIMT warps)
constexpr long long WAIT_DEFAULT = 4000000000LL;  // bound of a wait unless the caller sets one (~2 s)

struct TcParams {
  int S, NH, nb, dk, dv, DHQK, DHV, retention, dtype;
  int G, seg_chunks, n_tiles;
  const float *ig, *fg;
  const float *C0, *n0, *m0;  // initial state (snapshots where needed), may be NULL
  const __nv_bfloat16* og;
  __nv_bfloat16* h;
  float *C_out, *n_out, *m_out;
  float *dC, *dn, *segA, *segB;  // workspace: summaries of segments 0..G-2
  // workspace: prepared gate planes [BH][sp] (sp = G * seg_chunks * L, one row per (b, h)):
  // b_t (inclusive cumulative log f inside the chunk), X_t = itilde_t - b_t and its running
  // maximum inside the chunk; per chunk [BH][ncp] its total log f and max X
  float *gb, *gx, *gxc, *cg, *cxm;
  int sp, ncp;
  unsigned int* err;
  long long wait;  // bound of every mbarrier wait, SM cycles
  // scalar normaliser with a learnable bias (NULL: the vector normaliser n . q): bias [NH];
  // then n0 / n_out hold one value per (batch, head) and dn one value per (slice, segment)
  const float* nbias;
  // reversed sequence (token S-1 first): chunk c of the processing order is the original chunk
  // nck_all-1-c (rows aligned to 64 from the start), its tokens taken from the last row back
  int rev, nck_all;
  // segments: segment 0 has seg0_chunks chunks, the others seg_chunks (the last ends with the
  // sequence); every segment but the last is summarised by phase A, segment 0 in ups units
  // (halves when ups = 2), the others in one: NU units in all, by CTAs of dv / n_tiles_a value
  // rows each
  int seg0_chunks, ups, NU, n_tiles_a;
  int BH, slices;  // batch x heads, slices (BH x num_blocks): extents for the bounds-checked build
};

// Processing-order chunks [s0, s1) of segment g.
__device__ __forceinline__ void seg_range(const TcParams& p, int g, int& s0, int& s1) {
  s0 = g == 0 ? 0 : p.seg0_chunks + (g - 1) * p.seg_chunks;
  s1 = g == p.G - 1 ? p.nck_all : s0 + (g == 0 ? p.seg0_chunks : p.seg_chunks);
  s1 = min(s1, p.nck_all);
  s0 = min(s0, s1);
}
// Processing-order chunks [u0, u1) of summary unit j: units 0 .. ups-1 are the parts of
// segment 0, unit ups - 1 + g is segment g >= 1.
__device__ __forceinline__ void unit_range(const TcParams& p, int j, int& u0, int& u1) {
  int s0, s1;
  if (j < p.ups) {
    seg_range(p, 0, s0, s1);
    const int n = s1 - s0;
    u0 = s0 + j * n / p.ups;
    u1 = s0 + (j + 1) * n / p.ups;
  } else {
    seg_range(p, j - p.ups + 1, u0, u1);
  }
}
// Summary units before segment g.
__device__ __forceinline__ int units_before(const TcParams& p, int g) { return g == 0 ? 0 : p.ups + g - 1; }

// First original row of processing-order chunk c (global chunk index).
__device__ __forceinline__ int chunk_row0(const TcParams& p, int c) {
  return p.rev ? L * (p.nck_all - 1 - c) : L * c;
}
// Shared-memory row of position t (processing order) inside a chunk tile (the tile holds the
// chunk's rows in original order).
__device__ __forceinline__ int tile_row(const TcParams& p, int t) { return p.rev ? L - 1 - t : t; }
// The same with the direction known at compile time (the walk's per-chunk code).
template <bool REV>
__device__ __forceinline__ int chunk_row0_c(const TcParams& p, int c) {
  return REV ? L * (p.nck_all - 1 - c) : L * c;
}
template <bool REV>
__device__ __forceinline__ int tile_row_c(int t) {
  return REV ? L - 1 - t : t;
}

// A 64-column tile of q, k, v or h at (column x of the head row, token row, head bh).  Blocks
// narrower than 64 columns (pad) are addressed as block blk of a {width, nb, S, BH} tensor: the
// load fills the missing columns with zeros, the store writes only the block's columns.
__device__ __forceinline__ void tile_load(void* dst, const CUtensorMap* map, bool pad, int x, int blk, int row, int bh,
                                          uint64_t* bar) {
  if (pad)
    tma_load_4d(dst, map, 0, blk, row, bh, bar);
  else
    tma_load_3d(dst, map, x, row, bh, bar);
}
__device__ __forceinline__ void tile_store(const CUtensorMap* map, const void* src, bool pad, int x, int blk, int row,
                                           int bh) {
  if (pad)
    tma_store_4d(map, src, 0, blk, row, bh);
  else
    tma_store_3d(map, src, x, row, bh);
}

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
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 u;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr));
  return u;
}
__device__ __forceinline__ void st_shared_v4u(uint32_t addr, uint4 u) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w) : "memory");
}
// Scales the 8 bf16 of a 16-byte chunk by w with packed bf16 multiplies: w is rounded to
// bf16 once and each product rounded to bf16 (relative error <= 2^-8 per element, against
// 2^-9 for an fp32 product rounded once), at a quarter of the instructions.
__device__ __forceinline__ uint4 scale_bf16x8(uint4 u, float w) {
  const __nv_bfloat162 w2 = __float2bfloat162_rn(w);
  __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int j = 0; j < 4; ++j) b2[j] = __hmul2(b2[j], w2);
  return u;
}

// Gate values of token t (global index) for head `head`: (log f, itilde).
__device__ __forceinline__ void gate_vals(const TcParams& p, size_t tok, int head, float& lf, float& li) {
  if (p.retention) {
    lf = retention_log_gamma(head);
    li = 0.f;
  } else {
    if (!in_bounds(p.err, BS_GATE_INPUT, (long long)tok, (long long)p.BH * p.S)) {
      lf = 0.f;
      li = -INFINITY;
      return;
    }
    lf = log_sigmoid(p.fg[tok]);
    li = p.ig[tok];
  }
}

// n as the B operand of warp-level m16n8k16 MMAs for n . q_t: n = hi + lo (two bf16 values,
// so the products keep fp32 accuracy) in columns 0 and 1 of B.  Lane 4j + t (j = 0 hi, 1 lo,
// t = (k%8)/2) holds, for each 16-row step kk = k/16, the pairs (16kk+2t, +1) and
// (16kk+2t+8, +9); a lane's DK/4 values are contiguous, lanes DK/4 + 8 apart (16 bytes of
// padding put the eight lanes' loads in different banks).
template <int DK>
__device__ __forceinline__ void store_nfrag(__nv_bfloat16* nf, int k, float v) {
  const int kk = k >> 4, r = k & 15;
  const int i = ((r & 7) >> 1) * (DK / 4 + 8) + kk * 4 + ((r >> 3) << 1) + (r & 1);
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  nf[i] = hi;
  nf[i + 4 * (DK / 4 + 8)] = __float2bfloat16_rn(v - __bfloat162float(hi));
}
// bf16 pair (a, b) split as hi + lo: returns hi, lo in *lo
__device__ __forceinline__ uint32_t split_bf16x2(float a, float b, uint32_t* lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 f = __bfloat1622float2(h);
  *lo = pack_bf16(a - f.x, b - f.y);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Slow path of a warp's barrier wait (the phase was not complete when the warp tested it):
// every lane polls with the bounded wait unless a failure is already recorded; returns the
// warp's verdict and records a failure.  Out of line, so the per-chunk code keeps only the
// test and the vote.
__device__ __noinline__ bool warp_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                            long long limit) {
  const bool ok = !*abort_flag && mbar_wait(bar, parity, limit);
  if (!ok) *abort_flag = 1;
  return __all_sync(0xffffffffu, ok);
}
// The same for up to three barriers (unused ones null): each round tests all of them at once,
// so the warp resumes one shared-memory round trip after the last phase completes.
__device__ __noinline__ bool warp_wait_slow3(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, uint64_t* b2,
                                             uint32_t p2, volatile int* abort_flag, long long limit) {
  bool ok = !*abort_flag;
  const long long t0 = clock64();
  while (ok) {
    const bool x = mbar_test_wait(b0, p0), y = b1 == nullptr || mbar_test_wait(b1, p1),
               z = b2 == nullptr || mbar_test_wait(b2, p2);
    if (x && y && z) break;
    if (clock64() - t0 > limit) ok = false;
  }
  if (!ok) *abort_flag = 1;
  return __all_sync(0xffffffffu, ok);
}

// ---- rarely taken walk steps, kept out of line so that the per-chunk code stays compact
// (it is executed once per chunk by each role and must stay in the instruction cache).
// rows row0 .. row0+rows-1 of a 64 x DK bf16 tile (128-byte swizzled 64-column blocks), row t
// scaled by w[t]; the threads gt = 0..nthreads-1 share the work
template <int DK>
__device__ __noinline__ void scale_rows_bf16(uint32_t base_u, const float* w, int gt, int nthreads, int row0,
                                             int rows) {
  constexpr int NCH = DK / 8;  // 16-byte chunks per row
  for (int i = gt; i < rows * NCH; i += nthreads) {
    const int row = row0 + i / NCH, ch = i % NCH;
    const uint32_t a = base_u + (ch >> 3) * 8192 + row * 128 + ((ch & 7) << 4);
    st_shared_v4u(a, scale_bf16x8(ld_shared_v4(a), w[row]));
  }
}
// the DK fp32 columns of this thread's TMEM lane (address taddr) scaled by f; called by the
// whole warp
template <int DK>
__device__ __noinline__ void scale_tmem_lane(uint32_t taddr, float f) {
  for (int c0 = 0; c0 < DK; c0 += 32) {
    float r[32];
    tmem_ld32(taddr + c0, r);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] *= f;
    tmem_st16(taddr + c0, *reinterpret_cast<float(*)[16]>(r));
    tmem_st16(taddr + c0 + 16, *reinterpret_cast<float(*)[16]>(r + 16));
  }
  tmem_wait_st();
}
// h tile staged in shared memory (64 tokens x DVT values, 128-byte swizzled 64-value blocks)
// multiplied by the output gate og[t][d] (og points at token t0, value column v0; row stride
// ld), tokens t < Lc; the 128 threads of the output group share the work
template <int DVT>
__device__ __noinline__ void apply_ogate(uint32_t hs_u, const __nv_bfloat16* og, size_t ld, int Lc, int gt,
                                         int ncol) {
  constexpr int NCH = DVT / 8;
  for (int i = gt; i < Lc * NCH; i += 128) {
    const int t = i / NCH, d = 8 * (i % NCH);
    if (d >= ncol) continue;  // columns past a narrow block
    const uint32_t a = hs_u + (d >> 6) * 8192 + t * 128 + ((((d & 63) >> 3) ^ (t & 7)) << 4);
    uint4 h = ld_shared_v4(a);
    const uint4 o = *reinterpret_cast<const uint4*>(og + t * ld + d);
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&h);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = __bfloat1622float2(h2[j]), y = __bfloat1622float2(o2[j]);
      h2[j] = __floats2bfloat162_rn(x.x * y.x, x.y * y.y);
    }
    st_shared_v4u(a, h);
  }
}

}  // namespace

// ===================================================================== gate preparation
// One warp per (b, h, chunk): the within-chunk scans both kernels below need, computed once.
// Token t of the chunk (lane t/2): b_t = sum_{s<=t} log f_s, X_t = itilde_t - b_t,
// Xc_t = max_{s<=t} X_s.  Tokens past the end of the sequence carry log f = 0 and
// itilde = -inf (b and Xc keep the last token's values, X = -inf), so consumers need no
// bounds logic; the chunk totals are the values of token 63.
__global__ void __launch_bounds__(256) tc_gate_prep_kernel(TcParams p, int BH) {
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long wid = (long long)blockIdx.x * 8 + warp;
  if (wid >= (long long)BH * p.ncp) return;
  const int bh = (int)(wid / p.ncp), c = (int)(wid % p.ncp);
  if (c >= p.nck_all) return;
  const int t0 = c * L;  // processing order
  const int row0 = chunk_row0(p, c);
  const size_t tok = (size_t)bh * p.S;
  const int ta = 2 * lane, tb = ta + 1;
  // original rows of positions ta, tb (reversed: from the chunk's last row back; rows past the
  // end are the identity step, first in the chunk when reversed)
  const int ra = row0 + tile_row(p, ta), rb = row0 + tile_row(p, tb);
  float lfa = 0.f, lfb = 0.f, lia = -INFINITY, lib = -INFINITY;
  if (ra < p.S) gate_vals(p, tok + ra, bh % p.NH, lfa, lia);
  if (rb < p.S) gate_vals(p, tok + rb, bh % p.NH, lfb, lib);
  float isum = lfa + lfb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, isum, o);
    if (lane >= o) isum += u;
  }
  float esum = __shfl_up_sync(0xffffffffu, isum, 1);
  if (lane == 0) esum = 0.f;
  const float ba = esum + lfa, bb = ba + lfb;
  const float xa = lia - ba, xb = lib - bb;
  float mx = fmaxf(xa, xb);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, mx, o);
    if (lane >= o) mx = fmaxf(mx, u);
  }
  float ex = __shfl_up_sync(0xffffffffu, mx, 1);
  if (lane == 0) ex = -INFINITY;
  const float xca = fmaxf(ex, xa), xcb = fmaxf(xca, xb);
  const size_t r = (size_t)bh * p.sp + t0 + ta;
  if (in_bounds(p.err, BS_GATE_PLANES, (long long)r + 1, (long long)p.BH * p.sp)) {
    *reinterpret_cast<float2*>(p.gb + r) = make_float2(ba, bb);
    *reinterpret_cast<float2*>(p.gx + r) = make_float2(xa, xb);
    *reinterpret_cast<float2*>(p.gxc + r) = make_float2(xca, xcb);
  }
  if (lane == 31 && in_bounds(p.err, BS_GATE_CHUNK, (long long)bh * p.ncp + c, (long long)p.BH * p.ncp)) {
    p.cg[(size_t)bh * p.ncp + c] = bb;
    p.cxm[(size_t)bh * p.ncp + c] = xcb;
  }
}

// ===================================================================== phase A
// CTA = (value rows [DVA r, DVA r + DVA), summary unit j, slice): the zero-start contribution of
// the unit's chunks (a segment or half a segment, see seg_range / unit_range) to those rows of
// the state.  192 threads in three roles, NS TMA stages of (K, V) with per-stage barriers:
//   warp 0     producer: TMA loads of stage c % NS once the MMAs of chunk c - NS are done,
//              then the chunk's weights omega_s (second arrival on the stage's full barrier)
//   warp 1     MMA warp: D[rows, dk] += (V o omega)^T K once the SIMT group has scaled V; with
//              DVA = 256 two M = 128 accumulators fill the tensor memory and share each K tile
//   warps 2-5  SIMT group: V rows scaled in place by omega, dn partials (this CTA's share of
//              the key columns); at the end the TMEM accumulators and dn go to global memory
// The roles only meet at mbarriers, so the SIMT work of later stages overlaps the MMAs.
template <int DK, int DVA>
struct SegCfg {
  static constexpr int NACC = DVA == 256 ? 2 : 1;       // accumulators
  static constexpr int MA = DVA == 256 ? 128 : DVA;     // MMA M
  static constexpr int KB = DK * 128, VB = DVA * 128;   // bytes of one K / V chunk tile
  static constexpr int STAGE = KB + VB;
  static constexpr int NS = STAGE * 4 <= 200 * 1024 ? 4 : 3;  // TMA stages
  static constexpr int BYTES_FIXED = NS * STAGE + (128 * 8 + NS * L) * 4 + 1024;
};

template <int DK, int DVA, bool PAD>
__global__ void __launch_bounds__(NTA, 1)
    tc_segment_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV, TcParams p) {
  using CF = SegCfg<DK, DVA>;
  constexpr int KB = CF::KB, VB = CF::VB, NS = CF::NS, NACC = CF::NACC, MA = CF::MA;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage i: K at sm + i*(KB+VB), V right after it
  float* dnp = reinterpret_cast<float*>(sm + NS * (KB + VB));  // [128 * 8] partial sums of dn
  float* omb = dnp + 128 * 8;                                   // [NS][L] weights of the stage's chunk
  float* coff = omb + NS * L;                                   // [unit chunks]
  __shared__ uint64_t full[NS], scaled[NS], mma_done[NS], all_done, drain;
  __shared__ uint32_t tmem_base;
  __shared__ float red[NTA / 32];
  __shared__ volatile int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, j = blockIdx.y, slice = blockIdx.z;
  const int blk = slice % p.nb, bh = slice / p.nb;
  int u0, u1;
  unit_range(p, j, u0, u1);  // processing-order chunks of this unit (all full: it precedes the last segment)
  const int nck = u1 - u0;
  const int T0 = u0 * L;
  const int v0 = tile * DVA;
  // this CTA accumulates dn over key columns [dn0, min(DK, dn0 + dnw)), dnw a multiple of 8
  const int dnw = ((DK + p.n_tiles_a - 1) / p.n_tiles_a + 7) / 8 * 8;
  const int dn0 = tile * dnw;
  const bool do_dn = !p.retention && !p.nbias && dn0 < DK;

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 2);  // the TMA arrival (with its bytes) and the weights
      mbar_init(&scaled[i], 4);
      mbar_init(&mma_done[i], 1);
    }
    mbar_init(&all_done, 1);
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&mapK);
    prefetch_tensormap(&mapV);
  }
  if (warp == 0) tmem_alloc(&tmem_base, NACC * DK);
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;

  auto issue = [&](int c) {  // one lane
    const int st = c % NS;
    uint8_t* kb = sm + st * (KB + VB);
    const int row0 = chunk_row0(p, u0 + c);
    mbar_arrive_expect_tx(&full[st], KB + VB);
    for (int jj = 0; jj < DK / 64; ++jj)
      if (tma_box_ok(p.err, BS_SEG_TMA, blk * p.dk + 64 * jj, row0, 8, p.DHQK, p.S, L, false) &&
          in_bounds(p.err, BS_SEG_TMA, bh, p.BH))
        tile_load(kb + jj * 8192, &mapK, PAD && p.dk < DK, blk * p.dk + 64 * jj, blk, row0, bh, &full[st]);
    for (int jj = 0; jj < DVA / 64; ++jj)
      if (tma_box_ok(p.err, BS_SEG_TMA, blk * p.dv + v0 + 64 * jj, row0, 8, p.DHV, p.S, L, false))
        tile_load(kb + KB + jj * 8192, &mapV, PAD && p.dv < DVA, blk * p.dv + v0 + 64 * jj, blk, row0, bh, &full[st]);
  };
  // K and V are inputs: the first stages load while the previous kernel finishes
  int n_issued = 0;  // chunks whose loads thread 0 has issued
  if (tid == 0)
    for (int c = 0; c < NS && c < nck; ++c) {
      issue(c);
      n_issued = c + 1;
    }

  grid_dep_wait();  // the gate planes come from the preparation kernel
  grid_dep_launch();  // after the wait: a dependent grid that starts now finds the gate planes complete
  // ---- gates: Gtot = sum of the chunk totals, and for token s of chunk c the log weight
  // Gtot - G_s + itilde_s = Gtot - Gpre_c + X_s (Gpre_c: totals of the earlier chunks of the
  // unit); M = its maximum = max_c (Gtot - Gpre_c + max X of chunk c); omega_s = e^{. - M}
  {
    const size_t crow = (size_t)bh * p.ncp + (size_t)u0;
    float total = 0.f, Mg = -INFINITY;
    // chunk totals in passes of NTA (a unit has at most a few hundred chunks)
    for (int base = 0; base < nck; base += NTA) {
      const int c = base + tid;
      const bool cin = c < nck && in_bounds(p.err, BS_SEG_CHUNK, (long long)(crow + c), (long long)p.BH * p.ncp);
      const float gcv = cin ? p.cg[crow + c] : 0.f;
      const float xmv = cin ? p.cxm[crow + c] : -INFINITY;
      float inc = gcv;
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
      }
      __syncthreads();
      if (lane == 31) red[warp] = inc;
      __syncthreads();
      float wexcl = 0.f, ptotal = 0.f;
      for (int w = 0; w < NTA / 32; ++w) {
        if (w < warp) wexcl += red[w];
        ptotal += red[w];
      }
      // gpre relative to the unit start: earlier passes' total plus this pass's exclusive sum
      const float gpre = total + wexcl + inc - gcv;
      if (c < nck) coff[c] = gpre;  // provisional: Gpre_c; turned into Gtot - Gpre_c - M below
      float lm = c < nck ? xmv - gpre : -INFINITY;  // max_c (X max of chunk c - Gpre_c)
      for (int o = 16; o >= 1; o >>= 1) lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, o));
      __syncthreads();
      if (lane == 0) red[warp] = lm;
      __syncthreads();
      for (int w = 0; w < NTA / 32; ++w) Mg = fmaxf(Mg, red[w]);
      total += ptotal;
    }
    Mg += total;  // M = Gtot + max_c (X max - Gpre_c)
    if (p.retention) Mg = 0.f;
    __syncthreads();
    for (int c = tid; c < nck; c += NTA) coff[c] = total - coff[c] - Mg;
    if (tile == 0 && blk == 0 && tid == 0 &&
        in_bounds(p.err, BS_SEG_SCALARS, (long long)bh * p.NU + j, (long long)p.BH * p.NU)) {
      p.segA[(size_t)bh * p.NU + j] = total;
      p.segB[(size_t)bh * p.NU + j] = Mg;
    }
    __syncthreads();
  }
  // warp-uniform test of a barrier, bounded wait out of line when the phase is not complete
  auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_test_wait(bar, parity)) || warp_wait_slow(bar, parity, &abort_flag, p.wait);
  };

  if (warp == 0) {
    // =============================================================== producer
    // omega_s = e^{coff_c + X_s}: lane -> tokens 2 lane, 2 lane + 1 (X of the next chunk
    // prefetched into registers)
    const float* gxr = p.gx + (size_t)bh * p.sp + T0 + 2 * lane;
    const long long gxr0 = (long long)bh * p.sp + T0 + 2 * lane, gx_ext = (long long)p.BH * p.sp;
    float2 gxn = make_float2(-INFINITY, -INFINITY);
    if (in_bounds(p.err, BS_SEG_CHUNK, gxr0 + 1, gx_ext)) gxn = *reinterpret_cast<const float2*>(gxr);
    float osum = 0.f;  // scalar normaliser: this lane's share of the unit's sum of weights
    for (int c = 0; c < nck; ++c) {
      const int st = c % NS;
      if (c >= NS) {
        // the stage's previous chunk has been read by its MMAs (and by the SIMT group before)
        if (!warp_wait(&mma_done[st], ((c / NS) - 1) & 1)) break;
        if (lane == 0) {
          issue(c);
          n_issued = c + 1;
        }
      }
      const float cf = coff[c];
      const float2 om2 = make_float2(expf(cf + gxn.x), expf(cf + gxn.y));
      if (p.rev)  // positions 2 lane, 2 lane + 1 are tile rows 63 - 2 lane, 62 - 2 lane
        *reinterpret_cast<float2*>(omb + st * L + L - 2 - 2 * lane) = make_float2(om2.y, om2.x);
      else
        *reinterpret_cast<float2*>(omb + st * L + 2 * lane) = om2;
      osum += om2.x + om2.y;
      if (c + 1 < nck && in_bounds(p.err, BS_SEG_CHUNK, gxr0 + (long long)(c + 1) * L + 1, gx_ext))
        gxn = *reinterpret_cast<const float2*>(gxr + (size_t)(c + 1) * L);
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[st]);
    }
    if (p.nbias && !p.retention) {  // dn of the scalar normaliser: sum over the unit of omega_s
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) osum += __shfl_xor_sync(0xffffffffu, osum, o);
      if (lane == 0 && tile == 0 && !abort_flag &&
          in_bounds(p.err, BS_SEG_DN, ((long long)slice * p.NU + j) * p.dk, (long long)p.slices * p.NU * p.dk))
        p.dn[((size_t)slice * p.NU + j) * p.dk] = osum;
    }
  } else if (warp == 1) {
    // =============================================================== MMA warp
    const uint32_t idesc = idesc_bf16(MA, DK, 1, 1);
    for (int c = 0; c < nck; ++c) {
      const int st = c % NS;
      uint8_t* Kst = sm + st * (KB + VB);
      const uint64_t bd = smem_desc_sw128(smem_u32(Kst), 8192, 1024);
      const uint64_t ad0 = smem_desc_sw128(smem_u32(Kst + KB), 8192, 1024);
      if (!warp_wait(&scaled[st], (c / NS) & 1)) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < L / 16; ++ks)
#pragma unroll
          for (int a = 0; a < NACC; ++a)  // accumulator a: value rows 128 a .. (two 64-row blocks of V on)
            mma_bf16_ss(tm + a * DK, ad0 + (uint64_t)(ks * 128) + (uint64_t)((a * 16384) >> 4),
                        bd + (uint64_t)(ks * 128), idesc, (c > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&mma_done[st]);
        if (c == nck - 1) mma_commit(&all_done);
      }
      __syncwarp();
    }
  } else {
    // =============================================================== SIMT group
    const int gt = tid - 64;  // 0..127
    // dn partials: thread -> (column group of 8 inside this CTA's columns, row group)
    const int ncg = dnw / 8 < 128 ? dnw / 8 : 128, nrg = 128 / ncg, rows_per = (L + nrg - 1) / nrg;
    const int cg = gt % ncg, rg = gt / ncg;
    const int dcol = dn0 + 8 * cg;  // first of this thread's 8 columns
    float2 dacc[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) dacc[jj] = make_float2(0.f, 0.f);
    for (int c = 0; c < nck; ++c) {
      const int st = c % NS;
      uint8_t* Kst = sm + st * (KB + VB);
      const float* om = omb + st * L;
      // a failed wait leaves the loop of no warp: it runs on (later waits return at once)
      // and the error flag reports it
      if (!__all_sync(0xffffffffu, mbar_test_wait(&full[st], (c / NS) & 1)))
        warp_wait_slow(&full[st], (c / NS) & 1, &abort_flag, p.wait);
      {
        // V rows scaled in place by omega (loads batched ahead of the stores, in passes of 8)
        constexpr int NV = L * (DVA / 8) / 128;
        constexpr int NB = NV < 8 ? NV : 8;
        const uint32_t v_u = smem_u32(Kst + KB);
#pragma unroll
        for (int k0 = 0; k0 < NV; k0 += NB) {
          uint4 u[NB];
          float wr[NB];
          int offs[NB];
#pragma unroll
          for (int k = 0; k < NB; ++k) {
            const int i = (k0 + k) * 128 + gt;
            const int row = i / (DVA / 8), ch = i % (DVA / 8);
            offs[k] = (ch >> 3) * 8192 + row * 128 + ((ch & 7) << 4);
            u[k] = ld_shared_v4(v_u + offs[k]);
            wr[k] = om[row];
          }
#pragma unroll
          for (int k = 0; k < NB; ++k) st_shared_v4u(v_u + offs[k], scale_bf16x8(u[k], wr[k]));
        }
      }
      if (do_dn && rg < nrg && dcol < DK) {
        const uint8_t* kt = Kst + (dcol >> 6) * 8192;
        const int s1 = min(L, (rg + 1) * rows_per);
#pragma unroll 4
        for (int s = rg * rows_per; s < s1; ++s) {
          const uint4 u = *reinterpret_cast<const uint4*>(kt + sw128_offset(s, dcol & 63));
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
          const float w = om[s];
          const float2 w2 = make_float2(w, w);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) dacc[jj] = __ffma2_rn(__bfloat1622float2(b2[jj]), w2, dacc[jj]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&scaled[st]);
    }
    // ---- epilogue: the accumulators (warp w reads TMEM lane quarter w % 4) and dn
    if (!__all_sync(0xffffffffu, mbar_test_wait(&all_done, 0))) warp_wait_slow(&all_done, 0, &abort_flag, p.wait);
    tc_fence_after();
    const int quarter = warp & 3;
    const int row = acc_row<MA>(quarter, lane);
#pragma unroll 1
    for (int a = 0; a < NACC; ++a) {
      float* dst = row >= 0 ? p.dC + (((size_t)slice * p.NU + j) * p.dv + v0 + a * MA + row) * p.dk : nullptr;
#pragma unroll 1
      for (int c0 = 0; c0 < DK; c0 += 32) {
        float r[32];
        tmem_ld32(tm + ((uint32_t)(32 * quarter) << 16) + a * DK + c0, r);
        tmem_wait_ld();
        // (rows and columns past a narrow block's dv x dk are padding)
        const int ncol = PAD ? min(32, p.dk - c0) : 32;
        if (dst && !abort_flag && (!PAD || v0 + a * MA + row < p.dv) && ncol > 0 &&
            in_bounds(p.err, BS_SEG_DC,
                      (((long long)slice * p.NU + j) * p.dv + v0 + a * MA + row) * p.dk + c0 + ncol - 1,
                      (long long)p.slices * p.NU * p.dv * p.dk))
#pragma unroll
          for (int jj = 0; jj < 32; jj += 4)
            if (jj < ncol)
              *reinterpret_cast<float4*>(dst + c0 + jj) = make_float4(r[jj], r[jj + 1], r[jj + 2], r[jj + 3]);
      }
    }
    if (do_dn) {
      *reinterpret_cast<float4*>(dnp + gt * 8) = make_float4(dacc[0].x, dacc[0].y, dacc[1].x, dacc[1].y);
      *reinterpret_cast<float4*>(dnp + gt * 8 + 4) = make_float4(dacc[2].x, dacc[2].y, dacc[3].x, dacc[3].y);
      named_bar(1, 128);
      for (int col = gt; col < ncg * 8 && dn0 + col < (PAD ? p.dk : DK); col += 128) {
        float x = 0.f;
        for (int r = 0; r < nrg; ++r) x += dnp[(r * ncg + col / 8) * 8 + (col & 7)];
        if (!abort_flag && in_bounds(p.err, BS_SEG_DN, ((long long)slice * p.NU + j) * p.dk + dn0 + col,
                                     (long long)p.slices * p.NU * p.dk))
          p.dn[((size_t)slice * p.NU + j) * p.dk + dn0 + col] = x;
      }
    }
  }
  // Drain before TMEM is freed and the CTA exits: every MMA issued and every TMA load issued has
  // completed (after an expired wait the loops above may have stopped early).  These waits use
  // the default bound whatever the caller's limit: they end as soon as the copies land.
  if (warp == 1) {
    if (elect_one()) mma_commit(&drain);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    bool ok = mbar_wait(&drain, 0, WAIT_DEFAULT);
    for (int st = 0; st < NS; ++st)
      if (n_issued > st) {
        const int c_last = st + NS * ((n_issued - 1 - st) / NS);
        ok = mbar_wait(&full[st], (c_last / NS) & 1, WAIT_DEFAULT) && ok;
      }
    if (!ok) abort_flag = 1;
    if (abort_flag) atomicOr(p.err, 1u);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, NACC * DK);
}

// ===================================================================== phase C
// Warp-specialised walk: 15 warps.
//   warp 0       producer: TMA loads of Q/K/V (two stages) and the per-chunk gate quantities
//                (up to four chunks ahead)
//   warp 1       chain MMAs: the chunk's update (C += (V o u)^T K) and read-out (H = Cb Q^T)
//   warp 2       output MMAs: P V (H += V^T P^T), then S = Q K^T of the next chunk
//   warps 3-6    state group: bf16 snapshot of C into TMEM (the read-out operand), then
//                V o u of the next chunk while the MMAs run
//   warps 7-10   output group: P, denominators, h (TMA store)
//   warps 11-14  n group: n . q_t, Q scaling (guarded chunks only), n update
// MMAs are issued by warps that do nothing else: an issuing warp stalls for about the time
// its MMAs take to execute, which would hold up a SIMT group.  Each issuing warp is
// converged and one elected lane issues, with descriptors computed by the whole warp (an
// MMA issued with per-lane operands from divergent code costs ~100 cycles more); the
// elected lane is the same one every time, so each commit tracks all of the warp's earlier
// MMAs.  The producer has the lowest warp id: a warp scheduler favours its older warps, and
// the groups' long instruction runs would otherwise keep it waiting for issue slots.  A
// group's warps cover the four TMEM lane quarters (warp % 4).  Waits are mbarriers, every
// one bounded; a group decides to abort as one.
//
// Lazily scaled state.  TMEM holds C_st with C_unstabilised = e^{lam} C_st (n likewise),
// lam a scalar every role tracks identically.  With X_s = itilde_s - b_s (b the inclusive
// cumulative log f inside the chunk) and S = Q K^T:
//   h_t (stabilised numerator) = E_t [ C_st q_t + sum_{s<=t} u_s S_ts v_s ],
//   E_t = e^{b_t + lam - m_t},  u_s = e^{X_s - lam},
//   C_st <- C_st + (V o u)^T K,  lam <- lam + g      (g = b of the chunk's last token)
// so C is never rescaled in place: the chunk recurrence is one TMEM snapshot and two MMAs.
// lam is moved up to the stabiliser m_c (one extra TMEM pass over C) when m_c - lam > 20.
// A chunk with max_s X_s - lam > 60 (an input gate far above the running stabiliser) is
// "guarded": it uses the per-element stabilised form instead (C rescaled to units of
// e^{m}, Q scaled by e^{b_t + m_c - m_t}, P = S o e^{b_t - m_t + X_s}, update weights
// e^{g + X_s - m_next}); every fp32 / bf16 value then stays within e^{+-60} of 1.
constexpr int NTW = 480;
constexpr int NGB = 4;                             // gate buffers
constexpr int WG_STATE = 1, WG_OUT = 2, WG_N = 3;  // named barrier ids of the 128-thread groups
constexpr float LAM_RENORM = 20.f;       // renormalise lam when the stabiliser is this far above
constexpr float U_MAX_LOG = 60.f;        // largest log u_s a fast chunk may use

template <int DK, int DVT>
struct WalkSmem {
  static constexpr int QB = DK * 128, KB = DK * 128, VB = DVT * 128, PB = 64 * 128, HB = DVT * 128;
  static constexpr int STAGE = QB + KB + VB;
  static constexpr int OVW = 2 * STAGE, OP = OVW + VB, OH = OP + PB;
  static constexpr int OF = OH + HB;  // floats start here
  // n as a bf16 pair (hi + lo) in warp-MMA fragment order: 8 lanes x (DK/4 + 8 padding)
  static constexpr int NFRAG = 8 * (DK / 4 + 8);
  // n [DK], n fragments [2 buffers][NFRAG bf16], gate buffers [NGB][8][L], row sums / reciprocal
  // denominators [2][L], gate scalars [NGB][8]
  static constexpr int NF = DK + NFRAG + NGB * 8 * L + 2 * L + NGB * 8;
  static constexpr int BYTES = OF + NF * 4 + 1024;  // + alignment slack
};

// Per-chunk quantities (NGB buffers), written by the producer except nq (state group).
//   al, be : log2 row / column factors of P (fast: 0 and log2 u_s; guarded: (b_t - m_t) log2 e
//            and X_s log2 e); be = -inf for tokens past the end
//   u      : weight of v_s k_s in the update (and of k_s in the n update)
//   E, F   : h_t = E_t H_t / max(|E_t rowsum_t + F_t nq_t|, e^{-m_t}),  nq_t = n_st . q_t
//   emt    : e^{-m_t};  sq : Q scale of a guarded chunk
//   scal   : [0] flags (bit 0 guarded, bit 1 rewrite C), [1] scale of the bf16 snapshot,
//            [2] scale of the C rewrite, [3] scale of n before the n update,
//            [4] e^{lam - m} after the chunk (final-state scale)
struct GateBuf {
  float *al, *be, *u, *E, *F, *emt, *sq, *nq;
  float* scal;
};
constexpr int GF_GUARD = 1, GF_STORE_C = 2;

struct WalkBars {
  uint64_t full[2], empty[2], s_full[2], gfull[NGB], gempty[NGB], q_ready[NGB];
  uint64_t cb_ready, vw_full, upd_done, ro_done, h_empty, s_empty, p_full, mm_done;
  uint64_t drain;  // both MMA warps' last commits, before TMEM is freed
  uint64_t comp;   // the summary tiles of the start state (prologue)
};

template <int DK, int DVT, bool SN, bool REV, bool PAD>
__global__ void __launch_bounds__(NTW, 1)
    tc_walk_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapH,
                   const __grid_constant__ CUtensorMap mapS, TcParams p) {
  using SM = WalkSmem<DK, DVT>;
  // TMEM columns: C fp32 [DK], bf16 snapshot of C as MMA operand [DK/2], S [64], H [64]
  constexpr uint32_t TM_C = 0, TM_CB = DK, TM_S = DK + DK / 2, TM_H = TM_S + 64;
  constexpr uint32_t TM_COLS = (TM_H + 64 <= 256) ? 256 : 512;
  constexpr float LOG2E = 1.4426950408889634f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Vw = sm + SM::OVW;
  float* nvec = reinterpret_cast<float*>(sm + SM::OF);
  __nv_bfloat16* nfrag = reinterpret_cast<__nv_bfloat16*>(nvec + DK);  // [2][NFRAG]
  float* gmem = nvec + DK + SM::NFRAG;
  float* rsum = gmem + NGB * 8 * L;
  float* rden = rsum + L;
  float* gscal = rden + L;  // [NGB][8]
  auto gbuf = [&](int gi) {
    float* base = gmem + gi * 8 * L;
    return GateBuf{base,         base + L,     base + 2 * L, base + 3 * L, base + 4 * L,
                   base + 5 * L, base + 6 * L, base + 7 * L, gscal + 8 * gi};
  };
  __shared__ WalkBars bars;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ volatile int group_flag[2];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // segment slowest in the grid: the CTAs of segment 0, which need no summary, are dispatched first
  const int tile = blockIdx.x, slice = blockIdx.y, g = blockIdx.z;
  const int blk = slice % p.nb, bh = slice / p.nb;
  const int v0 = tile * DVT;
  int s0, s1;
  seg_range(p, g, s0, s1);  // this segment's processing-order chunks
  const int T0 = s0 * L;
  const int nck = s1 - s0;
  const bool ret = p.retention != 0;
  const bool last_seg = g == p.G - 1;
  const uint32_t sm_u = smem_u32(sm);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.full[i], 1);
      mbar_init(&bars.empty[i], 3);
      mbar_init(&bars.s_full[i], 1);
    }
    for (int i = 0; i < NGB; ++i) {
      mbar_init(&bars.gfull[i], 1);
      mbar_init(&bars.gempty[i], 6);  // four state warps, the n and output groups
      mbar_init(&bars.q_ready[i], 4);
    }
    mbar_init(&bars.cb_ready, 8);  // the state and n groups' warps
    mbar_init(&bars.vw_full, 4);
    mbar_init(&bars.upd_done, 1);
    mbar_init(&bars.ro_done, 1);
    mbar_init(&bars.h_empty, 4);
    mbar_init(&bars.s_empty, 4);
    mbar_init(&bars.p_full, 4);
    mbar_init(&bars.mm_done, 1);
    mbar_init(&bars.drain, 2);
    mbar_init(&bars.comp, 1);
    abort_flag = 0;
    group_flag[0] = group_flag[1] = 0;
    fence_mbar_init();
    prefetch_tensormap(&mapQ);
    prefetch_tensormap(&mapK);
    prefetch_tensormap(&mapV);
    prefetch_tensormap(&mapH);
    if (p.NU > 0) prefetch_tensormap(&mapS);
  }
  if (warp == 0) tmem_alloc(&tmem_base, TM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;

  // Summaries and gate planes come from the kernels before this one.  Segment 0 needs no summary:
  // when segment summaries run (the previous kernel, which signals its dependents only after its
  // own wait for the gate preparation), its CTAs start walking while the summaries are computed.
  if (g > 0 || p.NU == 0) grid_dep_wait();
  // ---- start state of the segment (see the file header); warps 3-10 fill TMEM and n.
  // It is stabilised at m_start, so lam starts at m_start.
  float m_start = ret ? 0.f : (p.m0 && in_bounds(p.err, BS_WALK_START, bh, p.BH) ? p.m0[bh] : 0.f);
  const float m_init = m_start;
  float gsum = 0.f;
  int nun = units_before(p, g);  // summary units before this segment
  if (nun > 0 && !in_bounds(p.err, BS_WALK_START, (long long)bh * p.NU + nun - 1, (long long)p.BH * p.NU)) nun = 0;
  for (int j = 0; j < nun; ++j) {
    const float A = p.segA[(size_t)bh * p.NU + j], Bm = p.segB[(size_t)bh * p.NU + j];
    if (!ret) m_start = fmaxf(A + m_start, Bm);
    gsum += A;
  }
  const float wc0 = expf(gsum + m_init - m_start);
  // Weights of the earlier units' summaries at m_start, once (the gate buffers are free until
  // the producer's first chunk).
  float* pw = gmem;  // [nun]
  if (tid == 0) {
    float after = gsum;
    for (int j = 0; j < nun; ++j) {
      after -= p.segA[(size_t)bh * p.NU + j];
      pw[j] = expf(p.segB[(size_t)bh * p.NU + j] + after - m_start);
    }
  }
  __syncthreads();
  // The start state of this CTA's rows, wc0 C0 + sum_j pw_j dC_j, into TMEM: wc0 C0 (or zeros)
  // first, then each earlier unit's tile rows land in the stage area (free until the producer's
  // first load) through TMA, 32-column boxes with 128-byte swizzle so that the 32 lanes of a warp
  // read 32 rows at one column without bank conflicts, and the warps owning the TMEM lanes add
  // them in.  The loads of a unit are all in flight at once.
  if (warp >= 3 && warp < 11) {
    const int quarter = warp & 3, half = (warp - 3) >> 2;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const int row = acc_row<DVT>(quarter, lane);
    for (int c0 = half * (DK / 2); c0 < (half + 1) * (DK / 2); c0 += 16) {
      float r[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) r[jj] = 0.f;
      if (row >= 0 && p.C0 && (!PAD || (v0 + row < p.dv && c0 < p.dk)) &&  // (narrow blocks: padding stays zero)
          in_bounds(p.err, BS_WALK_START, ((long long)slice * p.dv + v0 + row) * p.dk + c0 + 15,
                    (long long)p.slices * p.dv * p.dk)) {
        const float4* src = reinterpret_cast<const float4*>(p.C0 + ((size_t)slice * p.dv + v0 + row) * p.dk + c0);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float4 x = src[jj];
          r[4 * jj] = wc0 * x.x;
          r[4 * jj + 1] = wc0 * x.y;
          r[4 * jj + 2] = wc0 * x.z;
          r[4 * jj + 3] = wc0 * x.w;
        }
      }
      tmem_st16(tm + lane_off + TM_C + c0, r);
    }
    tmem_wait_st();
  }
  static_assert(DVT * DK * 4 <= 2 * SM::STAGE, "a summary tile fits the stage area");
  for (int j = 0; j < nun; ++j) {
    if (tid == 0) {
      const int ncb = PAD ? min(DK, p.dk + 31) / 32 : DK / 32;  // 32-column boxes holding the block's columns
      mbar_arrive_expect_tx(&bars.comp, (uint32_t)((DVT + 63) / 64 * ncb * 8192));
      const int r0 = ((int)slice * p.NU + j) * p.dv + v0;
      for (int rb = 0; rb < (DVT + 63) / 64; ++rb)
        for (int cb = 0; cb < ncb; ++cb)
          if (tma_box_ok(p.err, BS_WALK_SUM_TMA, 32 * cb, r0 + 64 * rb, 4, p.dk, (long long)p.slices * p.NU * p.dv,
                         64, true))  // held to a store's rule: the tile must start inside the summaries
            tma_load_2d(sm + (rb * (DK / 32) + cb) * 8192, &mapS, 32 * cb, r0 + 64 * rb, &bars.comp);
    }
    if (!mbar_wait(&bars.comp, j & 1, p.wait)) {  // give up on the data, but let the copies land
      abort_flag = 1;
      mbar_wait(&bars.comp, j & 1, WAIT_DEFAULT);
    }
    if (warp >= 3 && warp < 11) {
      const int quarter = warp & 3, half = (warp - 3) >> 2;
      const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
      const int row = acc_row<DVT>(quarter, lane);
      const int rr = row & 63;
      const float w = pw[j];
      tc_fence_after();
      for (int c0 = half * (DK / 2); c0 < (half + 1) * (DK / 2); c0 += 32) {
        float r[32];
        tmem_ld32(tm + lane_off + TM_C + c0, r);
        tmem_wait_ld();
        if (row >= 0 && (!PAD || (v0 + row < p.dv && c0 < p.dk))) {  // (narrow blocks: padding stays zero)
          const uint8_t* box = sm + ((row >> 6) * (DK / 32) + (c0 >> 5)) * 8192 + rr * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 x = *reinterpret_cast<const float4*>(box + ((k ^ (rr & 7)) << 4));
            r[4 * k] += w * x.x;
            r[4 * k + 1] += w * x.y;
            r[4 * k + 2] += w * x.z;
            r[4 * k + 3] += w * x.w;
          }
        }
        tmem_st16(tm + lane_off + TM_C + c0, *reinterpret_cast<float(*)[16]>(r));
        tmem_st16(tm + lane_off + TM_C + c0 + 16, *reinterpret_cast<float(*)[16]>(r + 16));
      }
      tmem_wait_st();
      tc_fence_before();
    }
    fence_proxy_async_smem();  // the reads of the stage area come before the next TMA writes
    __syncthreads();           // the stage area takes the next unit
  }
  // n (vector, or the scalar normaliser's one value per head) the same way, by the other warps
  if (warp >= 11 || warp < 3) {
    const int nt2 = warp >= 11 ? tid - 352 : 128 + tid;  // 0..223
    if (SN) {
      if (nt2 == 0) {
        float x = p.n0 && in_bounds(p.err, BS_WALK_START, bh, p.BH) ? wc0 * p.n0[bh] : 0.f;
        for (int jg = 0; jg < nun; ++jg)
          if (in_bounds(p.err, BS_WALK_START, ((long long)slice * p.NU + jg) * p.dk, (long long)p.slices * p.NU * p.dk))
            x += pw[jg] * p.dn[((size_t)slice * p.NU + jg) * p.dk];
        nvec[0] = x;
      }
    } else if (!ret)
      for (int col = nt2; col < DK; col += 224) {
        if (PAD && col >= p.dk) {  // padding of a narrow block
          nvec[col] = 0.f;
          store_nfrag<DK>(nfrag, col, 0.f);
          continue;
        }
        float x = p.n0 && in_bounds(p.err, BS_WALK_START, (long long)slice * p.dk + col, (long long)p.slices * p.dk)
                      ? wc0 * p.n0[(size_t)slice * p.dk + col]
                      : 0.f;
        for (int jg = 0; jg < nun; ++jg)
          if (in_bounds(p.err, BS_WALK_START, ((long long)slice * p.NU + jg) * p.dk + col,
                        (long long)p.slices * p.NU * p.dk))
            x += pw[jg] * p.dn[((size_t)slice * p.NU + jg) * p.dk + col];
        nvec[col] = x;
        store_nfrag<DK>(nfrag, col, x);
      }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // group-uniform bounded wait: the group's first thread waits, the group follows its verdict
  auto group_wait = [&](uint64_t* bar, uint32_t parity, int gi, bool first) -> bool {
    if (first && (abort_flag || !mbar_wait(bar, parity, p.wait))) {
      group_flag[gi] = 1;
      abort_flag = 1;
    }
    named_bar(gi == 0 ? WG_STATE : WG_OUT, 128);
    return group_flag[gi] == 0;
  };
  // warp-uniform bounded wait.  Every lane tests the barrier and a vote makes the verdict, so
  // a phase that is already complete costs one shared-memory round trip (a lane-0 wait
  // followed by a shuffle costs several, and under the SIMT groups' load each takes hundreds
  // of cycles); otherwise the lanes poll with the bounded wait.
  auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_test_wait(bar, parity)) || warp_wait_slow(bar, parity, &abort_flag, p.wait);
  };
  // wait of one warp of a SIMT group.  Warps of a group wait independently (no verdict is
  // shared), so group code never leaves its loop on a failed wait: it runs on, every later
  // wait returns at once, and the error flag reports the failure.  Named barriers stay only
  // where data crosses warps.
  auto gwait = [&](uint64_t* bar, uint32_t parity) {
    if (!__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) warp_wait_slow(bar, parity, &abort_flag, p.wait);
  };
  // two barriers tested at once (both tests in flight together)
  auto warp_wait2 = [&](uint64_t* b1, uint32_t p1, uint64_t* b2, uint32_t p2) -> bool {
    const bool x = mbar_test_wait(b1, p1), y = mbar_test_wait(b2, p2);
    if (__all_sync(0xffffffffu, x && y)) return true;
    return warp_wait_slow3(b1, p1, b2, p2, nullptr, 0, &abort_flag, p.wait);
  };
  int n_issued = 0;  // chunks whose Q/K/V loads the producer (thread 0) has issued
  const uint32_t id_s = idesc_bf16(64, 64, 0, 0);
  const uint32_t id_ro = idesc_bf16(DVT, 64, 0, 0);
  const uint32_t id_pv = idesc_bf16(DVT, 64, 1, 0);
  const uint32_t id_up = idesc_bf16(DVT, DK, 1, 1);
  // The issue helpers take descriptors computed by the whole (converged) warp, so the
  // elected lane only adds constant offsets.
  // S = Q K^T into the S columns; q_k, k_k: K-major descriptors of the chunk's Q and K
  auto issue_s = [&](uint64_t q_k, uint64_t k_k, int b) {
#pragma unroll 1
    for (int k = 0; k < DK; k += 16) {
      const uint64_t off = (uint64_t)(((k >> 6) * 8192 + (k & 63) * 2) >> 4);
      mma_bf16_ss(tm + TM_S, q_k + off, k_k + off, id_s, k > 0 ? 1u : 0u);
    }
    mma_commit(&bars.s_full[b]);
  };
  // read-out H = Cb Q^T (A = the bf16 snapshot in TMEM); releases stage b with the update
  auto issue_readout = [&](uint64_t q_k, int b) {
#pragma unroll 4
    for (int k = 0; k < DK; k += 16)
      mma_bf16_ts(tm + TM_H, tm + TM_CB + k / 2, q_k + (uint64_t)(((k >> 6) * 8192 + (k & 63) * 2) >> 4), id_ro,
                  k > 0 ? 1u : 0u);
    mma_commit(&bars.ro_done);
    mma_commit(&bars.empty[b]);
  };
  auto desc_k = [&](int c, int part) {  // part 0: Q, 1: K of chunk c's stage, K-major
    return smem_desc_sw128(sm_u + (c & 1) * SM::STAGE + part * SM::QB, 16, 1024);
  };
  // bf16 snapshot of C into TMEM for this warp's lanes, columns [c_lo, c_lo + DK/2) (the state
  // and n groups take one half each).  When lam moves (rare) C is first rescaled in place to
  // the snapshot's units, and after the snapshot to the units of the update.
  auto snapshot_half = [&](const GateBuf& G, int flags, uint32_t lane_off, int c_lo) {
    constexpr int HALF = DK / 2, SB = HALF >= 64 ? 64 : 32;
    const float cbs = G.scal[1], csc = G.scal[2];
    if (flags & GF_STORE_C) scale_tmem_lane<HALF>(tm + lane_off + TM_C + c_lo, cbs);
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_lo + HALF; c0 += SB) {
      float r[SB];
#pragma unroll
      for (int h2 = 0; h2 < SB / 32; ++h2)
        tmem_ld32(tm + lane_off + TM_C + c0 + 32 * h2, *reinterpret_cast<float(*)[32]>(r + 32 * h2));
      tmem_wait_ld();
      float pk[16];
#pragma unroll
      for (int h2 = 0; h2 < SB / 32; ++h2) {
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = __uint_as_float(pack_bf16(r[32 * h2 + 2 * j], r[32 * h2 + 2 * j + 1]));
        tmem_st16(tm + lane_off + TM_CB + c0 / 2 + 16 * h2, pk);
      }
    }
    if ((flags & GF_STORE_C) && csc != cbs) {
      tmem_wait_st();
      scale_tmem_lane<HALF>(tm + lane_off + TM_C + c_lo, csc / cbs);
    }
    tmem_wait_st();
  };

  if (warp == 0) {
    // =============================================================== producer
    // gate values of the next chunk are loaded into registers right after this chunk's
    // hand-off, so their latency never sits in front of an mbarrier arrive
    float pba = 0.f, pbb = 0.f, pxa = 0.f, pxb = 0.f, pca = 0.f, pcb = 0.f, pg = 0.f, pxm = 0.f;
    auto fetch_gates = [&](int c) {
      const size_t r = (size_t)bh * p.sp + T0 + c * L + 2 * lane;
      const size_t cr = (size_t)bh * p.ncp + (size_t)s0 + c;
      if (!in_bounds(p.err, BS_WALK_GATES, (long long)r + 1, (long long)p.BH * p.sp) ||
          !in_bounds(p.err, BS_WALK_GATES, (long long)cr, (long long)p.BH * p.ncp))
        return;
      // (L2 loads: segment 0 may read them before its grid has waited on the previous kernel)
      const float2 b2 = __ldcg(reinterpret_cast<const float2*>(p.gb + r));
      const float2 x2 = __ldcg(reinterpret_cast<const float2*>(p.gx + r));
      const float2 c2 = __ldcg(reinterpret_cast<const float2*>(p.gxc + r));
      pba = b2.x;
      pbb = b2.y;
      pxa = x2.x;
      pxb = x2.y;
      pca = c2.x;
      pcb = c2.y;
      pg = __ldcg(p.cg + cr);
      pxm = __ldcg(p.cxm + cr);
    };
    if (nck > 0) fetch_gates(0);
    float mc = m_start, lam = m_start;
    for (int c = 0; c < nck; ++c) {
      const int b = c & 1, gi = c % NGB;
      // operands of chunk c into stage b once its previous user (chunk c-2) released it
      if (!warp_wait(&bars.empty[b], ((c >> 1) & 1) ^ 1)) break;
      if (lane == 0) {
        uint8_t* base = sm + b * SM::STAGE;
        const int t0 = chunk_row0_c<REV>(p, s0 + c);
        mbar_arrive_expect_tx(&bars.full[b], SM::STAGE);
        for (int j = 0; j < DK / 64; ++j)
          if (tma_box_ok(p.err, BS_WALK_TMA, blk * p.dk + 64 * j, t0, 8, p.DHQK, p.S, L, false) &&
              in_bounds(p.err, BS_WALK_TMA, bh, p.BH)) {
            tile_load(base + j * 8192, &mapQ, PAD && p.dk < DK, blk * p.dk + 64 * j, blk, t0, bh, &bars.full[b]);
            tile_load(base + SM::QB + j * 8192, &mapK, PAD && p.dk < DK, blk * p.dk + 64 * j, blk, t0, bh, &bars.full[b]);
          }
        for (int j = 0; j < DVT / 64; ++j)
          if (tma_box_ok(p.err, BS_WALK_TMA, blk * p.dv + v0 + 64 * j, t0, 8, p.DHV, p.S, L, false))
            tile_load(base + SM::QB + SM::KB + j * 8192, &mapV, PAD && p.dv < DVT, blk * p.dv + v0 + 64 * j, blk, t0, bh,
                      &bars.full[b]);
        n_issued = c + 1;
      }
      // gate quantities of chunk c into buffer gi (lane: tokens 2 lane, 2 lane + 1)
      if (!warp_wait(&bars.gempty[gi], ((c / NGB) & 1) ^ 1)) break;
      GateBuf G = gbuf(gi);
      const int ta = 2 * lane, tb = 2 * lane + 1;
      const float ba = pba, bb = pbb, xa = pxa, xb = pxb, gtot = pg, xmax = pxm;
      // m_t = b_t + max(m_c, Xc_t): the stabiliser recurrence unrolled over the chunk
      const float ma = ret ? 0.f : ba + fmaxf(mc, pca);
      const float mb = ret ? 0.f : bb + fmaxf(mc, pcb);
      const float mn = ret ? 0.f : gtot + fmaxf(mc, xmax);
      const bool renorm = mc - lam > LAM_RENORM;
      const float lam_eff = renorm ? mc : lam;
      const bool guard = !ret && xmax - lam_eff > U_MAX_LOG;
      float nu, csc, lam_next;
      if (guard) {
        nu = expf(lam - mc);
        csc = expf(lam + gtot - mn);
        lam_next = mn;
      } else {
        nu = renorm ? expf(lam - mc) : 1.f;
        csc = nu;
        lam_next = lam_eff + gtot;
      }
      // tokens past the end have X = -inf: weight 0, column factor 0
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int t = tile_row_c<REV>(h2 ? tb : ta);  // the token's row in the chunk tiles
        const float bt = h2 ? bb : ba, mt = h2 ? mb : ma, xt = h2 ? xb : xa;
        if (guard) {
          const float sint = expf(bt + mc - mt);
          G.al[t] = (bt - mt) * LOG2E;
          G.be[t] = xt * LOG2E;
          G.u[t] = expf(gtot + xt - mn);
          G.E[t] = 1.f;
          G.F[t] = sint * nu;
          G.sq[t] = sint;
        } else {
          const float et = expf(bt + lam_eff - mt);
          G.al[t] = 0.f;
          G.be[t] = (xt - lam_eff) * LOG2E;
          G.u[t] = expf(xt - lam_eff);
          G.E[t] = et;
          G.F[t] = et * nu;
          G.sq[t] = 1.f;
        }
        G.emt[t] = expf(-mt);
      }
      if (lane == 0) {
        G.scal[0] = __int_as_float((guard ? GF_GUARD : 0) | ((guard || renorm) ? GF_STORE_C : 0));
        G.scal[1] = nu;
        G.scal[2] = csc;
        G.scal[3] = csc;
        G.scal[4] = expf(lam_next - mn);
      }
      mc = mn;
      lam = lam_next;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.gfull[gi]);
      if (c + 1 < nck) fetch_gates(c + 1);
    }
    if (lane == 0 && !abort_flag && last_seg && !ret && tile == 0 && blk == 0 && p.m_out &&
        in_bounds(p.err, BS_WALK_FINAL, bh, p.BH))
      p.m_out[bh] = mc;
  } else if (warp == 1) {
    // =============================================================== chain MMAs
    const uint64_t vw_mn = smem_desc_sw128(sm_u + SM::OVW, 8192, 1024);  // V o u, MN-major
    for (int c = 0; c < nck; ++c) {
      const int b = c & 1, gi = c % NGB;
      const uint64_t q_k = desc_k(c, 0);
      const uint64_t k_mn = smem_desc_sw128(sm_u + b * SM::STAGE + SM::QB, 8192, 1024);  // K, MN-major
      // update C += (V o u)^T K once the snapshot has read C and V o u is staged; whether the
      // previous h has left TMEM (for the read-out) is tested in the same batch
      bool h_free;
      {
        const bool x = mbar_test_wait(&bars.cb_ready, c & 1), y = mbar_test_wait(&bars.vw_full, c & 1),
                   z = mbar_test_wait(&bars.full[b], (c >> 1) & 1);
        h_free = c == 0 || mbar_test_wait(&bars.h_empty, (c - 1) & 1);
        if (!__all_sync(0xffffffffu, x && y && z) &&
            !warp_wait_slow3(&bars.cb_ready, c & 1, &bars.vw_full, c & 1, &bars.full[b], (c >> 1) & 1, &abort_flag, p.wait))
          break;
      }
      tc_fence_after();
      // the gate buffer is visible here through the state group's cb_ready, which it arrived
      // after reading the buffer; a guarded chunk scales Q before its read-out
      const int flags = __float_as_int(gbuf(gi).scal[0]);
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < L / 16; ++ks)
          mma_bf16_ss(tm + TM_C, vw_mn + (uint64_t)(ks * 128), k_mn + (uint64_t)(ks * 128), id_up, 1u);
        mma_commit(&bars.upd_done);
      }
      __syncwarp();
      const bool guard = (flags & GF_GUARD) != 0;
      if (guard || !__all_sync(0xffffffffu, h_free)) {
        if (!warp_wait_slow3(&bars.h_empty, (c - 1) & 1, guard ? &bars.q_ready[gi] : nullptr, (c / NGB) & 1, nullptr, 0,
                             &abort_flag, p.wait))
          break;
        tc_fence_after();
      }
      if (elect_one()) issue_readout(q_k, b);
      __syncwarp();
    }
  } else if (warp == 2) {
    // =============================================================== output MMAs
    const uint64_t ps_k = smem_desc_sw128(sm_u + SM::OP, 16, 1024);  // P, K-major rows t
    if (nck > 0 && warp_wait(&bars.full[0], 0)) {
      const uint64_t q_k = desc_k(0, 0), k_k = desc_k(0, 1);
      tc_fence_after();
      if (elect_one()) issue_s(q_k, k_k, 0);
      __syncwarp();
      for (int c = 0; c < nck; ++c) {
        const int b = c & 1;
        // P V onto the read-out (same accumulator, issued by the chain warp)
        const uint64_t v_mn = smem_desc_sw128(sm_u + b * SM::STAGE + SM::QB + SM::KB, 8192, 1024);
        if (!warp_wait2(&bars.p_full, c & 1, &bars.ro_done, c & 1)) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < L / 16; ++ks)
            mma_bf16_ss(tm + TM_H, v_mn + (uint64_t)(ks * 128), ps_k + (uint64_t)(ks * 2), id_pv, 1u);
          mma_commit(&bars.mm_done);
          mma_commit(&bars.empty[b]);
        }
        __syncwarp();
        // S of the next chunk after this chunk's read-out and P V in the tensor pipe (the
        // recurrence's MMAs never queue behind it), once this chunk's S has left TMEM
        if (c + 1 < nck) {
          const uint64_t q_k1 = desc_k(c + 1, 0), k_k1 = desc_k(c + 1, 1);
          if (!warp_wait2(&bars.s_empty, c & 1, &bars.full[b ^ 1], ((c + 1) >> 1) & 1)) break;
          tc_fence_after();
          if (elect_one()) issue_s(q_k1, k_k1, b ^ 1);
          __syncwarp();
        }
      }
    }
  } else if (warp < 7) {
    // =============================================================== state group
    const int quarter = warp & 3;
    const int st = tid - 96;  // 0..127
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const bool first = st == 0;
    float fin = 1.f;
    // V o u of chunk c into the update operand buffer (loads batched ahead of the stores)
    auto scale_v = [&](int c) {
      const GateBuf G = gbuf(c % NGB);
      const uint32_t vs_u = sm_u + (c & 1) * SM::STAGE + SM::QB + SM::KB, vw_u2 = smem_u32(Vw);
      constexpr int NV = L * (DVT / 8) / 128;  // 16-byte chunks per thread
      constexpr int NB = NV < 4 ? NV : 4;       // per pass; the pass loop keeps the code small
#pragma unroll 1
      for (int k0 = 0; k0 < NV; k0 += NB) {
        uint4 u[NB];
        float wr[NB];
        int offs[NB];
#pragma unroll
        for (int k = 0; k < NB; ++k) {
          const int i = (k0 + k) * 128 + st;
          const int row = i / (DVT / 8), ch = i % (DVT / 8);
          offs[k] = (ch >> 3) * 8192 + row * 128 + ((ch & 7) << 4);
          u[k] = ld_shared_v4(vs_u + offs[k]);
          wr[k] = G.u[row];
        }
#pragma unroll
        for (int k = 0; k < NB; ++k) st_shared_v4u(vw_u2 + offs[k], scale_bf16x8(u[k], wr[k]));
      }
      fence_proxy_async_smem();
    };
    if (nck > 0) {
      gwait(&bars.gfull[0], 0);
      gwait(&bars.full[0], 0);
      scale_v(0);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.vw_full);  // this warp's share of V o u is stored
    }
    for (int c = 0; c < nck; ++c) {
      const int gi = c % NGB;
      const GateBuf G = gbuf(gi);
      // the gate values, and (the previous read-out has read the snapshot and the previous
      // update has written C)
      if (c > 0) {
        const bool x = mbar_test_wait(&bars.gfull[gi], (c / NGB) & 1), y = mbar_test_wait(&bars.ro_done, (c - 1) & 1);
        if (!__all_sync(0xffffffffu, x && y))
          warp_wait_slow3(&bars.gfull[gi], (c / NGB) & 1, &bars.ro_done, (c - 1) & 1, nullptr, 0, &abort_flag, p.wait);
      } else {
        gwait(&bars.gfull[gi], 0);
      }
      tc_fence_after();
      const int flags = __float_as_int(G.scal[0]);
      fin = G.scal[4];
      snapshot_half(G, flags, lane_off, 0);  // columns [0, DK/2); the n group takes the rest
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.cb_ready);  // this warp's lanes of the snapshot are written
        mbar_arrive(&bars.gempty[gi]);  // and it is done with the chunk's gate buffer
      }
      // V o u of the next chunk once this chunk's update has read the buffer
      if (c + 1 < nck) {
        const int c1 = c + 1, b1 = c1 & 1;
        const bool x = mbar_test_wait(&bars.gfull[c1 % NGB], (c1 / NGB) & 1),
                   y = mbar_test_wait(&bars.full[b1], (c1 >> 1) & 1), z = mbar_test_wait(&bars.upd_done, c & 1);
        if (!__all_sync(0xffffffffu, x && y && z))
          warp_wait_slow3(&bars.gfull[c1 % NGB], (c1 / NGB) & 1, &bars.full[b1], (c1 >> 1) & 1, &bars.upd_done, c & 1,
                          &abort_flag, p.wait);
        scale_v(c1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.vw_full);
      }
    }
    // final state after the last update, back in units of e^{m}.  ro_done is committed after
    // the chunk's update, and this group has waited for each of its phases in turn (a parity
    // wait on a barrier two phases behind would return at once).
    if (nck > 0 && group_wait(&bars.ro_done, (nck - 1) & 1, 0, first) && last_seg && p.C_out) {
      tc_fence_after();
      const int row = acc_row<DVT>(quarter, lane);
      for (int c0 = 0; c0 < DK; c0 += 32) {
        float r[32];
        tmem_ld32(tm + lane_off + TM_C + c0, r);
        tmem_wait_ld();
        const int ncol = PAD ? min(32, p.dk - c0) : 32;  // (narrow blocks: padding is not written)
        if (row >= 0 && (!PAD || v0 + row < p.dv) && ncol > 0 &&
            in_bounds(p.err, BS_WALK_FINAL, ((long long)slice * p.dv + v0 + row) * p.dk + c0 + ncol - 1,
                      (long long)p.slices * p.dv * p.dk)) {
          float* dst = p.C_out + ((size_t)slice * p.dv + v0 + row) * p.dk + c0;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            if (j < ncol)
              *reinterpret_cast<float4*>(dst + j) = make_float4(fin * r[j], fin * r[j + 1], fin * r[j + 2], fin * r[j + 3]);
        }
      }
    }
  } else if (warp < 11) {
    // =============================================================== output group
    const int quarter = warp & 3;
    const int gt = tid - 224;  // 0..127
    const bool first = gt == 0;
    const uint32_t ps_u = sm_u + SM::OP, hs_u = sm_u + SM::OH;
    const bool use_og = p.og != nullptr && !ret;
    const float nbias_h = SN && in_bounds(p.err, BS_WALK_BIAS, bh % p.NH, p.NH) ? p.nbias[bh % p.NH] : 0.f;
    for (int c = 0; c < nck; ++c) {
      const int b = c & 1, gi = c % NGB;
      const GateBuf G = gbuf(gi);
      const int t0 = chunk_row0_c<REV>(p, s0 + c);  // first original row of the chunk tile
      const int Lc = min(L, p.S - t0);                        // rows of the tile inside the sequence
      const size_t tok0 = (size_t)bh * p.S + t0;
      // P = S o e^{al_t + be_s} (bf16, rows t, 128-byte swizzled) and its row sums, once the
      // chunk's gate values are written (the producer loads a stage before it writes them)
      // and P V of the previous chunk is done with the P buffer
      {
        const bool x = c == 0 || mbar_test_wait(&bars.mm_done, (c - 1) & 1),
                   y = mbar_test_wait(&bars.s_full[b], (c >> 1) & 1), z = mbar_test_wait(&bars.gfull[gi], (c / NGB) & 1);
        if (!__all_sync(0xffffffffu, x && y && z))
          warp_wait_slow3(&bars.s_full[b], (c >> 1) & 1, &bars.gfull[gi], (c / NGB) & 1,
                          c > 0 ? &bars.mm_done : nullptr, (c - 1) & 1, &abort_flag, p.wait);
      }
      tc_fence_after();
      {
        // 16x256b load: thread -> rows 16q + lane/4 and +8, column pairs 8j + 2(lane%4)
        const int r_lo = 16 * quarter + (lane >> 2), r_hi = r_lo + 8, cp = 2 * (lane & 3);
        float r[32], f_lo[16], f_hi[16];
        tmem_ld16x256_x8(tm + ((uint32_t)(32 * quarter) << 16) + TM_S, r);
        // element factors: u_s in a fast chunk (column factors only), e^{al_t + be_s} in a
        // guarded one
        if (!(__float_as_int(G.scal[0]) & GF_GUARD)) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float2 u2 = *reinterpret_cast<const float2*>(G.u + 8 * j + cp);
            f_lo[2 * j] = f_hi[2 * j] = u2.x;
            f_lo[2 * j + 1] = f_hi[2 * j + 1] = u2.y;
          }
        } else {
          const float al_lo = G.al[r_lo], al_hi = G.al[r_hi];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float2 be2 = *reinterpret_cast<const float2*>(G.be + 8 * j + cp);
            f_lo[2 * j] = exp2f(al_lo + be2.x);
            f_lo[2 * j + 1] = exp2f(al_lo + be2.y);
            f_hi[2 * j] = exp2f(al_hi + be2.x);
            f_hi[2 * j + 1] = exp2f(al_hi + be2.y);
          }
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_empty);  // this warp's rows of S have left TMEM
        float rs_lo = 0.f, rs_hi = 0.f;
        uint32_t plo[8], phi[8];
        // columns kept (causal): forward s <= t for rows inside the sequence; reversed, the tile rows
        // hold the positions backwards, so s >= t (rows past the end are identity steps there, whose
        // columns carry factor 0 and whose h is not stored)
        const int lim_lo = REV ? r_lo : (r_lo < Lc ? r_lo : -1), lim_hi = REV ? r_hi : (r_hi < Lc ? r_hi : -1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int s0 = 8 * j + cp;
          const float2 pa = __fmul2_rn(make_float2(r[2 * j], r[2 * j + 1]), make_float2(f_lo[2 * j], f_lo[2 * j + 1]));
          const float2 pb =
              __fmul2_rn(make_float2(r[16 + 2 * j], r[16 + 2 * j + 1]), make_float2(f_hi[2 * j], f_hi[2 * j + 1]));
          const bool ka0 = REV ? s0 >= lim_lo : s0 <= lim_lo, ka1 = REV ? s0 + 1 >= lim_lo : s0 + 1 <= lim_lo;
          const bool kb0 = REV ? s0 >= lim_hi : s0 <= lim_hi, kb1 = REV ? s0 + 1 >= lim_hi : s0 + 1 <= lim_hi;
          const float a0 = ka0 ? pa.x : 0.f;
          const float a1 = ka1 ? pa.y : 0.f;
          const float b0 = kb0 ? pb.x : 0.f;
          const float b1 = kb1 ? pb.y : 0.f;
          if (SN) {  // scalar normaliser: sums of the weights themselves (no q . k factor)
            rs_lo += (ka0 ? f_lo[2 * j] : 0.f) + (ka1 ? f_lo[2 * j + 1] : 0.f);
            rs_hi += (kb0 ? f_hi[2 * j] : 0.f) + (kb1 ? f_hi[2 * j + 1] : 0.f);
          } else {
            rs_lo += a0 + a1;
            rs_hi += b0 + b1;
          }
          plo[j] = pack_bf16(a0, a1);
          phi[j] = pack_bf16(b0, b1);
        }
        // matrices (rows lo, cols 8j), (rows hi, 8j), (lo, 8j+8), (hi, 8j+8) per instruction
        const int mrow = 16 * quarter + ((lane >> 3) & 1) * 8 + (lane & 7), mcol = lane >> 4;
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          const int cb = j + mcol;
          stmatrix_x4(ps_u + mrow * 128 + ((cb ^ (mrow & 7)) << 4), plo[j], phi[j], plo[j + 1], phi[j + 1]);
        }
        rs_lo += __shfl_xor_sync(0xffffffffu, rs_lo, 1);
        rs_lo += __shfl_xor_sync(0xffffffffu, rs_lo, 2);
        rs_hi += __shfl_xor_sync(0xffffffffu, rs_hi, 1);
        rs_hi += __shfl_xor_sync(0xffffffffu, rs_hi, 2);
        if ((lane & 3) == 0) {
          rsum[r_lo] = rs_lo;
          rsum[r_hi] = rs_hi;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full);  // this warp's rows of P are stored
      // reciprocal denominators times the output scale E_t (nq_t from the state group, the row
      // sums from all warps of this group)
      gwait(&bars.q_ready[gi], (c / NGB) & 1);
      named_bar(WG_OUT, 128);
      if (gt < L) {
        const int t = gt;
        const float e = G.E[t];
        if (SN)  // max(|n' + bias e^{-m}|, e^{-m}) in stabilised units
          rden[t] = e / fmaxf(fabsf(e * rsum[t] + G.F[t] * G.nq[t] + nbias_h * G.emt[t]), G.emt[t]);
        else
          rden[t] = ret ? e : e / fmaxf(fabsf(e * rsum[t] + G.F[t] * G.nq[t]), G.emt[t]);
      }
      // h_t = H_t rden_t (x o_t): H leaves TMEM first, then 8x8 tiles are stored transposed
      // into the 128-byte swizzled staging tile and TMA-stored
      if (first) bulk_wait_read_all();
      named_bar(WG_OUT, 128);  // rden is written and the previous h tile has left the staging tile
      gwait(&bars.mm_done, c & 1);
      tc_fence_after();
      {
        constexpr int NH = DVT == 128 ? 2 : 1;  // 16-lane halves of this warp's quarter
        float r[32], r2[32];
        tmem_ld16x256_x8(tm + ((uint32_t)(32 * quarter) << 16) + TM_H, r);
        if (NH == 2) tmem_ld16x256_x8(tm + ((uint32_t)(32 * quarter + 16) << 16) + TM_H, r2);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.h_empty);  // this warp's lanes of H have left TMEM
        const int cp = 2 * (lane & 3);
        float s0[8], s1[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 rd = *reinterpret_cast<const float2*>(rden + 8 * j + cp);
          s0[j] = rd.x;
          s1[j] = rd.y;
        }
        // one loop body for both halves (the second half's registers move into r), which
        // keeps this hot code short
#pragma unroll 1
        for (int hf = 0; hf < NH; ++hf) {
          if (hf == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = r2[j];
          }
          // value rows of this half: base + lane/4 (r[2j], r[2j+1]) and base + lane/4 + 8 (r[16+..])
          const int base = DVT == 128 ? 32 * quarter + 16 * hf : 16 * quarter;
          uint32_t plo[8], phi[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float2 sc = make_float2(s0[j], s1[j]);
            const float2 x = __fmul2_rn(make_float2(r[2 * j], r[2 * j + 1]), sc);
            const float2 y = __fmul2_rn(make_float2(r[16 + 2 * j], r[16 + 2 * j + 1]), sc);
            plo[j] = pack_bf16(x.x, x.y);
            phi[j] = pack_bf16(y.x, y.y);
          }
          // transposed: matrices (values lo, tokens 8j), (hi, 8j), (lo, 8j+8), (hi, 8j+8)
          const int d0 = base + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            const int t = 8 * (j + (lane >> 4)) + (lane & 7);
            const uint32_t addr = hs_u + (d0 >> 6) * 8192 + t * 128 + ((((d0 & 63) >> 3) ^ (t & 7)) << 4);
            if (in_bounds(p.err, BS_WALK_H_STAGE, (long long)(addr - hs_u) + 15, (DVT / 64) * 8192))
              stmatrix_x4_trans(addr, plo[j], phi[j], plo[j + 1], phi[j + 1]);
          }
        }
      }
      if (use_og) {  // h <- h o o_t on the staged tile
        named_bar(WG_OUT, 128);
        // (the largest index it reads: its last row's last column)
        const int ncol = PAD ? min(DVT, p.dv - v0) : DVT;  // (narrow blocks: only the block's columns)
        if (in_bounds(p.err, BS_WALK_OGATE, (long long)(tok0 + Lc - 1) * p.DHV + blk * p.dv + v0 + ncol - 1,
                      (long long)p.BH * p.S * p.DHV))
          apply_ogate<DVT>(hs_u, p.og + tok0 * p.DHV + (size_t)blk * p.dv + v0, p.DHV, Lc, gt, ncol);
      }
      fence_proxy_async_smem();
      named_bar(WG_OUT, 128);
      if (first) {
        for (int j = 0; j < DVT / 64; ++j)
          if (tma_box_ok(p.err, BS_WALK_H_TMA, blk * p.dv + v0 + 64 * j, t0, 8, p.DHV, p.S, L, true) &&
              in_bounds(p.err, BS_WALK_H_TMA, bh, p.BH))
            tile_store(&mapH, sm + SM::OH + j * 8192, PAD && p.dv < DVT, blk * p.dv + v0 + 64 * j, blk, t0, bh);
        bulk_commit();
        mbar_arrive(&bars.gempty[gi]);
      }
    }
    if (first) bulk_wait_all();
  } else {
    // =============================================================== n group
    const int nt = tid - 352, wq = nt >> 5;  // 0..127, 0..3
    const bool first = nt == 0;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    float fin = 1.f;
    float n_sc = SN ? nvec[0] : 0.f;  // scalar normaliser (lazily scaled like n)
    for (int c = 0; c < nck; ++c) {
      const int b = c & 1, gi = c % NGB;
      const GateBuf G = gbuf(gi);
      uint8_t* Qs = sm + b * SM::STAGE;
      uint8_t* Ks = Qs + SM::QB;
      // the upper half of the snapshot first: it is on the recurrence's path, n is not
      {
        const bool x = mbar_test_wait(&bars.gfull[gi], (c / NGB) & 1),
                   y = c == 0 || mbar_test_wait(&bars.ro_done, (c - 1) & 1);
        if (!__all_sync(0xffffffffu, x && y))
          warp_wait_slow3(&bars.gfull[gi], (c / NGB) & 1, c > 0 ? &bars.ro_done : nullptr, (c - 1) & 1, nullptr, 0,
                          &abort_flag, p.wait);
      }
      tc_fence_after();
      const int flags = __float_as_int(G.scal[0]);
      snapshot_half(G, flags, lane_off, DK / 2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.cb_ready);
      if (!__all_sync(0xffffffffu, mbar_test_wait(&bars.full[b], (c >> 1) & 1)))
        warp_wait_slow(&bars.full[b], (c >> 1) & 1, &abort_flag, p.wait);
      const bool guard = (flags & GF_GUARD) != 0;
      fin = G.scal[4];
      if (SN) {
        if (nt < L) G.nq[nt] = n_sc;  // scalar normaliser: the chunk's start value for every token
      } else if (!ret) {
        // nq_t = n_st . q_t for this warp's 16 tokens as warp-level MMAs: A = the Q rows
        // (ldmatrix from the swizzled tile), B = n as hi + lo in columns 0 and 1 (lanes 0-7)
        const int mi = lane >> 3, arow = 16 * wq + (mi & 1) * 8 + (lane & 7);
        const uint32_t a_row = smem_u32(Qs) + arow * 128;
        const __nv_bfloat16* nf = nfrag + (c & 1) * SM::NFRAG + (lane & 7) * (DK / 4 + 8);
        float d[4][4] = {};
#pragma unroll
        for (int kk = 0; kk < DK / 16; kk += 2) {
          const uint4 bv = *reinterpret_cast<const uint4*>(nf + 4 * kk);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int col = 16 * (kk + h2) + (mi >> 1) * 8;
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a_row + (col >> 6) * 8192 + ((((col & 63) >> 3) ^ (arow & 7)) << 4), a0, a1, a2, a3);
            const uint32_t b0 = lane < 8 ? (h2 ? bv.z : bv.x) : 0u, b1 = lane < 8 ? (h2 ? bv.w : bv.y) : 0u;
            mma_m16n8k16_bf16(d[(kk + h2) & 3], a0, a1, a2, a3, b0, b1);
          }
        }
        if ((lane & 3) == 0) {
          const int t = 16 * wq + (lane >> 2);
          G.nq[t] = ((d[0][0] + d[1][0]) + (d[2][0] + d[3][0])) + ((d[0][1] + d[1][1]) + (d[2][1] + d[3][1]));
          G.nq[t + 8] = ((d[0][2] + d[1][2]) + (d[2][2] + d[3][2])) + ((d[0][3] + d[1][3]) + (d[2][3] + d[3][3]));
        }
      }
      if (guard) {
        // guarded chunk: Q <- e^{b_t+m_c-m_t} Q once the S MMA has read the raw Q, then the
        // read-out with the scaled Q.  A warp's n . q read exactly the 16 rows it scales.
        gwait(&bars.s_full[b], (c >> 1) & 1);
        scale_rows_bf16<DK>(smem_u32(Qs), G.sq, lane, 32, 16 * wq, 16);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.q_ready[gi]);  // this warp's tokens: n . q (and scaled Q)
      if (SN) {
        // n <- ns n + sum_s u_s, the same in every thread of the group (no shared state)
        const float2 u2 = *reinterpret_cast<const float2*>(G.u + 2 * lane);
        float us = u2.x + u2.y;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) us += __shfl_xor_sync(0xffffffffu, us, o);
        n_sc = G.scal[3] * n_sc + us;
      } else if (!ret) {
        // n <- ns n + K^T u for this warp's DK/4 entries of n as warp-level MMAs: A = K^T
        // (ldmatrix.trans of the swizzled K tile), B = u as hi + lo in columns 0 and 1 (lanes 0-7)
        constexpr int MT = DK / 64;  // 16-entry tiles per warp
        const int mi = lane >> 3, tq = lane & 3, k0 = (DK / 4) * wq;
        uint32_t ub[L / 16][2];
#pragma unroll
        for (int ks = 0; ks < L / 16; ++ks) {
          const float2 x = *reinterpret_cast<const float2*>(G.u + 16 * ks + 2 * tq);
          const float2 y = *reinterpret_cast<const float2*>(G.u + 16 * ks + 2 * tq + 8);
          uint32_t xl, yl;
          const uint32_t xh = split_bf16x2(x.x, x.y, &xl), yh = split_bf16x2(y.x, y.y, &yl);
          ub[ks][0] = lane < 4 ? xh : lane < 8 ? xl : 0u;
          ub[ks][1] = lane < 4 ? yh : lane < 8 ? yl : 0u;
        }
        const uint32_t ks_u = smem_u32(Ks);
        float d[MT][4] = {};
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int ks = 0; ks < L / 16; ++ks) {
            const int srow = 16 * ks + (mi >> 1) * 8 + (lane & 7), m = k0 + 16 * mt + (mi & 1) * 8;
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(ks_u + (m >> 6) * 8192 + srow * 128 + ((((m & 63) >> 3) ^ (srow & 7)) << 4), a0, a1, a2,
                              a3);
            mma_m16n8k16_bf16(d[mt], a0, a1, a2, a3, ub[ks][0], ub[ks][1]);
          }
        if (tq == 0) {
          const float ns = G.scal[3];
          __nv_bfloat16* nf = nfrag + ((c + 1) & 1) * SM::NFRAG;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int k = k0 + 16 * mt + (lane >> 2) + 8 * h2;
              const float v = ns * nvec[k] + (d[mt][2 * h2] + d[mt][2 * h2 + 1]);
              nvec[k] = v;
              store_nfrag<DK>(nf, k, v);
            }
        }
      }
      named_bar(WG_N, 128);  // n updated for the next chunk; the group is done with the stage
      if (first) {
        mbar_arrive(&bars.empty[b]);
        mbar_arrive(&bars.gempty[gi]);
      }
    }
    // final n after the last update, back in units of e^{m}
    if (SN) {
      if (nck > 0 && last_seg && tile == 0 && blk == 0 && p.n_out && !abort_flag && nt == 0 &&
          in_bounds(p.err, BS_WALK_FINAL, bh, p.BH))
        p.n_out[bh] = fin * n_sc;
    } else if (nck > 0 && last_seg && !ret && tile == 0 && p.n_out && !abort_flag)
      for (int col = nt; col < (PAD ? p.dk : DK); col += 128)
        if (in_bounds(p.err, BS_WALK_FINAL, (long long)slice * p.dk + col, (long long)p.slices * p.dk))
          p.n_out[(size_t)slice * p.dk + col] = fin * nvec[col];
  }

  // Drain before TMEM is freed and the CTA exits: every MMA issued and every Q/K/V load issued
  // has completed (after an expired wait the role loops may have stopped early; the h stores
  // were waited for by the output group).  Default bound whatever the caller's limit.
  if (warp == 1 || warp == 2) {
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    bool ok = mbar_wait(&bars.drain, 0, WAIT_DEFAULT);
    for (int b = 0; b < 2; ++b)
      if (n_issued > b) {
        const int c_last = b + 2 * ((n_issued - 1 - b) / 2);
        ok = mbar_wait(&bars.full[b], (c_last >> 1) & 1, WAIT_DEFAULT) && ok;
      }
    if (!ok) abort_flag = 1;
    if (abort_flag) atomicOr(p.err, 2u);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, TM_COLS);
}

// ===================================================================== host side
bool tc_supported(int dtype, int chunk, int dk, int dv, int DHQK, int DHV) {
  if (dtype != 1 || chunk != L) return false;
  // block widths below 64 run padded to 64 (zero-filled columns / rows)
  if (dk != 64 && dk != 128 && dk != 256 && !(dk < 64 && dk % 8 == 0)) return false;
  if (dv % 64 != 0 && !(dv < 64 && dv % 8 == 0 && dk <= 64)) return false;
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
  pl.n_tiles = (dv + pl.dvt - 1) / pl.dvt;  // (a block narrower than 64 is one padded tile)
  const int chunks = (S + L - 1) / L;
  const long long base = (long long)B * NH * nb * pl.n_tiles;
  int G = base > 0 ? (int)(num_sms / base) : 1;
  if (G < 1) G = 1;
  // at least 4 chunks per segment, segments no longer than 8192 tokens (phase A keeps one
  // fp32 exponent offset per chunk of its segment in shared memory)
  if (G > chunks / 4) G = chunks / 4 > 0 ? chunks / 4 : 1;
  // up to 8 chunks one segment: the summaries' own launch and the composition cost more than
  // they save (8 chunks of 64-wide heads, one segment against two: 0.024 -> 0.021-0.022 ms)
  if (chunks <= 8) G = 1;
  while ((chunks + G - 1) / G * L > 8192) ++G;
  pl.seg_chunks = chunks > 0 ? (chunks + G - 1) / G : 1;
  pl.G = chunks > 0 ? (chunks + pl.seg_chunks - 1) / pl.seg_chunks : 1;
  pl.seg0_chunks = pl.seg_chunks;
  // phase A: CTAs of the walk's value tile, segment 0 summarised in two halves when that still
  // fits one wave
  pl.dva = pl.dvt;
  pl.n_tiles_a = pl.n_tiles;
  pl.ups = 1;
  pl.NU = pl.G - 1;
  if (pl.G > 1 && pl.seg_chunks >= 8) {
    // Segment 0 needs no summary and walks while the others are summarised, so it gets more
    // chunks.  Cost model in units of one walk chunk (measured on the large head: ~2.7 us per walk
    // chunk, ~1.05 us per summary chunk, ~1.5 us per summary composed into a start state, segment 0
    // starting ~6 us and phase A ~3 us after the call starts):
    //   end of segment 0     = 2.2 + s0
    //   end of the others    = 1.1 + a * (longest unit) + 0.55 * (units composed) + s
    // over s0 with s = ceil((chunks - s0) / (G - 1)), the two-unit split of segment 0 taken when
    // its CTAs fit one wave.  a, a summary chunk over a walk chunk, is 0.39 for 256-wide keys and
    // larger for narrower ones, whose walk chunk is shorter (0.54 fits 64-wide heads: the best
    // segment-0 length of 32 chunks in two segments measured 21, both modes); in between linear.
    const double a_sum = 0.39 + 0.15 * (256 - (dk < 64 ? 64 : dk > 256 ? 256 : dk)) / 192.0;
    const long long slices_l = (long long)B * NH * nb;
    // split segment 0 in two summary units only when the summary CTAs (G units: 2 + (G - 2)) and
    // segment 0's walk CTAs run at the same time: together one wave
    const bool can_split = (long long)(pl.G + 1) * pl.n_tiles * slices_l <= num_sms;
    double best = 1e30;
    int best_s0 = pl.seg_chunks, best_s = pl.seg_chunks, best_ups = 1;
    for (int s0 = pl.seg_chunks; s0 <= 2 * pl.seg_chunks && s0 <= 128 && s0 < chunks; ++s0) {
      const int s = (chunks - s0 + pl.G - 2) / (pl.G - 1);
      if (s < 4) break;
      for (int ups = 1; ups <= (can_split ? 2 : 1); ++ups) {
        const int longest = (s0 + ups - 1) / ups > s ? (s0 + ups - 1) / ups : s;
        const int composed = ups + pl.G - 2;
        const double others = 1.1 + a_sum * longest + 0.55 * composed + s;
        const double first = 2.2 + s0;
        const double cost = others > first ? others : first;
        if (cost < best - 1e-9) {
          best = cost;
          best_s0 = s0;
          best_s = s;
          best_ups = ups;
        }
      }
    }
    pl.seg0_chunks = best_s0;
    pl.seg_chunks = best_s;
    pl.ups = best_ups;
    while (pl.G > 1 && pl.seg0_chunks + (pl.G - 2) * pl.seg_chunks >= chunks) --pl.G;  // last segment non-empty
    pl.NU = pl.G > 1 ? pl.ups + pl.G - 2 : 0;
    if (pl.G == 1) pl.ups = 1;
  }
  return pl;
}

size_t tc_workspace_bytes(const TcPlan& pl, long long BH, int nb, int dk, int dv) {
  const long long slices = BH * nb;
  const size_t NU = pl.NU;
  size_t off = 256;  // error word
  off += ((size_t)slices * NU * dv * dk * 4 + 255) / 256 * 256;
  off += ((size_t)slices * NU * dk * 4 + 255) / 256 * 256;
  off += 2 * (((size_t)BH * NU * 4 + 255) / 256 * 256);
  const size_t ncp = (size_t)pl.seg0_chunks + (size_t)(pl.G - 1) * pl.seg_chunks, sp = ncp * L;
  off += 3 * (((size_t)BH * sp * 4 + 255) / 256 * 256);
  off += 2 * (((size_t)BH * ncp * 4 + 255) / 256 * 256);
  return off;
}

// Launch that may overlap the previous kernel of the stream (programmatic stream
// serialization); the kernel waits (griddepcontrol.wait) before it reads that kernel's results.
template <typename... KArgs, typename... Args>
static cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t stream,
                                    Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int DK, int DVA, bool PAD>
static cudaError_t launch_segment(const TcPlan& pl, const TcParams& prm, const CUtensorMap& mk, const CUtensorMap& mv,
                                  long long slices, cudaStream_t stream) {
  const int smemA = SegCfg<DK, DVA>::BYTES_FIXED + pl.seg0_chunks * 4;  // + one offset per chunk of a unit
  cudaError_t e = cudaFuncSetAttribute(tc_segment_kernel<DK, DVA, PAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smemA);
  if (e != cudaSuccess) return e;
  dim3 gridA(pl.n_tiles_a, pl.NU, (unsigned)slices);
  return launch_dependent(tc_segment_kernel<DK, DVA, PAD>, gridA, dim3(NTA), smemA, stream, mk, mv, prm);
}

template <int DK, int DVT, bool SN, bool REV, bool PAD>
static cudaError_t launch_tc_dk(const TcPlan& pl, const TcParams& prm, const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, const CUtensorMap& mh, const CUtensorMap& ms, long long slices,
                                cudaStream_t stream, cudaEvent_t ev0, cudaEvent_t ev1) {
  cudaError_t e;
  const long long BH = slices / prm.nb;
  tc_gate_prep_kernel<<<(unsigned)((BH * prm.ncp + 7) / 8), 256, 0, stream>>>(prm, (int)BH);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (pl.NU > 0) {
    e = pl.dva == 256   ? launch_segment<DK, 256, false>(pl, prm, mk, mv, slices, stream)
        : pl.dva == 128 ? launch_segment<DK, 128, PAD>(pl, prm, mk, mv, slices, stream)
                        : launch_segment<DK, 64, PAD>(pl, prm, mk, mv, slices, stream);
    if (e != cudaSuccess) return e;
  }
  const int smemC = WalkSmem<DK, DVT>::BYTES;
  e = cudaFuncSetAttribute(tc_walk_kernel<DK, DVT, SN, REV, PAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smemC);
  if (e != cudaSuccess) return e;
  if (ev0) cudaEventRecord(ev0, stream);
  dim3 gridC(pl.n_tiles, (unsigned)slices, pl.G);
  e = launch_dependent(tc_walk_kernel<DK, DVT, SN, REV, PAD>, gridC, dim3(NTW), smemC, stream, mq, mk, mv, mh, ms, prm);
  if (ev1) cudaEventRecord(ev1, stream);
  return e;
}

cudaError_t launch_tc(const WalkArgs& a, const TcPlan& pl, void* ws, cudaStream_t stream, cudaEvent_t ev0,
                      cudaEvent_t ev1) {
  const long long BH = (long long)a.B * a.NH, slices = BH * a.nb;
  if (slices == 0 || a.S == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mh;
  // blocks narrower than 64 columns: 4-D maps {block width, nb, S, BH} (tiles zero-padded to 64)
  const bool qk_ok = a.dk < 64 ? make_map_bf16_blocks(&mq, a.q, a.dk, a.nb, a.S, BH, L) &&
                                     make_map_bf16_blocks(&mk, a.k, a.dk, a.nb, a.S, BH, L)
                               : make_map_bf16_3d(&mq, a.q, a.DHQK, a.S, BH, L) &&
                                     make_map_bf16_3d(&mk, a.k, a.DHQK, a.S, BH, L);
  const bool vh_ok = a.dv < 64 ? make_map_bf16_blocks(&mv, a.v, a.dv, a.nb, a.S, BH, L) &&
                                     make_map_bf16_blocks(&mh, a.h, a.dv, a.nb, a.S, BH, L)
                               : make_map_bf16_3d(&mv, a.v, a.DHV, a.S, BH, L) &&
                                     make_map_bf16_3d(&mh, a.h, a.DHV, a.S, BH, L);
  if (!qk_ok || !vh_ok) return cudaErrorInvalidValue;
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
  const size_t NU = pl.NU;
  prm.seg0_chunks = pl.seg0_chunks;
  prm.ups = pl.ups;
  prm.NU = pl.NU;
  prm.n_tiles_a = pl.n_tiles_a;
  prm.err = reinterpret_cast<unsigned int*>(w);
  size_t off = 256;
  prm.dC = reinterpret_cast<float*>(w + off);
  off += ((size_t)slices * NU * a.dv * a.dk * 4 + 255) / 256 * 256;
  prm.dn = reinterpret_cast<float*>(w + off);
  off += ((size_t)slices * NU * a.dk * 4 + 255) / 256 * 256;
  prm.segA = reinterpret_cast<float*>(w + off);
  off += ((size_t)BH * NU * 4 + 255) / 256 * 256;
  prm.segB = reinterpret_cast<float*>(w + off);
  off += ((size_t)BH * NU * 4 + 255) / 256 * 256;
  prm.ncp = pl.seg0_chunks + (pl.G - 1) * pl.seg_chunks;
  // the segment summaries [slices * NU * dv rows][dk] fp32, read back by the walk through TMA
  CUtensorMap ms;
  memset(&ms, 0, sizeof(ms));
  if (pl.NU > 0 && !make_map_f32_2d(&ms, prm.dC, (uint64_t)a.dk, (uint64_t)slices * pl.NU * a.dv, 64))
    return cudaErrorInvalidValue;
  prm.sp = prm.ncp * L;
  prm.wait = a.wait_cycles > 0 ? a.wait_cycles : WAIT_DEFAULT;
  prm.nbias = a.retention ? nullptr : a.nbias;
  prm.rev = a.reverse ? 1 : 0;
  prm.nck_all = (a.S + L - 1) / L;
  float** planes[5] = {&prm.gb, &prm.gx, &prm.gxc, &prm.cg, &prm.cxm};
  for (int i = 0; i < 5; ++i) {
    *planes[i] = reinterpret_cast<float*>(w + off);
    off += ((size_t)BH * (i < 3 ? prm.sp : prm.ncp) * 4 + 255) / 256 * 256;
  }
  prm.BH = BH;
  prm.slices = (int)slices;
  // the error word and, for the bounds-checked build, its record (bytes 16..39)
  cudaError_t e = cudaMemsetAsync(w, 0, 64, stream);
  if (e != cudaSuccess) return e;
  const int dkp = a.dk < 64 ? 64 : a.dk;  // key width of the kernels (narrow blocks padded)
  const bool pad = a.dk < 64 || a.dv < 64;  // kernels that mask the padding of narrow blocks
#define MLSTM_TC_DISPATCH(SNV, REVV)                                                                       \
  do {                                                                                                   \
    if (a.dk == 256 && pl.dvt == 128)                                                                    \
      return launch_tc_dk<256, 128, SNV, REVV, false>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1);       \
    if (a.dk == 256 && pl.dvt == 64)                                                                     \
      return launch_tc_dk<256, 64, SNV, REVV, false>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1);        \
    if (a.dk == 128 && pl.dvt == 128)                                                                    \
      return launch_tc_dk<128, 128, SNV, REVV, false>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1);       \
    if (a.dk == 128 && pl.dvt == 64)                                                                     \
      return launch_tc_dk<128, 64, SNV, REVV, false>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1);        \
    if (dkp == 64 && pl.dvt == 128)                                                                      \
      return pad ? launch_tc_dk<64, 128, SNV, REVV, true>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1) \
                 : launch_tc_dk<64, 128, SNV, REVV, false>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1); \
    if (dkp == 64 && pl.dvt == 64)                                                                       \
      return pad ? launch_tc_dk<64, 64, SNV, REVV, true>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1) \
                 : launch_tc_dk<64, 64, SNV, REVV, false>(pl, prm, mq, mk, mv, mh, ms, slices, stream, ev0, ev1); \
  } while (0)
  // walk variants: the vector normaliser forward and reversed, the scalar normaliser forward
  if (prm.nbias && !prm.rev) MLSTM_TC_DISPATCH(true, false);
  else if (!prm.nbias && prm.rev) MLSTM_TC_DISPATCH(false, true);
  else if (!prm.nbias) MLSTM_TC_DISPATCH(false, false);
#undef MLSTM_TC_DISPATCH
  return cudaErrorInvalidValue;
}

}  // namespace mlstm
