// Internal launch interface between the C ABI (mlstm_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace mlstm {

// Arguments of the chunkwise walk kernels (one per prefill, shared by all variants).
struct WalkArgs {
  int B, NH, S, DHQK, DHV, chunk, nb, retention;
  int dk, dv;                // per-block key / value widths
  int dv_tile;               // value rows of the state per CTA
  int dtype;                 // 0 fp32, 1 bf16
  const void *q, *k, *v, *og;
  const float *ig, *fg;
  const float *C0;           // initial state [BH*nb, dv, dk] (may be NULL = zeros)
  const float *n_init;       // [BH*nb, dk] snapshot of n0 (never NULL for mLSTM)
  const float *m_init;       // [BH] snapshot of m0 (never NULL for mLSTM)
  const float *m_tok;        // [BH, S] stabiliser per token (mLSTM)
  const float *nbias;        // [NH]: scalar normaliser with this bias (NULL = vector n . q);
                             // then n_init / n_out hold one value per (batch, head)
  void *h;
  float *C_out, *n_out, *m_out;
  long long wait_cycles;     // bound of each device-side wait (tensor-core path); 0 = default
  int reverse;               // tensor-core path: the reversed sequence read in place (token S-1 first)
};

// The steps either side of retention (msr.cu): the rotation Theta of q and k by position
// (in place allowed: qo == q, ko == k), and the per-head GroupNorm + SiLU gate (y == h
// allowed).  *_supported: the head width fits the kernel's vector layout.
bool theta_rotate_supported(int D, int dtype);
bool gn_gate_supported(int DHV, int dtype);
cudaError_t launch_theta_rotate(int B, int NH, int S, int D, int dtype, const void* q, const void* k, void* qo,
                                void* ko, const long long* pos0, float base, cudaStream_t stream);
cudaError_t launch_gn_gate(long long rows, int NH, int S, int DHV, int dtype, const void* h, const void* g,
                           const float* w, const float* b, float eps, void* y, cudaStream_t stream);

// Gated DeltaNet-2 (gdn2.cu).  q, k [B,H,T,K], v [B,H,T,V] (dtype 0 fp32, 1 bf16); g (log
// decay), b (erase gate) [B,H,T,K] and w (write gate) [B,H,T,V] fp32; S0, S_out [B,H,K,V] fp32
// (S0 NULL = zeros, S_out NULL = not written, S_out == S0 in place); o [B,H,T,V] dtype.
struct Gdn2Args {
  int B, H, T, K, V, dtype;
  long long wait;  // bound of the tensor-core chunk kernels' waits (SM cycles), 0 = default
  int nsm;         // SMs of the device (set by the tensor-core chunk launcher)
  const void *q, *k, *v;
  const float *g, *b, *w;
  const float* S0;
  void* o;
  float* S_out;
};
bool gdn2_recurrent_supported(int K);
// value-tile width of the chunk scan kernel for these sizes (0 = unsupported)
int gdn2_chunk_vtile(int L, int K, int V);
// workspace of the chunk mode: one prepared slot per (batch, head, chunk)
size_t gdn2_chunk_workspace_bytes(long long BH, int T, int L, int K);
// mode 0: fused recurrent (token by token); 1: chunk of `chunk` tokens (needs ws)
cudaError_t launch_gdn2(const Gdn2Args& a, int mode, int chunk, void* ws, cudaStream_t stream);
// chunk mode on the tensor cores (gdn2_tc.cu): bf16, chunk 64, K 128, V 64 or 128, T > 0.  Its
// workspace starts with a GDN2_TC_HEADER-byte header whose first word is the error word of the
// bounded waits (bit 0: a wait ran out), then one slot per (batch x head, chunk).
constexpr size_t GDN2_TC_HEADER = 256;
bool gdn2_tc_supported(int chunk, int K, int V, int dtype, int T);
size_t gdn2_tc_workspace_bytes(long long BH, int T, int V);
cudaError_t launch_gdn2_tc(const Gdn2Args& a, void* ws, cudaStream_t stream);

cudaError_t launch_gate_prep(int BH, int S, int n_per_head, const float* ig, const float* fg,
                             const float* m0, const float* n0, float* m_tok, float* m_init,
                             float* n_init, cudaStream_t stream);

// SIMT fp32 chunkwise walk.  Returns cudaErrorInvalidValue if the shapes need more shared
// memory than a CTA has.
size_t simt_walk_smem_bytes(int chunk, int dk, int dv_tile);
int simt_walk_pick_tile(int chunk, int dk, int dv);
cudaError_t launch_simt_walk(const WalkArgs& a, cudaStream_t stream);

// Tensor-core (tcgen05) chunkwise prefill: bf16, chunk 64, block key width 64/128/256,
// block value width a multiple of 64.
struct TcPlan {
  int dvt;          // value rows per walk CTA (MMA M): 128 or 64
  int n_tiles;      // value tiles per block
  int G;            // sequence segments per (batch, head, block)
  int seg_chunks;   // chunks per segment (segments 1 .. G-1)
  int seg0_chunks;  // chunks of segment 0
  int dva;          // value rows per segment-summary CTA (64, 128 or 256)
  int n_tiles_a;    // summary CTAs per block and unit
  int ups;          // summary units per segment (1 or 2)
  int NU;           // summary units: ups * (G - 1)
};
bool tc_supported(int dtype, int chunk, int dk, int dv, int DHQK, int DHV);
int tc_num_sms();
TcPlan tc_plan(int B, int NH, int S, int nb, int dk, int dv, int num_sms);
size_t tc_workspace_bytes(const TcPlan& pl, long long BH, int nb, int dk, int dv);
// ws: workspace of at least tc_workspace_bytes bytes; its first 4 bytes become an error
// word (0 = ok; nonzero = a bounded wait expired), cleared on the stream before the kernels.  ev0/ev1 (may be NULL) are recorded
// around the walk kernel.
cudaError_t launch_tc(const WalkArgs& a, const TcPlan& pl, void* ws, cudaStream_t stream, cudaEvent_t ev0,
                      cudaEvent_t ev1);

// Decode step.
struct StepArgs {
  int B, NH, DHQK, DHV, nb, retention, dtype;
  int dk, dv;
  const void *q, *k, *v, *og;
  const float *ig, *fg;
  float *C, *n, *m;
  void *h;
};
bool step_supported_dk(int dk);
cudaError_t launch_step(const StepArgs& a, cudaStream_t stream);

// dst[bh][S-1-t] = src[bh][t] for [BH, S, row_bytes] tensors (row_bytes a multiple of 2).
cudaError_t launch_reverse_rows(const void* src, void* dst, long long BH, long long S, long long row_bytes,
                                cudaStream_t stream);

// Backward (gradients of h and of the final state).  One CTA per (batch, head).
struct BwdArgs {
  int B, NH, S, DHQK, DHV, nb, retention, dtype;
  int dk, dv;
  const void *q, *k, *v, *og, *dh;
  const float *ig, *fg, *C0, *n0, *m0, *dC, *dn;
  float *dq, *dk_out, *dv_out, *dig, *dfg, *dog, *dC0, *dn0, *dm0;
  float* ws;  // bwd_workspace_bytes
};
size_t bwd_smem_bytes(int dk, int dv);
size_t bwd_workspace_bytes(long long BH, int S, int nb);
bool bwd_supported(int dk, int dv, int dtype);
cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream);

}  // namespace mlstm
