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
  void *h;
  float *C_out, *n_out, *m_out;
};

cudaError_t launch_gate_prep(int BH, int S, int n_per_head, const float* ig, const float* fg,
                             const float* m0, const float* n0, float* m_tok, float* m_init,
                             float* n_init, cudaStream_t stream);

// SIMT fp32 chunkwise walk.  Returns cudaErrorInvalidValue if the shapes need more shared
// memory than a CTA has.
size_t simt_walk_smem_bytes(int chunk, int dk, int dv_tile);
int simt_walk_pick_tile(int chunk, int dk, int dv);
cudaError_t launch_simt_walk(const WalkArgs& a, cudaStream_t stream);

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

}  // namespace mlstm
