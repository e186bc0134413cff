// C ABI of libmlstm (declared in include/mlstm.h): host-side validation, workspace
// layout and kernel dispatch.  No entry point allocates, frees or synchronises.
#include <stdint.h>
#include <string.h>

#include "bounds.cuh"
#include "kernels.h"
#include "mlstm.h"

namespace {

using namespace mlstm;

struct FwdShape {
  int B, NH, S, DHQK, DHV, chunk, nb, dk, dv, retention, dtype;
  size_t esize;
  long long BH;
  bool tc;     // tensor-core path
  TcPlan tcp;  // its plan
};

mlstm_status_t check_fwd(const mlstm_fwd_params_t* p, FwdShape* s) {
  if (!p) return MLSTM_ERR_NULL;
  if (p->dtype != MLSTM_F32 && p->dtype != MLSTM_BF16) return MLSTM_ERR_DTYPE;
  if (p->B < 0 || p->NH < 0 || p->S < 0 || p->DHQK < 1 || p->DHV < 1 || p->chunk < 1 || p->num_blocks < 1)
    return MLSTM_ERR_SHAPE;
  if (p->DHQK % p->num_blocks || p->DHV % p->num_blocks) return MLSTM_ERR_SHAPE;
  s->B = p->B;
  s->NH = p->NH;
  s->S = p->S;
  s->DHQK = p->DHQK;
  s->DHV = p->DHV;
  s->chunk = p->chunk;
  s->nb = p->num_blocks;
  s->dk = p->DHQK / p->num_blocks;
  s->dv = p->DHV / p->num_blocks;
  s->retention = p->retention ? 1 : 0;
  s->dtype = p->dtype == MLSTM_BF16 ? 1 : 0;
  s->esize = p->dtype == MLSTM_BF16 ? 2 : 4;
  s->BH = (long long)p->B * p->NH;
  // grid limits of the kernels
  if (s->BH * s->nb > 65535LL || s->BH > (1LL << 31) / 1024) return MLSTM_ERR_SHAPE;
  if ((long long)s->S * s->BH > (1LL << 40)) return MLSTM_ERR_SHAPE;
  s->tc = tc_supported(s->dtype, s->chunk, s->dk, s->dv, s->DHQK, s->DHV);
  if (s->tc) {
    s->tcp = tc_plan(s->B, s->NH, s->S, s->nb, s->dk, s->dv, tc_num_sms());
    if ((long long)s->tcp.G * s->tcp.n_tiles > 65535 || s->BH * s->nb > 65535) return MLSTM_ERR_SHAPE;
  } else if (s->S > 0 && s->BH > 0 && simt_walk_pick_tile(s->chunk, s->dk, s->dv) == 0) {
    return MLSTM_ERR_SHAPE;
  }
  return MLSTM_OK;
}

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

struct WsLayout {
  size_t m_tok, m_init, n_init, total;
  size_t tc, c_init;  // tensor-core path: its own area, snapshot of C0
};

// scalar_n: the scalar-normaliser variant (n0 one value per (batch, head)); tensor-core path only
WsLayout fwd_layout(const FwdShape& s, bool scalar_n = false) {
  WsLayout w = {0, 0, 0, 0, 0, 0};
  if (s.BH == 0) return w;
  if (s.tc) {
    size_t off = 0;
    w.tc = off;
    off = align_up(off + tc_workspace_bytes(s.tcp, s.BH, s.nb, s.dk, s.dv));
    if (!s.retention) {
      w.n_init = off;
      off = align_up(off + sizeof(float) * (size_t)s.BH * (scalar_n ? 1 : (size_t)s.nb * s.dk));
      w.m_init = off;
      off = align_up(off + sizeof(float) * (size_t)s.BH);
    }
    if (s.tcp.G > 1) {
      w.c_init = off;
      off = align_up(off + sizeof(float) * (size_t)s.BH * s.nb * s.dv * s.dk);
    }
    w.total = off;
    return w;
  }
  if (s.retention) return w;
  size_t off = 0;
  w.m_tok = off;
  off = align_up(off + sizeof(float) * (size_t)s.BH * s.S);
  w.m_init = off;
  off = align_up(off + sizeof(float) * (size_t)s.BH);
  w.n_init = off;
  off = align_up(off + sizeof(float) * (size_t)s.BH * s.nb * s.dk);
  w.total = off;
  return w;
}

bool misaligned(const void* p) { return ((uintptr_t)p & 15) != 0; }

struct Range {
  const void* p;
  size_t n;
};
bool overlaps(Range a, Range b) {
  if (!a.p || !b.p || a.n == 0 || b.n == 0) return false;
  const uintptr_t a0 = (uintptr_t)a.p, b0 = (uintptr_t)b.p;
  return a0 < b0 + b.n && b0 < a0 + a.n;
}

// GroupNorm + SiLU gate applied to h after the recurrence: one more kernel over h in place
struct GnArgs {
  const void* g;
  const float *w, *b;
  float eps;
};

mlstm_status_t fwd_impl(const mlstm_fwd_params_t* p, const void* q, const void* k, const void* v,
                        const float* igate, const float* fgate, const void* ogate, const float* C0,
                        const float* n0, const float* m0, void* h, float* C_out, float* n_out, float* m_out,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream, cudaEvent_t ev0,
                        cudaEvent_t ev1, bool launch = true, const GnArgs* gn = nullptr,
                        const float* nbias = nullptr, bool reverse = false) {
  // reverse: the reversed sequence read in place by the tensor-core kernels (the caller checks
  // that the tensor-core path runs)
  // nbias != NULL: the scalar normaliser with this bias [NH] (tensor-core path only; n0 / n_out
  // one value per (batch, head)); the caller has validated it
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  const bool scalar_n = nbias != nullptr;
  if (scalar_n && (!s.tc || s.retention)) return MLSTM_ERR_SHAPE;
  const bool ret = s.retention != 0;
  if (ret) {
    igate = fgate = nullptr;
    ogate = nullptr;
    n0 = m0 = nullptr;
    n_out = m_out = nullptr;
  }
  const size_t tok = (size_t)s.BH * s.S;
  const size_t bq = tok * s.DHQK * s.esize, bv = tok * s.DHV * s.esize, bg = tok * sizeof(float);
  const size_t bC = (size_t)s.BH * s.nb * s.dv * s.dk * sizeof(float);
  const size_t bn = (size_t)s.BH * (scalar_n ? 1 : (size_t)s.nb * s.dk) * sizeof(float);
  const size_t bm = (size_t)s.BH * sizeof(float);
  if (tok > 0) {
    if (!q || !k || !v || !h) return MLSTM_ERR_NULL;
    if (!ret && (!igate || !fgate)) return MLSTM_ERR_NULL;
  }
  const void* all[] = {q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, workspace};
  for (const void* ptr : all)
    if (ptr && misaligned(ptr)) return MLSTM_ERR_ALIGN;
  const WsLayout ws = fwd_layout(s, scalar_n);
  if (ws.total > 0 && (!workspace || workspace_bytes < ws.total)) return MLSTM_ERR_WORKSPACE;

  // aliasing: outputs may not overlap inputs, except the exact in-place state aliases
  const Range in_q{q, bq}, in_k{k, bq}, in_v{v, bv}, in_ig{igate, bg}, in_fg{fgate, bg}, in_o{ogate, bv};
  const Range in_C{C0, bC}, in_n{n0, bn}, in_m{m0, bm};
  const Range out_h{h, bv}, out_C{C_out, bC}, out_n{n_out, bn}, out_m{m_out, bm};
  const Range wsr{workspace, ws.total};
  const Range inputs[] = {in_q, in_k, in_v, in_ig, in_fg, in_o};
  const Range outs[] = {out_h, out_C, out_n, out_m, wsr};
  for (const Range& o : outs) {
    for (const Range& i : inputs)
      if (overlaps(o, i)) return MLSTM_ERR_ALIAS;
  }
  for (int a = 0; a < 5; ++a)
    for (int b = a + 1; b < 5; ++b)
      if (overlaps(outs[a], outs[b])) return MLSTM_ERR_ALIAS;
  const Range states_in[] = {in_C, in_n, in_m};
  const Range states_out[] = {out_C, out_n, out_m};
  for (const Range& si : states_in) {
    if (overlaps(out_h, si) || overlaps(wsr, si)) return MLSTM_ERR_ALIAS;
    for (int j = 0; j < 3; ++j) {
      const Range& so = states_out[j];
      const bool exact = so.p == si.p && so.n == si.n && (&si - states_in) == j;
      if (overlaps(so, si) && !exact) return MLSTM_ERR_ALIAS;
    }
  }
  if (s.BH == 0 || !launch) return MLSTM_OK;

  cudaError_t e = cudaSuccess;
  if (s.S == 0) {  // nothing to read: the final state is the initial state
    if (C_out && C_out != C0)
      e = C0 ? cudaMemcpyAsync(C_out, C0, bC, cudaMemcpyDeviceToDevice, stream) : cudaMemsetAsync(C_out, 0, bC, stream);
    if (e == cudaSuccess && n_out && n_out != n0)
      e = n0 ? cudaMemcpyAsync(n_out, n0, bn, cudaMemcpyDeviceToDevice, stream) : cudaMemsetAsync(n_out, 0, bn, stream);
    if (e == cudaSuccess && m_out && m_out != m0)
      e = m0 ? cudaMemcpyAsync(m_out, m0, bm, cudaMemcpyDeviceToDevice, stream) : cudaMemsetAsync(m_out, 0, bm, stream);
    return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
  }

  char* wsb = static_cast<char*>(workspace);
  WalkArgs a;
  memset(&a, 0, sizeof(a));
  a.B = s.B;
  a.NH = s.NH;
  a.S = s.S;
  a.DHQK = s.DHQK;
  a.DHV = s.DHV;
  a.chunk = s.chunk;
  a.nb = s.nb;
  a.retention = s.retention;
  a.dk = s.dk;
  a.dv = s.dv;
  a.dtype = s.dtype;
  a.q = q;
  a.k = k;
  a.v = v;
  a.og = ogate;
  a.ig = igate;
  a.fg = fgate;
  a.C0 = C0;
  a.h = h;
  a.C_out = C_out;
  a.n_out = n_out;
  a.m_out = m_out;
  a.wait_cycles = p->wait_limit_cycles;
  a.nbias = nbias;
  a.reverse = reverse ? 1 : 0;
  if (s.tc) {
    // snapshots: the walk writes n_out / m_out (and C_out across segments) while other
    // CTAs may still read n0 / m0 / C0, which the caller may have aliased to them
    if (!ret && n0) {
      e = cudaMemcpyAsync(wsb + ws.n_init, n0, bn, cudaMemcpyDeviceToDevice, stream);
      a.n_init = reinterpret_cast<const float*>(wsb + ws.n_init);
    }
    if (e == cudaSuccess && !ret && m0) {
      e = cudaMemcpyAsync(wsb + ws.m_init, m0, bm, cudaMemcpyDeviceToDevice, stream);
      a.m_init = reinterpret_cast<const float*>(wsb + ws.m_init);
    }
    if (e == cudaSuccess && C0 && C_out == C0 && s.tcp.G > 1) {
      e = cudaMemcpyAsync(wsb + ws.c_init, C0, bC, cudaMemcpyDeviceToDevice, stream);
      a.C0 = reinterpret_cast<const float*>(wsb + ws.c_init);
    }
    if (e != cudaSuccess) return MLSTM_ERR_CUDA;
    e = launch_tc(a, s.tcp, wsb + ws.tc, stream, ev0, ev1);
    if (e == cudaSuccess && gn)
      e = launch_gn_gate((long long)s.BH * s.S, s.NH, s.S, s.DHV, s.dtype, h, gn->g, gn->w, gn->b, gn->eps, h, stream);
    return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
  }
  if (!ret) {
    a.m_tok = reinterpret_cast<const float*>(wsb + ws.m_tok);
    a.m_init = reinterpret_cast<const float*>(wsb + ws.m_init);
    a.n_init = reinterpret_cast<const float*>(wsb + ws.n_init);
    e = launch_gate_prep((int)s.BH, s.S, s.nb * s.dk, igate, fgate, m0, n0, reinterpret_cast<float*>(wsb + ws.m_tok),
                         reinterpret_cast<float*>(wsb + ws.m_init), reinterpret_cast<float*>(wsb + ws.n_init),
                         stream);
    if (e != cudaSuccess) return MLSTM_ERR_CUDA;
  }
  a.dv_tile = simt_walk_pick_tile(s.chunk, s.dk, s.dv);
  if (ev0 && cudaEventRecord(ev0, stream) != cudaSuccess) return MLSTM_ERR_CUDA;
  e = launch_simt_walk(a, stream);
  if (e != cudaSuccess) return MLSTM_ERR_CUDA;
  if (ev1 && cudaEventRecord(ev1, stream) != cudaSuccess) return MLSTM_ERR_CUDA;
  if (gn && launch_gn_gate((long long)s.BH * s.S, s.NH, s.S, s.DHV, s.dtype, h, gn->g, gn->w, gn->b, gn->eps, h,
                           stream) != cudaSuccess)
    return MLSTM_ERR_CUDA;
  return MLSTM_OK;
}

// Workspace of the multi-scale retention block: rotated q and k, then the forward's own.
struct MsrLayout {
  size_t qr, kr, fwd, total;
};
MsrLayout msr_layout(const FwdShape& s) {
  MsrLayout r = {0, 0, 0, 0};
  const size_t bq = (size_t)s.BH * s.S * s.DHQK * s.esize;
  r.fwd = 0;  // first, so that its error word sits at the start (mlstm_fwd_chunkwise_status)
  r.qr = align_up(fwd_layout(s).total);
  r.kr = r.qr + align_up(bq);
  r.total = r.kr + align_up(bq);
  return r;
}

bool finite_nonneg(float x) { return x >= 0.f && x <= 3.4e38f; }

// Sizes of the element-wise entries (rotation, GroupNorm): no recurrence kernel involved, so
// only the dimensions themselves and the grid limits are checked.
mlstm_status_t check_dims(const mlstm_fwd_params_t* p, FwdShape* s) {
  if (!p) return MLSTM_ERR_NULL;
  if (p->dtype != MLSTM_F32 && p->dtype != MLSTM_BF16) return MLSTM_ERR_DTYPE;
  if (p->B < 0 || p->NH < 0 || p->S < 0 || p->DHQK < 1 || p->DHV < 1) return MLSTM_ERR_SHAPE;
  memset(s, 0, sizeof(*s));
  s->B = p->B;
  s->NH = p->NH;
  s->S = p->S;
  s->DHQK = p->DHQK;
  s->DHV = p->DHV;
  s->dtype = p->dtype == MLSTM_BF16 ? 1 : 0;
  s->esize = p->dtype == MLSTM_BF16 ? 2 : 4;
  s->BH = (long long)p->B * p->NH;
  if (s->B > 65535 || (long long)s->S * s->BH > (1LL << 40)) return MLSTM_ERR_SHAPE;
  return MLSTM_OK;
}

// Sizes of a backward call; MLSTM_OK when the kernel supports them.
mlstm_status_t check_bwd(const mlstm_fwd_params_t* p, FwdShape* s) {
  if (!p) return MLSTM_ERR_NULL;
  if (p->dtype != MLSTM_F32 && p->dtype != MLSTM_BF16) return MLSTM_ERR_DTYPE;
  if (p->B < 0 || p->NH < 0 || p->S < 0 || p->DHQK < 1 || p->DHV < 1 || p->num_blocks < 1)
    return MLSTM_ERR_SHAPE;
  if (p->DHQK % p->num_blocks || p->DHV % p->num_blocks) return MLSTM_ERR_SHAPE;
  memset(s, 0, sizeof(*s));
  s->B = p->B;
  s->NH = p->NH;
  s->S = p->S;
  s->DHQK = p->DHQK;
  s->DHV = p->DHV;
  s->nb = p->num_blocks;
  s->dk = p->DHQK / p->num_blocks;
  s->dv = p->DHV / p->num_blocks;
  s->retention = p->retention ? 1 : 0;
  s->dtype = p->dtype == MLSTM_BF16 ? 1 : 0;
  s->esize = p->dtype == MLSTM_BF16 ? 2 : 4;
  s->BH = (long long)p->B * p->NH;
  if (s->BH > 0x7fffffffLL || (long long)s->S * s->BH > (1LL << 40)) return MLSTM_ERR_SHAPE;
  if (!bwd_supported(s->dk, s->dv, s->dtype)) return MLSTM_ERR_SHAPE;
  return MLSTM_OK;
}

}  // namespace

extern "C" {

int mlstm_abi_version(void) { return (2 << 16) | 3; }

const char* mlstm_status_string(mlstm_status_t s) {
  switch (s) {
    case MLSTM_OK: return "ok";
    case MLSTM_ERR_NULL: return "a required pointer is NULL";
    case MLSTM_ERR_SHAPE: return "a size is negative, inconsistent or unsupported";
    case MLSTM_ERR_DTYPE: return "unsupported dtype";
    case MLSTM_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case MLSTM_ERR_WORKSPACE: return "workspace missing or too small";
    case MLSTM_ERR_CUDA: return "CUDA runtime error at launch";
    case MLSTM_ERR_ALIAS: return "an output overlaps an input";
    case MLSTM_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case MLSTM_ERR_BOUNDS: return "an access failed its bounds check and was skipped";
  }
  return "unknown status";
}

size_t mlstm_fwd_chunkwise_workspace_size(const mlstm_fwd_params_t* p) {
  FwdShape s;
  if (check_fwd(p, &s) != MLSTM_OK) return 0;
  return fwd_layout(s).total;
}

mlstm_status_t mlstm_fwd_chunkwise_plan(const mlstm_fwd_params_t* p, mlstm_fwd_plan_t* plan) {
  if (!plan) return MLSTM_ERR_NULL;
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  memset(plan, 0, sizeof(*plan));
  if (s.tc) {
    plan->tensor_core = 1;
    plan->segments = s.tcp.G;
    plan->dv_tile = s.tcp.dvt;
    plan->ctas_main = (int)(s.tcp.n_tiles * s.tcp.G * s.BH * s.nb);
    plan->kernels = (s.BH == 0 || s.S == 0) ? 0 : (s.tcp.G > 1 ? 3 : 2);
    plan->workspace_bytes = fwd_layout(s).total;
    plan->seg0_chunks = s.tcp.seg0_chunks;
    plan->seg_chunks = s.tcp.seg_chunks;
    plan->summary_units = s.tcp.NU;
    return MLSTM_OK;
  }
  plan->tensor_core = 0;
  plan->segments = 1;
  plan->dv_tile = simt_walk_pick_tile(s.chunk, s.dk, s.dv);
  plan->ctas_main = plan->dv_tile > 0 ? (int)(((s.dv + plan->dv_tile - 1) / plan->dv_tile) * s.BH * s.nb) : 0;
  plan->kernels = (s.BH == 0 || s.S == 0) ? 0 : (s.retention ? 1 : 2);
  plan->workspace_bytes = fwd_layout(s).total;
  return MLSTM_OK;
}

mlstm_status_t mlstm_fwd_chunkwise(const mlstm_fwd_params_t* p, const void* q, const void* k, const void* v,
                                   const float* igate, const float* fgate, const void* ogate, const float* C0,
                                   const float* n0, const float* m0, void* h, float* C_out, float* n_out,
                                   float* m_out, void* workspace, size_t workspace_bytes, mlstm_stream_t stream) {
  return fwd_impl(p, q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, workspace, workspace_bytes,
                  (cudaStream_t)stream, nullptr, nullptr);
}

mlstm_status_t mlstm_fwd_chunkwise_timed(const mlstm_fwd_params_t* p, const void* q, const void* k, const void* v,
                                         const float* igate, const float* fgate, const void* ogate, const float* C0,
                                         const float* n0, const float* m0, void* h, float* C_out, float* n_out,
                                         float* m_out, void* workspace, size_t workspace_bytes,
                                         mlstm_stream_t stream, mlstm_event_t main_begin, mlstm_event_t main_end) {
  return fwd_impl(p, q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, workspace, workspace_bytes,
                  (cudaStream_t)stream, (cudaEvent_t)main_begin, (cudaEvent_t)main_end);
}

// Error word of the tensor-core kernels (0 = every bounded wait succeeded), read after the
// stream's work has finished.  `ws` is the forward's workspace (its error word comes first).
static mlstm_status_t read_error_word(const FwdShape& s, const void* ws, cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MLSTM_ERR_CUDA;
  if (!s.tc || s.BH == 0 || s.S == 0) return MLSTM_OK;  // no bounded waits ran
  unsigned int word = 0;
  const char* base = static_cast<const char*>(ws) + fwd_layout(s).tc;
  if (cudaMemcpy(&word, base, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MLSTM_ERR_CUDA;
  // bits 0, 1: a wait ran out (segment summaries, walk); bit 2: a bounds check failed
  return word == 0 ? MLSTM_OK : (word & 4u) ? MLSTM_ERR_BOUNDS : MLSTM_ERR_TIMEOUT;
}

mlstm_status_t mlstm_fwd_chunkwise_status(const mlstm_fwd_params_t* p, const void* workspace,
                                          mlstm_stream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  if (s.tc && s.BH > 0 && s.S > 0 && !workspace) return MLSTM_ERR_NULL;
  return read_error_word(s, workspace, (cudaStream_t)stream);
}

int mlstm_bounds_checked(void) { return mlstm::kBoundsChecked ? 1 : 0; }

mlstm_status_t mlstm_fwd_chunkwise_bounds_record(const mlstm_fwd_params_t* p, const void* workspace,
                                                 mlstm_stream_t stream, int* site, long long* index,
                                                 long long* extent) {
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  if (s.tc && s.BH > 0 && s.S > 0 && !workspace) return MLSTM_ERR_NULL;
  mlstm::BoundsRecord r = {};
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLSTM_ERR_CUDA;
  if (mlstm::kBoundsChecked && s.tc && s.BH > 0 && s.S > 0) {
    const char* base = static_cast<const char*>(workspace) + fwd_layout(s).tc + 16;
    if (cudaMemcpy(&r, base, sizeof(r), cudaMemcpyDeviceToHost) != cudaSuccess) return MLSTM_ERR_CUDA;
  }
  if (site) *site = r.count ? r.site : 0;
  if (index) *index = r.count ? r.index : 0;
  if (extent) *extent = r.count ? r.extent : 0;
  return MLSTM_OK;
}

// Workspace of the reversed-sequence pass: the forward's, then reversed copies of the
// inputs and of h.
struct RevLayout {
  size_t fwd, q, k, v, o, ig, fg, h, total;
};
RevLayout rev_layout(const FwdShape& s) {
  RevLayout r = {};
  const size_t tok = (size_t)s.BH * s.S;
  const size_t bq = tok * s.DHQK * s.esize, bv = tok * s.DHV * s.esize, bg = tok * sizeof(float);
  r.fwd = 0;  // the forward's own workspace comes first
  size_t off = align_up(fwd_layout(s).total);
  r.q = off;
  off = align_up(off + bq);
  r.k = off;
  off = align_up(off + bq);
  r.v = off;
  off = align_up(off + bv);
  if (!s.retention) {
    r.o = off;
    off = align_up(off + bv);
    r.ig = off;
    off = align_up(off + bg);
    r.fg = off;
    off = align_up(off + bg);
  }
  r.h = off;
  off = align_up(off + bv);
  r.total = off;
  return r;
}

size_t mlstm_fwd_chunkwise_reversed_workspace_size(const mlstm_fwd_params_t* p) {
  FwdShape s;
  if (check_fwd(p, &s) != MLSTM_OK) return 0;
  // the tensor-core kernels read the sequence backwards in place; the SIMT path runs on copies
  return s.BH == 0 || s.S == 0 || s.tc ? fwd_layout(s).total : rev_layout(s).total;
}

mlstm_status_t mlstm_fwd_chunkwise_reversed(const mlstm_fwd_params_t* p, const void* q, const void* k,
                                            const void* v, const float* igate, const float* fgate,
                                            const void* ogate, const float* C0, const float* n0, const float* m0,
                                            void* h, float* C_out, float* n_out, float* m_out, void* workspace,
                                            size_t workspace_bytes, mlstm_stream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  if (s.BH == 0 || s.S == 0)  // nothing to reverse
    return fwd_impl(p, q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, workspace,
                    workspace_bytes, cs, nullptr, nullptr);
  if (s.tc)  // the tensor-core kernels take the chunks and their rows backwards, no copies
    return fwd_impl(p, q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, workspace,
                    workspace_bytes, cs, nullptr, nullptr, true, nullptr, nullptr, true);
  const RevLayout r = rev_layout(s);
  const size_t fwd_bytes = fwd_layout(s).total;
  // the caller's buffers, validated as for the forward (with the forward's part of the workspace)
  st = fwd_impl(p, q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, workspace,
                workspace_bytes, cs, nullptr, nullptr, false);
  if (st != MLSTM_OK) return st;
  if (!workspace || workspace_bytes < r.total) return MLSTM_ERR_WORKSPACE;
  const bool ret = s.retention != 0;
  if (ret) {
    igate = fgate = nullptr;
    ogate = nullptr;
  }
  const size_t tok = (size_t)s.BH * s.S;
  const size_t bq = tok * s.DHQK * s.esize, bv = tok * s.DHV * s.esize, bg = tok * sizeof(float);
  const size_t bC = (size_t)s.BH * s.nb * s.dv * s.dk * sizeof(float);
  const size_t bn = (size_t)s.BH * s.nb * s.dk * sizeof(float), bm = (size_t)s.BH * sizeof(float);
  const Range wsr{workspace, r.total};
  const Range user[] = {{q, bq},   {k, bq},    {v, bv},     {igate, bg}, {fgate, bg}, {ogate, bv}, {C0, bC},
                        {n0, bn},  {m0, bm},   {h, bv},     {C_out, bC}, {n_out, bn}, {m_out, bm}};
  for (const Range& u : user)
    if (overlaps(wsr, u)) return MLSTM_ERR_ALIAS;
  char* w = static_cast<char*>(workspace);
  void *qr = w + r.q, *kr = w + r.k, *vr = w + r.v, *hr = w + r.h;
  void* orv = (!ret && ogate) ? static_cast<void*>(w + r.o) : nullptr;
  float* igr = ret ? nullptr : reinterpret_cast<float*>(w + r.ig);
  float* fgr = ret ? nullptr : reinterpret_cast<float*>(w + r.fg);
  const long long BH = s.BH, S = s.S;
  cudaError_t e = launch_reverse_rows(q, qr, BH, S, (long long)s.DHQK * s.esize, cs);
  if (e == cudaSuccess) e = launch_reverse_rows(k, kr, BH, S, (long long)s.DHQK * s.esize, cs);
  if (e == cudaSuccess) e = launch_reverse_rows(v, vr, BH, S, (long long)s.DHV * s.esize, cs);
  if (e == cudaSuccess && orv) e = launch_reverse_rows(ogate, orv, BH, S, (long long)s.DHV * s.esize, cs);
  if (e == cudaSuccess && igr) e = launch_reverse_rows(igate, igr, BH, S, 4, cs);
  if (e == cudaSuccess && fgr) e = launch_reverse_rows(fgate, fgr, BH, S, 4, cs);
  if (e != cudaSuccess) return MLSTM_ERR_CUDA;
  st = fwd_impl(p, qr, kr, vr, igr, fgr, orv, C0, n0, m0, hr, C_out, n_out, m_out, w + r.fwd, fwd_bytes, cs, nullptr,
                nullptr);
  if (st != MLSTM_OK) return st;
  return launch_reverse_rows(hr, h, BH, S, (long long)s.DHV * s.esize, cs) == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}

// Workspace of the scalar-normaliser prefill (SIMT walk): per-token stabiliser and snapshots
// of m0 and of the per-head n0.
// On the tensor-core path (bf16, chunk 64, the shapes it covers) the walk's own workspace with
// per-head n0 instead.
static size_t scalar_norm_ws(const FwdShape& s) {
  if (s.BH == 0 || s.S == 0) return 0;
  if (s.tc) return fwd_layout(s, true).total;
  return align_up(sizeof(float) * (size_t)s.BH * s.S) + 2 * align_up(sizeof(float) * (size_t)s.BH);
}

size_t mlstm_fwd_chunkwise_scalar_normaliser_workspace_size(const mlstm_fwd_params_t* p) {
  FwdShape s;
  if (check_fwd(p, &s) != MLSTM_OK || p->retention) return 0;
  return scalar_norm_ws(s);
}

mlstm_status_t mlstm_fwd_chunkwise_scalar_normaliser(const mlstm_fwd_params_t* p, const void* q, const void* k,
                                                     const void* v, const float* igate, const float* fgate,
                                                     const void* ogate, const float* bias, const float* C0,
                                                     const float* n0, const float* m0, void* h, float* C_out,
                                                     float* n_out, float* m_out, void* workspace,
                                                     size_t workspace_bytes, mlstm_stream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  if (p->retention) return MLSTM_ERR_SHAPE;  // retention has no normaliser
  if (s.BH > 0 && s.S > 0 && !s.tc && simt_walk_pick_tile(s.chunk, s.dk, s.dv) == 0) return MLSTM_ERR_SHAPE;
  const size_t tok = (size_t)s.BH * s.S;
  const size_t bq = tok * s.DHQK * s.esize, bv = tok * s.DHV * s.esize, bg = tok * sizeof(float);
  const size_t bC = (size_t)s.BH * s.nb * s.dv * s.dk * sizeof(float), bh4 = (size_t)s.BH * sizeof(float);
  if (tok > 0 && (!q || !k || !v || !h || !igate || !fgate || !bias)) return MLSTM_ERR_NULL;
  const void* all[] = {q, k, v, igate, fgate, ogate, bias, C0, n0, m0, h, C_out, n_out, m_out, workspace};
  for (const void* ptr : all)
    if (ptr && misaligned(ptr)) return MLSTM_ERR_ALIGN;
  const size_t need = scalar_norm_ws(s);
  const Range inputs[] = {{q, bq}, {k, bq}, {v, bv}, {igate, bg}, {fgate, bg}, {ogate, bv}, {bias, (size_t)s.NH * 4}};
  const Range outs[] = {{h, bv}, {C_out, bC}, {n_out, bh4}, {m_out, bh4}, {workspace, need}};
  for (const Range& o : outs)
    for (const Range& i : inputs)
      if (overlaps(o, i)) return MLSTM_ERR_ALIAS;
  for (int a = 0; a < 5; ++a)
    for (int b = a + 1; b < 5; ++b)
      if (overlaps(outs[a], outs[b])) return MLSTM_ERR_ALIAS;
  const Range states_in[] = {{C0, bC}, {n0, bh4}, {m0, bh4}};
  for (int i = 0; i < 3; ++i) {
    if (overlaps(outs[0], states_in[i]) || overlaps(outs[4], states_in[i])) return MLSTM_ERR_ALIAS;
    for (int j = 1; j < 4; ++j) {
      const bool exact = outs[j].p == states_in[i].p && outs[j].n == states_in[i].n && j == i + 1;
      if (overlaps(outs[j], states_in[i]) && !exact) return MLSTM_ERR_ALIAS;
    }
  }
  if (need > 0 && (!workspace || workspace_bytes < need)) return MLSTM_ERR_WORKSPACE;
  if (s.BH == 0) return MLSTM_OK;
  cudaStream_t cs = (cudaStream_t)stream;
  if (s.tc && s.S > 0)  // tensor-core kernels with the scalar normaliser
    return fwd_impl(p, q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, workspace,
                    workspace_bytes, cs, nullptr, nullptr, true, nullptr, bias);
  cudaError_t e = cudaSuccess;
  if (s.S == 0) {  // the final state is the initial state
    if (C_out && C_out != C0)
      e = C0 ? cudaMemcpyAsync(C_out, C0, bC, cudaMemcpyDeviceToDevice, cs) : cudaMemsetAsync(C_out, 0, bC, cs);
    if (e == cudaSuccess && n_out && n_out != n0)
      e = n0 ? cudaMemcpyAsync(n_out, n0, bh4, cudaMemcpyDeviceToDevice, cs) : cudaMemsetAsync(n_out, 0, bh4, cs);
    if (e == cudaSuccess && m_out && m_out != m0)
      e = m0 ? cudaMemcpyAsync(m_out, m0, bh4, cudaMemcpyDeviceToDevice, cs) : cudaMemsetAsync(m_out, 0, bh4, cs);
    return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
  }
  char* w = static_cast<char*>(workspace);
  float* m_tok = reinterpret_cast<float*>(w);
  float* m_init = reinterpret_cast<float*>(w + align_up(sizeof(float) * tok));
  float* n_init = reinterpret_cast<float*>(w + align_up(sizeof(float) * tok) + align_up(bh4));
  e = launch_gate_prep((int)s.BH, s.S, 1, igate, fgate, m0, n0, m_tok, m_init, n_init, cs);
  if (e != cudaSuccess) return MLSTM_ERR_CUDA;
  WalkArgs a;
  memset(&a, 0, sizeof(a));
  a.B = s.B;
  a.NH = s.NH;
  a.S = s.S;
  a.DHQK = s.DHQK;
  a.DHV = s.DHV;
  a.chunk = s.chunk;
  a.nb = s.nb;
  a.retention = 0;
  a.dk = s.dk;
  a.dv = s.dv;
  a.dtype = s.dtype;
  a.q = q;
  a.k = k;
  a.v = v;
  a.og = ogate;
  a.ig = igate;
  a.fg = fgate;
  a.C0 = C0;
  a.n_init = n_init;
  a.m_init = m_init;
  a.m_tok = m_tok;
  a.nbias = bias;
  a.h = h;
  a.C_out = C_out;
  a.n_out = n_out;
  a.m_out = m_out;
  a.dv_tile = simt_walk_pick_tile(s.chunk, s.dk, s.dv);
  return launch_simt_walk(a, cs) == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}

size_t mlstm_bwd_workspace_size(const mlstm_fwd_params_t* p) {
  FwdShape s;
  if (check_bwd(p, &s) != MLSTM_OK) return 0;
  return bwd_workspace_bytes(s.BH, s.S, s.nb);
}

mlstm_status_t mlstm_bwd(const mlstm_fwd_params_t* p, const void* q, const void* k, const void* v,
                         const float* igate, const float* fgate, const void* ogate, const float* C0,
                         const float* n0, const float* m0, const void* dh, const float* dC, const float* dn,
                         float* dq, float* dk, float* dv, float* digate, float* dfgate, float* dogate,
                         float* dC0, float* dn0, float* dm0, void* workspace, size_t workspace_bytes,
                         mlstm_stream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_bwd(p, &s);
  if (st != MLSTM_OK) return st;
  const bool ret = s.retention != 0;
  if (ret) {
    igate = fgate = nullptr;
    ogate = nullptr;
    n0 = m0 = dn = nullptr;
    digate = dfgate = dogate = dn0 = dm0 = nullptr;
  }
  if (!ogate) dogate = nullptr;
  const size_t BH = (size_t)s.BH, S = (size_t)s.S;
  const bool work = BH > 0 && S > 0;
  if (work) {
    if (!q || !k || !v || !dh || !dq || !dk || !dv) return MLSTM_ERR_NULL;
    if (!ret && (!igate || !fgate)) return MLSTM_ERR_NULL;
  }
  const void* all[] = {q,  k,  v,  igate,  fgate,  ogate,  C0,  n0,  m0,  dh,  dC,
                       dn, dq, dk, dv, digate, dfgate, dogate, dC0, dn0, dm0, workspace};
  for (const void* ptr : all)
    if (ptr && misaligned(ptr)) return MLSTM_ERR_ALIGN;
  const size_t es = s.esize, nbs = BH * s.nb;
  const size_t cbytes = nbs * s.dv * s.dk * 4, nbytes = nbs * s.dk * 4;
  const Range ins[] = {{q, BH * S * s.DHQK * es}, {k, BH * S * s.DHQK * es}, {v, BH * S * s.DHV * es},
                       {igate, BH * S * 4},       {fgate, BH * S * 4},       {ogate, BH * S * s.DHV * es},
                       {C0, cbytes},              {n0, nbytes},              {m0, BH * 4},
                       {dh, BH * S * s.DHV * es}, {dC, cbytes},              {dn, nbytes}};
  const Range outs[] = {{dq, BH * S * s.DHQK * 4}, {dk, BH * S * s.DHQK * 4}, {dv, BH * S * s.DHV * 4},
                        {digate, BH * S * 4},      {dfgate, BH * S * 4},      {dogate, BH * S * s.DHV * 4},
                        {dC0, cbytes},             {dn0, nbytes},             {dm0, BH * 4}};
  const int nout = (int)(sizeof(outs) / sizeof(outs[0]));
  const size_t need = bwd_workspace_bytes(s.BH, s.S, s.nb);
  const Range rws{need > 0 ? workspace : nullptr, need};
  for (int a = 0; a < nout; ++a) {
    for (const Range& i : ins)
      if (overlaps(outs[a], i)) return MLSTM_ERR_ALIAS;
    for (int b = a + 1; b < nout; ++b)
      if (overlaps(outs[a], outs[b])) return MLSTM_ERR_ALIAS;
    if (overlaps(outs[a], rws)) return MLSTM_ERR_ALIAS;
  }
  // (an empty sequence still needs it: the cluster kernel keeps each block's final-state terms
  // there for the gate-gradient kernel)
  if (need > 0 && (!workspace || workspace_bytes < need)) return MLSTM_ERR_WORKSPACE;
  cudaStream_t cs = (cudaStream_t)stream;
  if (BH == 0) return MLSTM_OK;  // with S == 0 the kernel still forms the initial-state gradients
  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.B = s.B;
  a.NH = s.NH;
  a.S = s.S;
  a.DHQK = s.DHQK;
  a.DHV = s.DHV;
  a.nb = s.nb;
  a.retention = s.retention;
  a.dtype = s.dtype;
  a.dk = s.dk;
  a.dv = s.dv;
  a.q = q;
  a.k = k;
  a.v = v;
  a.og = ogate;
  a.dh = dh;
  a.ig = igate;
  a.fg = fgate;
  a.C0 = C0;
  a.n0 = n0;
  a.m0 = m0;
  a.dC = dC;
  a.dn = dn;
  a.dq = dq;
  a.dk_out = dk;
  a.dv_out = dv;
  a.dig = digate;
  a.dfg = dfgate;
  a.dog = dogate;
  a.dC0 = dC0;
  a.dn0 = dn0;
  a.dm0 = dm0;
  a.ws = static_cast<float*>(workspace);
  return launch_bwd(a, cs) == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}

mlstm_status_t mlstm_step(const mlstm_step_params_t* p, const void* q, const void* k, const void* v,
                          const float* igate, const float* fgate, const void* ogate, float* C, float* n, float* m,
                          void* h, mlstm_stream_t stream) {
  if (!p) return MLSTM_ERR_NULL;
  if (p->dtype != MLSTM_F32 && p->dtype != MLSTM_BF16) return MLSTM_ERR_DTYPE;
  if (p->B < 0 || p->NH < 0 || p->DHQK < 1 || p->DHV < 1 || p->num_blocks < 1) return MLSTM_ERR_SHAPE;
  if (p->DHQK % p->num_blocks || p->DHV % p->num_blocks || p->num_blocks > 8) return MLSTM_ERR_SHAPE;
  const int dk = p->DHQK / p->num_blocks, dv = p->DHV / p->num_blocks;
  if (!step_supported_dk(dk)) return MLSTM_ERR_SHAPE;
  const long long BHll = (long long)p->B * p->NH;
  if (BHll * 8 > (1LL << 31) - 1) return MLSTM_ERR_SHAPE;
  const size_t BH = (size_t)BHll;
  const bool ret = p->retention != 0;
  if (ret) {
    igate = fgate = nullptr;
    ogate = nullptr;
    n = m = nullptr;
  }
  if (BH > 0) {
    if (!q || !k || !v || !C || !h) return MLSTM_ERR_NULL;
    if (!ret && (!igate || !fgate || !n || !m)) return MLSTM_ERR_NULL;
  }
  const void* all[] = {q, k, v, igate, fgate, ogate, C, n, m, h};
  for (const void* ptr : all)
    if (ptr && misaligned(ptr)) return MLSTM_ERR_ALIGN;
  const size_t es = p->dtype == MLSTM_BF16 ? 2 : 4;
  const Range rq{q, BH * p->DHQK * es}, rk{k, BH * p->DHQK * es}, rv{v, BH * p->DHV * es};
  const Range rig{igate, BH * 4}, rfg{fgate, BH * 4}, ro{ogate, BH * p->DHV * es};
  const Range rC{C, (size_t)BH * p->num_blocks * dv * dk * 4}, rn{n, (size_t)BH * p->num_blocks * dk * 4};
  const Range rm{m, BH * 4}, rh{h, BH * p->DHV * es};
  const Range ins[] = {rq, rk, rv, rig, rfg, ro};
  const Range outs[] = {rC, rn, rm, rh};
  for (int a = 0; a < 4; ++a) {
    for (const Range& i : ins)
      if (overlaps(outs[a], i)) return MLSTM_ERR_ALIAS;
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a], outs[b])) return MLSTM_ERR_ALIAS;
  }
  if (BH == 0) return MLSTM_OK;
  StepArgs a;
  memset(&a, 0, sizeof(a));
  a.B = p->B;
  a.NH = p->NH;
  a.DHQK = p->DHQK;
  a.DHV = p->DHV;
  a.nb = p->num_blocks;
  a.retention = ret ? 1 : 0;
  a.dtype = p->dtype == MLSTM_BF16 ? 1 : 0;
  a.dk = dk;
  a.dv = dv;
  a.q = q;
  a.k = k;
  a.v = v;
  a.og = ogate;
  a.ig = igate;
  a.fg = fgate;
  a.C = C;
  a.n = n;
  a.m = m;
  a.h = h;
  return launch_step(a, (cudaStream_t)stream) == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}


mlstm_status_t mlstm_theta_rotate(const mlstm_fwd_params_t* p, const void* q, const void* k, const long long* pos0,
                                  float theta_base, void* q_out, void* k_out, cudaStream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_dims(p, &s);
  if (st != MLSTM_OK) return st;
  if (!theta_rotate_supported(s.DHQK, s.dtype) || !(theta_base > 0.f) || !finite_nonneg(theta_base))
    return MLSTM_ERR_SHAPE;
  const size_t bq = (size_t)s.BH * s.S * s.DHQK * s.esize;
  if (bq == 0) return MLSTM_OK;
  if (!q || !k || !q_out || !k_out) return MLSTM_ERR_NULL;
  const void* all[] = {q, k, q_out, k_out, pos0};
  for (const void* ptr : all)
    if (ptr && ((uintptr_t)ptr & (ptr == pos0 ? 7 : 15))) return MLSTM_ERR_ALIGN;
  const Range rq{q, bq}, rk{k, bq}, oq{q_out, bq}, ok{k_out, bq}, rp{pos0, (size_t)s.B * 8};
  // in place only exactly (q_out == q, k_out == k); no other overlap
  if ((overlaps(oq, rq) && q_out != q) || overlaps(oq, rk) || overlaps(ok, rq) || (overlaps(ok, rk) && k_out != k) ||
      overlaps(oq, ok) || overlaps(oq, rp) || overlaps(ok, rp))
    return MLSTM_ERR_ALIAS;
  return launch_theta_rotate(s.B, s.NH, s.S, s.DHQK, s.dtype, q, k, q_out, k_out, pos0, theta_base,
                             (cudaStream_t)stream) == cudaSuccess
             ? MLSTM_OK
             : MLSTM_ERR_CUDA;
}

mlstm_status_t mlstm_group_norm_gate(const mlstm_fwd_params_t* p, const void* h, const void* g, const float* weight,
                                     const float* bias, float eps, void* y, cudaStream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_dims(p, &s);
  if (st != MLSTM_OK) return st;
  if (!gn_gate_supported(s.DHV, s.dtype) || !finite_nonneg(eps)) return MLSTM_ERR_SHAPE;
  const size_t bv = (size_t)s.BH * s.S * s.DHV * s.esize, bw = (size_t)s.NH * s.DHV * sizeof(float);
  if (bv == 0) return MLSTM_OK;
  if (!h || !y) return MLSTM_ERR_NULL;
  const void* all[] = {h, g, weight, bias, y};
  for (const void* ptr : all)
    if (ptr && misaligned(ptr)) return MLSTM_ERR_ALIGN;
  const Range rh{h, bv}, ry{y, bv}, rg{g, bv}, rw{weight, bw}, rb{bias, bw};
  if ((overlaps(ry, rh) && y != h) || overlaps(ry, rg) || overlaps(ry, rw) || overlaps(ry, rb)) return MLSTM_ERR_ALIAS;
  return launch_gn_gate((long long)s.BH * s.S, s.NH, s.S, s.DHV, s.dtype, h, g, weight, bias, eps, y,
                        (cudaStream_t)stream) == cudaSuccess
             ? MLSTM_OK
             : MLSTM_ERR_CUDA;
}

size_t mlstm_fwd_chunkwise_msr_workspace_size(const mlstm_fwd_params_t* p) {
  FwdShape s;
  if (check_fwd(p, &s) != MLSTM_OK) return 0;
  return msr_layout(s).total;
}

mlstm_status_t mlstm_fwd_chunkwise_msr(const mlstm_fwd_params_t* p, const void* q, const void* k, const void* v,
                                       const float* igate, const float* fgate, const long long* pos0,
                                       float theta_base, const void* g, const float* gn_weight,
                                       const float* gn_bias, float eps, const float* C0, const float* n0,
                                       const float* m0, void* y, float* C_out, float* n_out, float* m_out,
                                       void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  if (!theta_rotate_supported(s.DHQK, s.dtype) || !gn_gate_supported(s.DHV, s.dtype) || !(theta_base > 0.f) ||
      !finite_nonneg(theta_base) || !finite_nonneg(eps))
    return MLSTM_ERR_SHAPE;
  const MsrLayout r = msr_layout(s);
  const size_t tok = (size_t)s.BH * s.S;
  const size_t bq = tok * s.DHQK * s.esize, bv = tok * s.DHV * s.esize, bw = (size_t)s.NH * s.DHV * sizeof(float);
  if (tok > 0 && (!q || !k)) return MLSTM_ERR_NULL;
  const void* extra[] = {g, gn_weight, gn_bias, workspace};
  for (const void* ptr : extra)
    if (ptr && misaligned(ptr)) return MLSTM_ERR_ALIGN;
  if (pos0 && ((uintptr_t)pos0 & 7)) return MLSTM_ERR_ALIGN;
  // the block's own inputs must not overlap what the forward writes (y, state, workspace)
  const size_t bC = (size_t)s.BH * s.nb * s.dv * s.dk * sizeof(float);
  const size_t bn = s.retention ? 0 : (size_t)s.BH * s.nb * s.dk * sizeof(float), bm = s.retention ? 0 : (size_t)s.BH * 4;
  const Range outs[] = {{y, bv}, {C_out, bC}, {n_out, bn}, {m_out, bm}, {workspace, r.total}};
  const Range ins[] = {{g, bv}, {gn_weight, bw}, {gn_bias, bw}, {pos0, (size_t)s.B * 8}, {q, bq}, {k, bq}};
  for (const Range& o : outs)
    for (const Range& i : ins)
      if (overlaps(o, i)) return MLSTM_ERR_ALIAS;
  if (r.total > 0 && (!workspace || workspace_bytes < r.total)) return MLSTM_ERR_WORKSPACE;
  char* w = static_cast<char*>(workspace);
  void* qr = tok ? w + r.qr : nullptr;
  void* kr = tok ? w + r.kr : nullptr;
  // validate the forward (with the rotated copies as its q, k) before launching anything
  const GnArgs gn{g, gn_weight, gn_bias, eps};
  st = fwd_impl(p, qr, kr, v, igate, fgate, nullptr, C0, n0, m0, y, C_out, n_out, m_out, w ? w + r.fwd : nullptr,
                workspace_bytes > r.fwd ? workspace_bytes - r.fwd : 0, (cudaStream_t)stream, nullptr, nullptr, false,
                &gn);
  if (st != MLSTM_OK || s.BH == 0) return st;
  if (s.S > 0 && launch_theta_rotate(s.B, s.NH, s.S, s.DHQK, s.dtype, q, k, qr, kr, pos0, theta_base,
                                     (cudaStream_t)stream) != cudaSuccess)
    return MLSTM_ERR_CUDA;
  return fwd_impl(p, qr, kr, v, igate, fgate, nullptr, C0, n0, m0, y, C_out, n_out, m_out, w + r.fwd,
                  workspace_bytes - r.fwd, (cudaStream_t)stream, nullptr, nullptr, true, &gn);
}


size_t mlstm_gdn2_workspace_size(const mlstm_gdn2_params_t* p) {
  if (!p || p->mode != MLSTM_GDN2_CHUNK || p->B < 0 || p->H < 0 || p->T < 0 || p->K < 1) return 0;
  if (p->chunk < 4 || p->chunk > 64 || p->chunk % 4) return 0;
  if (gdn2_tc_supported(p->chunk, p->K, p->V, p->dtype == MLSTM_BF16 ? 1 : 0, p->T))
    return gdn2_tc_workspace_bytes((long long)p->B * p->H, p->T, p->V);
  return gdn2_chunk_workspace_bytes((long long)p->B * p->H, p->T, p->chunk, p->K);
}

mlstm_status_t mlstm_gdn2_status(const mlstm_gdn2_params_t* p, const void* workspace, mlstm_stream_t stream) {
  if (!p) return MLSTM_ERR_NULL;
  if (p->dtype != MLSTM_F32 && p->dtype != MLSTM_BF16) return MLSTM_ERR_DTYPE;
  if (p->B < 0 || p->H < 0 || p->T < 0 || p->K < 1 || p->V < 1) return MLSTM_ERR_SHAPE;
  if (p->mode != MLSTM_GDN2_RECURRENT && p->mode != MLSTM_GDN2_CHUNK) return MLSTM_ERR_SHAPE;
  const bool tc = p->mode == MLSTM_GDN2_CHUNK && (long long)p->B * p->H > 0 &&
                  gdn2_tc_supported(p->chunk, p->K, p->V, p->dtype == MLSTM_BF16 ? 1 : 0, p->T);
  if (tc && !workspace) return MLSTM_ERR_NULL;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLSTM_ERR_CUDA;
  if (!tc) return MLSTM_OK;  // no bounded waits ran
  unsigned int word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MLSTM_ERR_CUDA;
  return word == 0 ? MLSTM_OK : (word & 4u) ? MLSTM_ERR_BOUNDS : MLSTM_ERR_TIMEOUT;
}

mlstm_status_t mlstm_gdn2_fwd(const mlstm_gdn2_params_t* p, const void* q, const void* k, const void* v,
                              const float* g, const float* b, const float* w, const float* S0, void* o,
                              float* S_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!p) return MLSTM_ERR_NULL;
  if (p->dtype != MLSTM_F32 && p->dtype != MLSTM_BF16) return MLSTM_ERR_DTYPE;
  if (p->B < 0 || p->H < 0 || p->T < 0 || p->K < 1 || p->V < 1) return MLSTM_ERR_SHAPE;
  if (p->mode != MLSTM_GDN2_RECURRENT && p->mode != MLSTM_GDN2_CHUNK) return MLSTM_ERR_SHAPE;
  const long long BH = (long long)p->B * p->H;
  if (BH > 65535 || (long long)p->T * BH > (1LL << 40)) return MLSTM_ERR_SHAPE;
  if (p->mode == MLSTM_GDN2_RECURRENT ? !gdn2_recurrent_supported(p->K) : gdn2_chunk_vtile(p->chunk, p->K, p->V) == 0)
    return MLSTM_ERR_SHAPE;
  const size_t es = p->dtype == MLSTM_BF16 ? 2 : 4, tok = (size_t)BH * p->T;
  const size_t bq = tok * p->K * es, bv = tok * p->V * es, bg = tok * p->K * 4, bw = tok * p->V * 4;
  const size_t bS = (size_t)BH * p->K * p->V * 4;
  if (tok > 0 && (!q || !k || !v || !g || !b || !w || !o)) return MLSTM_ERR_NULL;
  const void* all[] = {q, k, v, g, b, w, S0, o, S_out, workspace};
  for (const void* ptr : all)
    if (ptr && misaligned(ptr)) return MLSTM_ERR_ALIGN;
  const size_t need = mlstm_gdn2_workspace_size(p);
  const Range ins[] = {{q, bq}, {k, bq}, {v, bv}, {g, bg}, {b, bg}, {w, bw}};
  const Range ro{o, bv}, rS{S_out, bS}, r0{S0, bS}, rw{workspace, need};
  for (const Range& i : ins)
    if (overlaps(ro, i) || overlaps(rS, i) || overlaps(rw, i)) return MLSTM_ERR_ALIAS;
  if (overlaps(ro, rS) || overlaps(ro, r0) || (overlaps(rS, r0) && S_out != S0)) return MLSTM_ERR_ALIAS;
  if (overlaps(rw, ro) || overlaps(rw, rS) || overlaps(rw, r0)) return MLSTM_ERR_ALIAS;
  if (need > 0 && (!workspace || workspace_bytes < need)) return MLSTM_ERR_WORKSPACE;
  if (BH == 0) return MLSTM_OK;
  Gdn2Args a;
  a.B = p->B, a.H = p->H, a.T = p->T, a.K = p->K, a.V = p->V, a.dtype = p->dtype == MLSTM_BF16 ? 1 : 0;
  a.wait = p->wait_limit_cycles > 0 ? p->wait_limit_cycles : 0;
  a.nsm = 0;
  a.q = q, a.k = k, a.v = v, a.g = g, a.b = b, a.w = w, a.S0 = S0, a.o = o, a.S_out = S_out;
  if (p->T == 0) {  // the final state is the initial state
    cudaError_t e = cudaSuccess;
    if (S_out && S_out != S0)
      e = S0 ? cudaMemcpyAsync(S_out, S0, bS, cudaMemcpyDeviceToDevice, (cudaStream_t)stream)
             : cudaMemsetAsync(S_out, 0, bS, (cudaStream_t)stream);
    return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
  }
  if (p->mode == MLSTM_GDN2_CHUNK && gdn2_tc_supported(p->chunk, p->K, p->V, a.dtype, p->T))
    return launch_gdn2_tc(a, workspace, (cudaStream_t)stream) == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
  return launch_gdn2(a, p->mode, p->chunk, workspace, (cudaStream_t)stream) == cudaSuccess ? MLSTM_OK
                                                                                             : MLSTM_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Prefill without a caller workspace.  Some callers cannot call cudaMalloc at all
// (their host framework owns every byte of device memory, or an allocation's implicit
// device synchronisation is not acceptable where they run), so this entry point takes
// its scratch memory from a fixed buffer compiled into the library instead.
//
// The buffer is a file-scope __device__ array: every GPU that loads the library holds
// MLSTM_NOALLOC_SCRATCH_BYTES of it until the process exits.  All calls share it and it
// keeps whatever the previous call left there; the kernels write every scratch byte they
// read except the error word, which each call clears on its stream.  Two calls whose
// GPU work overlaps (different streams, or different host threads) race on the buffer.
#include <mutex>

#define MLSTM_NOALLOC_SCRATCH_BYTES (32u << 20)

static __device__ __align__(256) unsigned char g_noalloc_scratch[MLSTM_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The host-side name of a
// __device__ array is only a stand-in, so the address is looked up once per device,
// with that device current, and cached.  (A cudaDeviceReset would make the cached
// address stale; the library's users do not reset devices while it is loaded.)
mlstm_status_t noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLSTM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MLSTM_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return MLSTM_OK;
}

}  // namespace

extern "C" {

size_t mlstm_noalloc_scratch_bytes(void) { return MLSTM_NOALLOC_SCRATCH_BYTES; }

mlstm_status_t mlstm_fwd_chunkwise_noalloc(const mlstm_fwd_params_t* p, const void* q, const void* k, const void* v,
                                           const float* igate, const float* fgate, const void* ogate,
                                           const float* C0, const float* n0, const float* m0, void* h, float* C_out,
                                           float* n_out, float* m_out, mlstm_stream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  const size_t need = fwd_layout(s).total;
  if (need > MLSTM_NOALLOC_SCRATCH_BYTES) return MLSTM_ERR_WORKSPACE;  // too large for the built-in buffer
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != MLSTM_OK) return st;
  return fwd_impl(p, q, k, v, igate, fgate, ogate, C0, n0, m0, h, C_out, n_out, m_out, scratch,
                  MLSTM_NOALLOC_SCRATCH_BYTES, (cudaStream_t)stream, nullptr, nullptr);
}

mlstm_status_t mlstm_fwd_chunkwise_noalloc_status(const mlstm_fwd_params_t* p, mlstm_stream_t stream) {
  FwdShape s;
  mlstm_status_t st = check_fwd(p, &s);
  if (st != MLSTM_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != MLSTM_OK) return st;
  return read_error_word(s, scratch, (cudaStream_t)stream);
}

}  // extern "C"
