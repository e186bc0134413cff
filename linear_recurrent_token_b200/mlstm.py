"""Python binding of libmlstm (include/mlstm.h): argument marshalling only.

Every step of the recurrence runs in the library's CUDA kernels.  PyTorch only
provides device memory (outputs and workspace are allocated here with
torch.empty when the caller does not pass them) and the current CUDA stream.
There is no CPU fallback: if the compiled library is missing or no CUDA device
is present, these functions raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmlstm.so")
# the bounds-checked debug build of the same library (include/mlstm.h, mlstm_bounds_checked)
LIB_CHECKED_PATH = os.path.join(_PKG, "libmlstm_checked.so")

MLSTM_F32, MLSTM_BF16 = 0, 1
_DTYPES = {torch.float32: MLSTM_F32, torch.bfloat16: MLSTM_BF16}


class FwdParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("NH", ctypes.c_int), ("S", ctypes.c_int), ("DHQK", ctypes.c_int),
                ("DHV", ctypes.c_int), ("chunk", ctypes.c_int), ("num_blocks", ctypes.c_int),
                ("dtype", ctypes.c_int), ("retention", ctypes.c_int), ("wait_limit_cycles", ctypes.c_longlong)]


class StepParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("NH", ctypes.c_int), ("DHQK", ctypes.c_int), ("DHV", ctypes.c_int),
                ("num_blocks", ctypes.c_int), ("dtype", ctypes.c_int), ("retention", ctypes.c_int)]


class Gdn2Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("K", ctypes.c_int),
                ("V", ctypes.c_int), ("dtype", ctypes.c_int), ("mode", ctypes.c_int), ("chunk", ctypes.c_int),
                ("wait_limit_cycles", ctypes.c_longlong)]


GDN2_RECURRENT, GDN2_CHUNK = 0, 1


class FwdPlan(ctypes.Structure):
    _fields_ = [("tensor_core", ctypes.c_int), ("segments", ctypes.c_int), ("dv_tile", ctypes.c_int),
                ("ctas_main", ctypes.c_int), ("kernels", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t),
                ("seg0_chunks", ctypes.c_int), ("seg_chunks", ctypes.c_int), ("summary_units", ctypes.c_int)]


class MlstmError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: status {status} ({status_string(status)})")
        self.status = status


_libs = {}
_use_checked = False


def lib():
    """The loaded libmlstm.so, or libmlstm_checked.so inside `with bounds_checked():` (raises if
    it has not been built)."""
    path = LIB_CHECKED_PATH if _use_checked else LIB_PATH
    if path not in _libs:
        _libs[path] = _load(path)
    return _libs[path]


@contextlib.contextmanager
def bounds_checked():
    """Every call made inside the block goes to libmlstm_checked.so, the bounds-checked debug
    build (its status calls return 9 = MLSTM_ERR_BOUNDS when a check failed; bounds_record
    says where).  Not thread-safe: it switches the library for the whole module."""
    global _use_checked
    prev = _use_checked
    _use_checked = True
    try:
        yield lib()
    finally:
        _use_checked = prev


def _load(path):
    """Loads one build of the library and declares the C signatures."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m linear_recurrent_token_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(path)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.mlstm_fwd_chunkwise_workspace_size.argtypes = [ctypes.POINTER(FwdParams)]
    L.mlstm_fwd_chunkwise_workspace_size.restype = Z
    L.mlstm_fwd_chunkwise_plan.argtypes = [ctypes.POINTER(FwdParams), ctypes.POINTER(FwdPlan)]
    L.mlstm_fwd_chunkwise_plan.restype = I
    L.mlstm_fwd_chunkwise.argtypes = [ctypes.POINTER(FwdParams)] + [P] * 14 + [Z, P]
    L.mlstm_fwd_chunkwise.restype = I
    L.mlstm_fwd_chunkwise_timed.argtypes = [ctypes.POINTER(FwdParams)] + [P] * 14 + [Z, P, P, P]
    L.mlstm_fwd_chunkwise_timed.restype = I
    L.mlstm_fwd_chunkwise_noalloc.argtypes = [ctypes.POINTER(FwdParams)] + [P] * 13 + [P]
    L.mlstm_fwd_chunkwise_noalloc.restype = I
    L.mlstm_fwd_chunkwise_status.argtypes = [ctypes.POINTER(FwdParams), P, P]
    L.mlstm_fwd_chunkwise_status.restype = I
    L.mlstm_fwd_chunkwise_noalloc_status.argtypes = [ctypes.POINTER(FwdParams), P]
    L.mlstm_fwd_chunkwise_noalloc_status.restype = I
    L.mlstm_bounds_checked.argtypes = []
    L.mlstm_bounds_checked.restype = I
    LL = ctypes.c_longlong
    L.mlstm_fwd_chunkwise_bounds_record.argtypes = [ctypes.POINTER(FwdParams), P, P, ctypes.POINTER(I),
                                                    ctypes.POINTER(LL), ctypes.POINTER(LL)]
    L.mlstm_fwd_chunkwise_bounds_record.restype = I
    L.mlstm_noalloc_scratch_bytes.argtypes = []
    L.mlstm_noalloc_scratch_bytes.restype = Z
    L.mlstm_fwd_chunkwise_reversed_workspace_size.argtypes = [ctypes.POINTER(FwdParams)]
    L.mlstm_fwd_chunkwise_reversed_workspace_size.restype = Z
    L.mlstm_fwd_chunkwise_reversed.argtypes = [ctypes.POINTER(FwdParams)] + [P] * 14 + [Z, P]
    L.mlstm_fwd_chunkwise_reversed.restype = I
    L.mlstm_fwd_chunkwise_scalar_normaliser_workspace_size.argtypes = [ctypes.POINTER(FwdParams)]
    L.mlstm_fwd_chunkwise_scalar_normaliser_workspace_size.restype = Z
    L.mlstm_fwd_chunkwise_scalar_normaliser.argtypes = [ctypes.POINTER(FwdParams)] + [P] * 15 + [Z, P]
    L.mlstm_fwd_chunkwise_scalar_normaliser.restype = I
    F = ctypes.c_float
    L.mlstm_theta_rotate.argtypes = [ctypes.POINTER(FwdParams), P, P, P, F, P, P, P]
    L.mlstm_theta_rotate.restype = I
    L.mlstm_group_norm_gate.argtypes = [ctypes.POINTER(FwdParams), P, P, P, P, F, P, P]
    L.mlstm_group_norm_gate.restype = I
    L.mlstm_fwd_chunkwise_msr_workspace_size.argtypes = [ctypes.POINTER(FwdParams)]
    L.mlstm_fwd_chunkwise_msr_workspace_size.restype = Z
    L.mlstm_fwd_chunkwise_msr.argtypes = [ctypes.POINTER(FwdParams), P, P, P, P, P, P, F, P, P, P, F, P, P, P,
                                          P, P, P, P, P, Z, P]
    L.mlstm_fwd_chunkwise_msr.restype = I
    L.mlstm_gdn2_workspace_size.argtypes = [ctypes.POINTER(Gdn2Params)]
    L.mlstm_gdn2_workspace_size.restype = Z
    L.mlstm_gdn2_fwd.argtypes = [ctypes.POINTER(Gdn2Params)] + [P] * 10 + [Z, P]
    L.mlstm_gdn2_status.argtypes = [ctypes.POINTER(Gdn2Params), P, P]
    L.mlstm_gdn2_status.restype = I
    L.mlstm_gdn2_fwd.restype = I
    L.mlstm_bwd_workspace_size.argtypes = [ctypes.POINTER(FwdParams)]
    L.mlstm_bwd_workspace_size.restype = Z
    L.mlstm_bwd.argtypes = [ctypes.POINTER(FwdParams)] + [P] * 22 + [Z, P]
    L.mlstm_bwd.restype = I
    L.mlstm_step.argtypes = [ctypes.POINTER(StepParams)] + [P] * 10 + [P]
    L.mlstm_step.restype = I
    L.mlstm_status_string.argtypes = [I]
    L.mlstm_status_string.restype = ctypes.c_char_p
    L.mlstm_abi_version.argtypes = []
    L.mlstm_abi_version.restype = I
    return L


def status_string(status: int) -> str:
    return lib().mlstm_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}") from None


def fwd_params(B, NH, S, DHQK, DHV, chunk=64, num_blocks=1, dtype=torch.bfloat16, retention=False,
               wait_limit_cycles: int = 0) -> FwdParams:
    return FwdParams(int(B), int(NH), int(S), int(DHQK), int(DHV), int(chunk), int(num_blocks),
                     _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype), int(bool(retention)),
                     int(wait_limit_cycles))


def fwd_status(params: FwdParams, workspace=None, stream=None, noalloc: bool = False) -> int:
    """Outcome of the bounded device-side waits of the last prefill with these params and this
    workspace (mlstm_fwd_chunkwise_status; noalloc=True: of the last mlstm_fwd_chunkwise_noalloc,
    mlstm_fwd_chunkwise_noalloc_status).  Synchronises the stream.  Returns the status code:
    0 = ok, 8 = a wait ran out (MLSTM_ERR_TIMEOUT), 9 = a check of the bounds-checked build
    failed (MLSTM_ERR_BOUNDS)."""
    if noalloc:
        return int(lib().mlstm_fwd_chunkwise_noalloc_status(ctypes.byref(params), _stream_ptr(stream)))
    return int(lib().mlstm_fwd_chunkwise_status(ctypes.byref(params), _ptr(workspace), _stream_ptr(stream)))


def bounds_record(params: FwdParams, workspace, stream=None):
    """First failed check of the last prefill with this workspace in the bounds-checked build
    (mlstm_fwd_chunkwise_bounds_record): (site, index, extent), site 0 when none failed."""
    site, index, extent = ctypes.c_int(0), ctypes.c_longlong(0), ctypes.c_longlong(0)
    st = lib().mlstm_fwd_chunkwise_bounds_record(ctypes.byref(params), _ptr(workspace), _stream_ptr(stream),
                                                 ctypes.byref(site), ctypes.byref(index), ctypes.byref(extent))
    if st != 0:
        raise MlstmError(st, "mlstm_fwd_chunkwise_bounds_record")
    return site.value, index.value, extent.value


def workspace_size(params: FwdParams) -> int:
    return int(lib().mlstm_fwd_chunkwise_workspace_size(ctypes.byref(params)))


def plan(params: FwdParams) -> dict:
    out = FwdPlan()
    st = lib().mlstm_fwd_chunkwise_plan(ctypes.byref(params), ctypes.byref(out))
    if st != 0:
        raise MlstmError(st, "mlstm_fwd_chunkwise_plan")
    return {name: getattr(out, name) for name, _ in FwdPlan._fields_}


def fwd_chunkwise(q, k, v, igate=None, fgate=None, ogate=None, C0=None, n0=None, m0=None, *,
                  chunk: int = 64, num_blocks: int = 1, retention: bool = False,
                  h=None, C_out=None, n_out=None, m_out=None, workspace=None,
                  return_state: bool = True, stream=None, events=None, reverse: bool = False,
                  wait_limit_cycles: int = 0):
    """Chunkwise-parallel prefill (mlstm_fwd_chunkwise).  CUDA tensors, contiguous.

    q, k [B,NH,S,DHQK], v [B,NH,S,DHV] (fp32 or bf16); igate, fgate [B,NH,S] fp32;
    ogate [B,NH,S,DHV] or None; C0 [B,NH,nb,DHV/nb,DHQK/nb], n0 [B,NH,nb,DHQK/nb],
    m0 [B,NH] fp32 or None (zeros).  Returns (h, C, n, m); n, m are None in
    retention mode and the state is None when return_state is False.
    ``events`` = (begin, end) torch.cuda.Event pair recorded around the main kernel.
    ``reverse``: the reversed-sequence pass (mlstm_fwd_chunkwise_reversed): token S-1 first,
    h at the original positions, the final state after token 0.
    """
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = int(num_blocks)
    p = fwd_params(B, NH, S, DHQK, DHV, chunk, nb, q.dtype, retention, wait_limit_cycles)
    dev = q.device
    if h is None:
        h = torch.empty((B, NH, S, DHV), dtype=q.dtype, device=dev)
    if return_state and C_out is None:
        C_out = torch.empty((B, NH, nb, DHV // nb, DHQK // nb), dtype=torch.float32, device=dev)
    if return_state and not retention:
        if n_out is None:
            n_out = torch.empty((B, NH, nb, DHQK // nb), dtype=torch.float32, device=dev)
        if m_out is None:
            m_out = torch.empty((B, NH), dtype=torch.float32, device=dev)
    ws_bytes = reversed_workspace_size(p) if reverse else workspace_size(p)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = [ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(ogate),
            _ptr(C0), _ptr(n0), _ptr(m0), _ptr(h), _ptr(C_out), _ptr(n_out), _ptr(m_out),
            _ptr(workspace), ctypes.c_size_t(ws_len), _stream_ptr(stream)]
    if reverse:
        if events is not None:
            raise ValueError("events are not supported with reverse=True")
        st = lib().mlstm_fwd_chunkwise_reversed(*args)
        if st != 0:
            raise MlstmError(st, "mlstm_fwd_chunkwise_reversed")
        return (h, C_out, None, None) if retention else (h, C_out, n_out, m_out)
    if events is None:
        st = lib().mlstm_fwd_chunkwise(*args)
    else:
        for e in events:  # torch creates the CUDA event lazily, on its first record
            if e.cuda_event == 0:
                e.record(stream)
        st = lib().mlstm_fwd_chunkwise_timed(*args, ctypes.c_void_p(events[0].cuda_event),
                                             ctypes.c_void_p(events[1].cuda_event))
    if st != 0:
        raise MlstmError(st, "mlstm_fwd_chunkwise")
    if retention:
        return h, C_out, None, None
    return h, C_out, n_out, m_out


def fwd_chunkwise_scalar_normaliser(q, k, v, igate, fgate, bias, ogate=None, C0=None, n0=None, m0=None, *,
                                    chunk: int = 64, num_blocks: int = 1, workspace=None, stream=None):
    """The prefill with a scalar normaliser and a learnable bias
    (mlstm_fwd_chunkwise_scalar_normaliser): bias [NH] fp32, n0 [B,NH] fp32 or None.
    Returns (h, C, n [B,NH], m [B,NH])."""
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = int(num_blocks)
    p = fwd_params(B, NH, S, DHQK, DHV, chunk, nb, q.dtype, False)
    dev = q.device
    h = torch.empty((B, NH, S, DHV), dtype=q.dtype, device=dev)
    C_out = torch.empty((B, NH, nb, DHV // nb, DHQK // nb), dtype=torch.float32, device=dev)
    n_out = torch.empty((B, NH), dtype=torch.float32, device=dev)
    m_out = torch.empty((B, NH), dtype=torch.float32, device=dev)
    ws_bytes = int(lib().mlstm_fwd_chunkwise_scalar_normaliser_workspace_size(ctypes.byref(p)))
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mlstm_fwd_chunkwise_scalar_normaliser(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(ogate), _ptr(bias), _ptr(C0),
        _ptr(n0), _ptr(m0), _ptr(h), _ptr(C_out), _ptr(n_out), _ptr(m_out), _ptr(workspace), ctypes.c_size_t(ws_len),
        _stream_ptr(stream))
    if st != 0:
        raise MlstmError(st, "mlstm_fwd_chunkwise_scalar_normaliser")
    return h, C_out, n_out, m_out


def theta_rotate(q, k, pos0=None, theta_base: float = 10000.0, *, q_out=None, k_out=None, stream=None):
    """The rotation Theta of q and k by position (mlstm_theta_rotate): q, k [B,NH,S,DHQK];
    pos0 [B] int64 (position of token 0 of each sequence) or None.  q_out / k_out may be q / k
    (in place).  Returns (q_out, k_out)."""
    B, NH, S, DHQK = q.shape
    p = fwd_params(B, NH, S, DHQK, DHQK, 64, 1, q.dtype, True)
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    st = lib().mlstm_theta_rotate(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(pos0), ctypes.c_float(theta_base),
                                  _ptr(q_out), _ptr(k_out), _stream_ptr(stream))
    if st != 0:
        raise MlstmError(st, "mlstm_theta_rotate")
    return q_out, k_out


def group_norm_gate(h, g=None, weight=None, bias=None, eps: float = 1e-5, *, y=None, stream=None):
    """Per-head GroupNorm of h [B,NH,S,DHV] and the SiLU gate g (mlstm_group_norm_gate);
    weight, bias [NH*DHV] fp32 or None.  y may be h (in place).  Returns y."""
    B, NH, S, DHV = h.shape
    p = fwd_params(B, NH, S, DHV, DHV, 64, 1, h.dtype, True)
    y = torch.empty_like(h) if y is None else y
    st = lib().mlstm_group_norm_gate(ctypes.byref(p), _ptr(h), _ptr(g), _ptr(weight), _ptr(bias),
                                     ctypes.c_float(eps), _ptr(y), _stream_ptr(stream))
    if st != 0:
        raise MlstmError(st, "mlstm_group_norm_gate")
    return y


def msr_workspace_size(params: FwdParams) -> int:
    return int(lib().mlstm_fwd_chunkwise_msr_workspace_size(ctypes.byref(params)))


def fwd_chunkwise_msr(q, k, v, igate=None, fgate=None, g=None, gn_weight=None, gn_bias=None, C0=None, n0=None,
                      m0=None, *, pos0=None, theta_base: float = 10000.0, eps: float = 1e-5, chunk: int = 64,
                      num_blocks: int = 1, retention: bool = True, y=None, workspace=None, stream=None):
    """The multi-scale retention block in one call (mlstm_fwd_chunkwise_msr): rotate q, k,
    the recurrence, GroupNorm and the SiLU gate.  Returns (y, C, n, m); n, m None in
    retention mode."""
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = int(num_blocks)
    p = fwd_params(B, NH, S, DHQK, DHV, chunk, nb, q.dtype, retention)
    dev = q.device
    y = torch.empty((B, NH, S, DHV), dtype=q.dtype, device=dev) if y is None else y
    C_out = torch.empty((B, NH, nb, DHV // nb, DHQK // nb), dtype=torch.float32, device=dev)
    n_out = None if retention else torch.empty((B, NH, nb, DHQK // nb), dtype=torch.float32, device=dev)
    m_out = None if retention else torch.empty((B, NH), dtype=torch.float32, device=dev)
    ws_bytes = msr_workspace_size(p)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mlstm_fwd_chunkwise_msr(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(pos0), ctypes.c_float(theta_base),
        _ptr(g), _ptr(gn_weight), _ptr(gn_bias), ctypes.c_float(eps), _ptr(C0), _ptr(n0), _ptr(m0), _ptr(y),
        _ptr(C_out), _ptr(n_out), _ptr(m_out), _ptr(workspace), ctypes.c_size_t(ws_len), _stream_ptr(stream))
    if st != 0:
        raise MlstmError(st, "mlstm_fwd_chunkwise_msr")
    return y, C_out, n_out, m_out


def gdn2_workspace_size(params: Gdn2Params) -> int:
    return int(lib().mlstm_gdn2_workspace_size(ctypes.byref(params)))


def gdn2_params(q, v, mode: str = "recurrent", chunk: int = 64, wait_limit_cycles: int = 0) -> Gdn2Params:
    B, H, T, K = q.shape
    return Gdn2Params(int(B), int(H), int(T), int(K), int(v.shape[-1]), _dtype_code(q),
                      GDN2_CHUNK if mode == "chunk" else GDN2_RECURRENT, int(chunk), int(wait_limit_cycles))


def gdn2_status(q, v, workspace, *, mode: str = "chunk", chunk: int = 64, stream=None) -> int:
    """Outcome of the bounded waits of the last gdn2_fwd with this workspace (mlstm_gdn2_status;
    synchronises): 0 ok, 8 a wait ran out (MLSTM_ERR_TIMEOUT)."""
    p = gdn2_params(q, v, mode, chunk)
    return int(lib().mlstm_gdn2_status(ctypes.byref(p), _ptr(workspace), _stream_ptr(stream)))


def gdn2_fwd(q, k, v, g, b, w, S0=None, *, mode: str = "recurrent", chunk: int = 64, o=None, S_out=None,
             return_state: bool = True, workspace=None, stream=None, wait_limit_cycles: int = 0):
    """Gated DeltaNet-2 (mlstm_gdn2_fwd): q, k [B,H,T,K], v [B,H,T,V] (fp32 or bf16); g, b
    [B,H,T,K] and w [B,H,T,V] fp32; S0 [B,H,K,V] fp32 or None.  mode "recurrent" or "chunk".
    S_out may be S0 (in place: the decode step).  Returns (o, S_out)."""
    B, H, T, K = q.shape
    V = v.shape[-1]
    p = gdn2_params(q, v, mode, chunk, wait_limit_cycles)
    if o is None:
        o = torch.empty((B, H, T, V), dtype=q.dtype, device=q.device)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, K, V), dtype=torch.float32, device=q.device)
    ws_bytes = gdn2_workspace_size(p)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mlstm_gdn2_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0),
                              _ptr(o), _ptr(S_out), _ptr(workspace), ctypes.c_size_t(ws_len), _stream_ptr(stream))
    if st != 0:
        raise MlstmError(st, "mlstm_gdn2_fwd")
    return o, S_out


def reversed_workspace_size(params: FwdParams) -> int:
    return int(lib().mlstm_fwd_chunkwise_reversed_workspace_size(ctypes.byref(params)))


def scalar_normaliser_workspace_size(params: FwdParams) -> int:
    return int(lib().mlstm_fwd_chunkwise_scalar_normaliser_workspace_size(ctypes.byref(params)))


def bwd_workspace_size(params: FwdParams) -> int:
    return int(lib().mlstm_bwd_workspace_size(ctypes.byref(params)))


def bwd(q, k, v, dh, igate=None, fgate=None, ogate=None, C0=None, n0=None, m0=None, dC=None, dn=None, *,
        num_blocks: int = 1, retention: bool = False, workspace=None, stream=None):
    """Backward of the recurrence (mlstm_bwd).  CUDA tensors, contiguous; the forward's inputs
    plus dh [B,NH,S,DHV] (the input dtype) and optional dC, dn (gradients of the final state,
    fp32).  Returns a dict of fp32 gradients dq, dk, dv, di, df (None in retention mode), do
    (None without ogate), dC0, dn0 and dm0 (the last two None in retention mode)."""
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = int(num_blocks)
    p = fwd_params(B, NH, S, DHQK, DHV, 64, nb, q.dtype, retention)
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dq": torch.empty((B, NH, S, DHQK), **f32), "dk": torch.empty((B, NH, S, DHQK), **f32),
           "dv": torch.empty((B, NH, S, DHV), **f32),
           "di": None if retention else torch.empty((B, NH, S), **f32),
           "df": None if retention else torch.empty((B, NH, S), **f32),
           "do": torch.empty((B, NH, S, DHV), **f32) if (ogate is not None and not retention) else None,
           "dC0": torch.empty((B, NH, nb, DHV // nb, DHQK // nb), **f32),
           "dn0": None if retention else torch.empty((B, NH, nb, DHQK // nb), **f32),
           "dm0": None if retention else torch.empty((B, NH), **f32)}
    ws_bytes = bwd_workspace_size(p)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mlstm_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(ogate),
                         _ptr(C0), _ptr(n0), _ptr(m0), _ptr(dh), _ptr(dC), _ptr(dn),
                         _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["di"]), _ptr(out["df"]),
                         _ptr(out["do"]), _ptr(out["dC0"]), _ptr(out["dn0"]), _ptr(out["dm0"]),
                         _ptr(workspace), ctypes.c_size_t(ws_len), _stream_ptr(stream))
    if st != 0:
        raise MlstmError(st, "mlstm_bwd")
    return out


def fwd_chunkwise_noalloc(q, k, v, igate=None, fgate=None, ogate=None, C0=None, n0=None, m0=None, *,
                          chunk: int = 64, num_blocks: int = 1, retention: bool = False,
                          h=None, C_out=None, n_out=None, m_out=None, stream=None):
    """mlstm_fwd_chunkwise_noalloc: the prefill with the library's built-in scratch buffer
    instead of a workspace (for callers that cannot allocate device memory).  Outputs not
    passed in are allocated here with torch, as in fwd_chunkwise; the library allocates
    nothing.  The call runs with q's device current (the library uses the buffer of the
    current device) and, unless a stream is given, on that device's current stream.  Calls
    that overlap on the GPU share the buffer and race."""
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = int(num_blocks)
    p = fwd_params(B, NH, S, DHQK, DHV, chunk, nb, q.dtype, retention)
    dev = q.device
    if h is None:
        h = torch.empty((B, NH, S, DHV), dtype=q.dtype, device=dev)
    if C_out is None:
        C_out = torch.empty((B, NH, nb, DHV // nb, DHQK // nb), dtype=torch.float32, device=dev)
    if not retention:
        if n_out is None:
            n_out = torch.empty((B, NH, nb, DHQK // nb), dtype=torch.float32, device=dev)
        if m_out is None:
            m_out = torch.empty((B, NH), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        cs = _stream_ptr(stream if stream is not None else torch.cuda.current_stream(dev))
        st = lib().mlstm_fwd_chunkwise_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate),
                                               _ptr(ogate), _ptr(C0), _ptr(n0), _ptr(m0), _ptr(h), _ptr(C_out),
                                               _ptr(n_out), _ptr(m_out), cs)
    if st != 0:
        raise MlstmError(st, "mlstm_fwd_chunkwise_noalloc")
    if retention:
        return h, C_out, None, None
    return h, C_out, n_out, m_out


def step(q, k, v, igate, fgate, C, n, m, ogate=None, *, num_blocks: int = 1, retention: bool = False,
         h=None, stream=None):
    """One decode step (mlstm_step), updating C, n, m in place.  Returns h [B,NH,DHV].

    q, k [B,NH,DHQK]; v [B,NH,DHV]; igate, fgate [B,NH] fp32; C [B,NH,nb,DHV/nb,DHQK/nb],
    n [B,NH,nb,DHQK/nb], m [B,NH] fp32 (n, m, gates may be None in retention mode).
    """
    B, NH, DHQK = q.shape
    DHV = v.shape[-1]
    p = StepParams(int(B), int(NH), int(DHQK), int(DHV), int(num_blocks), _dtype_code(q), int(bool(retention)))
    if h is None:
        h = torch.empty((B, NH, DHV), dtype=q.dtype, device=q.device)
    st = lib().mlstm_step(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(ogate),
                          _ptr(C), _ptr(n), _ptr(m), _ptr(h), _stream_ptr(stream))
    if st != 0:
        raise MlstmError(st, "mlstm_step")
    return h
