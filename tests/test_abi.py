"""The C ABI without a GPU: the library loads, exports every declared symbol and
rejects invalid arguments on the host before anything is enqueued."""
import ctypes
import re

import pytest
import torch

from linear_recurrent_token_b200 import build, mlstm
from tests.conftest import ROOT

HEADER = f"{ROOT}/include/mlstm.h"

# Fake, 16-byte aligned, never dereferenced: every call below fails validation first.
A, B_, C_, D_, E_, F_, G_, H_ = (0x100000 * (i + 1) for i in range(8))


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mlstm_[a-z_]+)\s*\(", text)))


def test_library_builds_and_exports_every_declared_symbol():
    build.build()
    lib = mlstm.lib()
    names = declared_functions()
    assert "mlstm_fwd_chunkwise" in names and "mlstm_step" in names
    for name in names:
        assert hasattr(lib, name), name


def test_bounds_checked_build_loads_and_exports_every_declared_symbol():
    build.build()
    assert mlstm.lib().mlstm_bounds_checked() == 0
    with mlstm.bounds_checked() as lib:
        assert mlstm.lib() is lib and lib.mlstm_bounds_checked() == 1
        for name in declared_functions():
            assert hasattr(lib, name), name
        assert lib.mlstm_abi_version() == mlstm_default_abi()
        # argument validation is the same library code
        assert lib.mlstm_fwd_chunkwise_status(None, ctypes.c_void_p(G_), ctypes.c_void_p(0)) == 1
    assert mlstm.lib().mlstm_bounds_checked() == 0


def mlstm_default_abi():
    return mlstm.lib().mlstm_abi_version()


def test_status_strings_and_version():
    for code in range(10):
        assert mlstm.status_string(code) != "unknown status"
    assert mlstm.status_string(8) == "a bounded device-side wait ran out"
    assert mlstm.status_string(9) == "an access failed its bounds check and was skipped"
    assert mlstm.status_string(99) == "unknown status"
    assert mlstm.lib().mlstm_abi_version() >> 16 == 2


def test_params_struct_matches_header_layout():
    # nine ints, then the 64-bit wait limit at offset 40 (C alignment of long long)
    assert ctypes.sizeof(mlstm.FwdParams) == 48
    assert mlstm.FwdParams.wait_limit_cycles.offset == 40
    assert mlstm.fwd_params(1, 1, 1, 16, 16).wait_limit_cycles == 0
    # GDN-2: eight ints, then its wait limit at offset 32
    assert ctypes.sizeof(mlstm.Gdn2Params) == 40
    assert mlstm.Gdn2Params.wait_limit_cycles.offset == 32
    assert mlstm.Gdn2Params(1, 1, 1, 128, 128, 1, 1, 64).wait_limit_cycles == 0


def test_status_calls_validate_before_touching_the_device():
    P = ctypes.c_void_p
    L = mlstm.lib()
    assert L.mlstm_fwd_chunkwise_status(None, P(G_), P(0)) == 1
    assert L.mlstm_fwd_chunkwise_status(ctypes.byref(params(B=-1)), P(G_), P(0)) == 2
    assert L.mlstm_fwd_chunkwise_status(ctypes.byref(params(dtype=7)), P(G_), P(0)) == 3
    tc = mlstm.fwd_params(1, 2, 640, 128, 128, 64, 1, torch.bfloat16, False)
    assert mlstm.plan(tc)["tensor_core"] == 1
    assert L.mlstm_fwd_chunkwise_status(ctypes.byref(tc), None, P(0)) == 1  # its error word lives there
    assert L.mlstm_fwd_chunkwise_noalloc_status(None, P(0)) == 1
    I, LL = ctypes.c_int(5), ctypes.c_longlong(5)
    assert L.mlstm_fwd_chunkwise_bounds_record(None, P(G_), P(0), None, None, None) == 1
    assert L.mlstm_fwd_chunkwise_bounds_record(ctypes.byref(params(B=-1)), P(G_), P(0), ctypes.byref(I),
                                               ctypes.byref(LL), None) == 2
    assert L.mlstm_fwd_chunkwise_bounds_record(ctypes.byref(tc), None, P(0), None, None, None) == 1


def fwd(p, q=A, k=B_, v=C_, ig=D_, fg=E_, og=None, C0=None, n0=None, m0=None, h=F_, C=None, n=None, m=None,
        ws=G_, ws_bytes=1 << 40):
    P = ctypes.c_void_p
    return mlstm.lib().mlstm_fwd_chunkwise(ctypes.byref(p), q, k, v, ig, fg, og, C0, n0, m0, h, C, n, m, ws,
                                           ctypes.c_size_t(ws_bytes), P(0))


def params(**kw):
    base = dict(B=2, NH=2, S=64, DHQK=16, DHV=16, chunk=16, num_blocks=1, dtype=torch.float32, retention=False)
    base.update(kw)
    return mlstm.fwd_params(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 2), (dict(S=-1), 2), (dict(DHQK=0), 2), (dict(chunk=0), 2),
    (dict(num_blocks=3), 2), (dict(num_blocks=0), 2), (dict(dtype=7), 3),
])
def test_fwd_rejects_bad_params(kw, status):
    assert fwd(params(**kw)) == status


def test_fwd_null_pointers():
    p = params()
    assert fwd(p, q=None) == 1
    assert fwd(p, h=None) == 1
    assert fwd(p, ig=None) == 1
    assert fwd(p, fg=None) == 1


def test_fwd_null_params():
    P = ctypes.c_void_p
    st = mlstm.lib().mlstm_fwd_chunkwise(None, A, B_, C_, D_, E_, None, None, None, None, F_, None, None,
                                         None, G_, ctypes.c_size_t(1 << 30), P(0))
    assert st == 1


def test_fwd_misaligned_pointer():
    assert fwd(params(), q=A + 8) == 4
    assert fwd(params(), C=H_ + 4) == 4


def test_fwd_workspace_checks():
    p = params()
    need = mlstm.workspace_size(p)
    assert need > 0
    assert fwd(p, ws=None) == 5
    assert fwd(p, ws_bytes=need - 1) == 5


def test_fwd_aliasing():
    p = params()
    # h on top of q
    assert fwd(p, h=A) == 7
    # final state partially overlapping the initial state (not an exact in-place alias)
    assert fwd(p, C0=H_, C=H_ + 256) == 7
    # workspace on top of v
    assert fwd(p, ws=C_) == 7


def test_workspace_size_and_plan():
    for kw in (dict(), dict(retention=True), dict(S=0), dict(B=0)):
        p = params(**kw)
        plan = mlstm.plan(p)
        assert plan["workspace_bytes"] == mlstm.workspace_size(p)
    assert mlstm.workspace_size(params(retention=True)) == 0  # retention needs no gate workspace
    assert mlstm.workspace_size(params(B=-1)) == 0
    big = mlstm.fwd_params(1, 8, 8192, 256, 512, 64, 1, torch.bfloat16, False)
    assert mlstm.workspace_size(big) >= 8 * 8192 * 4


def step_call(p, q=A, k=B_, v=C_, ig=D_, fg=E_, og=None, C=F_, n=G_, m=H_, h=0x9000000):
    return mlstm.lib().mlstm_step(ctypes.byref(p), q, k, v, ig, fg, og, C, n, m, h, ctypes.c_void_p(0))


def sparams(**kw):
    base = dict(B=2, NH=2, DHQK=16, DHV=16, num_blocks=1, dtype=0, retention=0)
    base.update(kw)
    return mlstm.StepParams(*[int(base[k]) for k in ("B", "NH", "DHQK", "DHV", "num_blocks", "dtype", "retention")])


@pytest.mark.parametrize("kw,status", [
    (dict(DHQK=24), 2),            # block key width 24 is not a supported power of two
    (dict(num_blocks=3), 2), (dict(num_blocks=16, DHQK=64, DHV=64), 2), (dict(B=-2), 2), (dict(dtype=5), 3),
])
def test_step_rejects_bad_params(kw, status):
    assert step_call(sparams(**kw)) == status


def test_step_null_and_alias():
    assert step_call(sparams(), C=None) == 1
    assert step_call(sparams(), n=None) == 1
    assert step_call(sparams(), h=F_) == 7        # h on top of C
    assert step_call(sparams(), C=A) == 7         # state on top of q
    assert step_call(sparams(), q=A + 4) == 4


# ---------------------------------------------------------------- backward
def bwd_call(p, q=A, k=B_, v=C_, ig=D_, fg=E_, og=None, C0=None, n0=None, m0=None, dh=F_, dC=None, dn=None,
             dq=0x9000000, dk=0xA000000, dv=0xB000000, di=None, df=None, do=None, dC0=None, dn0=None, dm0=None,
             ws=0xC000000, ws_bytes=1 << 40):
    return mlstm.lib().mlstm_bwd(ctypes.byref(p), q, k, v, ig, fg, og, C0, n0, m0, dh, dC, dn, dq, dk, dv, di, df,
                                 do, dC0, dn0, dm0, ws, ctypes.c_size_t(ws_bytes), ctypes.c_void_p(0))


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 2), (dict(S=-1), 2), (dict(DHQK=0), 2), (dict(num_blocks=3), 2), (dict(dtype=7), 3),
    (dict(DHQK=512, DHV=16), 2),              # block key width above 256
    (dict(DHQK=256, DHV=256), 2),             # state of one block beyond shared memory
])
def test_bwd_rejects_bad_params(kw, status):
    assert bwd_call(params(**kw)) == status


def test_bwd_null_align_alias_workspace():
    p = params()
    assert bwd_call(p, dh=None) == 1
    assert bwd_call(p, fg=None) == 1
    assert bwd_call(p, dq=None) == 1
    # gates are ignored in retention mode: validation passes them and stops at the (too small)
    # workspace, so nothing is launched with these fake pointers
    assert bwd_call(params(retention=True), ig=None, fg=None, ws_bytes=16) == 5
    assert bwd_call(p, q=A + 8) == 4
    assert bwd_call(p, dq=A) == 7                  # dq on top of q
    assert bwd_call(p, dk=0x9000000) == 7          # dk on top of dq
    assert bwd_call(p, ws=0x9000000) == 7          # workspace on top of dq
    assert bwd_call(p, ws_bytes=16) == 5
    assert bwd_call(p, ws=None) == 5
    # per batch x head: max(8 S floats (SIMT kernels), 6 S nb + 2 S + 2 nb floats (cluster kernel))
    assert mlstm.bwd_workspace_size(p) == 2 * 2 * max(8 * 64, 6 * 64 + 2 * 64 + 2) * 4
    big = mlstm.fwd_params(1, 8, 8192, 256, 512, 64, 1, torch.bfloat16, False)
    assert mlstm.bwd_workspace_size(big) == 8 * max(8 * 8192, 6 * 8192 + 2 * 8192 + 2) * 4
    blocks = mlstm.fwd_params(4, 4, 512, 64, 64, 64, 2, torch.bfloat16, False)
    assert mlstm.bwd_workspace_size(blocks) == 16 * (6 * 512 * 2 + 2 * 512 + 2 * 2) * 4
    # an empty sequence still needs the per-(batch x head, block) final-state terms
    assert mlstm.bwd_workspace_size(params(S=0)) == 2 * 2 * 2 * 4
    assert bwd_call(params(S=0), ws=None) == 5
    assert mlstm.bwd_workspace_size(params(DHQK=512)) == 0


# ---------------------------------------------------------------- reversed-sequence pass
def rev_call(p, q=A, k=B_, v=C_, ig=D_, fg=E_, og=None, C0=None, n0=None, m0=None, h=F_, C=None, n=None, m=None,
             ws=G_, ws_bytes=1 << 40):
    return mlstm.lib().mlstm_fwd_chunkwise_reversed(ctypes.byref(p), q, k, v, ig, fg, og, C0, n0, m0, h, C, n, m, ws,
                                                    ctypes.c_size_t(ws_bytes), ctypes.c_void_p(0))


def test_reversed_validates_like_the_forward_and_checks_its_workspace():
    p = params()
    assert rev_call(params(B=-1)) == 2
    assert rev_call(p, q=None) == 1
    assert rev_call(p, h=A) == 7                     # h on top of q
    assert rev_call(p, q=A + 8) == 4
    need = mlstm.reversed_workspace_size(p)
    # the reversed copies of q, k, v, gates, o and h come on top of the forward's workspace
    tok = 2 * 2 * 64
    assert need >= mlstm.workspace_size(p) + 2 * tok * 16 * 4 + 3 * tok * 16 * 4 + 2 * tok * 4
    assert rev_call(p, ws_bytes=need - 1) == 5
    assert rev_call(p, ws=C_ - 256) == 7             # workspace overlapping v
    assert mlstm.reversed_workspace_size(params(S=0)) == mlstm.workspace_size(params(S=0))


# ---------------------------------------------------------------- scalar-normaliser prefill
def sn_call(p, q=A, k=B_, v=C_, ig=D_, fg=E_, og=None, bias=0xD000000, C0=None, n0=None, m0=None, h=F_, C=None, n=None,
            m=None, ws=G_, ws_bytes=1 << 40):
    return mlstm.lib().mlstm_fwd_chunkwise_scalar_normaliser(ctypes.byref(p), q, k, v, ig, fg, og, bias, C0, n0, m0,
                                                             h, C, n, m, ws, ctypes.c_size_t(ws_bytes),
                                                             ctypes.c_void_p(0))


def test_scalar_normaliser_validation():
    p = params()
    assert sn_call(params(retention=True)) == 2        # retention has no normaliser
    assert sn_call(p, bias=None) == 1
    assert sn_call(p, fg=None) == 1
    assert sn_call(p, bias=0xD000000 + 4) == 4
    assert sn_call(p, h=A) == 7
    assert sn_call(p, n=0xD000000) == 7                 # n_out on top of the bias
    # an in-place state passes the alias checks and stops at the (too small) workspace
    assert sn_call(p, C=0xE000000, C0=0xE000000, ws_bytes=16) == 5
    need = mlstm.lib().mlstm_fwd_chunkwise_scalar_normaliser_workspace_size(ctypes.byref(p))
    assert need > 0 and sn_call(p, ws_bytes=need - 1) == 5


# ---------------------------------------------------------------- multi-scale retention block
def rot_call(p, q=A, k=B_, pos0=None, base=10000.0, qo=C_, ko=D_):
    return mlstm.lib().mlstm_theta_rotate(ctypes.byref(p), q, k, pos0, ctypes.c_float(base), qo, ko,
                                          ctypes.c_void_p(0))


def gn_call(p, h=A, g=B_, w=None, b=None, eps=1e-5, y=C_):
    return mlstm.lib().mlstm_group_norm_gate(ctypes.byref(p), h, g, w, b, ctypes.c_float(eps), y, ctypes.c_void_p(0))


def msr_call(p, q=A, k=B_, v=C_, ig=D_, fg=E_, pos0=None, base=10000.0, g=H_, w=None, b=None, eps=1e-5, C0=None,
             n0=None, m0=None, y=F_, C=None, n=None, m=None, ws=G_, ws_bytes=1 << 40):
    return mlstm.lib().mlstm_fwd_chunkwise_msr(ctypes.byref(p), q, k, v, ig, fg, pos0, ctypes.c_float(base), g, w, b,
                                               ctypes.c_float(eps), C0, n0, m0, y, C, n, m, ws,
                                               ctypes.c_size_t(ws_bytes), ctypes.c_void_p(0))


def test_theta_rotate_validation():
    # every call here fails validation: none reaches a launch
    p = params()
    assert rot_call(params(DHQK=18)) == 2                   # not a whole number of 16-byte vectors
    assert rot_call(params(DHQK=12, dtype=torch.bfloat16)) == 2   # 12 bf16 = 1.5 vectors
    assert rot_call(p, base=0.0) == 2 and rot_call(p, base=float("nan")) == 2
    assert rot_call(p, q=None) == 1 and rot_call(p, ko=None) == 1
    assert rot_call(p, q=A + 4) == 4 and rot_call(p, pos0=E_ + 4) == 4
    assert rot_call(p, qo=A + 16) == 7                      # overlaps q without being q
    assert rot_call(p, qo=B_) == 7 and rot_call(p, ko=C_) == 7
    assert rot_call(p, pos0=C_) == 7                        # positions under an output


def test_group_norm_gate_validation():
    p = params()
    assert gn_call(params(DHV=24)) == 2                     # 6 vectors per row: not a power of two
    assert gn_call(p, eps=-1.0) == 2
    assert gn_call(p, h=None) == 1 and gn_call(p, y=None) == 1
    assert gn_call(p, w=E_ + 8) == 4
    assert gn_call(p, y=B_) == 7 and gn_call(p, y=A + 16) == 7
    assert gn_call(p, w=C_ + 16) == 7                       # weights under y


def test_msr_block_validation_and_workspace():
    p = params(retention=True)
    need = mlstm.msr_workspace_size(p)
    tok = 2 * 2 * 64
    assert need >= mlstm.workspace_size(p) + 2 * tok * 16 * 4
    assert msr_call(p, ws_bytes=need - 1) == 5
    assert msr_call(params(DHQK=18, retention=True)) == 2
    assert msr_call(params(DHV=24, retention=True)) == 2
    assert msr_call(p, q=None) == 1
    assert msr_call(p, g=F_) == 7                           # gate under y
    assert msr_call(p, ws=A) == 7                           # workspace under q
    assert msr_call(p, pos0=G_ + 8) == 7                    # positions inside the workspace
    assert msr_call(p, g=H_ + 4) == 4
    assert msr_call(params(), ig=None, ws_bytes=16) == 5  # mLSTM mode: workspace checked first


# ---------------------------------------------------------------- Gated DeltaNet-2
def gdn2_call(B=2, H=2, T=16, K=64, V=64, dtype=0, mode=0, chunk=16, q=A, k=B_, v=C_, g=D_, b=E_, w=F_, S0=None,
              o=G_, S=None, ws=None, ws_bytes=0):
    p = mlstm.Gdn2Params(B, H, T, K, V, dtype, mode, chunk)
    return mlstm.lib().mlstm_gdn2_fwd(ctypes.byref(p), q, k, v, g, b, w, S0, o, S, ws, ctypes.c_size_t(ws_bytes),
                                      ctypes.c_void_p(0))


def test_gdn2_validation():
    # every call here fails validation: none reaches a launch
    assert gdn2_call(K=48) == 2                     # recurrent: K in {32, 64, 128, 256}
    assert gdn2_call(mode=1, chunk=66) == 2         # chunk length over 64
    assert gdn2_call(mode=1, chunk=6) == 2          # not a multiple of 4
    assert gdn2_call(mode=2) == 2 and gdn2_call(dtype=5) == 3 and gdn2_call(T=-1) == 2
    assert gdn2_call(q=None) == 1 and gdn2_call(w=None) == 1 and gdn2_call(o=None) == 1
    assert gdn2_call(g=D_ + 4) == 4
    assert gdn2_call(o=A) == 7                      # o on top of q
    assert gdn2_call(S=G_ + 64) == 7                # state inside o
    assert gdn2_call(S0=H_, S=H_ + 16) == 7         # state overlapping the initial state, not equal
    assert gdn2_call(S0=G_, S=None) == 7            # initial state under o
    # chunk mode: one prepared slot per (batch, head, chunk) of 4 L K + 4 L^2 + K floats
    p = mlstm.Gdn2Params(2, 2, 16, 64, 64, 0, 1, 8)
    assert mlstm.gdn2_workspace_size(p) == 2 * 2 * 2 * (4 * 8 * 64 + 4 * 64 + 64) * 4
    assert mlstm.gdn2_workspace_size(mlstm.Gdn2Params(2, 2, 16, 64, 64, 0, 0, 8)) == 0
    assert gdn2_call(mode=1, chunk=8) == 5                          # no workspace
    assert gdn2_call(mode=1, chunk=8, ws=H_, ws_bytes=16) == 5      # too small
    assert gdn2_call(mode=1, chunk=8, ws=A, ws_bytes=1 << 30) == 7  # workspace over q
    # the tensor-core chunk path (bf16, chunk 64, K 128, V 64 / 128): a 256-byte header (the
    # error word of its bounded waits), then per (batch, head, chunk) a slot of Wk, Qw, Kt, nBt
    # (4 x 16 KiB), U, Ur, Ou (3 x 128 V bytes) and e^{G_L} (512 bytes)
    for V in (64, 128):
        tc = mlstm.Gdn2Params(2, 3, 130, 128, V, 1, 1, 64)
        assert mlstm.gdn2_workspace_size(tc) == 256 + 6 * 3 * (65536 + 384 * V + 512)
    P = ctypes.c_void_p
    L = mlstm.lib()
    assert L.mlstm_gdn2_status(None, P(G_), P(0)) == 1
    assert L.mlstm_gdn2_status(ctypes.byref(mlstm.Gdn2Params(2, 3, 130, 128, 128, 5, 1, 64)), P(G_), P(0)) == 3
    assert L.mlstm_gdn2_status(ctypes.byref(mlstm.Gdn2Params(2, 3, -1, 128, 128, 1, 1, 64)), P(G_), P(0)) == 2
    assert L.mlstm_gdn2_status(ctypes.byref(mlstm.Gdn2Params(2, 3, 130, 128, 128, 1, 1, 64)), None, P(0)) == 1


def test_header_is_plain_c(tmp_path):
    """include/mlstm.h is a C header: it compiles as pedantic C99 with no CUDA headers and
    declares every type the entry points use."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "mlstm.h"\n'
                   "int main(void) {\n"
                   "  mlstm_fwd_params_t f; mlstm_step_params_t s; mlstm_gdn2_params_t g; mlstm_fwd_plan_t p;\n"
                   "  (void)f; (void)s; (void)g; (void)p;\n"
                   "  return (int)MLSTM_OK + (int)MLSTM_GDN2_CHUNK * 0;\n"
                   "}\n")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", f"{ROOT}/include",
                        "-fsyntax-only", str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.parametrize("shape", [
    # B, NH, S, DHQK, DHV, nb, retention
    (1, 8, 8192, 256, 512, 1, False),   # the large head
    (8, 8, 2048, 64, 64, 1, True),      # the retention workload
    (4, 4, 512, 64, 64, 2, False),      # 32 x 32 blocks (zero-padded tiles)
    (1, 2, 1000, 128, 256, 1, False),
    (2, 3, 70, 64, 64, 1, False),       # two chunks, ragged
    (1, 1, 64, 32, 32, 2, False),       # one chunk of 16 x 16 blocks
    (1, 4, 20000, 128, 128, 1, False),  # many short segments
])
def test_tensor_core_plan_covers_the_sequence(shape):
    """The tensor-core plan (host logic, no GPU): segments cover the chunks once, the last segment
    is not empty, one summary unit per segment but the last (segment 0 may be split in two), the
    walk's CTAs (value tiles x slices x heads x segments) fit the 148 SMs of a B200 when there is
    more than one segment, and the workspace holds the summaries."""
    B, NH, S, DHQK, DHV, nb, retention = shape
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, nb, torch.bfloat16, retention)
    pl = mlstm.plan(p)
    assert pl["tensor_core"] == 1, pl
    chunks = (S + 63) // 64
    G, s0, s = pl["segments"], pl["seg0_chunks"], pl["seg_chunks"]
    assert G >= 1
    if G > 1:
        assert s0 + (G - 2) * s < chunks <= s0 + (G - 1) * s, pl
        assert pl["summary_units"] >= G - 1 and pl["summary_units"] <= G, pl
    else:
        assert pl["summary_units"] == 0
    dk, dv = DHQK // nb, DHV // nb
    tiles = -(-dv // pl["dv_tile"])
    assert pl["ctas_main"] == B * NH * nb * tiles * G
    assert pl["ctas_main"] <= 148 or G == 1
    assert pl["workspace_bytes"] >= B * NH * nb * pl["summary_units"] * dv * dk * 4


def test_planner_choices_on_the_measured_workloads():
    """The plans the cost model gives the workloads it was measured on: the large head in four
    segments of 32 chunks (three summary units); 64-wide retention heads of 32 chunks in two
    segments with the longer first (21 + 11); sequences of at most 8 chunks in one segment (no
    summaries kernel)."""
    def plan(B, NH, S, DHQK, DHV, nb, ret):
        return mlstm.plan(mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, nb, torch.bfloat16, ret))
    pl = plan(1, 8, 8192, 256, 512, 1, False)
    assert (pl["segments"], pl["seg0_chunks"], pl["seg_chunks"], pl["summary_units"]) == (4, 32, 32, 3)
    pl = plan(8, 8, 2048, 64, 64, 1, True)
    assert (pl["segments"], pl["seg0_chunks"], pl["seg_chunks"], pl["summary_units"]) == (2, 21, 11, 1)
    for shape in ((4, 4, 512, 64, 64, 2, False), (8, 8, 512, 64, 64, 1, True), (1, 2, 450, 128, 128, 1, False)):
        pl = plan(*shape)
        assert pl["segments"] == 1 and pl["summary_units"] == 0 and pl["kernels"] == 2, (shape, pl)
