"""Host-side checks of the C ABI (no GPU): the library loads, exports exactly
the entry points include/rmm.h declares, and rejects bad problems on the host
before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

import input_adaptive_reduced_b200 as rmm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "rmm.h")).read()
    return sorted(set(re.findall(r"RMM_API\s+[\w\s\*]+?\b(rmm_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(rmm.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    out = subprocess.check_output(["nm", "-D", "--defined-only", rmm.library_path], text=True)
    exported = sorted(l.split()[-1] for l in out.splitlines() if l.split()[-1].startswith("rmm_"))
    assert exported == _declared()
    for name in _declared():
        assert getattr(rmm.lib, name) is not None


def test_no_cuda_runtime_symbols_leak():
    out = subprocess.check_output(["nm", "-D", "--defined-only", rmm.library_path], text=True)
    assert not [l for l in out.splitlines() if " cuda" in l]


def test_status_strings_and_version():
    assert rmm.rmm_status_string(rmm.RMM_OK) == "RMM_OK"
    assert rmm.rmm_status_string(rmm.RMM_ERR_TIMEOUT) == "RMM_ERR_TIMEOUT"
    assert rmm.rmm_status_string(99) == "RMM_ERR_UNKNOWN"
    assert re.fullmatch(r"\d+\.\d+\.\d+", rmm.rmm_version())


def test_problem_init_defaults():
    p = rmm.rmm_problem_init(rmm.RMM_QK, rmm.RMM_BF16, 10, 128, 40)
    assert (p.lda, p.ldb, p.ldy, p.heads, p.kv_heads, p.rho, p.alpha) == (128, 128, 40, 1, 1, 1.0, 1.0)
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, 10, 64, 40)
    assert p.ldb == 40


def _status(p):
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    s = rmm.lib.rmm_plan_create(ctypes.byref(h), ctypes.byref(p), ctypes.byref(ws))
    if h.value:
        rmm.lib.rmm_plan_destroy(h)
    return s


def _base():
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, 64, 256, 256)
    p.rho = 0.5
    return p


@pytest.mark.parametrize("field,value", [
    ("mode", 7), ("dtype", 5), ("n", -1), ("d", 0), ("d", 250), ("m", 12), ("lda", 200),
    ("lda", 260), ("ldy", 100), ("ldb", 100), ("heads", 0), ("kv_heads", 3), ("rho", 0.0),
    ("rho", 1.5), ("k", 300), ("k", -2), ("flags", 16), ("flags", 1),
    ("flags", 6),  # given scores together with given indices
])
def test_invalid_problems_are_rejected_on_the_host(field, value):
    p = _base()
    setattr(p, field, value)
    assert _status(p) == rmm.RMM_ERR_INVALID_ARG


def test_emitted_scores_need_a_linear_or_pv_output():
    """The output of QK is masked attention scores; its consumer is the
    softmax, which scores P itself: RMM_FLAG_EMIT_SCORES is rejected there."""
    p = rmm.rmm_problem_init(rmm.RMM_QK, rmm.RMM_BF16, 64, 128, 64)
    p.rho = 0.5
    p.flags = rmm.RMM_FLAG_EMIT_SCORES
    assert _status(p) == rmm.RMM_ERR_INVALID_ARG


def test_softmax_arguments_are_checked_on_the_host():
    ok = dict(heads=2, n=16, t=64, lds=64, stride_s=1024, ldp=64, stride_p=1024, flags=0)
    fake = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x100000)
    wsz = rmm.rmm_softmax_workspace_size(2, 16, 64)
    assert wsz >= 2 * 4 + 2 * 64 * 4

    def call(**kw):
        a = dict(ok, **kw)
        return rmm.lib.rmm_softmax_scores(fake, fake, fake, a["heads"], a["n"], a["t"], a["lds"], a["stride_s"],
                                          a["ldp"], a["stride_p"], a["flags"], kw.get("ws", ws),
                                          kw.get("wsz", wsz), None)
    assert call(t=60) == rmm.RMM_ERR_INVALID_ARG          # t not a multiple of 8
    assert call(lds=32) == rmm.RMM_ERR_INVALID_ARG        # row stride below t
    assert call(stride_p=100) == rmm.RMM_ERR_INVALID_ARG  # head stride below n * ldp
    assert call(flags=2) == rmm.RMM_ERR_INVALID_ARG       # only the causal flag
    assert call(t=8200, lds=8200, ldp=8200, stride_s=8200 * 16, stride_p=8200 * 16) == rmm.RMM_ERR_UNSUPPORTED
    assert call(wsz=wsz - 1) == rmm.RMM_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p(0x100010)) == rmm.RMM_ERR_WORKSPACE  # not 256-byte aligned
    assert call(n=0) == rmm.RMM_OK                        # nothing to do, nothing launched


def _pv(n, nk, flags):
    p = rmm.rmm_problem_init(rmm.RMM_PV, rmm.RMM_BF16, n, nk, 128)
    p.heads, p.kv_heads = 4, 2
    p.stride_a, p.stride_b, p.stride_y = n * nk, nk * 128, n * 128
    p.rho = 0.5
    p.flags = flags
    return p


def test_causal_pv_needs_one_query_per_token():
    """RMM_FLAG_CAUSAL on PV states P[i][t] = 0 for t > i, which needs n = n_k."""
    import torch
    assert _status(_pv(256, 512, rmm.RMM_FLAG_CAUSAL)) == rmm.RMM_ERR_INVALID_ARG
    want = rmm.RMM_OK if torch.cuda.is_available() else rmm.RMM_ERR_CUDA
    assert _status(_pv(512, 512, rmm.RMM_FLAG_CAUSAL)) == want
    assert _status(_pv(256, 512, 0)) == want


def test_valid_problem_reaches_the_device_query():
    # Validation passes, so the next step asks the CUDA runtime for the SM count:
    # OK on a GPU machine, RMM_ERR_CUDA where there is no device.
    import torch
    want = rmm.RMM_OK if torch.cuda.is_available() else rmm.RMM_ERR_CUDA
    assert _status(_base()) == want


def test_null_arguments():
    assert rmm.lib.rmm_plan_create(None, None, None) == rmm.RMM_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert rmm.lib.rmm_plan_create(ctypes.byref(h), None, None) == rmm.RMM_ERR_INVALID_ARG
    assert rmm.lib.rmm_plan_destroy(None) == rmm.RMM_OK
    assert rmm.lib.rmm_plan_k(None) == -1
    assert rmm.lib.rmm_plan_workspace_size(None) == 0
    assert rmm.lib.rmm_matmul(None, None, None, None, None, None, 0, None) == rmm.RMM_ERR_INVALID_ARG
    assert rmm.lib.rmm_select(None, None, None, None, None, 0, None) == rmm.RMM_ERR_INVALID_ARG


def test_attention_problems_are_checked_on_the_host():
    """rmm_attention sizes its workspace on the host and refuses what its
    kernels do not implement: d_h or d_v other than 128, n not a multiple of 8,
    strides below a row or a head, ratios outside (0, 1]."""
    p = rmm.rmm_attn_problem()
    p.heads, p.kv_heads, p.n, p.d_h, p.d_v = 4, 2, 256, 128, 128
    p.ldq = p.ldk = p.ldv = p.ldo = 128
    p.stride_q = p.stride_k = p.stride_v = p.stride_o = 256 * 128
    p.rho_d, p.rho_t, p.alpha = 0.5, 0.5, 0.125
    assert rmm.rmm_attention_workspace_size(p) > 4 * 256 * 128 * 2  # holds the masked Q
    for field, value in (("d_h", 64), ("d_v", 256), ("n", 250), ("kv_heads", 3), ("ldq", 100),
                         ("stride_o", 1000), ("rho_d", 0.0), ("rho_t", 1.5), ("flags", 2)):
        q = rmm.rmm_attn_problem.from_buffer_copy(p)
        setattr(q, field, value)
        assert rmm.rmm_attention_workspace_size(q) == 0, field
        assert rmm.lib.rmm_attention(ctypes.byref(q), None, None, None, None, None, None, None, 0, None) in (
            rmm.RMM_ERR_INVALID_ARG, rmm.RMM_ERR_UNSUPPORTED), field
