"""The C-ABI library loads, exports every entry point include/kda.h declares,
and rejects bad arguments synchronously (no GPU needed: argument checks run
before any CUDA call)."""
import ctypes
import os
import re

import pytest
import torch

from gated_delta_rule_61_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")
FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: checks fail first


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert set(_declared()) == set(kda.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = kda.lib()
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    for code in range(6):
        assert kda.status_string(code)
    assert kda.status_string(99) == "unknown status"
    assert kda.lib().kda_version() >= 100


def test_workspace_query():
    W = lambda n, H, has_cu, dtype=kda.KDA_BF16, chunk=64, d=128: kda.workspace_bytes(
        n, H, d, d, dtype, chunk, has_cu)
    slot = 128 * 128 * 4
    # order of packed sequences: one int32 each, 256-byte granules
    assert W(1024, 1, True) == 4096
    assert W(1025, 1, True) == 4096 + 256
    # few chains (<= 128): one hand-over slot per chain after the order
    assert W(64, 2, False) == 128 * slot
    assert W(64, 2, True) == 256 + 128 * slot
    assert W(1, 1, True) == 256 + slot
    assert W(129, 1, False) == 0
    assert W(0, 4, True) == 0
    # no workspace when the token-recurrent kernel serves the call
    assert W(4, 2, True, chunk=0) == 0
    assert W(4, 2, True, dtype=kda.KDA_F32) == 0
    assert W(4, 2, True, d=64) == 0


def _prefill(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, cu=None, n_seq=0, B=1, T=64,
             H=2, dk=128, dv=128, dtype=kda.KDA_BF16, chunk=64, o=FAKE, sT=None, ws=None,
             ws_bytes=0, stream=None)
    a.update(kw)
    return kda.lib().kda_prefill(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["cu"],
                                 a["n_seq"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                 a["dtype"], a["chunk"], a["o"], a["sT"], a["ws"],
                                 a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(B=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-5), kda.KDA_ERR_INVALID_ARG),
    (dict(dtype=7), kda.KDA_ERR_INVALID_ARG),
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=None), kda.KDA_ERR_INVALID_ARG),
    (dict(o=None), kda.KDA_ERR_INVALID_ARG),
    (dict(n_seq=3, B=2), kda.KDA_ERR_INVALID_ARG),
    (dict(cu=FAKE, B=2, n_seq=2), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(cu=FAKE, n_seq=4), kda.KDA_ERR_WORKSPACE),       # varlen needs its workspace
    (dict(cu=FAKE, n_seq=4, ws=FAKE, ws_bytes=16), kda.KDA_ERR_WORKSPACE),
    (dict(cu=FAKE, n_seq=4, ws=ctypes.c_void_p(0x10004), ws_bytes=1 << 24),
     kda.KDA_ERR_WORKSPACE),
    (dict(B=2), kda.KDA_ERR_WORKSPACE),                    # few chains: hand-over slots
    (dict(B=2, ws=FAKE, ws_bytes=2 * 2 * 65536 - 1), kda.KDA_ERR_WORKSPACE),
    # the chunked kernel moves its tensors in 16-byte vectors
    (dict(la=ctypes.c_void_p(0x10008)), kda.KDA_ERR_INVALID_ARG),
    (dict(k=ctypes.c_void_p(0x10008)), kda.KDA_ERR_INVALID_ARG),
    (dict(o=ctypes.c_void_p(0x10002)), kda.KDA_ERR_INVALID_ARG),
    (dict(sT=ctypes.c_void_p(0x10004)), kda.KDA_ERR_INVALID_ARG),
])
def test_prefill_rejects_bad_arguments(kw, status):
    assert _prefill(**kw) == status


def test_prefill_empty_is_ok_without_touching_memory():
    assert _prefill(B=0, T=0, q=None, k=None, v=None, la=None, beta=None, o=None) == kda.KDA_OK


def _decode(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, state=FAKE, B=2, H=2, dk=128, dv=128,
             dtype=kda.KDA_BF16, o=FAKE, stream=None)
    a.update(kw)
    return kda.lib().kda_decode_step(a["q"], a["k"], a["v"], a["la"], a["beta"], a["state"],
                                     a["B"], a["H"], a["dk"], a["dv"], a["dtype"], a["o"],
                                     a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(B=-2), kda.KDA_ERR_INVALID_ARG),
    (dict(dtype=3), kda.KDA_ERR_INVALID_ARG),
    (dict(state=None), kda.KDA_ERR_INVALID_ARG),
    (dict(o=None), kda.KDA_ERR_INVALID_ARG),
    (dict(state=ctypes.c_void_p(0x10004)), kda.KDA_ERR_INVALID_ARG),   # 16-byte alignment
    (dict(dk=100), kda.KDA_ERR_UNSUPPORTED),
    (dict(B=0), kda.KDA_OK),
])
def test_decode_rejects_bad_arguments(kw, status):
    assert _decode(**kw) == status


def _backward(**kw):
    a = dict(B=2, T=4, H=2, dk=128, dv=128, dtype=kda.KDA_BF16, gate=kda.KDA_GATE_CHANNEL,
             flags=0, ws=None, ws_bytes=0)
    a.update(kw)
    return kda.lib().kda_backward_ex(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, a["B"], a["T"],
                                     a["H"], a["dk"], a["dv"], a["dtype"], a["gate"], a["flags"],
                                     FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, a["ws"],
                                     a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(flags=8), kda.KDA_ERR_INVALID_ARG),         # not a prologue flag
    (dict(gate=7), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=100), kda.KDA_ERR_UNSUPPORTED),
    (dict(flags=7), kda.KDA_ERR_WORKSPACE),           # valid flags; no workspace given
    (dict(B=0, T=0), kda.KDA_OK),
])
def test_backward_rejects_bad_arguments(kw, status):
    assert _backward(**kw) == status


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_launch_without_device_reports_cuda_error():
    assert _decode() == kda.KDA_ERR_CUDA
    assert _prefill(chunk=0) == kda.KDA_ERR_CUDA
    # bf16 with dk = dv = 64 is served by the token-recurrent kernel (no workspace)
    assert _prefill(dk=64, dv=64) == kda.KDA_ERR_CUDA
    assert _prefill(B=2, ws=FAKE, ws_bytes=2 * 2 * 65536) == kda.KDA_ERR_CUDA


def test_python_wrapper_checks_shapes_before_the_library():
    q = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    with pytest.raises((ValueError, TypeError)):
        kda.prefill(q, q, q, torch.zeros(1, 4, 2, 64), torch.zeros(1, 4, 2))
    with pytest.raises(TypeError):
        kda.prefill(q.half(), q.half(), q.half(), torch.zeros(1, 4, 2, 128), torch.zeros(1, 4, 2))
