"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

libkda.so must load, export every entry point include/kda.h declares, and
reject bad arguments on the host before touching the device: the pointers
passed here are fake, so a call that got past validation would fail loudly.
"""
import ctypes
import os
import re

import pytest

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_158_b200 import build
    build.build()
    return _lib.lib()


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"KDA_API[^;(]*?\b(kda_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol(L):
    declared = _declared_symbols()
    assert {"kda_chunk_fwd", "kda_decode_step", "kda_gate_fwd"} <= declared
    for name in declared:
        assert hasattr(L, name), name
    assert set(_lib._SIGNATURES) == declared


def test_debug_library_exports_the_same_symbols_and_reports_its_checks(L):
    """libkda_debug.so (KDA_DEBUG_CHECKS) has the release ABI; only its
    kda_debug_checks_enabled answers 1, and its bounds selftest rejects bad
    arguments on the host like every other entry point."""
    D = _lib._load(_lib.DEBUG_LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(D, name), name
    assert D.kda_debug_checks_enabled() == 1
    assert L.kda_debug_checks_enabled() == 0
    assert D.kda_selftest_bounds_check(None, None) == kda.KDA_ERR_INVALID_ARG
    assert D.kda_selftest_bounds_check(FAKE + 4, None) == kda.KDA_ERR_MISALIGNED
    # the release build has no checks to exercise: refused before any launch
    assert L.kda_selftest_bounds_check(FAKE, None) == kda.KDA_ERR_UNSUPPORTED
    assert D.kda_status_string(8) == b"KDA_ERR_BOUNDS"


def test_status_strings(L):
    for code, name in [(0, "KDA_OK"), (1, "KDA_ERR_INVALID_ARG"), (2, "KDA_ERR_UNSUPPORTED"),
                       (3, "KDA_ERR_MISALIGNED"), (4, "KDA_ERR_WORKSPACE"), (5, "KDA_ERR_CUDA"),
                       (6, "KDA_ERR_TIMEOUT"), (7, "KDA_ERR_BAD_SEQLENS"),
                       (8, "KDA_ERR_BOUNDS")]:
        assert kda.kda_status_string(code) == name
    assert kda.kda_status_string(99) == "KDA_ERR_UNKNOWN"


def test_last_cuda_error_string_starts_clean(L):
    # host-only calls that fail validation never record a CUDA error
    assert kda.kda_last_cuda_error_string().startswith("cudaSuccess")


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced


def _chunk(L, **over):
    a = dict(q=FAKE, k=FAKE + 0x1000, v=FAKE + 0x2000, g=FAKE + 0x3000, beta=FAKE + 0x4000,
             dt=_lib.KDA_BF16, init=None, cu=None, nseq=0, B=2, T=64, H=4, dk=128, dv=128,
             scale=1.0, chunk=0, out=FAKE + 0x5000, final=None, ws=FAKE + 0x6000,
             ws_bytes=1 << 40, stream=None)
    a.update(over)
    return L.kda_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["dt"], a["init"],
                           a["cu"], a["nseq"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                           a["scale"], a["chunk"], a["out"], a["final"], a["ws"], a["ws_bytes"],
                           a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), _lib.KDA_ERR_INVALID_ARG),
    (dict(out=None), _lib.KDA_ERR_INVALID_ARG),
    (dict(ws=None), _lib.KDA_ERR_INVALID_ARG),
    (dict(B=0), _lib.KDA_ERR_INVALID_ARG),
    (dict(T=-1), _lib.KDA_ERR_INVALID_ARG),
    (dict(dt=7), _lib.KDA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.KDA_ERR_INVALID_ARG),
    (dict(dk=96), _lib.KDA_ERR_UNSUPPORTED),
    (dict(dv=256), _lib.KDA_ERR_UNSUPPORTED),
    (dict(chunk=48), _lib.KDA_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), _lib.KDA_ERR_MISALIGNED),
    (dict(final=FAKE + 0x7004), _lib.KDA_ERR_MISALIGNED),
    (dict(out=FAKE), _lib.KDA_ERR_INVALID_ARG),           # out aliases q
    (dict(cu=FAKE + 0x8000, nseq=3), _lib.KDA_ERR_INVALID_ARG),  # varlen needs B == 1
    (dict(cu=FAKE + 0x8000, nseq=0, B=1), _lib.KDA_ERR_INVALID_ARG),
    (dict(ws_bytes=16), _lib.KDA_ERR_WORKSPACE),
])
def test_chunk_fwd_rejects_on_host(L, over, code):
    assert _chunk(L, **over) == code


def test_workspace_size_positive(L):
    n = kda.kda_chunk_fwd_workspace_size(8, 4096, 32, 128, 128, 0, 0, _lib.KDA_BF16)
    assert n >= 256
    n2 = kda.kda_chunk_fwd_workspace_size(1, 1000, 16, 128, 128, 64, 0, _lib.KDA_BF16)
    assert n2 >= 256 + 64 * 4


@pytest.mark.parametrize("args,code", [
    ((None, FAKE, FAKE, FAKE, FAKE, 1, FAKE, 4, 2, 128, 128, 1.0, FAKE + 64, None), 1),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 1, FAKE, 4, 2, 100, 128, 1.0, FAKE + 64, None), 2),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 1, FAKE + 4, 4, 2, 128, 128, 1.0, FAKE + 64, None), 3),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 1, FAKE, 0, 2, 128, 128, 1.0, FAKE + 64, None), 1),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 1, FAKE + 64, 4, 2, 128, 128, 1.0, FAKE + 64, None), 1),
])
def test_decode_rejects_on_host(L, args, code):
    assert L.kda_decode_step(*args) == code


def test_gate_rejects_on_host(L):
    assert L.kda_gate_fwd(None, FAKE, -5.0, FAKE + 64, 10, 2, 32, None) == 1
    assert L.kda_gate_fwd(FAKE, FAKE + 16, 5.0, FAKE + 64, 10, 2, 32, None) == 1
    assert L.kda_gate_fwd(FAKE, FAKE + 16, -5.0, FAKE, 10, 2, 32, None) == 1
    assert L.kda_gate_fwd(FAKE + 4, FAKE + 16, -5.0, FAKE + 64, 10, 2, 32, None) == 3
    assert L.kda_gate_fwd(FAKE, FAKE + 16, -5.0, FAKE + 64, 0, 2, 32, None) == 0  # no-op


def test_device_status_rejects_null(L):
    assert L.kda_get_device_status(None, None, None) == 1
    assert L.kda_selftest_bounded_wait(None, 1000, None) == 1
    assert L.kda_selftest_bounded_wait(FAKE + 4, 1000, None) == 3


def test_gated_entries_reject_on_host(L):
    args = [FAKE, FAKE + 0x1000, FAKE + 0x2000, FAKE + 0x3000, FAKE + 0x9000, -5.0,
            FAKE + 0x4000, _lib.KDA_BF16, None, None, 0, 2, 64, 4, 128, 128, 1.0, 0,
            FAKE + 0x5000, None, FAKE + 0x6000, 1 << 40, None]
    bad = list(args); bad[4] = None           # A_log missing
    assert L.kda_chunk_fwd_gated(*bad) == _lib.KDA_ERR_INVALID_ARG
    bad = list(args); bad[5] = 5.0            # g_min must be negative
    assert L.kda_chunk_fwd_gated(*bad) == _lib.KDA_ERR_INVALID_ARG
    bad = list(args); bad[4] = FAKE + 0x9004  # misaligned A_log
    assert L.kda_chunk_fwd_gated(*bad) == _lib.KDA_ERR_MISALIGNED
    d = [FAKE, FAKE, FAKE, FAKE, None, -5.0, FAKE, 1, FAKE, 4, 2, 128, 128, 1.0, FAKE + 64, None]
    assert L.kda_decode_step_gated(*d) == _lib.KDA_ERR_INVALID_ARG
    d[4] = FAKE + 16
    d[5] = float("inf")
    assert L.kda_decode_step_gated(*d) == _lib.KDA_ERR_INVALID_ARG


def test_verify_replay_reject_on_host(L):
    v = [FAKE, FAKE, FAKE, FAKE, None, -5.0, FAKE, 1, FAKE + 64, 4, 2, 4, 128, 128, 1.0,
         FAKE + 128, None]
    bad = list(v); bad[11] = 0            # K = 0
    assert L.kda_decode_verify(*bad) == _lib.KDA_ERR_UNSUPPORTED
    bad = list(v); bad[11] = 17           # K above 16
    assert L.kda_decode_verify(*bad) == _lib.KDA_ERR_UNSUPPORTED
    bad = list(v); bad[15] = FAKE         # out aliases q
    assert L.kda_decode_verify(*bad) == _lib.KDA_ERR_INVALID_ARG
    r = [FAKE, FAKE, FAKE, None, -5.0, FAKE, 1, FAKE + 64, FAKE + 128, 4, 2, 4, 128, 128, None]
    bad = list(r); bad[8] = None          # accept_len missing
    assert L.kda_decode_replay(*bad) == _lib.KDA_ERR_INVALID_ARG
    bad = list(r); bad[8] = FAKE + 132    # misaligned accept_len
    assert L.kda_decode_replay(*bad) == _lib.KDA_ERR_MISALIGNED


def test_kcp_entries_reject_on_host(L):
    fake = 0x7F0000000000
    ptr = lambda i: fake + 0x1000 * i
    # fp32 inputs: only the bf16 tensor-core kernel has the transition mode
    assert L.kda_chunk_segment_transition(ptr(0), ptr(1), ptr(2), ptr(3), ptr(4), -5.0, ptr(5),
                                          kda.KDA_F32, 1, 64, 2, 128, 128, ptr(6), ptr(7),
                                          256, None) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_chunk_segment_transition(ptr(0), ptr(1), ptr(2), ptr(3), ptr(4), -5.0, ptr(5),
                                          kda.KDA_BF16, 1, 64, 2, 64, 64, ptr(6), ptr(7),
                                          256, None) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_chunk_segment_transition(ptr(0), ptr(1), ptr(2), ptr(3), None, -5.0, ptr(5),
                                          kda.KDA_BF16, 1, 64, 2, 128, 128, ptr(6), ptr(7),
                                          256, None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_segment_transition(ptr(0), ptr(1), ptr(2), ptr(3), ptr(4), -5.0, ptr(5),
                                          kda.KDA_BF16, 1, 64, 2, 128, 128, ptr(6), ptr(7),
                                          16, None) == kda.KDA_ERR_WORKSPACE
    assert L.kda_chunk_segment_transition(ptr(0), ptr(1), ptr(2), ptr(3), ptr(4), -5.0, ptr(5),
                                          kda.KDA_BF16, 1, 64, 2, 128, 128, ptr(0), ptr(7),
                                          256, None) == kda.KDA_ERR_INVALID_ARG
    # prefix: index must be in [0, count); 128 x 128 only; no aliasing
    assert L.kda_chunk_state_prefix(ptr(0), 3, 3, None, 1, 2, 128, 128, ptr(1), None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_state_prefix(ptr(0), 3, -1, None, 1, 2, 128, 128, ptr(1), None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_state_prefix(ptr(0), 3, 1, None, 1, 2, 64, 64, ptr(1), None) == \
        kda.KDA_ERR_UNSUPPORTED
    assert L.kda_chunk_state_prefix(ptr(0), 3, 1, ptr(1), 1, 2, 128, 128, ptr(1), None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_state_prefix(ptr(0) + 4, 3, 1, None, 1, 2, 128, 128, ptr(1), None) == \
        kda.KDA_ERR_MISALIGNED



def test_backward_entries_reject_on_host(L):
    ptr = lambda i: FAKE + 0x1000 * i
    ws = L.kda_recurrent_bwd_workspace_size(1, 100, 2, 128, 128, 0)
    # the device status word, then per (sequence, head) and 32-token chunk: its
    # start state, the gradient of its end state (64 KB each), three 32 x 32
    # key-side matrices and four 32 x dv intermediates (R, U, dU, W)
    per_chunk = (2 * 128 * 128 + 3 * 32 * 32 + 4 * 32 * 128) * 4
    assert ws == 256 + 2 * 4 * per_chunk
    assert L.kda_recurrent_bwd_workspace_size(1, 0, 2, 128, 128, 0) == 256
    assert L.kda_recurrent_bwd_workspace_size(1, 100, 2, 96, 128, 0) == 0
    # packed: 3 sequences in 100 tokens take at most ceil(100/32) + 3 chunks
    assert L.kda_recurrent_bwd_workspace_size(1, 100, 2, 128, 128, 3) == 256 + 256 + 2 * 7 * per_chunk
    assert L.kda_recurrent_bwd_workspace_size(2, 100, 2, 128, 128, 3) == 0  # packed needs B == 1

    def args(**over):
        a = dict(q=ptr(0), k=ptr(1), v=ptr(2), g=ptr(3), beta=ptr(4), dt=kda.KDA_BF16,
                 init=None, dout=ptr(5), dfinal=None, cu=None, nseq=0, B=1, T=100, H=2, dk=128,
                 dv=128, scale=1.0, dq=ptr(6), dko=ptr(7), dvo=ptr(8), dg=ptr(9), dbeta=ptr(10),
                 dinit=None, ws=ptr(11), wsb=ws, stream=None)
        a.update(over)
        return list(a.values())

    assert L.kda_recurrent_bwd(*args(dk=96)) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_recurrent_bwd(*args(dt=7)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_recurrent_bwd(*args(dout=None)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_recurrent_bwd(*args(B=0)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_recurrent_bwd(*args(scale=float("nan"))) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_recurrent_bwd(*args(wsb=ws - 16)) == kda.KDA_ERR_WORKSPACE
    assert L.kda_recurrent_bwd(*args(ws=None)) == kda.KDA_ERR_WORKSPACE
    assert L.kda_recurrent_bwd(*args(dg=ptr(9) + 4)) == kda.KDA_ERR_MISALIGNED
    assert L.kda_recurrent_bwd(*args(dq=ptr(0))) == kda.KDA_ERR_INVALID_ARG  # dq aliases q
    assert L.kda_recurrent_bwd(*args(dinit=ptr(11))) == kda.KDA_ERR_INVALID_ARG  # aliases ws
    assert L.kda_recurrent_bwd(*args(cu=ptr(12), nseq=0)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_recurrent_bwd(*args(cu=ptr(12), nseq=3, B=2)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_recurrent_bwd(*args(nseq=3)) == kda.KDA_ERR_INVALID_ARG  # counts without offsets
    assert L.kda_recurrent_bwd(*args(cu=ptr(12) + 4, nseq=3, wsb=10 ** 9)) == \
        kda.KDA_ERR_MISALIGNED
    # packed workspace is larger than the dense one for the same T
    assert L.kda_recurrent_bwd(*args(cu=ptr(12), nseq=3)) == kda.KDA_ERR_WORKSPACE
    # empty sequence with no d_init requested: nothing to do, nothing launched
    ws0 = L.kda_recurrent_bwd_workspace_size(1, 0, 2, 128, 128, 0)
    assert L.kda_recurrent_bwd(*args(T=0, q=None, k=None, v=None, g=None, beta=None, dout=None,
                                     dq=None, dko=None, dvo=None, dg=None, dbeta=None,
                                     wsb=ws0)) == kda.KDA_OK


def test_host_stream_entry_rejects_on_host(L):
    ptr = lambda i: FAKE + 0x1000 * i
    n = L.kda_chunk_fwd_gated_host_workspace_size(2, 4096, 4, 128, 128, kda.KDA_BF16)
    assert n > 0
    assert L.kda_chunk_fwd_gated_host_workspace_size(4, 4096, 4, 128, 128, kda.KDA_BF16) > n
    assert L.kda_chunk_fwd_gated_host_workspace_size(2, 4096, 4, 96, 128, kda.KDA_BF16) == 0
    assert L.kda_chunk_fwd_gated_host_workspace_size(2, 0, 4, 128, 128, kda.KDA_BF16) == 0

    def args(**over):
        a = dict(q=ptr(0), k=ptr(1), v=ptr(2), z=ptr(3), A_log=ptr(4), g_min=-5.0, beta=ptr(5),
                 dt=kda.KDA_BF16, init=None, B=2, T=4096, H=4, dk=128, dv=128, scale=1.0,
                 out=ptr(6), final=None, ws=ptr(16), wsb=n, stream=None, copy=None)
        a.update(over)
        return list(a.values())

    assert L.kda_chunk_fwd_gated_host(*args(out=None)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_fwd_gated_host(*args(A_log=None)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_fwd_gated_host(*args(g_min=0.5)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_fwd_gated_host(*args(dt=9)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_fwd_gated_host(*args(T=0)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_chunk_fwd_gated_host(*args(dv=48)) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_chunk_fwd_gated_host(*args(ws=ptr(16) + 16)) == kda.KDA_ERR_MISALIGNED
    assert L.kda_chunk_fwd_gated_host(*args(wsb=n - 1)) == kda.KDA_ERR_WORKSPACE
    assert L.kda_chunk_fwd_gated_host(*args(out=ptr(2))) == kda.KDA_ERR_INVALID_ARG  # aliases v


def test_gate_backward_rejects_on_host(L):
    ptr = lambda i: FAKE + 0x1000 * i
    n = L.kda_gate_bwd_workspace_size(4)
    assert n == 4 * 256 * 4 and L.kda_gate_bwd_workspace_size(0) == 0

    def args(**over):
        a = dict(z=ptr(0), A_log=ptr(1), g_min=-5.0, dg=ptr(2), dz=ptr(3), dA=ptr(4), rows=10,
                 H=4, dk=64, ws=ptr(5), wsb=n, stream=None)
        a.update(over)
        return list(a.values())

    assert L.kda_gate_bwd(*args(dg=None)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_gate_bwd(*args(g_min=1.0)) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_gate_bwd(*args(dk=96)) == kda.KDA_ERR_UNSUPPORTED      # not a power of two
    assert L.kda_gate_bwd(*args(dk=2048)) == kda.KDA_ERR_UNSUPPORTED
    assert L.kda_gate_bwd(*args(wsb=n - 4)) == kda.KDA_ERR_WORKSPACE
    assert L.kda_gate_bwd(*args(dz=ptr(3) + 8)) == kda.KDA_ERR_MISALIGNED
    assert L.kda_gate_bwd(*args(dz=ptr(0))) == kda.KDA_ERR_INVALID_ARG   # dz aliases z
    assert L.kda_gate_bwd(*args(dA=ptr(3))) == kda.KDA_ERR_INVALID_ARG   # dA_log aliases dz


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: without libkda.so every entry point raises."""
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libkda.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="libkda.so not found"):
        _lib.lib()
    with pytest.raises(RuntimeError):
        kda.kda_status_string(0)
