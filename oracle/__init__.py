"""fp64 CPU oracle for the KDA path -- TEST INFRASTRUCTURE.

Only tests/, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
import this package.  It shares no code with the CUDA path: the arithmetic is
the plain C in ``kda_oracle.c`` (compiled with gcc by ``oracle/build.py``);
this module only marshals numpy arrays.

Functions
---------
gate(z, A_log, g_min=-5.0)
    "NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Model Architecture > Kimi
    Delta Attention (KDA) > Lower-bounded decay: g = g_min * Sigmoid(e^{A_h} z).
forward(q, k, v, g, beta, ...)
    Same page and section, state-update equation: the sequential recurrence
    S_t = (I - b_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + b_t k_t v_t^T and
    o_t = scale * S_t^T q_t, token by token in fp64.
backward(q, k, v, g, beta, dout, ...)
    Gradients of a loss through that recurrence (reverse-mode chain rule on
    the same steps; the pages give the forward only), dense layout, fp64.
gate_backward(z, A_log, dg, g_min=-5.0)
    dz and dA_log from dg through the gate (chain rule of the gate formula).

Every function is pinned: gate and forward by tests/test_oracle_pins.py
(closed forms, invariants, brute-force product form, special cases), the two
backward functions by tests/test_oracle_backward_pins.py (central finite
differences of the forward functions, closed forms).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.kda_oracle_gate.restype = None
        lib.kda_oracle_gate.argtypes = [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_double, ctypes.c_void_p]
        lib.kda_oracle_gate_backward.restype = None
        lib.kda_oracle_gate_backward.argtypes = [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p]
        lib.kda_oracle_forward.restype = ctypes.c_int
        lib.kda_oracle_forward.argtypes = [
            ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_int]
        lib.kda_oracle_backward.restype = ctypes.c_int
        lib.kda_oracle_backward.argtypes = [
            ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def gate(z, A_log, g_min: float = -5.0):
    """g = g_min * sigmoid(exp(A_log[h]) * z) for z of shape [..., H, dk]."""
    z = _f64(z)
    A_log = _f64(A_log).reshape(-1)
    H, dk = z.shape[-2], z.shape[-1]
    assert A_log.shape[0] == H
    rows = int(np.prod(z.shape[:-2])) if z.ndim > 2 else 1
    out = np.empty_like(z)
    _load().kda_oracle_gate(rows, H, dk, _ptr(z), _ptr(A_log), float(g_min),
                            _ptr(out))
    return out


def gate_backward(z, A_log, dg, g_min: float = -5.0):
    """(dz, dA_log) for the gate g = g_min * sigmoid(exp(A_log[h]) * z), given
    dg of z's shape [..., H, dk]; fp64."""
    z = _f64(z)
    dg = _f64(dg)
    A_log = _f64(A_log).reshape(-1)
    H, dk = z.shape[-2], z.shape[-1]
    assert A_log.shape[0] == H and dg.shape == z.shape
    rows = int(np.prod(z.shape[:-2])) if z.ndim > 2 else 1
    dz = np.empty_like(z)
    dA = np.empty(H)
    _load().kda_oracle_gate_backward(rows, H, dk, _ptr(z), _ptr(A_log), float(g_min),
                                     _ptr(dg), _ptr(dz), _ptr(dA))
    return dz, dA


def forward(q, k, v, g, beta, init_state=None, cu_seqlens=None,
            scale: float = 1.0, units=None, nthreads=None, want_o=True):
    """Sequential fp64 KDA recurrence.

    Dense layout: q, k, g [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H].
    Varlen layout (cu_seqlens given): B == 1 and sequence n is tokens
    cu_seqlens[n] .. cu_seqlens[n+1]-1.  init_state is [N, H, dk, dv] or None.
    ``units`` optionally restricts the work to a list of (seq, head) pairs;
    the outputs of other units are left as NaN.

    Returns (o [B, T, H, dv] or None, final_state [N, H, dk, dv]).
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and g.shape == q.shape
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    if cu_seqlens is None:
        seq_off = np.arange(B + 1, dtype=np.int64) * T
    else:
        assert B == 1
        seq_off = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        assert seq_off[0] == 0 and seq_off[-1] == T
    N = seq_off.shape[0] - 1
    S0 = None if init_state is None else _f64(init_state)
    if S0 is not None:
        assert S0.shape == (N, H, dk, dv)
    o = np.full((B, T, H, dv), np.nan) if want_o else None
    S_out = np.full((N, H, dk, dv), np.nan)
    u = None
    nu = 0
    if units is not None:
        u = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 2))
        nu = u.shape[0]
    rc = _load().kda_oracle_forward(
        N, _ptr(seq_off), H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
        _ptr(beta), _ptr(S0), float(scale), _ptr(o), _ptr(S_out), _ptr(u), nu,
        int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return o, S_out


def backward(q, k, v, g, beta, dout, init_state=None, d_final=None, scale: float = 1.0):
    """Gradients of L = sum(o * dout) + sum(S_T * d_final) with respect to
    q, k, v, g, beta and the initial state, dense layout [B, T, H, *],
    in fp64.  Returns a dict with keys dq, dk, dv, dg, dbeta, dS0."""
    q, k, v, g, beta, dout = (_f64(a) for a in (q, k, v, g, beta, dout))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and g.shape == q.shape
    assert v.shape == (B, T, H, dv) and dout.shape == v.shape and beta.shape == (B, T, H)
    S0 = None if init_state is None else _f64(init_state)
    dF = None if d_final is None else _f64(d_final)
    for s_ in (S0, dF):
        if s_ is not None:
            assert s_.shape == (B, H, dk, dv)
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros_like(g), dbeta=np.zeros_like(beta),
               dS0=np.zeros((B, H, dk, dv)))
    rc = _load().kda_oracle_backward(
        B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
        _ptr(dout), _ptr(dF), float(scale), _ptr(out["dq"]), _ptr(out["dk"]),
        _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dS0"]))
    if rc != 0:
        raise MemoryError("oracle backward: out of memory")
    return out

