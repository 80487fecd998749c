"""ctypes binding of libkda's C ABI (include/kda.h): argument marshalling only.

Every function below has the name of the C entry point it calls, takes torch
tensors (device memory) and plain numbers, and passes their pointers, sizes
and the current CUDA stream through unchanged.  No computation happens here;
if libkda.so is missing or fails to load, every call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")
# the same sources built with device-side bounds checks (KDA_DEBUG_CHECKS)
DEBUG_LIB_PATH = os.path.join(_HERE, "libkda_debug.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_MISALIGNED = 3
KDA_ERR_WORKSPACE = 4
KDA_ERR_CUDA = 5
KDA_ERR_TIMEOUT = 6
KDA_ERR_BAD_SEQLENS = 7
KDA_ERR_BOUNDS = 8

KDA_F32 = 0
KDA_BF16 = 1

_VP = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "kda_status_string": (ctypes.c_char_p, [_I]),
    "kda_last_cuda_error_string": (ctypes.c_char_p, []),
    "kda_gate_fwd": (_I, [_VP, _VP, _F, _VP, _I64, _I, _I, _VP]),
    "kda_gate_bwd_workspace_size": (_SZ, [_I]),
    "kda_gate_bwd": (_I, [_VP, _VP, _F, _VP, _VP, _VP, _I64, _I, _I, _VP, _SZ, _VP]),
    "kda_chunk_fwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "kda_chunk_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _VP, _VP, _I, _I, _I, _I, _I, _I,
                           _F, _I, _VP, _VP, _VP, _SZ, _VP]),
    "kda_chunk_segment_transition": (_I, [_VP, _VP, _VP, _VP, _VP, _F, _VP, _I, _I, _I, _I, _I,
                                          _I, _VP, _VP, _SZ, _VP]),
    "kda_chunk_state_prefix": (_I, [_VP, _I, _I, _VP, _I, _I, _I, _I, _VP, _VP]),
    "kda_chunk_fwd_gated": (_I, [_VP, _VP, _VP, _VP, _VP, _F, _VP, _I, _VP, _VP, _I, _I, _I, _I,
                                 _I, _I, _F, _I, _VP, _VP, _VP, _SZ, _VP]),
    "kda_decode_step": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _VP, _I, _I, _I, _I, _F, _VP, _VP]),
    "kda_decode_step_gated": (_I, [_VP, _VP, _VP, _VP, _VP, _F, _VP, _I, _VP, _I, _I, _I, _I, _F,
                                   _VP, _VP]),
    "kda_chunk_fwd_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _VP, _VP, _I, _I, _I, _I, _I, _I,
                                   _F, _I, _VP, _VP, _VP]),
    "kda_decode_verify": (_I, [_VP, _VP, _VP, _VP, _VP, _F, _VP, _I, _VP, _I, _I, _I, _I, _I, _F,
                               _VP, _VP]),
    "kda_decode_replay": (_I, [_VP, _VP, _VP, _VP, _F, _VP, _I, _VP, _VP, _I, _I, _I, _I, _I,
                               _VP]),
    "kda_chunk_fwd_gated_host_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "kda_chunk_fwd_gated_host": (_I, [_VP, _VP, _VP, _VP, _VP, _F, _VP, _I, _VP, _I, _I, _I, _I,
                                      _I, _F, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "kda_recurrent_bwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "kda_recurrent_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _VP, _VP, _VP, _VP, _I, _I, _I, _I,
                               _I, _I, _F, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "kda_get_device_status": (_I, [_VP, _VP, ctypes.POINTER(ctypes.c_int32)]),
    "kda_noalloc_get_device_status": (_I, [ctypes.POINTER(ctypes.c_int32), _VP]),
    "kda_selftest_bounded_wait": (_I, [_VP, _I64, _VP]),
    "kda_debug_checks_enabled": (_I, []),
    "kda_selftest_bounds_check": (_I, [_VP, _VP]),
    "kda_set_wait_limit_ns": (_I, [_I64]),
}

_lib = None
_lib_path = LIB_PATH


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where} failed: {kda_status_string(status)} ({status})"
        if status == KDA_ERR_CUDA:
            msg += f" [{kda_last_cuda_error_string()}]"
        super().__init__(msg)


def _load(path):
    if not os.path.exists(path):
        raise RuntimeError(
            f"{os.path.basename(path)} not found at {path}; build it with "
            "`python -m gated_delta_rule_158_b200.build`")
    L = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


def lib():
    """The selected library, libkda.so unless select_library(debug=True) was
    called (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


def select_library(debug: bool):
    """Routes every call of this module to libkda_debug.so (debug=True) or
    libkda.so.  Returns the previously selected library's path."""
    global _lib, _lib_path
    prev = _lib_path
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if path != _lib_path or _lib is None:
        _lib = _load(path)
        _lib_path = path
    return prev


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("libkda takes contiguous tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported input dtype {t.dtype}")


def _check(status, where):
    if status != KDA_OK:
        raise KdaError(status, where)


def kda_status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def kda_last_cuda_error_string() -> str:
    return lib().kda_last_cuda_error_string().decode()


def kda_gate_fwd(z, A_log, g, g_min=-5.0, stream=None):
    """g = g_min * sigmoid(exp(A_log[h]) * z); z, g fp32 [..., H, dk]."""
    H, dk = z.shape[-2], z.shape[-1]
    rows = z.numel() // (H * dk) if z.numel() else 0
    _check(lib().kda_gate_fwd(_ptr(z), _ptr(A_log), float(g_min), _ptr(g), rows, H, dk,
                              _stream(stream)), "kda_gate_fwd")


def kda_gate_bwd_workspace_size(H) -> int:
    return int(lib().kda_gate_bwd_workspace_size(H))


def kda_gate_bwd(z, A_log, dg, dz, dA_log, workspace, g_min=-5.0, stream=None):
    """dz [..., H, dk] and dA_log [H] from dg through the gate
    g = g_min * sigmoid(exp(A_log[h]) * z); dz may be dg itself."""
    H, dk = z.shape[-2], z.shape[-1]
    rows = z.numel() // (H * dk) if z.numel() else 0
    _check(lib().kda_gate_bwd(_ptr(z), _ptr(A_log), float(g_min), _ptr(dg), _ptr(dz),
                              _ptr(dA_log), rows, H, dk, _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)),
           "kda_gate_bwd")


def kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs=0, chunk_size=0,
                                 in_dtype=KDA_BF16) -> int:
    return int(lib().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size,
                                                  in_dtype))


def kda_chunk_fwd(q, k, v, g, beta, out, workspace, init_state=None, cu_seqlens=None,
                  final_state=None, scale=1.0, chunk_size=0, stream=None):
    """Chunkwise forward; q, k, g [B,T,H,dk], v/out [B,T,H,dv], beta [B,T,H]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(lib().kda_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _dtype(q), _ptr(init_state),
        _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv, float(scale), int(chunk_size), _ptr(out),
        _ptr(final_state), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)), "kda_chunk_fwd")


def kda_chunk_fwd_noalloc(q, k, v, g, beta, out, init_state=None, cu_seqlens=None,
                          final_state=None, scale=1.0, chunk_size=0, stream=None):
    """kda_chunk_fwd using the library's built-in scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/kda.h)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(lib().kda_chunk_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _dtype(q), _ptr(init_state),
        _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv, float(scale), int(chunk_size), _ptr(out),
        _ptr(final_state), _stream(stream)), "kda_chunk_fwd_noalloc")


def kda_chunk_fwd_gated(q, k, v, z, A_log, beta, out, workspace, g_min=-5.0, init_state=None,
                        cu_seqlens=None, final_state=None, scale=1.0, chunk_size=0, stream=None):
    """kda_chunk_fwd with the gate fused in: z [B,T,H,dk] and A_log [H] replace g."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(lib().kda_chunk_fwd_gated(
        _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), float(g_min), _ptr(beta), _dtype(q),
        _ptr(init_state), _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv, float(scale),
        int(chunk_size), _ptr(out), _ptr(final_state), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)), "kda_chunk_fwd_gated")


def kda_chunk_segment_transition(q, k, v, z, A_log, beta, pairs, workspace, g_min=-5.0,
                                 stream=None):
    """Per (b, h) of the segment given: pairs[b, h, 0] = S~ (from a zero state),
    pairs[b, h, 1] = M (the segment's transition); pairs fp32 [B, H, 2, 128, 128]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(lib().kda_chunk_segment_transition(
        _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), float(g_min), _ptr(beta), _dtype(q),
        B, T, H, dk, dv, _ptr(pairs), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "kda_chunk_segment_transition")


def kda_chunk_state_prefix(pairs, index, state_out, init_state=None, stream=None):
    """Incoming state of segment `index` from the pairs [count, B, H, 2, dk, dv] of the
    segments in order: S_in[0] = init (or 0), S_in[r + 1] = S~_r + M_r S_in[r]."""
    count, B, H = pairs.shape[0], pairs.shape[1], pairs.shape[2]
    dk, dv = pairs.shape[-2], pairs.shape[-1]
    _check(lib().kda_chunk_state_prefix(_ptr(pairs), count, int(index), _ptr(init_state), B, H,
                                        dk, dv, _ptr(state_out), _stream(stream)),
           "kda_chunk_state_prefix")


def kda_decode_step_gated(q, k, v, z, A_log, beta, state, out, g_min=-5.0, scale=1.0,
                          stream=None):
    """kda_decode_step with the gate fused in: z [N,H,dk] and A_log [H] replace g."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    _check(lib().kda_decode_step_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log),
                                       float(g_min), _ptr(beta), _dtype(q), _ptr(state), N, H,
                                       dk, dv, float(scale), _ptr(out), _stream(stream)),
           "kda_decode_step_gated")


def kda_decode_step(q, k, v, g, beta, state, out, scale=1.0, stream=None):
    """One decode step; q, k, g [N,H,dk], v/out [N,H,dv], beta [N,H], state in place."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    _check(lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _dtype(q),
                                 _ptr(state), N, H, dk, dv, float(scale), _ptr(out),
                                 _stream(stream)), "kda_decode_step")


def kda_decode_verify(q, k, v, g, beta, state, out, A_log=None, g_min=-5.0, scale=1.0,
                      stream=None):
    """Outputs of K draft tokens per sequence, state read only.  q, k, g
    [N,K,H,dk], v/out [N,K,H,dv], beta [N,K,H]; g is z when A_log is given."""
    N, K, H, dk = q.shape
    dv = v.shape[-1]
    _check(lib().kda_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(A_log),
                                   float(g_min), _ptr(beta), _dtype(q), _ptr(state), N, H, K, dk,
                                   dv, float(scale), _ptr(out), _stream(stream)),
           "kda_decode_verify")


def kda_decode_replay(k, v, g, beta, state, accept_len, A_log=None, g_min=-5.0, stream=None):
    """Apply each sequence's first accept_len[n] tokens to the state in place."""
    N, K, H, dk = k.shape
    dv = v.shape[-1]
    _check(lib().kda_decode_replay(_ptr(k), _ptr(v), _ptr(g), _ptr(A_log), float(g_min),
                                   _ptr(beta), _dtype(k), _ptr(state), _ptr(accept_len), N, H, K,
                                   dk, dv, _stream(stream)), "kda_decode_replay")


def kda_chunk_fwd_gated_host_workspace_size(B, T, H, dk, dv, in_dtype=KDA_BF16) -> int:
    return int(lib().kda_chunk_fwd_gated_host_workspace_size(B, T, H, dk, dv, in_dtype))


def kda_chunk_fwd_gated_host(q, k, v, z, A_log, beta, out, workspace, g_min=-5.0,
                             init_state=None, final_state=None, scale=1.0, stream=None,
                             copy_stream=None):
    """Gated chunked prefill of a dense batch in host memory (CPU tensors,
    page-locked for overlap): q, k [B,T,H,dk], v [B,T,H,dv], z [B,T,H,dk]
    fp32, A_log [H], beta [B,T,H]; out [B,T,H,dv] and final_state
    [B,H,dk,dv] are host tensors written by the time `stream` reaches the end
    of the call's work.  workspace is a device uint8 tensor."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t in (q, k, v, z, A_log, beta, out, init_state, final_state):
        if t is not None and t.is_cuda:
            raise ValueError("kda_chunk_fwd_gated_host takes host tensors")
    _check(lib().kda_chunk_fwd_gated_host(
        _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), float(g_min), _ptr(beta), _dtype(q),
        _ptr(init_state), B, T, H, dk, dv, float(scale), _ptr(out), _ptr(final_state),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
        None if copy_stream is None else _stream(copy_stream)), "kda_chunk_fwd_gated_host")


def kda_recurrent_bwd_workspace_size(B, T, H, dk, dv, num_seqs=0) -> int:
    return int(lib().kda_recurrent_bwd_workspace_size(B, T, H, dk, dv, num_seqs))


def kda_recurrent_bwd(q, k, v, g, beta, dout, grads, workspace, init_state=None, d_final=None,
                      cu_seqlens=None, scale=1.0, stream=None):
    """Gradients through the recurrence.  q, k, g [B,T,H,dk]; v, dout
    [B,T,H,dv]; beta [B,T,H]; cu_seqlens (int32 [N+1], B == 1) for a packed
    batch.  `grads` is a dict of fp32 output tensors dq, dk, dg [B,T,H,dk],
    dv [B,T,H,dv], dbeta [B,T,H] and optionally d_init [N,H,dk,dv]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(lib().kda_recurrent_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _dtype(q), _ptr(init_state), _ptr(dout),
        _ptr(d_final), _ptr(cu_seqlens), N, B, T, H, dk, dv, float(scale), _ptr(grads["dq"]),
        _ptr(grads["dk"]), _ptr(grads["dv"]), _ptr(grads["dg"]), _ptr(grads["dbeta"]),
        _ptr(grads.get("d_init")), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)), "kda_recurrent_bwd")


def kda_get_device_status(workspace, stream=None):
    """(status, detail) recorded on the device in this workspace; syncs the stream."""
    detail = ctypes.c_int32(0)
    st = lib().kda_get_device_status(_ptr(workspace), _stream(stream), ctypes.byref(detail))
    return int(st), int(detail.value)


def kda_noalloc_get_device_status(stream=None):
    """(status, detail) that the last kda_chunk_fwd_noalloc call on the current
    device recorded in the library's built-in scratch; syncs the stream."""
    detail = ctypes.c_int32(0)
    st = lib().kda_noalloc_get_device_status(ctypes.byref(detail), _stream(stream))
    return int(st), int(detail.value)


def kda_set_wait_limit_ns(limit_ns):
    """Diagnostic: bound of the chunk kernel's internal waits (default 2e9 ns)."""
    _check(lib().kda_set_wait_limit_ns(int(limit_ns)), "kda_set_wait_limit_ns")


def kda_debug_checks_enabled() -> bool:
    return bool(lib().kda_debug_checks_enabled())


def kda_selftest_bounds_check(workspace, stream=None):
    _check(lib().kda_selftest_bounds_check(_ptr(workspace), _stream(stream)),
           "kda_selftest_bounds_check")


def kda_selftest_bounded_wait(workspace, spin_limit_ns, stream=None):
    _check(lib().kda_selftest_bounded_wait(_ptr(workspace), int(spin_limit_ns),
                                           _stream(stream)), "kda_selftest_bounded_wait")
