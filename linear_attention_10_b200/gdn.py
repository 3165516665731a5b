"""Thin Python binding of libgdn.so (ctypes).  Argument marshalling only: every step of the
computation runs in the library's CUDA kernels; torch provides device memory and streams.

The functions carry the C names: ``gdn_chunk_prefill``, ``gdn_decode_step``,
``gdn_get_device_status``.  If the compiled library is missing or cannot be loaded, every call
raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_F32, GDN_BF16 = 0, 1
GDN_QK_L2NORM = 0x100           # flag in the dtype argument: q, k raw, normalised by the library
CHUNK = 32

# symbols declared in include/gdn.h
EXPORTS = (
    "gdn_status_string",
    "gdn_last_error",
    "gdn_version",
    "gdn_chunk_prefill_workspace_bytes",
    "gdn_chunk_prefill_workspace_bytes_ex",
    "gdn_chunk_prefill",
    "gdn_chunk_prefill_cuts",
    "gdn_chunk_prefill_noalloc",
    "gdn_decode_step",
    "gdn_decode_verify",
    "gdn_decode_verify_tree",
    "gdn_get_device_status",
    "gdn_selftest_wait_timeout",
    "gdn_profile_start",
    "gdn_profile_stop",
)

_lib = None


class GdnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        detail = ""
        try:
            d = lib().gdn_last_error()
            if d:
                detail = " [%s]" % d.decode()
        except Exception:  # pragma: no cover
            pass
        super().__init__("%s failed: %s (%d)%s" % (what, status_string(code), code, detail))


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libgdn.so is not built (%s); run `python -m linear_attention_10_b200.build`"
                           % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.gdn_status_string.argtypes = [i32]
    L.gdn_status_string.restype = ctypes.c_char_p
    L.gdn_version.argtypes = []
    L.gdn_version.restype = i32
    L.gdn_last_error.argtypes = []
    L.gdn_last_error.restype = ctypes.c_char_p
    L.gdn_chunk_prefill_workspace_bytes.argtypes = [i64, i32, i32, i32, i32]
    L.gdn_chunk_prefill_workspace_bytes.restype = sz
    L.gdn_chunk_prefill_workspace_bytes_ex.argtypes = [i64, i32, i32, i32, i32, i32]
    L.gdn_chunk_prefill_workspace_bytes_ex.restype = sz
    L.gdn_chunk_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, i32, i32, i32, i32,
                                    vp, sz, vp]
    L.gdn_chunk_prefill.restype = i32
    L.gdn_chunk_prefill_cuts.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, i32, vp, vp, vp, vp, i32, i32, i32,
                                         i32, vp, sz, vp]
    L.gdn_chunk_prefill_cuts.restype = i32
    L.gdn_chunk_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, i32, i32, i32, i32, vp]
    L.gdn_chunk_prefill_noalloc.restype = i32
    L.gdn_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]
    L.gdn_decode_step.restype = i32
    L.gdn_decode_verify.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    L.gdn_decode_verify.restype = i32
    L.gdn_decode_verify_tree.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    L.gdn_decode_verify_tree.restype = i32
    L.gdn_get_device_status.argtypes = [vp]
    L.gdn_get_device_status.restype = i32
    L.gdn_selftest_wait_timeout.argtypes = [i64, vp]
    L.gdn_selftest_wait_timeout.restype = i32
    L.gdn_profile_start.argtypes = []
    L.gdn_profile_start.restype = i32
    L.gdn_profile_stop.argtypes = [i32, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_int)]
    L.gdn_profile_stop.restype = i32
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().gdn_status_string(int(code)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise TypeError("q/k/v must be float32 or bfloat16, got %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, shape, dtype, dev):
    if not t.is_cuda or t.device != dev:
        raise ValueError("%s must be on %s" % (name, dev))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if t.dtype != dtype:
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def workspace_bytes(total_tokens: int, num_seqs: int, H: int, dk: int, dv: int, dtype_code: Optional[int] = None) -> int:
    """Workspace of a prefill call (num_seqs counts segments: sequences plus cut points); with a
    dtype code carrying GDN_QK_L2NORM the normalised q/k copies are included."""
    if dtype_code is None:
        return int(lib().gdn_chunk_prefill_workspace_bytes(int(total_tokens), int(num_seqs), int(H), int(dk),
                                                            int(dv)))
    return int(lib().gdn_chunk_prefill_workspace_bytes_ex(int(total_tokens), int(num_seqs), int(H), int(dk), int(dv),
                                                           int(dtype_code)))


def gdn_chunk_prefill(q, k, v, g, beta, cu_seqlens=None, state_in=None, out=None, state_out=None,
                      workspace=None, num_seqs: Optional[int] = None, stream=None, output_final_state=True,
                      normalize_qk=False):
    """Chunked gated-delta-rule prefill over packed sequences.

    q, k ``[T, H, dk]``; v ``[T, H, dv]`` (fp32 or bf16, same dtype); g, beta ``[T, H]`` fp32;
    cu_seqlens int32 ``[N + 1]`` on the device (or None with ``num_seqs`` equal-length sequences);
    state_in fp32 ``[N, H, dv, dk]`` or None.  Returns ``(out, state_out)``; buffers not given are
    allocated with torch.  ``state_out`` may be ``state_in`` (in-place resume).
    """
    T, H, dk = q.shape
    dv = v.shape[2]
    dev = q.device
    dt = q.dtype
    N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else int(num_seqs or 1)
    _check(q, "q", (T, H, dk), dt, dev)
    _check(k, "k", (T, H, dk), dt, dev)
    _check(v, "v", (T, H, dv), dt, dev)
    _check(g, "g", (T, H), torch.float32, dev)
    _check(beta, "beta", (T, H), torch.float32, dev)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    if state_in is not None:
        _check(state_in, "state_in", (N, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((T, H, dv), dtype=dt, device=dev)
    _check(out, "out", (T, H, dv), dt, dev)
    if state_out is None and output_final_state:
        state_out = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if state_out is not None:
        _check(state_out, "state_out", (N, H, dv, dk), torch.float32, dev)
    code = _dtype_code(q) | (GDN_QK_L2NORM if normalize_qk else 0)
    need = workspace_bytes(T, N, H, dk, dv, code)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    rc = lib().gdn_chunk_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, T,
                                 _ptr(state_in), _ptr(out), _ptr(state_out), H, dk, dv, code,
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_chunk_prefill")
    return out, state_out


def gdn_chunk_prefill_cuts(q, k, v, g, beta, cuts, cu_seqlens=None, state_in=None, out=None, state_out=None,
                           snapshots=None, workspace=None, num_seqs: Optional[int] = None, stream=None,
                           output_final_state=True, normalize_qk=False):
    """``gdn_chunk_prefill`` that also returns the state at each cut point: ``cuts`` int32 ``[n]`` on
    the device (strictly increasing token offsets, each strictly inside a sequence).  Returns
    ``(out, state_out, snapshots [n, H, dv, dk])``."""
    T, H, dk = q.shape
    dv = v.shape[2]
    dev = q.device
    dt = q.dtype
    N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else int(num_seqs or 1)
    nc = int(cuts.numel())
    _check(q, "q", (T, H, dk), dt, dev)
    _check(k, "k", (T, H, dk), dt, dev)
    _check(v, "v", (T, H, dv), dt, dev)
    _check(g, "g", (T, H), torch.float32, dev)
    _check(beta, "beta", (T, H), torch.float32, dev)
    _check(cuts, "cuts", (nc,), torch.int32, dev)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    if state_in is not None:
        _check(state_in, "state_in", (N, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((T, H, dv), dtype=dt, device=dev)
    _check(out, "out", (T, H, dv), dt, dev)
    if state_out is None and output_final_state:
        state_out = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if state_out is not None:
        _check(state_out, "state_out", (N, H, dv, dk), torch.float32, dev)
    if snapshots is None:
        snapshots = torch.empty((max(nc, 1), H, dv, dk), dtype=torch.float32, device=dev)[:nc]
    _check(snapshots, "snapshots", (nc, H, dv, dk), torch.float32, dev)
    code = _dtype_code(q) | (GDN_QK_L2NORM if normalize_qk else 0)
    need = workspace_bytes(T, N + nc, H, dk, dv, code)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    rc = lib().gdn_chunk_prefill_cuts(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, T,
                                      _ptr(cuts), nc, _ptr(state_in), _ptr(out), _ptr(state_out), _ptr(snapshots),
                                      H, dk, dv, code, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_chunk_prefill_cuts")
    return out, state_out, snapshots


def gdn_decode_step(q, k, v, g, beta, state, out=None, stream=None, normalize_qk=False):
    """One recurrent step for B sequences: q, k ``[B, H, dk]``, v ``[B, H, dv]``, g, beta ``[B, H]``,
    state fp32 ``[B, H, dv, dk]`` updated in place.  Returns ``out [B, H, dv]``."""
    B, H, dk = q.shape
    dv = v.shape[2]
    dev, dt = q.device, q.dtype
    _check(q, "q", (B, H, dk), dt, dev)
    _check(k, "k", (B, H, dk), dt, dev)
    _check(v, "v", (B, H, dv), dt, dev)
    _check(g, "g", (B, H), torch.float32, dev)
    _check(beta, "beta", (B, H), torch.float32, dev)
    _check(state, "state", (B, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, dv), dtype=dt, device=dev)
    _check(out, "out", (B, H, dv), dt, dev)
    code = _dtype_code(q) | (GDN_QK_L2NORM if normalize_qk else 0)
    rc = lib().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(out),
                               B, H, dk, dv, code, _stream_ptr(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_decode_step")
    return out


def gdn_decode_verify(q, k, v, g, beta, state_in, states_out=None, out=None, want_states=True, stream=None,
                      normalize_qk=False):
    """Tk speculative tokens per sequence through the recurrence: q, k ``[B, Tk, H, dk]``, v
    ``[B, Tk, H, dv]``, g, beta ``[B, Tk, H]``, state_in fp32 ``[B, H, dv, dk]`` (read only).
    Returns ``(out [B, Tk, H, dv], states_out [B, Tk, H, dv, dk] or None)``."""
    B, Tk, H, dk = q.shape
    dv = v.shape[3]
    dev, dt = q.device, q.dtype
    _check(q, "q", (B, Tk, H, dk), dt, dev)
    _check(k, "k", (B, Tk, H, dk), dt, dev)
    _check(v, "v", (B, Tk, H, dv), dt, dev)
    _check(g, "g", (B, Tk, H), torch.float32, dev)
    _check(beta, "beta", (B, Tk, H), torch.float32, dev)
    _check(state_in, "state_in", (B, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, Tk, H, dv), dtype=dt, device=dev)
    _check(out, "out", (B, Tk, H, dv), dt, dev)
    if states_out is None and want_states:
        states_out = torch.empty((B, Tk, H, dv, dk), dtype=torch.float32, device=dev)
    if states_out is not None:
        _check(states_out, "states_out", (B, Tk, H, dv, dk), torch.float32, dev)
    rc = lib().gdn_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in),
                                 None if states_out is None else _ptr(states_out), _ptr(out),
                                 B, Tk, H, dk, dv, _dtype_code(q) | (GDN_QK_L2NORM if normalize_qk else 0),
                                 _stream_ptr(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_decode_verify")
    return out, states_out


def gdn_decode_verify_tree(q, k, v, g, beta, parents, state_in, states_out=None, out=None, stream=None,
                           normalize_qk=False):
    """Tk drafted tokens per sequence verified as a tree: token t continues from the state after token
    ``parents[b, t]`` (an earlier token) or from state_in when that is -1.  Shapes as
    ``gdn_decode_verify`` plus parents int32 ``[B, Tk]`` on the device.  Returns ``(out [B, Tk, H,
    dv], states_out [B, Tk, H, dv, dk])``; a parent that is not -1 or an earlier token is reported by
    ``gdn_get_device_status`` as GDN_ERR_BAD_PARENTS."""
    B, Tk, H, dk = q.shape
    dv = v.shape[3]
    dev, dt = q.device, q.dtype
    _check(q, "q", (B, Tk, H, dk), dt, dev)
    _check(k, "k", (B, Tk, H, dk), dt, dev)
    _check(v, "v", (B, Tk, H, dv), dt, dev)
    _check(g, "g", (B, Tk, H), torch.float32, dev)
    _check(beta, "beta", (B, Tk, H), torch.float32, dev)
    _check(parents, "parents", (B, Tk), torch.int32, dev)
    _check(state_in, "state_in", (B, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, Tk, H, dv), dtype=dt, device=dev)
    _check(out, "out", (B, Tk, H, dv), dt, dev)
    if states_out is None:
        states_out = torch.empty((B, Tk, H, dv, dk), dtype=torch.float32, device=dev)
    _check(states_out, "states_out", (B, Tk, H, dv, dk), torch.float32, dev)
    rc = lib().gdn_decode_verify_tree(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(parents),
                                      _ptr(state_in), _ptr(states_out), _ptr(out), B, Tk, H, dk, dv,
                                      _dtype_code(q) | (GDN_QK_L2NORM if normalize_qk else 0), _stream_ptr(stream))
    if rc != 0:
        raise GdnError(rc, "gdn_decode_verify_tree")
    return out, states_out


def gdn_get_device_status(stream=None) -> int:
    """Synchronise ``stream`` and return (and clear) the device status word."""
    return int(lib().gdn_get_device_status(_stream_ptr(stream)))


def gdn_profile_start() -> None:
    """Start per-kernel event timing of the library's launches (measurement aid)."""
    rc = lib().gdn_profile_start()
    if rc != 0:
        raise GdnError(rc, "gdn_profile_start")


def gdn_profile_stop(max_kernels: int = 16) -> dict:
    """Stop timing; returns ``{kernel_name: (total_ms, launches)}``."""
    names = ctypes.create_string_buffer(64 * max_kernels)
    ms = (ctypes.c_double * max_kernels)()
    cnt = (ctypes.c_int * max_kernels)()
    n = lib().gdn_profile_stop(max_kernels, names, ms, cnt)
    if n < 0:
        raise GdnError(n, "gdn_profile_stop")
    res = {}
    for i in range(min(n, max_kernels)):
        nm = names.raw[64 * i:64 * (i + 1)].split(b"\0", 1)[0].decode()
        res[nm] = (float(ms[i]), int(cnt[i]))
    return res
