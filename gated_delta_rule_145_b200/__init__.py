"""B200 (sm_100a) gated delta rule forward pass: Python binding of libgdr.so.

The binding only marshals arguments: every step of the computation runs in the CUDA
kernels of ``libgdr.so`` (built in-tree by ``build.py``).  There is no CPU or PyTorch
fallback: importing works without a GPU, but every call needs the library and CUDA
tensors, and fails loudly otherwise.

The functions named ``gdr_*`` mirror the C ABI in ``include/gdr.h`` one to one
(pointer arguments take torch tensors, None or raw integer addresses).  ``prefill``
and ``decode_step`` are conveniences that check tensors and allocate the outputs.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "GdrError", "library", "gdr_prefill_chunked", "gdr_prefill_chunked_f32",
    "gdr_prefill_recurrent", "gdr_prefill_recurrent_f32", "gdr_decode_step",
    "gdr_decode_step_f32", "gdr_status_string", "gdr_device_status", "prefill", "decode_step", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdr.so")

GDR_OK = 0
GDR_ERR_NULL = -1
GDR_ERR_SHAPE = -2
GDR_ERR_UNSUPPORTED = -3
GDR_ERR_ALIGN = -4
GDR_ERR_OOM = -5
GDR_ERR_CUDA = -6
GDR_ERR_TIMEOUT = -7
GDR_ERR_TOO_LARGE = -8


class GdrError(RuntimeError):
    def __init__(self, name, status):
        super().__init__(f"{name} returned {status}: {gdr_status_string(status)}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int

_SIGS = {
    "gdr_prefill_chunked": [_P] * 11 + [_I] * 7 + [_P],
    "gdr_prefill_chunked_f32": [_P] * 11 + [_I] * 7 + [_P],
    "gdr_prefill_chunked_noalloc": [_P] * 11 + [_I] * 7 + [_P],
    "gdr_prefill_recurrent": [_P] * 11 + [_I] * 6 + [_P],
    "gdr_prefill_recurrent_f32": [_P] * 11 + [_I] * 6 + [_P],
    "gdr_decode_step": [_P] * 9 + [_I] * 5 + [_P],
    "gdr_decode_step_f32": [_P] * 9 + [_I] * 5 + [_P],
    "gdr_gla_prefill_chunked": [_P] * 11 + [_I] * 7 + [_P],
    "gdr_gla_prefill_chunked_f32": [_P] * 11 + [_I] * 7 + [_P],
    "gdr_gla_prefill_recurrent": [_P] * 11 + [_I] * 6 + [_P],
    "gdr_gla_prefill_recurrent_f32": [_P] * 11 + [_I] * 6 + [_P],
    "gdr_gla_decode_step": [_P] * 9 + [_I] * 5 + [_P],
    "gdr_gla_decode_step_f32": [_P] * 9 + [_I] * 5 + [_P],
    "gdr_short_conv_silu": [_P] * 6 + [_I] * 4 + [_P],
    "gdr_gated_rmsnorm": [_P] * 4 + [ctypes.c_longlong, _I, ctypes.c_float, _P],
    "gdr_gated_rmsnorm_f32": [_P] * 4 + [ctypes.c_longlong, _I, ctypes.c_float, _P],
    "gdr_prefill_segment_maps": [_P] * 10 + [_I] * 7 + [_P],
    "gdr_segment_combine": [_P] * 5 + [_I] * 4 + [_P],
    "gdr_prefill_chunked_cp": [_P] * 10 + [_I] * 7 + [_P],
    "gdr_prefill_chunked_host": [_P] * 10 + [_I] * 8 + [_P],
}


def library():
    """The loaded libgdr.so (ctypes).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m gated_delta_rule_145_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = _I
        lib.gdr_device_status.argtypes = [_P]
        lib.gdr_device_status.restype = _I
        lib.gdr_selftest_bounded_wait.argtypes = [_P]
        lib.gdr_selftest_bounded_wait.restype = _I
        lib.gdr_status_string.argtypes = [_I]
        lib.gdr_status_string.restype = ctypes.c_char_p
        lib.gdr_release_workspace.argtypes = []
        lib.gdr_release_workspace.restype = None
        _lib = lib
    return _lib


def gdr_status_string(status: int) -> str:
    return library().gdr_status_string(int(status)).decode()


def gdr_device_status(stream=None) -> int:
    """Synchronise `stream` and return the device-side status (GDR_OK or an error code)."""
    return library().gdr_device_status(_stream(stream))


def gdr_selftest_bounded_wait(stream=None) -> int:
    """Enqueue the failure-detection self-test (see include/gdr.h); gdr_device_status then
    reports GDR_ERR_TIMEOUT once its bounded wait has given up."""
    return library().gdr_selftest_bounded_wait(_stream(stream))


def gdr_release_workspace() -> None:
    """Return the workspace memory cached by earlier chunked prefill calls."""
    library().gdr_release_workspace()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return _P(x)
    return _P(x.data_ptr())


def _stream(s):
    if s is None:
        import torch

        return _P(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return _P(s)
    return _P(s.cuda_stream)


def _call(name, ptrs, ints, stream, check):
    fn = getattr(library(), name)
    status = fn(*[_ptr(p) for p in ptrs], *[int(i) for i in ints], _stream(stream))
    if check and status != GDR_OK:
        raise GdrError(name, status)
    return status


def gdr_prefill_chunked(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, cu_seqlens,
                        B, T, Hk, Hv, dk, dv, chunk, stream=None, check=True):
    return _call("gdr_prefill_chunked",
                 (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, cu_seqlens),
                 (B, T, Hk, Hv, dk, dv, chunk), stream, check)


def gdr_prefill_chunked_noalloc(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state,
                                cu_seqlens, B, T, Hk, Hv, dk, dv, chunk, stream=None, check=True):
    """gdr_prefill_chunked on the library's fixed scratch: no device memory is allocated
    (bf16, dk = dv = 128, chunk 32; see include/gdr.h for the size limit)."""
    return _call("gdr_prefill_chunked_noalloc",
                 (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, cu_seqlens),
                 (B, T, Hk, Hv, dk, dv, chunk), stream, check)


def gdr_prefill_chunked_host(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, B,
                             T, Hk, Hv, dk, dv, chunk=32, seg_tokens=0, stream=None,
                             check=True):
    """gdr_prefill_chunked from and to HOST buffers (pinned CPU tensors or raw addresses),
    the copies overlapped with the kernels; complete once `stream` is."""
    return _call("gdr_prefill_chunked_host",
                 (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state),
                 (B, T, Hk, Hv, dk, dv, chunk, seg_tokens), stream, check)


def gdr_prefill_segment_maps(q, k, v, a, b, A_log, dt_bias, phi, nmap, cu_seqlens, B, T, Hk,
                             Hv, dk, dv, chunk, stream=None, check=True):
    """Per-segment state maps S_end = phi S_start + nmap of B segments (include/gdr.h)."""
    return _call("gdr_prefill_segment_maps",
                 (q, k, v, a, b, A_log, dt_bias, phi, nmap, cu_seqlens),
                 (B, T, Hk, Hv, dk, dv, chunk), stream, check)


def gdr_segment_combine(phi, nmap, init_state, seg_init, final_state, G, Hv, dk, dv,
                        stream=None, check=True):
    """Composes G segment maps in order into start states and the final state."""
    return _call("gdr_segment_combine", (phi, nmap, init_state, seg_init, final_state),
                 (G, Hv, dk, dv), stream, check)


def gdr_prefill_chunked_cp(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, T, Hk,
                           Hv, dk, dv, chunk, nseg, stream=None, check=True):
    """One sequence cut into at most nseg segments processed side by side on this GPU."""
    return _call("gdr_prefill_chunked_cp",
                 (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state),
                 (T, Hk, Hv, dk, dv, chunk, nseg), stream, check)


def gdr_prefill_chunked_f32(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state,
                            cu_seqlens, B, T, Hk, Hv, dk, dv, chunk, stream=None, check=True):
    return _call("gdr_prefill_chunked_f32",
                 (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, cu_seqlens),
                 (B, T, Hk, Hv, dk, dv, chunk), stream, check)


def gdr_prefill_recurrent(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state,
                          cu_seqlens, B, T, Hk, Hv, dk, dv, stream=None, check=True):
    return _call("gdr_prefill_recurrent",
                 (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, cu_seqlens),
                 (B, T, Hk, Hv, dk, dv), stream, check)


def gdr_prefill_recurrent_f32(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state,
                              cu_seqlens, B, T, Hk, Hv, dk, dv, stream=None, check=True):
    return _call("gdr_prefill_recurrent_f32",
                 (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, cu_seqlens),
                 (B, T, Hk, Hv, dk, dv), stream, check)


def gdr_decode_step(q, k, v, a, b, A_log, dt_bias, state, out, B, Hk, Hv, dk, dv, stream=None,
                    check=True):
    return _call("gdr_decode_step", (q, k, v, a, b, A_log, dt_bias, state, out),
                 (B, Hk, Hv, dk, dv), stream, check)


def gdr_decode_step_f32(q, k, v, a, b, A_log, dt_bias, state, out, B, Hk, Hv, dk, dv,
                        stream=None, check=True):
    return _call("gdr_decode_step_f32", (q, k, v, a, b, A_log, dt_bias, state, out),
                 (B, Hk, Hv, dk, dv), stream, check)


# ------------------------------------------------------------------------- conveniences


def _check_tensors(tensors, dtype):
    import torch

    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        want = dtype if name in ("q", "k", "v", "a", "b") else (
            torch.int32 if name == "cu_seqlens" else torch.float32)
        if t.dtype != want:
            raise ValueError(f"{name} must be {want}, got {t.dtype}")


def _gla_wrapper(name, nptr):
    """Mirror of the C entry point `name`: nptr pointer arguments, then the sizes."""
    def fn(*args, stream=None, check=True):
        return _call(name, args[:nptr], args[nptr:], stream, check)
    fn.__name__ = name
    fn.__doc__ = f"{name}: the erase=False (gated linear attention) form; see include/gdr.h."
    return fn


gdr_gla_prefill_chunked = _gla_wrapper("gdr_gla_prefill_chunked", 11)
gdr_gla_prefill_chunked_f32 = _gla_wrapper("gdr_gla_prefill_chunked_f32", 11)
gdr_gla_prefill_recurrent = _gla_wrapper("gdr_gla_prefill_recurrent", 11)
gdr_gla_prefill_recurrent_f32 = _gla_wrapper("gdr_gla_prefill_recurrent_f32", 11)
gdr_gla_decode_step = _gla_wrapper("gdr_gla_decode_step", 9)
gdr_gla_decode_step_f32 = _gla_wrapper("gdr_gla_decode_step_f32", 9)


def gdr_short_conv_silu(x, weight, bias, conv_state_in, conv_state_out, y, B, T, C, width=4,
                        stream=None, check=True):
    """The four-tap causal convolution + SiLU before the rule (see include/gdr.h)."""
    return _call("gdr_short_conv_silu", (x, weight, bias, conv_state_in, conv_state_out, y),
                 (B, T, C, width), stream, check)


def _norm_call(name, o, z, weight, y, rows, d, eps, stream, check):
    fn = getattr(library(), name)
    status = fn(_ptr(o), _ptr(z), _ptr(weight), _ptr(y), ctypes.c_longlong(int(rows)), int(d),
                ctypes.c_float(eps), _stream(stream))
    if check and status != GDR_OK:
        raise GdrError(name, status)
    return status


def gdr_gated_rmsnorm(o, z, weight, y, rows, d, eps=1e-6, stream=None, check=True):
    """The gated RMS normalisation after the rule, bf16 gate (see include/gdr.h)."""
    return _norm_call("gdr_gated_rmsnorm", o, z, weight, y, rows, d, eps, stream, check)


def gdr_gated_rmsnorm_f32(o, z, weight, y, rows, d, eps=1e-6, stream=None, check=True):
    """The gated RMS normalisation after the rule, fp32 gate (see include/gdr.h)."""
    return _norm_call("gdr_gated_rmsnorm_f32", o, z, weight, y, rows, d, eps, stream, check)


def prefill(q, k, v, a, b, A_log, dt_bias, init_state=None, cu_seqlens=None, chunk=32,
            form="chunked", out=None, final_state=None, stream=None, erase=True):
    """Prefill over q, k [B, T, Hk, dk], v [B, T, Hv, dv], a, b [B, T, Hv] (bf16 or fp32).

    ``form`` is "chunked" (UT transform) or "recurrent".  With ``cu_seqlens`` (int32,
    device, [N + 1]) the tokens are packed along T (B must be 1) into N sequences.
    ``erase=False`` runs gated linear attention (the rule without its erase term).
    Returns (out [B, T, Hv, dv] fp32, final_state [Nseq, Hv, dk, dv] fp32).
    """
    import torch

    dtype = q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q, k, v, a, b must be bf16 or fp32")
    _check_tensors(dict(q=q, k=k, v=v, a=a, b=b, A_log=A_log, dt_bias=dt_bias,
                        init_state=init_state, cu_seqlens=cu_seqlens), dtype)
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    nseq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and B != 1:
        raise ValueError("packed sequences need B == 1")
    if out is None:
        out = torch.empty((B, T, Hv, dv), device=q.device, dtype=torch.float32)
    if final_state is None:
        final_state = torch.empty((nseq, Hv, dk, dv), device=q.device, dtype=torch.float32)
    f32 = dtype == torch.float32
    args = (q, k, v, a, b, A_log, dt_bias, init_state, out, final_state, cu_seqlens,
            nseq, B * T if cu_seqlens is not None else T, Hk, Hv, dk, dv)
    if form == "chunked":
        fn = ((gdr_prefill_chunked_f32 if f32 else gdr_prefill_chunked) if erase else
              (gdr_gla_prefill_chunked_f32 if f32 else gdr_gla_prefill_chunked))
        fn(*args, chunk, stream=stream)
    elif form == "recurrent":
        fn = ((gdr_prefill_recurrent_f32 if f32 else gdr_prefill_recurrent) if erase else
              (gdr_gla_prefill_recurrent_f32 if f32 else gdr_gla_prefill_recurrent))
        fn(*args, stream=stream)
    else:
        raise ValueError(f"unknown form {form!r}")
    return out, final_state


def decode_step(q, k, v, a, b, A_log, dt_bias, state, out=None, stream=None, erase=True):
    """One recurrent step: q, k [B, Hk, dk], v [B, Hv, dv], a, b [B, Hv]; ``state``
    [B, Hv, dk, dv] fp32 is updated in place (``erase=False``: gated linear attention).
    Returns out [B, Hv, dv] fp32."""
    import torch

    dtype = q.dtype
    _check_tensors(dict(q=q, k=k, v=v, a=a, b=b, A_log=A_log, dt_bias=dt_bias, state=state),
                   dtype)
    B, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if out is None:
        out = torch.empty((B, Hv, dv), device=q.device, dtype=torch.float32)
    f32 = dtype == torch.float32
    fn = ((gdr_decode_step_f32 if f32 else gdr_decode_step) if erase else
          (gdr_gla_decode_step_f32 if f32 else gdr_gla_decode_step))
    fn(q, k, v, a, b, A_log, dt_bias, state, out, B, Hk, Hv, dk, dv, stream=stream)
    return out
