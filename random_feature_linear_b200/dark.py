"""Python binding of the C ABI in include/dark.h (ctypes; marshalling only).

Every function here has the name of the C entry point it calls and does
nothing but convert arguments: torch tensors become device pointers, the
current torch stream becomes the cudaStream_t, statuses become exceptions.
All computation runs in the native library ``libdark.so``; importing this
module fails loudly if that library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdark.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m random_feature_linear_b200.build` "
        "(there is no fallback implementation)")
_lib = ctypes.CDLL(_LIB_PATH)

DARK_OK, DARK_ERR_INVALID_ARG, DARK_ERR_UNSUPPORTED, DARK_ERR_STALE_STATE = 0, 1, 2, 3
DARK_ERR_CUDA, DARK_ERR_NUMERIC, DARK_ERR_TIMEOUT = 4, 5, 6
DARK_F32, DARK_BF16 = 0, 1
DARK_CAUSAL, DARK_STABILISE, DARK_EXACT = 1, 2, 4
WS_HEADER_BYTES = 256

EXPORTS = ("dark_abi_version", "dark_status_string", "dark_projection_bytes",
           "dark_make_projection", "dark_attention_workspace_bytes", "dark_attention_fwd",
           "dark_state_init", "dark_decode_step", "dark_noalloc_scratch_bytes",
           "dark_attention_fwd_noalloc", "dark_cross_attention_workspace_bytes",
           "dark_cross_attention_fwd", "dark_cross_decode_step",
           "dark_attention_bwd_workspace_bytes", "dark_attention_bwd",
           "dark_sample_omega_workspace_bytes", "dark_sample_omega", "dark_redraw_schedule_init",
           "dark_redraw_on_forward", "dark_redraw_request", "dark_redraw_set_fixed",
           "dark_auto_uses_exact", "dark_set_test_stall_cycles")


class dark_projection(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int), ("m", ctypes.c_int), ("r", ctypes.c_int),
                ("d", ctypes.c_int), ("dtype", ctypes.c_int), ("generation", ctypes.c_uint64),
                ("w", ctypes.c_void_p)]


class dark_state(ctypes.Structure):
    _fields_ = [("kv", ctypes.c_void_p), ("z", ctypes.c_void_p), ("shift", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("m", ctypes.c_int), ("d", ctypes.c_int),
                ("generation", ctypes.c_uint64)]


class dark_redraw_schedule(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("draw", ctypes.c_uint64),
                ("interval", ctypes.c_int64), ("count", ctypes.c_int64), ("fixed", ctypes.c_int)]


_P = ctypes.POINTER
_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.dark_abi_version.restype = _i
_lib.dark_status_string.restype = ctypes.c_char_p
_lib.dark_set_test_stall_cycles.argtypes = [ctypes.c_longlong]
_lib.dark_set_test_stall_cycles.restype = None
_lib.dark_status_string.argtypes = [_i]
_lib.dark_projection_bytes.restype = _sz
_lib.dark_projection_bytes.argtypes = [_i, _i, _i, _i, _i]
_lib.dark_make_projection.restype = _i
_lib.dark_make_projection.argtypes = [_vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp,
                                      _P(dark_projection)]
_lib.dark_attention_workspace_bytes.restype = _sz
_lib.dark_attention_workspace_bytes.argtypes = [_P(dark_projection), _i, _i, _i, _i]
_lib.dark_attention_fwd.restype = _i
_lib.dark_attention_fwd.argtypes = [_P(dark_projection), _vp, _vp, _vp, _vp, _P(ctypes.c_int64),
                                    _P(ctypes.c_int64), _i, _i, _i, _vp, _i, _P(dark_state), _vp,
                                    _sz, _vp, _vp]
_lib.dark_noalloc_scratch_bytes.restype = _sz
_lib.dark_attention_fwd_noalloc.restype = _i
_lib.dark_attention_fwd_noalloc.argtypes = [_P(dark_projection), _vp, _vp, _vp, _vp,
                                            _P(ctypes.c_int64), _P(ctypes.c_int64), _i, _i, _i,
                                            _vp, _i, _P(dark_state), _vp, _vp]
_lib.dark_state_init.restype = _i
_lib.dark_state_init.argtypes = [_P(dark_projection), _P(dark_state), _vp]
_lib.dark_decode_step.restype = _i
_lib.dark_decode_step.argtypes = [_P(dark_projection), _P(dark_state), _vp, _vp, _vp, _vp, _vp,
                                  _vp, _vp]
_lib.dark_cross_attention_workspace_bytes.restype = _sz
_lib.dark_cross_attention_workspace_bytes.argtypes = [_P(dark_projection), _i, _i, _i, _i, _i]
_lib.dark_cross_attention_fwd.restype = _i
_lib.dark_cross_attention_fwd.argtypes = [_P(dark_projection), _vp, _P(ctypes.c_int64), _i, _vp,
                                          _vp, _vp, _P(ctypes.c_int64), _i, _vp, _vp,
                                          _P(ctypes.c_int64), _i, _i, _i, _P(dark_state), _vp,
                                          _sz, _vp, _vp]
_lib.dark_cross_decode_step.restype = _i
_lib.dark_cross_decode_step.argtypes = [_P(dark_projection), _P(dark_state), _vp, _vp, _vp, _vp]
_lib.dark_auto_uses_exact.restype = _i
_lib.dark_auto_uses_exact.argtypes = [_i, _i]
_lib.dark_sample_omega_workspace_bytes.restype = _sz
_lib.dark_sample_omega_workspace_bytes.argtypes = [_i, _i, _i, _i]
_lib.dark_sample_omega.restype = _i
_lib.dark_sample_omega.argtypes = [ctypes.c_uint64, ctypes.c_uint64, _i, _i, _i, _i, _vp, _vp, _sz,
                                   _vp]
_lib.dark_redraw_schedule_init.restype = _i
_lib.dark_redraw_schedule_init.argtypes = [_P(dark_redraw_schedule), ctypes.c_uint64,
                                           ctypes.c_int64, _i]
_lib.dark_redraw_on_forward.restype = _i
_lib.dark_redraw_on_forward.argtypes = [_P(dark_redraw_schedule), _i]
_lib.dark_redraw_request.restype = _i
_lib.dark_redraw_request.argtypes = [_P(dark_redraw_schedule), _i]
_lib.dark_redraw_set_fixed.restype = None
_lib.dark_redraw_set_fixed.argtypes = [_P(dark_redraw_schedule), _i]
_lib.dark_attention_bwd_workspace_bytes.restype = _sz
_lib.dark_attention_bwd_workspace_bytes.argtypes = [_i] * 8
_lib.dark_attention_bwd.restype = _i
_lib.dark_attention_bwd.argtypes = [_vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                    _P(ctypes.c_int64), _vp, _P(ctypes.c_int64), _i, _i, _i, _vp,
                                    _i, _vp, _vp, _vp, _P(ctypes.c_int64), _vp, _vp, _sz, _vp,
                                    _vp]


class DarkError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(dark_status_string(status))


def _check(status: int) -> None:
    if status != DARK_OK:
        raise DarkError(status)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _strides(given, *tensors):
    """Element strides {b, h, l} of [B][H][L][d] tensors for the C ABI: the given
    ones, else the tensors' own, which must agree and have a unit d stride."""
    if given is None:
        own = {tuple(t.stride()) for t in tensors}
        if len(own) != 1:
            raise ValueError("tensors sharing one stride argument have different strides")
        s = own.pop()
        if len(s) != 4 or s[3] != 1:
            raise ValueError("expected [B][H][L][d] tensors with a unit d stride")
        given = s[:3]
    return (ctypes.c_int64 * 3)(*given)


def _dense(t, name):
    """Arrays without stride arguments cross the ABI as dense row-major buffers."""
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _dptr(t, name) -> int | None:
    return _ptr(_dense(t, name))


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def library_path() -> str:
    return _LIB_PATH


def dark_abi_version() -> int:
    return _lib.dark_abi_version()


def dark_status_string(status: int) -> str:
    return _lib.dark_status_string(status).decode()


def dark_set_test_stall_cycles(cycles: int) -> None:
    """Testing hook of the device time-out path (0 turns it off); see dark.h."""
    _lib.dark_set_test_stall_cycles(int(cycles))


def dark_projection_bytes(heads: int, m: int, r: int, d: int, dtype: int) -> int:
    return _lib.dark_projection_bytes(heads, m, r, d, dtype)


def dark_make_projection(omega: torch.Tensor, geom: torch.Tensor, H: int, dtype: int,
                         w: torch.Tensor | None = None, stream=None) -> tuple:
    """omega [H_o, m, r] and geom [H_m, r, d] fp32 device tensors.

    Returns (dark_projection, w_buffer); keep the buffer alive while the
    projection is used.
    """
    assert omega.dtype == torch.float32 and geom.dtype == torch.float32
    omega, geom = omega.contiguous(), geom.contiguous()
    ho, m, r = omega.shape
    hg, r2, d = geom.shape
    assert r == r2
    heads = max(ho, hg)
    nbytes = dark_projection_bytes(heads, m, r, d, dtype)
    if w is None:
        w = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=omega.device)
    proj = dark_projection()
    _check(_lib.dark_make_projection(_ptr(omega), ho, _ptr(geom), hg, H, m, r, d, dtype,
                                     _ptr(w), w.numel() * w.element_size(), _stream(stream),
                                     ctypes.byref(proj)))
    return proj, w


def dark_attention_workspace_bytes(proj: dark_projection, B: int, H: int, L: int,
                                   flags: int) -> int:
    return _lib.dark_attention_workspace_bytes(ctypes.byref(proj), B, H, L, flags)


def make_state(proj: dark_projection, B: int, H: int, device, stabilised: bool = False):
    """Allocates (torch) the arrays of a dark_state; returns (state, tensors)."""
    kv = torch.zeros(B, H, proj.m, proj.d, dtype=torch.float32, device=device)
    z = torch.zeros(B, H, proj.m, dtype=torch.float32, device=device)
    sh = torch.zeros(B, H, dtype=torch.float32, device=device) if stabilised else None
    st = dark_state(kv.data_ptr(), z.data_ptr(), _ptr(sh), B, H, proj.m, proj.d, 0)
    return st, (kv, z, sh)


def dark_attention_fwd(proj: dark_projection, q, k, v, out, B: int, H: int, L: int,
                       key_mask=None, flags: int = 0, state_out: dark_state | None = None,
                       ws=None, dev_status=None, stream=None, qkv_strides=None,
                       out_strides=None) -> None:
    """q/k/v/out are device tensors viewed as [B][H][L][d] with the given element
    strides ({b, h, l}; None = the tensors' own). ws: a zero-initialised uint8 tensor."""
    _check(_lib.dark_attention_fwd(
        ctypes.byref(proj), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _strides(qkv_strides, q, k, v),
        _strides(out_strides, out), B, H, L, _dptr(key_mask, "key_mask"), flags,
        None if state_out is None else ctypes.byref(state_out), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def dark_noalloc_scratch_bytes() -> int:
    return _lib.dark_noalloc_scratch_bytes()


def dark_attention_fwd_noalloc(proj: dark_projection, q, k, v, out, B: int, H: int, L: int,
                               key_mask=None, flags: int = 0,
                               state_out: dark_state | None = None, dev_status=None,
                               stream=None, qkv_strides=None, out_strides=None) -> None:
    """dark_attention_fwd with the library's fixed scratch instead of a workspace."""
    _check(_lib.dark_attention_fwd_noalloc(
        ctypes.byref(proj), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _strides(qkv_strides, q, k, v),
        _strides(out_strides, out), B, H, L, _dptr(key_mask, "key_mask"), flags,
        None if state_out is None else ctypes.byref(state_out), _ptr(dev_status),
        _stream(stream)))


def dark_state_init(proj: dark_projection, st: dark_state, stream=None) -> None:
    _check(_lib.dark_state_init(ctypes.byref(proj), ctypes.byref(st), _stream(stream)))


def dark_decode_step(proj: dark_projection, st: dark_state, q_t, k_t, v_t, out_t, valid=None,
                     dev_status=None, stream=None) -> None:
    _check(_lib.dark_decode_step(ctypes.byref(proj), ctypes.byref(st), _dptr(q_t, "q_t"),
                                 _dptr(k_t, "k_t"), _dptr(v_t, "v_t"), _dptr(out_t, "out_t"),
                                 _dptr(valid, "valid"), _ptr(dev_status), _stream(stream)))


def dark_cross_attention_workspace_bytes(proj: dark_projection, B: int, H: int, Lq: int, Lk: int,
                                         flags: int) -> int:
    return _lib.dark_cross_attention_workspace_bytes(ctypes.byref(proj), B, H, Lq, Lk, flags)


def dark_cross_attention_fwd(proj: dark_projection, q, k, v, out, B: int, H: int, Lq: int, Lk: int,
                             query_mask=None, context_mask=None, flags: int = 0,
                             context_out: dark_state | None = None, ws=None, dev_status=None,
                             stream=None, q_strides=None, kv_strides=None,
                             out_strides=None) -> None:
    """q/out viewed as [B][H][Lq][d], k/v as [B][H][Lk][d] with the given element
    strides ({b, h, l}; None = the tensors' own). ws: a zero-initialised uint8 tensor."""
    _check(_lib.dark_cross_attention_fwd(
        ctypes.byref(proj), _ptr(q), _strides(q_strides, q), Lq, _dptr(query_mask, "query_mask"), _ptr(k), _ptr(v),
        _strides(kv_strides, k, v), Lk, _dptr(context_mask, "context_mask"), _ptr(out), _strides(out_strides, out),
        B, H, flags,
        None if context_out is None else ctypes.byref(context_out), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def dark_cross_decode_step(proj: dark_projection, context: dark_state, q_t, out_t,
                           dev_status=None, stream=None) -> None:
    _check(_lib.dark_cross_decode_step(ctypes.byref(proj), ctypes.byref(context),
                                       _dptr(q_t, "q_t"), _dptr(out_t, "out_t"), _ptr(dev_status),
                                       _stream(stream)))


def alloc_cross_workspace(proj: dark_projection, B: int, H: int, Lq: int, Lk: int, flags: int,
                          device):
    """A zero-filled workspace of the size dark_cross_attention_workspace_bytes asks for."""
    n = dark_cross_attention_workspace_bytes(proj, B, H, Lq, Lk, flags)
    return torch.zeros(max(n, WS_HEADER_BYTES), dtype=torch.uint8, device=device)


def dark_attention_bwd_workspace_bytes(heads_omega: int, heads_geom: int, m: int, r: int, d: int,
                                       B: int, H: int, L: int) -> int:
    return _lib.dark_attention_bwd_workspace_bytes(heads_omega, heads_geom, m, r, d, B, H, L)


def dark_attention_bwd(omega, geom, q, k, v, dout, dq, dk, dv, B: int, H: int, L: int,
                       dtype: int, key_mask=None, flags: int = 0, dgeom=None, ws=None,
                       dev_status=None, stream=None, qkv_strides=None, dout_strides=None,
                       grad_strides=None) -> None:
    """Gradients of sum(dout * out) of self-attention. omega: fp32 device tensor
    [H_o, m, r]; geom: fp32 [H_m, r, d]; q/k/v/dout/dq/dk/dv viewed as
    [B][H][L][d] with element strides ({b, h, l}; None = the tensors' own); dgeom: fp32
    [H_m, r, d] or None; ws: see alloc_bwd_workspace."""
    assert omega.dtype == torch.float32 and geom.dtype == torch.float32
    omega, geom = omega.contiguous(), geom.contiguous()
    if dgeom is not None:
        _dense(dgeom, "dgeom")
    ho, m, r = omega.shape
    hg, _, d = geom.shape
    _check(_lib.dark_attention_bwd(
        _ptr(omega), ho, _ptr(geom), hg, m, r, d, dtype, _ptr(q), _ptr(k), _ptr(v),
        _strides(qkv_strides, q, k, v), _ptr(dout), _strides(dout_strides, dout), B, H, L,
        _dptr(key_mask, "key_mask"), flags, _ptr(dq), _ptr(dk), _ptr(dv), _strides(grad_strides, dq, dk, dv),
        _ptr(dgeom), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def alloc_bwd_workspace(omega, geom, B: int, H: int, L: int, device):
    """A workspace of the size dark_attention_bwd_workspace_bytes asks for."""
    ho, m, r = omega.shape
    hg, _, d = geom.shape
    n = dark_attention_bwd_workspace_bytes(ho, hg, m, r, d, B, H, L)
    return torch.empty(max(n, WS_HEADER_BYTES), dtype=torch.uint8, device=device)


def alloc_workspace(proj: dark_projection, B: int, H: int, L: int, flags: int, device):
    """A zero-filled workspace of the size dark_attention_workspace_bytes asks for."""
    n = dark_attention_workspace_bytes(proj, B, H, L, flags)
    return torch.zeros(max(n, WS_HEADER_BYTES), dtype=torch.uint8, device=device)


def dark_auto_uses_exact(L: int, exact_threshold: int) -> bool:
    return bool(_lib.dark_auto_uses_exact(L, exact_threshold))


def dark_sample_omega_workspace_bytes(heads: int, m: int, r: int, orthogonal: bool) -> int:
    return _lib.dark_sample_omega_workspace_bytes(heads, m, r, int(orthogonal))


def dark_sample_omega(seed: int, draw: int, omega, orthogonal: bool = True, ws=None,
                      stream=None) -> None:
    """Fills the fp32 device tensor omega [heads, m, r] from (seed, draw)."""
    _dense(omega, "omega")
    assert omega.dtype == torch.float32 and omega.dim() == 3
    heads, m, r = omega.shape
    if orthogonal and ws is None:
        n = dark_sample_omega_workspace_bytes(heads, m, r, True)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=omega.device)
    _check(_lib.dark_sample_omega(seed, draw, heads, m, r, int(orthogonal), _ptr(omega), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream)))


class RedrawSchedule:
    """The library's redraw schedule (dark_redraw_schedule) with Python method names."""

    def __init__(self, seed: int, interval: int | None = None, deterministic: bool = False):
        self.s = dark_redraw_schedule()
        _check(_lib.dark_redraw_schedule_init(ctypes.byref(self.s), seed,
                                              0 if interval is None else interval,
                                              int(deterministic)))

    @property
    def draw(self) -> int:
        return self.s.draw

    def forward(self, training: bool) -> bool:
        return bool(_lib.dark_redraw_on_forward(ctypes.byref(self.s), int(training)))

    def redraw(self, force: bool = False) -> bool:
        return bool(_lib.dark_redraw_request(ctypes.byref(self.s), int(force)))

    def fix(self) -> None:
        _lib.dark_redraw_set_fixed(ctypes.byref(self.s), 1)

    def unfix(self) -> None:
        _lib.dark_redraw_set_fixed(ctypes.byref(self.s), 0)


def torch_dtype(dtype: int):
    return torch.bfloat16 if dtype == DARK_BF16 else torch.float32
