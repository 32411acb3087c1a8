"""Python binding of libssd_b200 (the C ABI in include/ssd.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity and their pointers are handed to the C library, which runs every
step of the computation in its CUDA kernels.  There is no fallback: if the
library is missing, loading it raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

# the library this binding loads: the in-package build, or the one SSD_B200_LIBRARY
# names (e.g. libssd_b200_debug.so from `build.py --debug`)
_LIB_PATH = os.environ.get("SSD_B200_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libssd_b200.so")
_lib = None

SSD_F32, SSD_BF16 = 0, 1
SSD_PATH_AUTO, SSD_PATH_SIMT, SSD_PATH_TC = -1, 0, 1
SSD_OPT_FORCE_PATH = 1
SSD_OPT_TC_UNIT_COLUMNS = 2
SSD_OPT_WAIT_LIMIT_US = 3
SSD_OPT_TEST_FORCE_TIMEOUT = 4
ERRORS = {
    0: "SSD_OK", -1: "SSD_ERR_INVALID_ARG", -2: "SSD_ERR_UNSUPPORTED", -3: "SSD_ERR_CUDA",
    -4: "SSD_ERR_TIMEOUT", -5: "SSD_ERR_OOM", -6: "SSD_ERR_BAD_SEQLENS",
    -7: "SSD_ERR_SCRATCH_TOO_SMALL", -8: "SSD_ERR_DEBUG_CHECK",
}
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

# every symbol include/ssd.h declares
ABI_SYMBOLS = (
    "ssd_validate_desc", "ssd_plan", "ssd_create", "ssd_set_option", "ssd_forward",
    "ssd_forward_host", "ssd_get_status", "ssd_destroy", "ssd_error_string", "ssd_version",
    "ssd_forward_noalloc", "ssd_step", "ssd_cp_logdecay", "ssd_cp_combine", "ssd_cp_correct",
    "ssd_backward", "ssd_feature_map_dim", "ssd_forward_ext", "ssd_debug_line", "ssd_debug_build",
)


class SSDError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {ERRORS.get(code, code)}")


class Desc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int32),
        ("headdim", ctypes.c_int32), ("dstate", ctypes.c_int32), ("ngroups", ctypes.c_int32),
        ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32), ("max_docs", ctypes.c_int32),
        ("flags", ctypes.c_int32),
    ]


class Plan(ctypes.Structure):
    _fields_ = [
        ("path", ctypes.c_int32), ("num_docs", ctypes.c_int32), ("num_chunks_max", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_int64), ("units", ctypes.c_int32), ("kernels", ctypes.c_int32),
    ]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libssd_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with "
                "`python -m structured_state_space_chunked_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.ssd_validate_desc.argtypes = [ctypes.POINTER(Desc)]
        L.ssd_plan.argtypes = [ctypes.POINTER(Desc), i32, i32, ctypes.POINTER(Plan)]
        L.ssd_create.argtypes = [ctypes.POINTER(Desc), ctypes.POINTER(vp)]
        L.ssd_set_option.argtypes = [vp, i32, i32]
        fwd = [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, vp, vp, vp]
        L.ssd_forward.argtypes = fwd
        L.ssd_forward_host.argtypes = fwd
        L.ssd_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp,
                                   vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.ssd_feature_map_dim.argtypes = [i32, i32]
        L.ssd_forward_ext.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32,
                                      vp, vp, vp]
        L.ssd_get_status.argtypes = [vp, vp]
        L.ssd_forward_noalloc.argtypes = [ctypes.POINTER(Desc), vp, vp, vp, vp, vp, vp, vp, i32,
                                          vp, vp, i32, vp, vp, vp, vp]
        L.ssd_forward_noalloc.restype = ctypes.c_int
        L.ssd_step.argtypes = [ctypes.POINTER(Desc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.ssd_step.restype = ctypes.c_int
        L.ssd_cp_logdecay.argtypes = [ctypes.POINTER(Desc), vp, vp, vp, vp, vp, vp]
        L.ssd_cp_combine.argtypes = [ctypes.POINTER(Desc), i32, i32, vp, vp, vp, vp, vp, vp]
        L.ssd_cp_correct.argtypes = [ctypes.POINTER(Desc), vp, vp, vp, vp, vp, vp]
        for name in ("ssd_cp_logdecay", "ssd_cp_combine", "ssd_cp_correct"):
            getattr(L, name).restype = ctypes.c_int
        L.ssd_destroy.argtypes = [vp]
        L.ssd_debug_line.argtypes = [vp]
        L.ssd_debug_line.restype = ctypes.c_int
        L.ssd_debug_build.restype = ctypes.c_int
        L.ssd_error_string.argtypes = [i32]
        L.ssd_error_string.restype = ctypes.c_char_p
        L.ssd_version.restype = ctypes.c_char_p
        for name in ("ssd_validate_desc", "ssd_plan", "ssd_create", "ssd_set_option",
                     "ssd_forward", "ssd_forward_host", "ssd_get_status", "ssd_destroy"):
            getattr(L, name).restype = ctypes.c_int
        del i64
        _lib = L
    return _lib


def _dt_code(dtype) -> int:
    if dtype == torch.bfloat16:
        return SSD_BF16
    if dtype == torch.float32:
        return SSD_F32
    raise TypeError(f"unsupported dtype {dtype}")


def make_desc(batch, seqlen, nheads, headdim, dstate, ngroups=1, dtype=torch.bfloat16,
              out_dtype=None, max_docs=0) -> Desc:
    return Desc(batch, seqlen, nheads, headdim, dstate, ngroups, _dt_code(dtype),
                _dt_code(out_dtype or dtype), max_docs, 0)


def validate_desc(desc: Desc) -> int:
    return int(lib().ssd_validate_desc(ctypes.byref(desc)))


def plan(desc: Desc, chunk_size: int, num_docs: int = 0) -> Plan:
    p = Plan()
    rc = lib().ssd_plan(ctypes.byref(desc), int(chunk_size), int(num_docs), ctypes.byref(p))
    if rc:
        raise SSDError(rc, "ssd_plan")
    return p


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class SSD:
    """A handle for one problem shape (``ssd_create`` / ``ssd_destroy``)."""

    def __init__(self, batch, seqlen, nheads, headdim, dstate, ngroups=1, dtype=torch.bfloat16,
                 out_dtype=None, max_docs=0, device=None):
        self.desc = make_desc(batch, seqlen, nheads, headdim, dstate, ngroups, dtype, out_dtype,
                              max_docs)
        self.dtype = dtype
        self.out_dtype = out_dtype or dtype
        device = torch.device("cuda") if device is None else torch.device(device)
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.device = device
        with torch.cuda.device(self.device):
            h = ctypes.c_void_p()
            rc = lib().ssd_create(ctypes.byref(self.desc), ctypes.byref(h))
            if rc:
                raise SSDError(rc, "ssd_create")
        self._h = h

    # -- options ---------------------------------------------------------------------
    def force_path(self, path: int) -> None:
        rc = lib().ssd_set_option(self._h, SSD_OPT_FORCE_PATH, int(path))
        if rc:
            raise SSDError(rc, "ssd_set_option")

    def tc_unit_columns(self, cols: int) -> None:
        """Column width (64 or 128) of the tensor-core kernel's work units."""
        rc = lib().ssd_set_option(self._h, SSD_OPT_TC_UNIT_COLUMNS, int(cols))
        if rc:
            raise SSDError(rc, "ssd_set_option")

    def wait_limit_us(self, us: int) -> None:
        """Bound (microseconds) of every device-side wait of the tensor-core kernel."""
        rc = lib().ssd_set_option(self._h, SSD_OPT_WAIT_LIMIT_US, int(us))
        if rc:
            raise SSDError(rc, "ssd_set_option")

    def force_timeout(self, on: bool) -> None:
        """Failure-path test: make the tensor-core kernel's first wait run out."""
        rc = lib().ssd_set_option(self._h, SSD_OPT_TEST_FORCE_TIMEOUT, int(bool(on)))
        if rc:
            raise SSDError(rc, "ssd_set_option")

    def plan(self, chunk_size: int, num_docs: int = 0) -> Plan:
        return plan(self.desc, chunk_size, num_docs)

    # -- checks ------------------------------------------------------------------------
    def _shapes(self, ndocs):
        d = self.desc
        return dict(
            x=(d.batch, d.seqlen, d.nheads, d.headdim), dt=(d.batch, d.seqlen, d.nheads),
            B=(d.batch, d.seqlen, d.ngroups, d.dstate), state=(ndocs, d.nheads, d.dstate, d.headdim),
        )

    def _check(self, name, t, shape, dtype, on_device=True):
        if t is None:
            return
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
        if t.dtype != dtype:
            raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if on_device and (t.device.type != "cuda" or t.device.index != self.device.index):
            raise ValueError(f"{name} must be on {self.device}")
        if not on_device and t.device.type != "cpu":
            raise ValueError(f"{name} must be a host tensor")

    def _prepare(self, x, dt, A, B, C, D, dt_bias, initial_states, cu_seqlens, num_docs, y,
                 final_states, return_final_states, on_device):
        ndocs = (num_docs if num_docs is not None else cu_seqlens.numel() - 1) \
            if cu_seqlens is not None else self.desc.batch
        s = self._shapes(ndocs)
        dev = self.device if on_device else torch.device("cpu")
        self._check("x", x, s["x"], self.dtype, on_device)
        self._check("dt", dt, s["dt"], self.dtype, on_device)
        self._check("B", B, s["B"], self.dtype, on_device)
        self._check("C", C, s["B"], self.dtype, on_device)
        for n, t in (("A", A), ("D", D), ("dt_bias", dt_bias)):
            self._check(n, t, (self.desc.nheads,), torch.float32, on_device)
        self._check("initial_states", initial_states, s["state"], torch.float32, on_device)
        if cu_seqlens is not None:
            self._check("cu_seqlens", cu_seqlens, (ndocs + 1,), torch.int32, on_device)
        if y is None:
            y = torch.empty(s["x"], dtype=self.out_dtype, device=dev,
                            pin_memory=(not on_device and torch.cuda.is_available()))
        self._check("y", y, s["x"], self.out_dtype, on_device)
        if final_states is None and return_final_states:
            final_states = torch.empty(s["state"], dtype=torch.float32, device=dev)
        self._check("final_states", final_states, s["state"], torch.float32, on_device)
        return ndocs, y, final_states

    # -- compute -----------------------------------------------------------------------
    def forward(self, x, dt, A, B, C, D=None, dt_bias=None, chunk_size=256, initial_states=None,
                cu_seqlens=None, num_docs=None, y=None, final_states=None,
                return_final_states=True, stream=None):
        """Enqueue ``ssd_forward`` on ``stream`` (default: torch's current stream)."""
        ndocs, y, final_states = self._prepare(x, dt, A, B, C, D, dt_bias, initial_states,
                                               cu_seqlens, num_docs, y, final_states,
                                               return_final_states, True)
        rc = lib().ssd_forward(self._h, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                               _ptr(dt_bias), int(chunk_size), _ptr(initial_states),
                               _ptr(cu_seqlens), int(ndocs if cu_seqlens is not None else 0),
                               _ptr(y), _ptr(final_states), _stream_ptr(stream))
        if rc:
            raise SSDError(rc, "ssd_forward")
        return y, final_states

    def forward_ext(self, x, dt, A, B, C, D=None, dt_bias=None, chunk_size=256,
                    feature_map=1, normalize=False, cu_seqlens=None, num_docs=None, y=None,
                    final_states=None, return_final_states=True, stream=None):
        """``ssd_forward_ext``: the scan with feature map ``feature_map`` (SSD_FMAP_*)
        on B and C and, with ``normalize``, division by the scan of a ones column.
        ``final_states`` has the mapped dstate."""
        ndocs, y, _ = self._prepare(x, dt, A, B, C, D, dt_bias, None, cu_seqlens, num_docs, y,
                                    None, False, True)
        n2 = feature_map_dim(feature_map, self.desc.dstate)
        shape = (ndocs, self.desc.nheads, n2, self.desc.headdim)
        if final_states is None and return_final_states:
            final_states = torch.empty(shape, dtype=torch.float32, device=self.device)
        self._check("final_states", final_states, shape, torch.float32)
        rc = lib().ssd_forward_ext(self._h, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                   _ptr(dt_bias), int(chunk_size), _ptr(cu_seqlens),
                                   int(ndocs if cu_seqlens is not None else 0), int(feature_map),
                                   int(bool(normalize)), _ptr(y), _ptr(final_states),
                                   _stream_ptr(stream))
        if rc:
            raise SSDError(rc, "ssd_forward_ext")
        return y, final_states

    def backward(self, x, dt, A, B, C, dy, D=None, dt_bias=None, initial_states=None,
                 dfinal_states=None, cu_seqlens=None, num_docs=None, stream=None):
        """Enqueue ``ssd_backward``: the gradient of sum <dy, y> + <dfinal_states,
        final_states> for the forward call with the same inputs.  Returns a dict of
        fp32 tensors: dx, ddt, dA, dB, dC, dD, ddt_bias, dinitial_states."""
        ndocs, _, _ = self._prepare(x, dt, A, B, C, D, dt_bias, initial_states, cu_seqlens,
                                    num_docs, dy, None, False, True)
        s = self._shapes(ndocs)
        self._check("dfinal_states", dfinal_states, s["state"], torch.float32)
        f32 = dict(dtype=torch.float32, device=self.device)
        H = self.desc.nheads
        g = {"dx": torch.empty(s["x"], **f32), "ddt": torch.empty(s["dt"], **f32),
             "dA": torch.empty(H, **f32), "dB": torch.empty(s["B"], **f32),
             "dC": torch.empty(s["B"], **f32), "dD": torch.empty(H, **f32),
             "ddt_bias": torch.empty(H, **f32), "dinitial_states": torch.empty(s["state"], **f32)}
        rc = lib().ssd_backward(self._h, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(dt_bias), _ptr(initial_states), _ptr(cu_seqlens),
                                int(ndocs if cu_seqlens is not None else 0), _ptr(dy),
                                _ptr(dfinal_states), _ptr(g["dx"]), _ptr(g["ddt"]), _ptr(g["dA"]),
                                _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["ddt_bias"]),
                                _ptr(g["dinitial_states"]), _stream_ptr(stream))
        if rc:
            raise SSDError(rc, "ssd_backward")
        return g

    def forward_host(self, x, dt, A, B, C, D=None, dt_bias=None, chunk_size=256,
                     initial_states=None, cu_seqlens=None, num_docs=None, y=None,
                     final_states=None, return_final_states=True, stream=None):
        """``ssd_forward_host``: host tensors in and out, copies and sync inside."""
        ndocs, y, final_states = self._prepare(x, dt, A, B, C, D, dt_bias, initial_states,
                                               cu_seqlens, num_docs, y, final_states,
                                               return_final_states, False)
        with torch.cuda.device(self.device):
            rc = lib().ssd_forward_host(self._h, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                        _ptr(D), _ptr(dt_bias), int(chunk_size),
                                        _ptr(initial_states), _ptr(cu_seqlens),
                                        int(ndocs if cu_seqlens is not None else 0), _ptr(y),
                                        _ptr(final_states), _stream_ptr(stream))
        if rc:
            raise SSDError(rc, "ssd_forward_host")
        return y, final_states

    def status(self, stream=None) -> int:
        """``ssd_get_status``: synchronise and return/clear the device status word."""
        return int(lib().ssd_get_status(self._h, _stream_ptr(stream)))

    def debug_line(self) -> int:
        """``ssd_debug_line``: source line of the first failed device-side check (debug
        builds; 0 when none failed or in a release build)."""
        return int(lib().ssd_debug_line(self._h))

    def close(self):
        if getattr(self, "_h", None):
            lib().ssd_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


SSD_FMAP_NONE, SSD_FMAP_SILU, SSD_FMAP_RELU, SSD_FMAP_BASED, SSD_FMAP_REBASED = 0, 1, 2, 3, 4


def feature_map_dim(kind: int, dstate: int) -> int:
    """``ssd_feature_map_dim``: dstate of the scan after feature map ``kind``."""
    n = int(lib().ssd_feature_map_dim(int(kind), int(dstate)))
    if n < 1:
        raise SSDError(-1, "ssd_feature_map_dim")
    return n


_cache = {}


def ssd_forward(x, dt, A, B, C, D=None, dt_bias=None, chunk_size=256, initial_states=None,
                cu_seqlens=None, return_final_states=True, path: int = SSD_PATH_AUTO, stream=None):
    """Functional form: y, final_states = SSD(...) with a cached handle per shape."""
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    max_docs = 0
    if cu_seqlens is not None:
        max_docs = max(1, cu_seqlens.numel() - 1)
    key = (bsz, L, H, P, N, G, x.dtype, max_docs, x.device.index, path)
    h = _cache.get(key)
    if h is None:
        h = SSD(bsz, L, H, P, N, G, x.dtype, None, max_docs, x.device)
        if path != SSD_PATH_AUTO:
            h.force_path(path)
        _cache[key] = h
    return h.forward(x, dt, A, B, C, D, dt_bias, chunk_size, initial_states, cu_seqlens,
                     return_final_states=return_final_states, stream=stream)


def ssd_step(x, dt, A, B, C, state, D=None, dt_bias=None, y=None, out_dtype=None, stream=None):
    """``ssd_step``: one decode token for every sequence, the state updated in place.

    x [b,H,P], dt [b,H], B/C [b,G,N] (bf16 or fp32, one dtype), A/D/dt_bias [H] fp32,
    state [b,H,N,P] fp32 (read and overwritten).  Returns y [b,H,P] in ``out_dtype``
    (default: x's dtype).
    """
    bsz, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if tuple(state.shape) != (bsz, H, N, P) or state.dtype != torch.float32:
        raise ValueError(f"state must be float32 {(bsz, H, N, P)}")
    for name, t in (("x", x), ("dt", dt), ("B", B), ("C", C), ("state", state)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    out_dtype = out_dtype or x.dtype
    if y is None:
        y = torch.empty(bsz, H, P, dtype=out_dtype, device=x.device)
    desc = make_desc(bsz, 1, H, P, N, G, x.dtype, out_dtype, 0)
    with torch.cuda.device(x.device):
        rc = lib().ssd_step(ctypes.byref(desc), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                            _ptr(D), _ptr(dt_bias), _ptr(state), _ptr(y), _stream_ptr(stream))
    if rc:
        raise SSDError(rc, "ssd_step")
    return y


# -- context-parallel device steps (see include/ssd.h) -----------------------------------

def _cp_desc(dt, nheads, headdim, dstate, ngroups, out_dtype):
    bsz, L = dt.shape[0], dt.shape[1]
    return make_desc(bsz, L, nheads, headdim, dstate, ngroups, dt.dtype, out_dtype, 0)


def cp_logdecay(dt, A, dt_bias=None, headdim=4, dstate=1, ngroups=1, stream=None):
    """``ssd_cp_logdecay``: (cs [b,L,H] fp32, logdecay [b,H] fp32) of this slice."""
    bsz, L, H = dt.shape
    cs = torch.empty(bsz, L, H, dtype=torch.float32, device=dt.device)
    ld = torch.empty(bsz, H, dtype=torch.float32, device=dt.device)
    desc = _cp_desc(dt, H, headdim, dstate, ngroups, dt.dtype)
    with torch.cuda.device(dt.device):
        rc = lib().ssd_cp_logdecay(ctypes.byref(desc), _ptr(dt), _ptr(A), _ptr(dt_bias),
                                   _ptr(cs), _ptr(ld), _stream_ptr(stream))
    if rc:
        raise SSDError(rc, "ssd_cp_logdecay")
    return cs, ld


def cp_combine(rank, local_final_all, logdecay_all, initial_states=None, dt_dtype=torch.bfloat16,
               stream=None):
    """``ssd_cp_combine``: (h_in, final_state) of ``rank`` from every rank's
    local final state [R,b,H,N,P] and log decay [R,b,H]."""
    R, bsz, H, N, P = local_final_all.shape
    h_in = torch.empty(bsz, H, N, P, dtype=torch.float32, device=local_final_all.device)
    fin = torch.empty_like(h_in)
    desc = make_desc(bsz, 1, H, P, N, 1, dt_dtype, dt_dtype, 0)
    with torch.cuda.device(local_final_all.device):
        rc = lib().ssd_cp_combine(ctypes.byref(desc), int(rank), int(R), _ptr(local_final_all),
                                  _ptr(logdecay_all), _ptr(initial_states), _ptr(h_in), _ptr(fin),
                                  _stream_ptr(stream))
    if rc:
        raise SSDError(rc, "ssd_cp_combine")
    return h_in, fin


def cp_correct(C, cs, h_in, y, status=None, stream=None):
    """``ssd_cp_correct``: y += exp(cs) C H_in, in place.  ``status`` is an optional
    one-element int32 device tensor that receives a device-side timeout code."""
    bsz, L, G, N = C.shape
    H, P = y.shape[2], y.shape[3]
    desc = make_desc(bsz, L, H, P, N, G, C.dtype, y.dtype, 0)
    with torch.cuda.device(y.device):
        rc = lib().ssd_cp_correct(ctypes.byref(desc), _ptr(C), _ptr(cs), _ptr(h_in), _ptr(y),
                                  _ptr(status), _stream_ptr(stream))
    if rc:
        raise SSDError(rc, "ssd_cp_correct")
    return y
