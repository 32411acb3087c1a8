"""ctypes driver for the float64 C oracle (``ssd_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).

``oracle_forward`` takes host arrays in any float dtype (the test harness passes
the values the GPU sees, already rounded to the device dtype), upcasts them to
float64, and returns float64 ``y`` and ``final_states``.  Documents are given
either implicitly (``batch`` rows of ``seqlen`` tokens) or by ``cu_seqlens``
(one packed row), exactly as the CUDA boundary takes them.
"""

from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ssd_oracle.c`` into ``libssd_oracle.so`` with gcc + OpenMP."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f = lib.ssd_oracle_forward
        f.restype = ctypes.c_int
        f.argtypes = [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ]
        f = lib.ssd_oracle_backward
        f.restype = ctypes.c_int
        f.argtypes = [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ]
        lib.ssd_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def oracle_threads() -> int:
    """OpenMP threads the oracle uses by default on this host."""
    return int(_load().ssd_oracle_max_threads())


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # a torch tensor (CPU); bf16 has no numpy dtype
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def oracle_forward(x, dt, A, B, C, D=None, dt_bias=None, initial_states=None,
                   cu_seqlens=None, heads=None, nthreads: int = 0):
    """Run the float64 recurrence.

    Shapes (batch mode):  x [b,L,H,P], dt [b,L,H], B/C [b,L,G,N].
    Shapes (packed mode, ``cu_seqlens`` given): the same with b == 1, and
    ``initial_states`` / the returned final states are per document.
    ``heads``: optional list of head indices; only those heads are computed
    (the other entries of ``y`` / ``final_states`` are returned as NaN).
    Returns ``(y [b,L,H,P] f64, final_states [ndocs,H,N,P] f64)``.
    """
    x = _f64(x)
    dt = _f64(dt)
    A = _f64(A)
    B = _f64(B)
    C = _f64(C)
    D = _f64(D)
    dt_bias = _f64(dt_bias)
    init = _f64(initial_states)
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    T = bsz * L
    if cu_seqlens is None:
        offsets = np.arange(bsz + 1, dtype=np.int64) * L
    else:
        if bsz != 1:
            raise ValueError("cu_seqlens requires a single packed row (batch == 1)")
        offsets = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    ndocs = len(offsets) - 1
    if init is not None and init.shape != (ndocs, H, N, P):
        raise ValueError(f"initial_states must be {(ndocs, H, N, P)}, got {init.shape}")
    sel = None
    if heads is not None:
        sel = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    y = np.full((T, H, P), np.nan)
    final = np.full((ndocs, H, N, P), np.nan)
    rc = _load().ssd_oracle_forward(
        T, H, P, N, G, ndocs, _ptr(offsets),
        _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(dt_bias), _ptr(init),
        _ptr(sel), 0 if sel is None else len(sel), _ptr(y), _ptr(final), int(nthreads),
    )
    if rc != 0:
        raise ValueError("ssd_oracle_forward rejected its arguments")
    return y.reshape(bsz, L, H, P), final


def oracle_step(state, x, dt, A, B, C, D=None, dt_bias=None):
    """One token of the recurrence for every sequence of a decode batch, in float64.

    The same definition as ``oracle_forward`` run for a single token from a given
    state: the recurrent (linear) mode of the selective SSM ("Transformers are
    SSMs", paperlayer.ai summary, §3.4.1; scalar-times-identity A, §2.4).
    Shapes: state [b,H,N,P], x [b,H,P], dt [b,H], B/C [b,G,N].  Returns
    ``(y [b,H,P] f64, new_state [b,H,N,P] f64)``.
    """
    s = _f64(state)
    x = _f64(x)
    dt = _f64(dt)
    A = _f64(A)
    B = _f64(B)
    C = _f64(C)
    bsz, H, N, P = s.shape
    G = B.shape[1]
    D = np.zeros(H) if D is None else _f64(D)
    bias = np.zeros(H) if dt_bias is None else _f64(dt_bias)
    g = np.arange(H) // (H // G)                      # contiguous group of each head
    delta = np.logaddexp(0.0, dt + bias[None, :])      # softplus
    decay = np.exp(delta * A[None, :])                 # [b, H]
    Bh, Ch = B[:, g, :], C[:, g, :]                    # [b, H, N]
    new = decay[:, :, None, None] * s + (delta[:, :, None, None] * Bh[:, :, :, None]) * x[:, :, None, :]
    y = np.einsum("bhn,bhnp->bhp", Ch, new) + D[None, :, None] * x
    return y, new


def oracle_backward(x, dt, A, B, C, dy, D=None, dt_bias=None, initial_states=None,
                    dfinal_states=None, cu_seqlens=None, heads=None, nthreads: int = 0):
    """Gradient of ``sum <dy, y> + <dfinal_states, final_states>`` with respect to
    every input of ``oracle_forward``, in float64: the chain rule taken backwards
    through the same sequential recurrence (``ssd_oracle_backward`` in the C file
    states each step).

    Shapes as for ``oracle_forward``; ``dy`` like ``x``; ``dfinal_states`` like the
    final states (None: zero).  ``heads`` restricts the computation to those heads:
    their per-head gradients are filled (the others stay NaN) and dB / dC hold only
    their share.  Returns a dict with dx, ddt, dA, dB, dC, dD, ddt_bias and
    dinitial_states (the gradient with respect to the initial states, present
    whether or not initial states were given)."""
    x = _f64(x)
    dt = _f64(dt)
    A = _f64(A)
    B = _f64(B)
    C = _f64(C)
    D = _f64(D)
    dt_bias = _f64(dt_bias)
    init = _f64(initial_states)
    dy = _f64(dy)
    dfin = _f64(dfinal_states)
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    T = bsz * L
    if cu_seqlens is None:
        offsets = np.arange(bsz + 1, dtype=np.int64) * L
    else:
        if bsz != 1:
            raise ValueError("cu_seqlens requires a single packed row (batch == 1)")
        offsets = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    ndocs = len(offsets) - 1
    for name, a in (("initial_states", init), ("dfinal_states", dfin)):
        if a is not None and a.shape != (ndocs, H, N, P):
            raise ValueError(f"{name} must be {(ndocs, H, N, P)}, got {a.shape}")
    if dy.shape != x.shape:
        raise ValueError("dy must have the shape of x")
    sel = None
    if heads is not None:
        sel = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    dx = np.full((T, H, P), np.nan)
    ddt = np.full((T, H), np.nan)
    dB = np.zeros((T, G, N))
    dC = np.zeros((T, G, N))
    dA_part = np.full((ndocs, H), np.nan)
    dD_part = np.full((ndocs, H), np.nan)
    db_part = np.full((ndocs, H), np.nan)
    dinit = np.full((ndocs, H, N, P), np.nan)
    rc = _load().ssd_oracle_backward(
        T, H, P, N, G, ndocs, _ptr(offsets),
        _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(dt_bias), _ptr(init),
        _ptr(dy), _ptr(dfin), _ptr(sel), 0 if sel is None else len(sel),
        _ptr(dx), _ptr(ddt), _ptr(dA_part), _ptr(dB), _ptr(dC), _ptr(dD_part), _ptr(db_part),
        _ptr(dinit), int(nthreads),
    )
    if rc == -2:
        raise MemoryError("ssd_oracle_backward ran out of host memory")
    if rc != 0:
        raise ValueError("ssd_oracle_backward rejected its arguments")
    return {
        "dx": dx.reshape(bsz, L, H, P), "ddt": ddt.reshape(bsz, L, H),
        "dA": dA_part.sum(axis=0), "dB": dB.reshape(bsz, L, G, N), "dC": dC.reshape(bsz, L, G, N),
        "dD": dD_part.sum(axis=0), "ddt_bias": db_part.sum(axis=0), "dinitial_states": dinit,
    }


FMAP_NONE, FMAP_SILU, FMAP_RELU, FMAP_BASED, FMAP_REBASED = 0, 1, 2, 3, 4


def oracle_feature_map(X, kind):
    """A kernel feature map on the last axis of X, in float64 ("Transformers are
    SSMs", paperlayer.ai summary: §7.3 feature maps, SiLU by default; App. D.4 the
    Based map, the second-order Taylor expansion of exp, and the ReBased map x (x) x).
    The outer products are flattened row-major."""
    X = _f64(X)
    if kind == FMAP_NONE:
        return X
    if kind == FMAP_SILU:
        return X / (1.0 + np.exp(-X))
    if kind == FMAP_RELU:
        return np.maximum(X, 0.0)
    outer = (X[..., :, None] * X[..., None, :]).reshape(*X.shape[:-1], -1)
    if kind == FMAP_REBASED:
        return outer
    if kind == FMAP_BASED:
        ones = np.ones(X.shape[:-1] + (1,))
        return np.concatenate([ones, X, outer / math.sqrt(2.0)], axis=-1)
    raise ValueError(f"unknown feature map {kind}")


def oracle_forward_ext(x, dt, A, B, C, D=None, dt_bias=None, feature_map=FMAP_SILU,
                       normalize=False, cu_seqlens=None):
    """The scan with the feature map on B and C and, optionally, the denominator
    normalisation of §7.3: the numerator is the scan on x with no skip term, the
    denominator the same scan on a column of ones (X augmented with ones), and
    y = num / den + D x.  Returns (y, final_states of the numerator)."""
    x64 = _f64(x)
    D64 = None if D is None else _f64(D)
    Bf = oracle_feature_map(B, feature_map)
    Cf = oracle_feature_map(C, feature_map)
    if not normalize:
        return oracle_forward(x64, dt, A, Bf, Cf, D64, dt_bias, cu_seqlens=cu_seqlens)
    num, fin = oracle_forward(x64, dt, A, Bf, Cf, None, dt_bias, cu_seqlens=cu_seqlens)
    den, _ = oracle_forward(np.ones(x64.shape[:-1] + (1,)), dt, A, Bf, Cf, None, dt_bias,
                            cu_seqlens=cu_seqlens)
    with np.errstate(invalid="ignore", divide="ignore"):
        y = num / den
    if D64 is not None:
        y = y + D64[None, None, :, None] * x64
    return y, fin
