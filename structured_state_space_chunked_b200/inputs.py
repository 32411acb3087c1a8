"""Seeded synthetic inputs for the SSD forward workloads.

This module holds no arithmetic of the method itself: it only draws random
numbers with the shapes and value distributions of the workloads and rounds
them once to the device dtype.  Both the CUDA path and the float64 oracle
consume exactly the tensors produced here.

Value recipe (every workload):
  * x ~ N(0, 1); B, C ~ N(0, 1) / sqrt(N); D ~ N(0, 1)
  * A[h] = -exp(U[0, ln 16])                       (negative, scalar per head)
  * dt_bias[h] = softplus^-1(u_h), u_h log-uniform in [1e-3, 1e-1]
  * dt ~ N(0, 1)   (so delta = softplus(dt + dt_bias) is centred on u_h)
  * initial states: zero, or N(0, 0.1^2) per (sequence, head) where asked
  * x, dt, B, C are rounded once (round-to-nearest-even) to the input dtype;
    A, D, dt_bias and states stay float32.
Packed variable-length workloads draw document lengths from a lognormal with
median 512 and sigma 1, clipped to [16, 8192]; the last document is cut so the
total is exact and a remainder shorter than 16 joins the previous document.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

BASE_SEED = 20240531


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk_size: int
    dtype: str = "bf16"          # "bf16" or "fp32": dtype of x, dt, B, C and y
    init: str = "zero"           # "zero" or "normal0.1"
    varlen_tokens: int = 0       # > 0: one packed row of this many tokens with documents
    seed: int = BASE_SEED

    @property
    def tokens(self) -> int:
        return self.varlen_tokens if self.varlen_tokens else self.batch * self.seqlen

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def workloads() -> List[Workload]:
    """The five workloads of the benchmark (the long-sequence one as a 3 x 3 sweep)."""
    out = [
        Workload("tiny_fp32_L256_H2_P16_N16", 1, 256, 2, 16, 16, 1, 64, "fp32", seed=BASE_SEED + 0),
        Workload("mamba2_130m_layer_b4_L2048", 4, 2048, 24, 64, 128, 1, 256, seed=BASE_SEED + 1),
        Workload("mamba2_2p7b_layer_b8_L4096", 8, 4096, 80, 64, 128, 1, 256, init="normal0.1",
                 seed=BASE_SEED + 2),
    ]
    k = 0
    for L in (2048, 16384, 65536):
        for N in (64, 128, 256):
            out.append(Workload(f"long_L{L}_H64_P128_N{N}_G8", 1, L, 64, 128, N, 8, 256,
                                seed=BASE_SEED + 3 + 100 * (k + 1)))
            k += 1
    out.append(Workload("varlen_32k_H32_P64_N128", 1, 32768, 32, 64, 128, 1, 256,
                        varlen_tokens=32768, seed=BASE_SEED + 4))
    return out


def workload(name: str) -> Workload:
    for w in workloads():
        if w.name == name:
            return w
    raise KeyError(name)


def doc_lengths(total: int, rng: np.random.Generator, median: float = 512.0,
                sigma: float = 1.0, lo: int = 16, hi: int = 8192) -> List[int]:
    """Lognormal document lengths that add up to exactly ``total``."""
    lens: List[int] = []
    acc = 0
    while acc < total:
        n = int(round(float(rng.lognormal(math.log(median), sigma))))
        n = min(max(n, lo), hi)
        lens.append(n)
        acc += n
    lens[-1] -= acc - total
    if lens[-1] < lo and len(lens) > 1:
        lens[-2] += lens.pop()
    return lens


def cu_seqlens_from_lengths(lens) -> np.ndarray:
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lens, dtype=np.int64))
    return cu


def _inv_softplus(u: np.ndarray) -> np.ndarray:
    # the dt_bias that puts softplus(dt_bias) at u (input preparation only)
    return u + np.log(-np.expm1(-u))


def make_inputs(w: Workload, device="cpu", heads_subset_seed: Optional[int] = None,
                cu_seqlens=None):
    """Draw the inputs of ``w``.  Returns a dict of torch tensors on ``device``.

    Keys: x [b,L,H,P], dt [b,L,H], A [H], B [b,L,G,N], C [b,L,G,N], D [H],
    dt_bias [H], initial_states [ndocs,H,N,P] or None, cu_seqlens int32 or None.
    """
    rng = np.random.default_rng(w.seed)
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    if w.varlen_tokens:
        b, L = 1, w.varlen_tokens
        if cu_seqlens is None:
            cu_seqlens = cu_seqlens_from_lengths(doc_lengths(L, rng))
    ndocs = (len(cu_seqlens) - 1) if cu_seqlens is not None else b
    dt_t = w.torch_dtype

    def normal(shape, scale=1.0):
        a = rng.standard_normal(size=shape, dtype=np.float32)
        if scale != 1.0:
            a *= np.float32(scale)
        return a

    x = normal((b, L, H, P))
    dt = normal((b, L, H))
    Bm = normal((b, L, G, N), 1.0 / math.sqrt(N))
    Cm = normal((b, L, G, N), 1.0 / math.sqrt(N))
    A = -np.exp(rng.uniform(0.0, math.log(16.0), size=H)).astype(np.float32)
    D = rng.standard_normal(size=H).astype(np.float32)
    u = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=H))
    dt_bias = _inv_softplus(u).astype(np.float32)
    init = None
    if w.init == "normal0.1":
        init = normal((ndocs, H, N, P), 0.1)

    def t(a, dtype):
        return torch.from_numpy(a).to(dtype).to(device)

    out = dict(
        x=t(x, dt_t), dt=t(dt, dt_t), A=t(A, torch.float32), B=t(Bm, dt_t), C=t(Cm, dt_t),
        D=t(D, torch.float32), dt_bias=t(dt_bias, torch.float32),
        initial_states=None if init is None else t(init, torch.float32),
        cu_seqlens=None if cu_seqlens is None else torch.from_numpy(
            np.asarray(cu_seqlens, dtype=np.int32)).to(device),
    )
    return out


def random_small(seed: int, dtype: str = "bf16", batch: int = 1, seqlen: int = 300,
                 nheads: int = 4, headdim: int = 64, dstate: int = 128, ngroups: int = 1,
                 chunk_size: int = 128, init: str = "zero", varlen_tokens: int = 0) -> Workload:
    """A small workload with the same value recipe (parity and edge-case tests)."""
    return Workload(f"small_s{seed}", batch, seqlen, nheads, headdim, dstate, ngroups,
                    chunk_size, dtype, init, varlen_tokens, seed)


def make_cotangents(w: Workload, ndocs: int, device="cpu", seed_offset: int = 1):
    """Cotangents for the backward pass of ``w``: dy [b,L,H,P] in the output dtype
    (standard normal) and dfinal_states [ndocs,H,N,P] fp32 (standard normal),
    from their own seeded stream."""
    rng = np.random.default_rng(w.seed + seed_offset)
    b, L = (1, w.varlen_tokens) if w.varlen_tokens else (w.batch, w.seqlen)
    dy = rng.standard_normal(size=(b, L, w.nheads, w.headdim), dtype=np.float32)
    dfin = rng.standard_normal(size=(ndocs, w.nheads, w.dstate, w.headdim), dtype=np.float32)
    return (torch.from_numpy(dy).to(w.torch_dtype).to(device),
            torch.from_numpy(dfin).to(device))
