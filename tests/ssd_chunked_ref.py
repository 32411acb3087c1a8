"""Test-only float64 implementations that are *not* the oracle's recurrence.

Two independent restatements of what the SSD layer computes, used to pin the
oracle ("Transformers are SSMs", paperlayer.ai summary):

* ``quadratic_form``: the materialised dual form.  The SSM is multiplication
  by a T x T lower-triangular semiseparable matrix, M[t,s] = (C_t . B_s) *
  L[t,s] * delta_s with the 1-semiseparable mask L[t,s] = prod_{k=s+1..t}
  exp(delta_k A) (§3.3, §3.4.2 quadratic mode, §5.1, §5.3).
* ``chunked``: the block-decomposed algorithm of §6: diagonal blocks by the
  quadratic form with zero initial state (§6.1), chunk states from the right
  factors (§6.2), a scalar scan of states across chunks (§6.2, App. B.3.2
  state-passing mode), and outputs from the left factors (§6.2).

Both take float64 numpy arrays for ONE document and ONE head:
  x [T,P], delta [T], a (=A[h]) scalar, Bm/Cm [T,N], D scalar, init [N,P] or None.
"""

import numpy as np


def quadratic_form(x, delta, a, Bm, Cm, D, init=None):
    T = x.shape[0]
    la = delta * a  # log of the per-step transition multiplier
    # L[t,s] = exp(sum_{k=s+1}^{t} la_k) for s <= t, else 0, built entry by entry
    L = np.zeros((T, T))
    for t in range(T):
        acc = 0.0
        L[t, t] = 1.0
        for s in range(t - 1, -1, -1):
            acc += la[s + 1]
            L[t, s] = np.exp(acc)
    M = (Cm @ Bm.T) * L * delta[None, :]
    y = M @ x + D * x
    final = (L[T - 1, :, None] * delta[:, None] * Bm).T @ x if T else None
    if init is not None:
        # the initial state decays through every step up to and including t
        dec = np.exp(np.cumsum(la))
        y = y + dec[:, None] * (Cm @ init)
        if T:
            final = final + dec[T - 1] * init
    if T == 0:
        final = init.copy() if init is not None else np.zeros((Bm.shape[1], x.shape[1]))
    return y, final


def chunked(x, delta, a, Bm, Cm, D, Q, init=None):
    T, P = x.shape
    N = Bm.shape[1]
    y = np.zeros((T, P))
    state = np.zeros((N, P)) if init is None else init.astype(np.float64).copy()
    for c0 in range(0, T, Q):
        c1 = min(c0 + Q, T)
        xs, ds, Bs, Cs = x[c0:c1], delta[c0:c1], Bm[c0:c1], Cm[c0:c1]
        cs = np.cumsum(ds * a)  # in-chunk cumulative log decay
        # diagonal block: quadratic form with zero initial state (§6.1)
        seg = cs[:, None] - cs[None, :]
        Lc = np.where(np.tril(np.ones((c1 - c0, c1 - c0), dtype=bool)), np.exp(np.minimum(seg, 0.0)), 0.0)
        y_diag = ((Cs @ Bs.T) * Lc * ds[None, :]) @ xs
        # left factors: contribution of the state entering the chunk (§6.2)
        y_off = np.exp(cs)[:, None] * (Cs @ state)
        y[c0:c1] = y_diag + y_off + D * xs
        # right factors: chunk state with no inputs before the chunk (§6.2)
        w = np.exp(cs[-1] - cs) * ds
        chunk_state = Bs.T @ (w[:, None] * xs)
        # scalar scan across chunks (state passing)
        state = np.exp(cs[-1]) * state + chunk_state
    return y, state
