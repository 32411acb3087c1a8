"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle (a sequential recurrence, "Transformers are SSMs",
paperlayer.ai summary, §3.4.1) against a different statement of the same
mathematics: the materialised quadratic (dual) form (§3.4.2, §5.1, §5.3), the
A = 0 closed form (App. B.1: the scan reduces to a cumulative sum; §4.2.1),
the chunked block decomposition (§6), document resets (§8.3), state hand-off
between workers (§8.2), hand-computed scan values (App. B.3.5) and closed
softplus values.  A dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.
"""

import math
import os

import numpy as np
import pytest

import oracle
from tests.ssd_chunked_ref import chunked, quadratic_form

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL = 1e-11


def _rand(seed, b=1, L=37, H=3, P=5, N=4, G=1, ndoc_init=None):
    r = np.random.default_rng(seed)
    x = r.standard_normal((b, L, H, P))
    dt = r.standard_normal((b, L, H))
    A = -np.exp(r.uniform(0, math.log(16), H))
    Bm = r.standard_normal((b, L, G, N)) / math.sqrt(N)
    Cm = r.standard_normal((b, L, G, N)) / math.sqrt(N)
    D = r.standard_normal(H)
    dt_bias = np.log(np.expm1(np.exp(r.uniform(math.log(1e-3), math.log(1e-1), H))))
    init = None
    if ndoc_init is not None:
        init = 0.1 * r.standard_normal((ndoc_init, H, N, P))
    return x, dt, A, Bm, Cm, D, dt_bias, init


def _delta(dt, bias):
    # library softplus (np.logaddexp), not the oracle's formula
    return np.logaddexp(0.0, dt + bias)


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


@pytest.mark.parametrize("seed,G,H", [(0, 1, 3), (1, 2, 4), (2, 4, 4)])
def test_oracle_equals_materialised_quadratic_form(seed, G, H):
    b, L, P, N = 2, 29, 5, 6
    x, dt, A, Bm, Cm, D, bias, init = _rand(seed, b, L, H, P, N, G, ndoc_init=b)
    y, fin = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, init)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            yq, fq = quadratic_form(x[bi, :, h], _delta(dt[bi, :, h], bias[h]), A[h],
                                    Bm[bi, :, g], Cm[bi, :, g], D[h], init[bi, h])
            assert _rel(y[bi, :, h], yq) < RTOL
            assert _rel(fin[bi, h], fq) < RTOL


def test_closed_form_when_A_is_zero():
    # A = 0: the transition multiplier is 1, the scan is a cumulative sum and the
    # state is init + sum_s delta_s * B_s (outer) x_s  ([N, P] orientation).
    r = np.random.default_rng(7)
    L, H, P, N = 23, 2, 3, 4
    x = r.standard_normal((1, L, H, P))
    delta = r.uniform(0.01, 2.0, (1, L, H))
    dt = np.log(np.expm1(delta))  # so that softplus(dt + 0) == delta
    A = np.zeros(H)
    Bm = r.standard_normal((1, L, 1, N))
    Cm = r.standard_normal((1, L, 1, N))
    D = r.standard_normal(H)
    init = r.standard_normal((1, H, N, P))
    y, fin = oracle.oracle_forward(x, dt, A, Bm, Cm, D, None, init)
    for h in range(H):
        outer = delta[0, :, h, None, None] * Bm[0, :, 0, :, None] * x[0, :, h, None, :]
        states = init[0, h][None] + np.cumsum(outer, axis=0)  # [L, N, P]
        yc = np.einsum("tn,tnp->tp", Cm[0, :, 0], states) + D[h] * x[0, :, h]
        assert _rel(y[0, :, h], yc) < RTOL
        assert _rel(fin[0, h], states[-1]) < RTOL


@pytest.mark.parametrize("z,expected", [(0.0, math.log(2.0)), (30.0, 30.0 + math.exp(-30.0)),
                                        (-30.0, math.exp(-30.0)), (1.0, math.log1p(math.e))])
def test_softplus_closed_values(z, expected):
    # one token, N = P = 1, B = C = x = 1, D = 0: y = delta = softplus(dt + dt_bias)
    one = np.ones((1, 1, 1, 1))
    y, _ = oracle.oracle_forward(one, np.full((1, 1, 1), z - 0.25), np.array([-1.0]),
                                 one, one, np.zeros(1), np.array([0.25]))
    assert abs(y[0, 0, 0, 0] - expected) <= 1e-15 * max(1.0, abs(expected))


def _read_scan_golden():
    rows = []
    with open(os.path.join(GOLDEN, "scalar_scan_assoc.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            rows.append(line.split())
    return rows


@pytest.mark.parametrize("row", _read_scan_golden(), ids=lambda r: r[0])
def test_scalar_scan_hand_values(row):
    kind, start = row[0], int(row[1])
    val = lambda s: None if s == "-" else float(s)
    a = [None, val(row[2]), val(row[3]), val(row[4])]
    bvals = [val(v) for v in row[5:9]]
    expected = [float(v) for v in row[9:]]
    # realise a_t = exp(delta_t * A) with A = -1 and b_t = delta_t * x_t
    A = np.array([-1.0])
    delta = np.array([1.0 if at is None else -math.log(at) for at in a])
    xs = np.array([0.0 if bt is None else bt / dl for bt, dl in zip(bvals, delta)])
    dt = np.log(np.expm1(delta)).reshape(1, 4, 1)
    one = np.ones((1, 4, 1, 1))
    cu = [0, start, 4] if start else [0, 4]
    y, _ = oracle.oracle_forward(xs.reshape(1, 4, 1, 1), dt, A, one, one, np.zeros(1), None,
                                 None, cu_seqlens=cu)
    got = y[0, start:, 0, 0]
    np.testing.assert_allclose(got, expected, rtol=1e-12, atol=0)
    assert kind in ("block2", "full")


@pytest.mark.parametrize("Q", [1, 3, 16, 20, 40, 41])
def test_chunked_decomposition_equals_oracle_for_every_chunk_size(Q):
    L = 40
    x, dt, A, Bm, Cm, D, bias, init = _rand(11, 1, L, 2, 4, 3, 1, ndoc_init=1)
    y, fin = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, init)
    for h in range(2):
        yc, fc = chunked(x[0, :, h], _delta(dt[0, :, h], bias[h]), A[h], Bm[0, :, 0],
                         Cm[0, :, 0], D[h], Q, init[0, h])
        assert _rel(y[0, :, h], yc) < RTOL
        assert _rel(fin[0, h], fc) < RTOL


def test_packed_documents_equal_separate_runs():
    lens = [5, 1, 17, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1])
    x, dt, A, Bm, Cm, D, bias, init = _rand(3, 1, T, 3, 4, 5, 1, ndoc_init=len(lens))
    y, fin = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, init, cu_seqlens=cu)
    for d in range(len(lens)):
        s, e = cu[d], cu[d + 1]
        ys, fs = oracle.oracle_forward(x[:, s:e], dt[:, s:e], A, Bm[:, s:e], Cm[:, s:e], D, bias,
                                       init[d:d + 1])
        assert _rel(y[:, s:e], ys) < 1e-15
        assert _rel(fin[d], fs[0]) < 1e-15


def test_perturbing_one_document_leaves_the_others_unchanged():
    lens = [12, 7, 10]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1])
    x, dt, A, Bm, Cm, D, bias, _ = _rand(4, 1, T, 2, 3, 4, 1)
    y0, f0 = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, cu_seqlens=cu)
    x2, B2 = x.copy(), Bm.copy()
    x2[:, cu[1]:cu[2]] += 5.0
    B2[:, cu[1]:cu[2]] *= -3.0
    y1, f1 = oracle.oracle_forward(x2, dt, A, B2, Cm, D, bias, cu_seqlens=cu)
    for d in (0, 2):
        assert np.array_equal(y0[:, cu[d]:cu[d + 1]], y1[:, cu[d]:cu[d + 1]])
        assert np.array_equal(f0[d], f1[d])
    assert not np.allclose(y0[:, cu[1]:cu[2]], y1[:, cu[1]:cu[2]])


@pytest.mark.parametrize("t0", [1, 13, 30])
def test_state_handoff_between_workers(t0):
    x, dt, A, Bm, Cm, D, bias, init = _rand(5, 1, 31, 2, 3, 4, 1, ndoc_init=1)
    y, fin = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, init)
    ya, fa = oracle.oracle_forward(x[:, :t0], dt[:, :t0], A, Bm[:, :t0], Cm[:, :t0], D, bias, init)
    yb, fb = oracle.oracle_forward(x[:, t0:], dt[:, t0:], A, Bm[:, t0:], Cm[:, t0:], D, bias, fa)
    assert _rel(np.concatenate([ya, yb], axis=1), y) < RTOL
    assert _rel(fb, fin) < RTOL


def test_group_to_head_mapping_is_contiguous():
    # H = 4, G = 2: heads 0,1 read group 0 and heads 2,3 read group 1
    x, dt, A, Bm, Cm, D, bias, _ = _rand(6, 1, 19, 4, 3, 5, 2)
    y, f = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias)
    expand = [0, 0, 1, 1]
    y4, f4 = oracle.oracle_forward(x, dt, A, Bm[:, :, expand], Cm[:, :, expand], D, bias)
    assert np.array_equal(y, y4) and np.array_equal(f, f4)


def test_degenerate_cases():
    x, dt, A, Bm, Cm, D, bias, init = _rand(8, 1, 21, 2, 3, 4, 1, ndoc_init=1)
    Dx = D[None, None, :, None] * x
    # C = 0: only the skip term is left
    y, _ = oracle.oracle_forward(x, dt, A, Bm, np.zeros_like(Cm), D, bias, init)
    assert np.array_equal(y, Dx)
    # B = 0 and no initial state: the state stays zero
    y, f = oracle.oracle_forward(x, dt, A, np.zeros_like(Bm), Cm, D, bias)
    assert np.array_equal(y, Dx) and not np.any(f)
    # transition multiplier 0 (A -> -inf): memoryless, y_t = (C_t.B_t) delta_t x_t + D x_t
    y, _ = oracle.oracle_forward(x, dt, np.full(2, -1e300), Bm, Cm, D, bias, init)
    delta = _delta(dt, bias[None, None, :])
    cb = np.einsum("ltn,ltn->lt", Cm[:, :, 0], Bm[:, :, 0])
    expect = (cb[:, :, None] * delta)[..., None] * x + Dx
    assert _rel(y, expect) < RTOL


def test_linearity_in_x():
    x, dt, A, Bm, Cm, D, bias, _ = _rand(9, 1, 25, 2, 3, 4, 1)
    x2 = np.random.default_rng(10).standard_normal(x.shape)
    y1, _ = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias)
    y2, _ = oracle.oracle_forward(x2, dt, A, Bm, Cm, D, bias)
    y3, _ = oracle.oracle_forward(2.0 * x - 3.0 * x2, dt, A, Bm, Cm, D, bias)
    assert _rel(y3, 2.0 * y1 - 3.0 * y2) < 1e-12


def test_head_subset_matches_full_run_and_empty_document_keeps_its_state():
    lens = [6, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x, dt, A, Bm, Cm, D, bias, init = _rand(12, 1, 15, 4, 3, 2, 2, ndoc_init=3)
    y, f = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, init, cu_seqlens=cu)
    ys, fs = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, init, cu_seqlens=cu, heads=[3, 1])
    for h in (1, 3):
        assert np.array_equal(ys[:, :, h], y[:, :, h]) and np.array_equal(fs[:, h], f[:, h])
    assert np.all(np.isnan(ys[:, :, 0])) and np.all(np.isnan(fs[:, 2]))
    assert np.array_equal(f[1], init[1])


def test_oracle_rejects_inconsistent_documents():
    x, dt, A, Bm, Cm, D, bias, _ = _rand(13, 1, 10, 2, 2, 2, 1)
    with pytest.raises(ValueError):
        oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, cu_seqlens=[0, 6, 4, 10])
    with pytest.raises(ValueError):
        oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, cu_seqlens=[0, 9])


@pytest.mark.parametrize("seed,G,H", [(21, 1, 3), (22, 2, 4)])
def test_decode_step_equals_the_sequential_recurrence(seed, G, H):
    # stepping token by token from an initial state gives the recurrence run by the
    # C oracle over the same sequence (outputs and final state)
    b, L = 3, 9
    x, dt, A, Bm, Cm, D, bias, init = _rand(seed, b, L, H, 5, 4, G, ndoc_init=b)
    y_ref, fin_ref = oracle.oracle_forward(x, dt, A, Bm, Cm, D, bias, init)
    state = init.copy()
    ys = []
    for t in range(L):
        y, state = oracle.oracle_step(state, x[:, t], dt[:, t], A, Bm[:, t], Cm[:, t], D, bias)
        ys.append(y)
    assert _rel(np.stack(ys, axis=1), y_ref) < RTOL
    assert _rel(state, fin_ref) < RTOL


def test_decode_step_from_zero_state_matches_quadratic_form():
    # from a zero state the stepped outputs are the rows of the materialised dual form
    H, P, N, L = 2, 3, 4, 11
    x, dt, A, Bm, Cm, D, bias, _ = _rand(23, 1, L, H, P, N, 1)
    state = np.zeros((1, H, N, P))
    ys = []
    for t in range(L):
        y, state = oracle.oracle_step(state, x[:, t], dt[:, t], A, Bm[:, t], Cm[:, t], D, bias)
        ys.append(y[0])
    ys = np.stack(ys)  # [L, H, P]
    for h in range(H):
        yq, fq = quadratic_form(x[0, :, h], _delta(dt[0, :, h], bias[h]), A[h], Bm[0, :, 0],
                                Cm[0, :, 0], D[h])
        assert _rel(ys[:, h], yq) < RTOL
        assert _rel(state[0, h], fq) < RTOL


# ---- the backward oracle ------------------------------------------------------------
# Pinned against central finite differences of oracle_forward (itself pinned above) and
# against torch.autograd of a plain float64 loop over tokens: two independent ways of
# differentiating the recurrence.

def _bwd_case(seed, varlen):
    r = np.random.default_rng(seed)
    H, P, N, G = 4, 3, 2, 2
    if varlen:
        cu = np.array([0, 4, 4, 11, 13], dtype=np.int64)   # an empty document too
        b, L = 1, 13
        ndocs = 4
    else:
        cu = None
        b, L = 2, 6
        ndocs = 2
    x, dt, A, Bm, Cm, D, bias, init = _rand(seed, b, L, H, P, N, G, ndoc_init=ndocs)
    A = -np.exp(r.uniform(-1.0, 1.0, H))       # decays of order one: every term is visible
    bias = r.uniform(-0.5, 0.5, H)
    init = r.standard_normal((ndocs, H, N, P))
    dy = r.standard_normal((b, L, H, P))
    dfin = r.standard_normal((ndocs, H, N, P))
    return dict(x=x, dt=dt, A=A, B=Bm, C=Cm, D=D, dt_bias=bias, initial_states=init), dy, dfin, cu


def _loss(inp, dy, dfin, cu):
    y, fin = oracle.oracle_forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                   inp["dt_bias"], inp["initial_states"], cu_seqlens=cu)
    return float(np.sum(dy * y) + np.sum(dfin * fin))


_BWD_KEYS = [("x", "dx"), ("dt", "ddt"), ("A", "dA"), ("B", "dB"), ("C", "dC"), ("D", "dD"),
             ("dt_bias", "ddt_bias"), ("initial_states", "dinitial_states")]


@pytest.mark.parametrize("varlen", [False, True], ids=["batch", "packed"])
def test_backward_equals_finite_differences_of_the_forward(varlen):
    inp, dy, dfin, cu = _bwd_case(7, varlen)
    g = oracle.oracle_backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"],
                               inp["dt_bias"], inp["initial_states"], dfin, cu_seqlens=cu)
    eps = 1e-6
    for key, gkey in _BWD_KEYS:
        base = inp[key]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            plus = {k: v.copy() for k, v in inp.items()}
            minus = {k: v.copy() for k, v in inp.items()}
            plus[key][idx] += eps
            minus[key][idx] -= eps
            fd[idx] = (_loss(plus, dy, dfin, cu) - _loss(minus, dy, dfin, cu)) / (2 * eps)
        assert _rel(g[gkey], fd) < 1e-7, key


def _torch_loss(t, dy, dfin, offsets, G):
    """Plain float64 loop over tokens, differentiated by torch.autograd."""
    import torch
    x, dt, A, Bm, Cm, D, bias, init = (t[k] for k in ("x", "dt", "A", "B", "C", "D", "dt_bias",
                                                      "initial_states"))
    b, L, H, P = x.shape
    xs, dts, Bs, Cs = (v.reshape(b * L, *v.shape[2:]) for v in (x, dt, Bm, Cm))
    dys = torch.from_numpy(dy).reshape(b * L, H, P)
    dfin_t = torch.from_numpy(dfin)
    loss = torch.zeros((), dtype=torch.float64)
    hpg = H // G
    for d in range(len(offsets) - 1):
        for h in range(H):
            g = h // hpg
            S = init[d, h]
            for tok in range(offsets[d], offsets[d + 1]):
                delta = torch.nn.functional.softplus(dts[tok, h] + bias[h])
                S = torch.exp(delta * A[h]) * S + delta * torch.outer(Bs[tok, g], xs[tok, h])
                y = Cs[tok, g] @ S + D[h] * xs[tok, h]
                loss = loss + torch.dot(dys[tok, h], y)
            loss = loss + torch.sum(dfin_t[d, h] * S)
    return loss


@pytest.mark.parametrize("varlen", [False, True], ids=["batch", "packed"])
def test_backward_equals_autograd_of_a_token_loop(varlen):
    import torch
    inp, dy, dfin, cu = _bwd_case(11, varlen)
    b, L = inp["x"].shape[:2]
    offsets = list(cu) if cu is not None else [i * L for i in range(b + 1)]
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in inp.items()}
    _torch_loss(t, dy, dfin, offsets, inp["B"].shape[2]).backward()
    g = oracle.oracle_backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"],
                               inp["dt_bias"], inp["initial_states"], dfin, cu_seqlens=cu)
    for key, gkey in _BWD_KEYS:
        assert _rel(g[gkey], t[key].grad.numpy()) < 1e-12, key


def test_backward_head_subset_matches_full_run():
    inp, dy, dfin, cu = _bwd_case(3, False)
    full = oracle.oracle_backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"],
                                  inp["dt_bias"], inp["initial_states"], dfin)
    part = oracle.oracle_backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"],
                                  inp["dt_bias"], inp["initial_states"], dfin, heads=[1, 2])
    for h in (1, 2):
        assert np.array_equal(part["dx"][:, :, h], full["dx"][:, :, h])
        assert np.array_equal(part["ddt"][:, :, h], full["ddt"][:, :, h])
        assert np.array_equal(part["dinitial_states"][:, h], full["dinitial_states"][:, h])
        assert part["dA"][h] == full["dA"][h]
    assert np.isnan(part["dx"][:, :, 0]).all()


# ---- feature maps and denominator normalisation ---------------------------------------

def test_pointwise_feature_maps_match_library_functions():
    from scipy.special import expit
    X = np.random.default_rng(1).standard_normal((5, 3, 7)) * 4
    assert np.allclose(oracle.oracle_feature_map(X, oracle.FMAP_SILU), X * expit(X), rtol=1e-14)
    assert np.array_equal(oracle.oracle_feature_map(X, oracle.FMAP_RELU), np.clip(X, 0, None))
    assert np.array_equal(oracle.oracle_feature_map(X, oracle.FMAP_NONE), X)


def test_based_and_rebased_maps_are_the_kernels_they_approximate():
    r = np.random.default_rng(2)
    a, b = r.standard_normal(6), r.standard_normal(6)
    dot = float(a @ b)
    fa, fb = (oracle.oracle_feature_map(v[None], oracle.FMAP_BASED)[0] for v in (a, b))
    assert fa.shape == (1 + 6 + 36,)
    assert abs(fa @ fb - (1 + dot + dot * dot / 2)) < 1e-12      # Taylor of exp to 2nd order
    ga, gb = (oracle.oracle_feature_map(v[None], oracle.FMAP_REBASED)[0] for v in (a, b))
    assert ga.shape == (36,)
    assert abs(ga @ gb - dot * dot) < 1e-12


def test_normalised_scan_equals_normalised_linear_attention_when_A_is_zero():
    """A = 0 removes the decay: y_t = sum_{s<=t} w_ts x_s / sum_{s<=t} w_ts with
    w_ts = delta_s <phi(C_t), phi(B_s)>, written out directly (plus D x)."""
    r = np.random.default_rng(3)
    L, H, P, N = 9, 2, 3, 8
    x = r.standard_normal((1, L, H, P))
    dt = r.standard_normal((1, L, H))
    A = np.zeros(H)
    Bm, Cm = r.standard_normal((1, L, 1, N)), r.standard_normal((1, L, 1, N))
    D = r.standard_normal(H)
    bias = r.uniform(-0.5, 0.5, H)
    for kind in (oracle.FMAP_RELU, oracle.FMAP_BASED, oracle.FMAP_REBASED):
        y, _ = oracle.oracle_forward_ext(x, dt, A, Bm, Cm, D, bias, kind, normalize=True)
        fB = oracle.oracle_feature_map(Bm[0, :, 0], kind)
        fC = oracle.oracle_feature_map(Cm[0, :, 0], kind)
        delta = np.logaddexp(0.0, dt[0] + bias)                         # [L, H]
        assert np.isfinite(y).mean() > 0.8      # ReLU can leave a token with no weight (0 / 0)
        for h in range(H):
            for t in range(L):
                w = np.array([delta[s, h] * (fC[t] @ fB[s]) for s in range(t + 1)])
                with np.errstate(invalid="ignore"):
                    ref = (w[:, None] * x[0, :t + 1, h]).sum(0) / w.sum() + D[h] * x[0, t, h]
                with np.errstate(invalid="ignore"):
                    assert np.allclose(y[0, t, h], ref, rtol=1e-11, atol=1e-12, equal_nan=True)


def test_normalised_scan_of_a_constant_input_returns_it():
    r = np.random.default_rng(4)
    L, H, P, N = 40, 3, 5, 4
    v = r.standard_normal(P)
    x = np.broadcast_to(v, (2, L, H, P)).copy()
    dt = r.standard_normal((2, L, H))
    A = -np.exp(r.uniform(0, 2, H))
    Bm, Cm = r.standard_normal((2, L, 1, N)), r.standard_normal((2, L, 1, N))
    for kind in (oracle.FMAP_RELU, oracle.FMAP_BASED, oracle.FMAP_REBASED):
        y, _ = oracle.oracle_forward_ext(x, dt, A, Bm, Cm, None, None, kind, normalize=True)
        ok = np.isfinite(y)
        assert ok.mean() > 0.9
        assert np.allclose(y[ok], np.broadcast_to(v, y.shape)[ok], rtol=1e-9)


def test_feature_map_without_normalisation_is_the_plain_scan_of_mapped_inputs():
    x, dt, A, Bm, Cm, D, bias, _ = _rand(5, 2, 21, 3, 4, 3, 1)
    y, fin = oracle.oracle_forward_ext(x, dt, A, Bm, Cm, D, bias, oracle.FMAP_SILU)
    y2, fin2 = oracle.oracle_forward(x, dt, A, Bm / (1 + np.exp(-Bm)), Cm / (1 + np.exp(-Cm)), D,
                                     bias)
    assert np.array_equal(y, y2) and np.array_equal(fin, fin2)
