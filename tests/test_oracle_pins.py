"""Pins that tie the fp64 oracle to facts other than itself (CPU only).

Each test names the passage of "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
(review page sections / equations) that fixes the expected behaviour. Together they are chosen so
that a plausible slip in the oracle -- decay applied after the read, erase gate on the wrong side,
write gate missing, output read before the update, a wrong sign or a transposed state -- fails at
least one of them (test_planted_mistakes_are_caught checks exactly that on mutated copies).
"""
from __future__ import annotations

import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from tests import chunkform_np

RNG = np.random.default_rng


def _rand_inputs(rng, B, T, H, dk, dv, *, neg_eig=False, s0=True, unit_k=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    la = -0.3 * np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dk))))
    if neg_eig:
        b = 2.0 * b
    w = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dv))))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None
    return q, k, v, la, b, w, S0


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# --- hand-worked example ---------------------------------------------------------------------

def _read_golden(name):
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    vals = {}
    for line in open(path):
        m = re.match(r"^(\w+)\s*=\s*([-0-9. ]+)$", line.strip())
        if m and not line.startswith("#"):
            vals[m.group(1)] = np.array([float(x) for x in m.group(2).split()])
    return vals


def test_hand_worked_eq10_example():
    """Two tokens worked by hand from Steps 1-5 (section "The Gated Delta Rule-2 State Update")."""
    g = _read_golden("eq10_hand_worked.txt")
    shp_k = (1, 2, 1, 2)
    q = g["q"].reshape(shp_k)
    k = g["k"].reshape(shp_k)
    b = g["b"].reshape(shp_k)
    la = np.log(g["alpha"]).reshape(shp_k)
    v = g["v"].reshape(shp_k)
    w = g["w"].reshape(shp_k)
    S0 = g["S0"].reshape(1, 1, 2, 2)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    np.testing.assert_allclose(o.reshape(-1), g["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(ST.reshape(-1), g["S_final"], rtol=0, atol=1e-12)
    # the decode entry point is the same step, one token at a time
    S = S0
    for t in range(2):
        ot, S = oracle.decode(q[:, t], k[:, t], v[:, t], la[:, t], b[:, t], w[:, t], S)
        np.testing.assert_allclose(ot.reshape(-1), g["o"][2 * t:2 * t + 2], atol=1e-12)
    np.testing.assert_allclose(S.reshape(-1), g["S_final"], atol=1e-12)


# --- reductions to earlier models ------------------------------------------------------------

def _kda_reference(q, k, v, la, beta, S0):
    """KDA (review, "Why this form": S = (I - beta k k^T) D S + beta k v^T), written independently."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = S0[bi, h].copy() if S0 is not None else np.zeros((dk, dv))
            for t in range(T):
                kk = k[bi, t, h][:, None]
                bt = beta[bi, t, h]
                S = (np.eye(dk) - bt * kk @ kk.T) @ np.diag(np.exp(la[bi, t, h])) @ S + bt * kk @ v[bi, t, h][None, :]
                o[bi, t, h] = S.T @ q[bi, t, h]
            ST[bi, h] = S
    return o, ST


def test_pin_kda_reduction():
    """b = w = beta*1 reduces Eq. 10 to KDA (review: tied-gate case of Eq. 10)."""
    rng = RNG(1)
    q, k, v, la, _, _, S0 = _rand_inputs(rng, 2, 9, 2, 5, 4)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((2, 9, 2))))
    b = np.repeat(beta[..., None], 5, axis=-1)
    w = np.repeat(beta[..., None], 4, axis=-1)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    o2, ST2 = _kda_reference(q, k, v, la, beta, S0)
    assert _rel(o, o2) < 1e-13 and _rel(ST, ST2) < 1e-13


def test_pin_gated_deltanet_reduction():
    """Additionally scalar alpha gives Gated DeltaNet: S = alpha (I - beta k k^T) S + beta k v^T."""
    rng = RNG(2)
    q, k, v, _, _, _, S0 = _rand_inputs(rng, 1, 11, 3, 6, 3)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, 11, 3))))
    alpha = np.exp(-0.5 * rng.random((1, 11, 3)))
    la = np.repeat(np.log(alpha)[..., None], 6, axis=-1)
    b = np.repeat(beta[..., None], 6, axis=-1)
    w = np.repeat(beta[..., None], 3, axis=-1)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    for h in range(3):
        S = S0[0, h].copy()
        for t in range(11):
            kk = k[0, t, h][:, None]
            S = alpha[0, t, h] * (np.eye(6) - beta[0, t, h] * kk @ kk.T) @ S + beta[0, t, h] * kk @ v[0, t, h][None, :]
            assert _rel(o[0, t, h], S.T @ q[0, t, h]) < 1e-13
        assert _rel(ST[0, h], S) < 1e-13


def test_pin_linear_attention_prefix_sum():
    """alpha = 1, b = 0: no decay and no erase, so S_t = S_0 + sum_{s<=t} k_s (w_s*v_s)^T (Eq. 1 with z)."""
    rng = RNG(3)
    q, k, v, _, _, w, S0 = _rand_inputs(rng, 2, 13, 2, 4, 5, unit_k=False)
    la = np.zeros_like(q)
    b = np.zeros_like(q)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    outer = np.einsum("bthi,bthj->bthij", k, w * v)
    S_all = S0[:, None] + np.cumsum(outer, axis=1)
    o_ref = np.einsum("bthij,bthi->bthj", S_all, q)
    assert _rel(o, o_ref) < 1e-13
    assert _rel(ST, S_all[:, -1]) < 1e-13


@pytest.mark.parametrize("decay", [0.0, 0.4])
def test_pin_projector_read_back(decay):
    """b = 1 and |k| = 1: the edit makes the new state read back z along k, k^T S_t = z_t^T
    (review, fast-weight section: the update corrects the read at k_t to the target z_t)."""
    rng = RNG(4)
    q, k, v, la, _, w, S0 = _rand_inputs(rng, 1, 1, 1, 6, 5)
    la = la * decay / 0.3
    b = np.ones_like(q)
    T = 7
    S = S0
    for t in range(T):
        q, k, v, la_t, _, w, _ = _rand_inputs(rng, 1, 1, 1, 6, 5, s0=False)
        o, S = oracle.fwd(q, k, v, la_t * decay / 0.3, b, w, S)
        lhs = np.einsum("i,ij->j", k[0, 0, 0], S[0, 0])
        np.testing.assert_allclose(lhs, (w * v)[0, 0, 0], atol=1e-13)


def test_pin_negative_eigenvalue_reflection():
    """b = 2, w = 0, alpha = 1, |k| = 1: I - 2 k k^T is a Householder reflection (eigenvalue -1,
    the [0, 2] erase-gate variant of Eq. 11), so the Frobenius norm of S never changes."""
    rng = RNG(5)
    q, k, v, _, _, _, S0 = _rand_inputs(rng, 1, 40, 2, 8, 6)
    la = np.zeros_like(q)
    b = 2.0 * np.ones_like(q)
    w = np.zeros_like(v)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    np.testing.assert_allclose(np.linalg.norm(ST, axis=(-2, -1)), np.linalg.norm(S0, axis=(-2, -1)), rtol=1e-13)
    # and it is not the identity: the state does move
    assert _rel(ST, S0) > 1e-2


def test_pin_transition_matrix_product():
    """S_T = M_T...M_1 S_0 + sum_t M_T...M_{t+1} k_t z_t^T with M_t = (I - k_t e_t^T) Diag(alpha_t)
    (Eq. 10 read as a product of per-token transition matrices), on tiny T and d."""
    rng = RNG(6)
    for T in (1, 2, 3, 4):
        q, k, v, la, b, w, S0 = _rand_inputs(rng, 1, T, 1, 4, 3, neg_eig=True)
        o, ST = oracle.fwd(q, k, v, la, b, w, S0)
        M = [(np.eye(4) - np.outer(k[0, t, 0], b[0, t, 0] * k[0, t, 0])) @ np.diag(np.exp(la[0, t, 0]))
             for t in range(T)]
        for t_end in range(1, T + 1):
            P = np.eye(4)
            for t in range(t_end):
                P = M[t] @ P
            S = P @ S0[0, 0]
            for t in range(t_end):
                Pt = np.eye(4)
                for s in range(t + 1, t_end):
                    Pt = M[s] @ Pt
                S = S + Pt @ np.outer(k[0, t, 0], w[0, t, 0] * v[0, t, 0])
            np.testing.assert_allclose(o[0, t_end - 1, 0], S.T @ q[0, t_end - 1, 0], atol=1e-13)
        np.testing.assert_allclose(ST[0, 0], S, atol=1e-13)


def test_pin_value_column_independence():
    """The value axis enters Eq. 10 only through z and r column by column, so running the oracle
    on a subset J of value channels reproduces those columns of o and S."""
    rng = RNG(7)
    q, k, v, la, b, w, S0 = _rand_inputs(rng, 2, 17, 2, 5, 6)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    J = [1, 4, 5]
    oJ, STJ = oracle.fwd(q, k, v[..., J], la, b, w[..., J], np.ascontiguousarray(S0[..., J]))
    assert _rel(oJ, o[..., J]) < 1e-14 and _rel(STJ, ST[..., J]) < 1e-14


def test_pin_fast_weight_stationarity():
    """The update is the minimiser of the local loss of the fast-weight section (Eq. 13):
    L(S) = |S - Sbar|_F^2 - 2 <S^T k, z - Sbar^T e>. Checked numerically: L at the oracle's S_1 is
    below L at random perturbations of it, and the perturbation cost is exactly |dS|_F^2."""
    rng = RNG(8)
    q, k, v, la, b, w, S0 = _rand_inputs(rng, 1, 1, 1, 5, 4)
    _, S1 = oracle.fwd(q, k, v, la, b, w, S0)
    Sbar = np.exp(la[0, 0, 0])[:, None] * S0[0, 0]
    kk, e, z = k[0, 0, 0], b[0, 0, 0] * k[0, 0, 0], w[0, 0, 0] * v[0, 0, 0]

    def L(S):
        return np.sum((S - Sbar) ** 2) - 2 * np.dot(S.T @ kk, z - Sbar.T @ e)

    base = L(S1[0, 0])
    for _ in range(5):
        d = rng.standard_normal(S1[0, 0].shape) * 1e-2
        np.testing.assert_allclose(L(S1[0, 0] + d) - base, np.sum(d * d), rtol=1e-8, atol=1e-15)


# --- backward ----------------------------------------------------------------------------------

def _loss(q, k, v, la, b, w, S0, dO, dST):
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    return float(np.sum(o * dO) + np.sum(ST * dST))


@pytest.mark.parametrize("neg_eig", [False, True])
def test_pin_finite_differences(neg_eig):
    """Every gradient of L = <o, dO> + <S_T, dS_T> matches central differences (h = 1e-6): the
    gradient-check protocol of the review's Appendix D.6 paragraph, in fp64."""
    rng = RNG(9 + neg_eig)
    B, T, H, dk, dv = 1, 6, 1, 3, 2
    q, k, v, la, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv, neg_eig=neg_eig)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    g = oracle.bwd(q, k, v, la, b, w, S0, dO, dST)
    args = {"q": q, "k": k, "v": v, "la": la, "b": b, "w": w, "S0": S0}
    names = {"q": "dq", "k": "dk", "v": "dv", "la": "dlog_alpha", "b": "db", "w": "dw", "S0": "dS0"}
    h = 1e-6
    for name, arr in args.items():
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            saved = arr[idx]
            arr[idx] = saved + h
            lp = _loss(**args, dO=dO, dST=dST)
            arr[idx] = saved - h
            lm = _loss(**args, dO=dO, dST=dST)
            arr[idx] = saved
            num[idx] = (lp - lm) / (2 * h)
        got = g[names[name]]
        assert _rel(got, num) < 1e-7, (name, _rel(got, num))


def test_pin_gradient_zero_upstream():
    """No upstream gradient -> all gradients vanish; dS_T alone -> dq = 0 and dS0 = prod of M_t^T."""
    rng = RNG(11)
    q, k, v, la, b, w, S0 = _rand_inputs(rng, 1, 5, 1, 3, 2)
    g = oracle.bwd(q, k, v, la, b, w, S0, None, None)
    assert all(np.all(x == 0) for x in g.values())
    dST = rng.standard_normal(S0.shape)
    g = oracle.bwd(q, k, v, la, b, w, S0, None, dST)
    assert np.all(g["dq"] == 0)
    P = np.eye(3)
    for t in range(5):
        P = (np.eye(3) - np.outer(k[0, t, 0], b[0, t, 0] * k[0, t, 0])) @ np.diag(np.exp(la[0, t, 0])) @ P
    np.testing.assert_allclose(g["dS0"][0, 0], P.T @ dST[0, 0], atol=1e-13)


# --- the chunkwise algebra ----------------------------------------------------------------------

@pytest.mark.parametrize("T,C", [(128, 64), (100, 64), (37, 16), (1, 64)])
def test_pin_chunk_form_matches_oracle(T, C):
    """An independent numpy restatement of the chunkwise WY algorithm (Eqs. 20-24 forward, gate-aware
    backward of Eqs. 64-65) equals the token recurrence to ~1e-12 (review, Appendix D.6: "agree to
    machine precision" in fp64), including a ragged last chunk."""
    rng = RNG(12)
    dk, dv = 8, 6
    q, k, v, la, b, w, S0 = _rand_inputs(rng, 1, T, 1, dk, dv, neg_eig=True)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    g = oracle.bwd(q, k, v, la, b, w, S0, dO, dST)
    sl = (0, slice(None), 0)
    oc, STc, _ = chunkform_np.chunk_fwd(q[sl], k[sl], v[sl], la[sl], b[sl], w[sl], S0[0, 0], C)
    assert _rel(oc, o[sl]) < 1e-11 and _rel(STc, ST[0, 0]) < 1e-11
    gc = chunkform_np.chunk_bwd(q[sl], k[sl], v[sl], la[sl], b[sl], w[sl], S0[0, 0], dO[sl], dST[0, 0], C)
    for name in ("dq", "dk", "dv", "db", "dw"):
        assert _rel(gc[name], g[name][sl]) < 1e-10, name
    assert _rel(gc["dla"], g["dlog_alpha"][sl]) < 1e-10
    assert _rel(gc["dS0"], g["dS0"][0, 0]) < 1e-10


def test_pin_relative_decay_factors():
    """The chunk form with decay factors relative to each channel's mid-chunk log-decay (the tensor-core
    kernels' algebra) equals the token recurrence to ~1e-10 in fp64, at mild and at strong decay; and in
    fp32 arithmetic at about -2 per token (G_C near -128 over a 64-row chunk) it stays finite and within
    fp32 rounding of the oracle, while the absolute factors e^{+-G} overflow."""
    rng = RNG(21)
    dk, dv, T, C = 8, 6, 150, 64
    q, k, v, la, b, w, S0 = _rand_inputs(rng, 1, T, 1, dk, dv, neg_eig=True)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    sl = (0, slice(None), 0)
    for scale in (None, 2.0):
        las = la if scale is None else -(1.6 + 0.8 * rng.random(la.shape))  # [-2.4, -1.6] per token
        o, ST = oracle.fwd(q, k, v, las, b, w, S0)
        g = oracle.bwd(q, k, v, las, b, w, S0, dO, dST)
        oc, STc, _ = chunkform_np.chunk_fwd(q[sl], k[sl], v[sl], las[sl], b[sl], w[sl], S0[0, 0], C, relative=True)
        assert _rel(oc, o[sl]) < 1e-10 and _rel(STc, ST[0, 0]) < 1e-10
        gc = chunkform_np.chunk_bwd(q[sl], k[sl], v[sl], las[sl], b[sl], w[sl], S0[0, 0], dO[sl], dST[0, 0], C,
                                    relative=True)
        for name in ("dq", "dk", "dv", "db", "dw"):
            assert _rel(gc[name], g[name][sl]) < 1e-9, (scale, name)
        assert _rel(gc["dla"], g["dlog_alpha"][sl]) < 1e-9
        assert _rel(gc["dS0"], g["dS0"][0, 0]) < 1e-9
    # fp32 arithmetic at the strong decay of the last case
    f32 = [x[sl].astype(np.float32) for x in (q, k, v, las, b, w)]
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        oa, _, _ = chunkform_np.chunk_fwd(*f32, S0[0, 0].astype(np.float32), C)
        orl, STr, _ = chunkform_np.chunk_fwd(*f32, S0[0, 0].astype(np.float32), C, relative=True)
    assert not np.all(np.isfinite(oa))  # e^{-G} of the absolute keys overflows fp32
    assert np.all(np.isfinite(orl)) and np.all(np.isfinite(STr))
    assert _rel(orl.astype(np.float64), o[sl]) < 1e-4 and _rel(STr.astype(np.float64), ST[0, 0]) < 1e-4


def test_oracle_thread_count_does_not_change_results():
    rng = RNG(13)
    q, k, v, la, b, w, S0 = _rand_inputs(rng, 3, 70, 3, 4, 4)
    o1, S1 = oracle.fwd(q, k, v, la, b, w, S0, nthreads=1)
    o4, S4 = oracle.fwd(q, k, v, la, b, w, S0, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(S1, S4)


# --- planted mistakes -----------------------------------------------------------------------------

_MUTANTS = {
    # decay applied after the read instead of before it (Step 1 / Step 2 order)
    "decay_after_read": ("r[j] += sbar[i * dv + j] * e;", "r[j] += S[i * dv + j] * e;"),
    # erase gate dropped from the read direction
    "no_erase_gate": ("double e = b[i] * k[i];", "double e = k[i];"),
    # write gate dropped
    "no_write_gate": ("z[j] = w[j] * v[j];", "z[j] = v[j];"),
    # output read from the pre-update state
    "output_before_update": ("o[j] += S[i * dv + j] * q[i];", "o[j] += sbar[i * dv + j] * q[i];"),
    # wrong sign of the residual
    "residual_sign": ("k[i] * (z[j] - r[j])", "k[i] * (r[j] - z[j])"),
    # adjoint: decay gradient missing the erase correction
    "adjoint_mu": ("mu[i * dv + j] = lam[i * dv + j] - e[i] * dd[j];", "mu[i * dv + j] = lam[i * dv + j];"),
    # adjoint: erase-gate gradient with the wrong factor
    "adjoint_db": ("dbp[i] = de[i] * k[i];", "dbp[i] = de[i] * b[i];"),
}


@pytest.mark.parametrize("mutant", sorted(_MUTANTS))
def test_planted_mistakes_are_caught(mutant, tmp_path, monkeypatch):
    """Plant one plausible mistake in a copy of the oracle's C source, rebuild it in a temporary
    directory, and check that at least one pin above fails on it."""
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdr2_oracle.c")).read()
    old, new = _MUTANTS[mutant]
    assert src.count(old) >= 1, mutant
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", str(so), str(mut), "-lm", "-lpthread"])
    import ctypes
    lib = ctypes.CDLL(str(so))
    lib.oracle_gdr2_fwd.argtypes = oracle._load().oracle_gdr2_fwd.argtypes
    lib.oracle_gdr2_bwd.argtypes = oracle._load().oracle_gdr2_bwd.argtypes
    lib.oracle_gdr2_decode.argtypes = oracle._load().oracle_gdr2_decode.argtypes
    monkeypatch.setattr(oracle, "_lib", lib)
    pins = [test_hand_worked_eq10_example, test_pin_kda_reduction, test_pin_linear_attention_prefix_sum,
            lambda: test_pin_projector_read_back(0.4), test_pin_transition_matrix_product,
            lambda: test_pin_finite_differences(True),
            lambda: test_pin_chunk_form_matches_oracle(37, 16)]
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught the planted mistake {mutant}"


# --- the chunk-level scan ------------------------------------------------------------------------

def test_pin_segment_scan_composition():
    """Eq. 23 is affine in the state entering a chunk, so a chain cut into segments composes as
    S_end = M S_start + N, with M the segment run from S = I without writes (z = 0) and N the run
    from S = 0. Forward: chaining the segments' (M, N) and rerunning each from its start state gives
    the whole chain's o and S_T. Backward: the gradient entering a segment's end obeys
    E_{s-1} = M_s^T E_s + dN_s (dN_s the segment's dS0 for dS_T = 0), and rerunning each segment
    from E_s gives the whole chain's gradients."""
    rng = RNG(13)
    T, dk, dv = 23, 4, 3
    q, k, v, la, b, w, S0 = _rand_inputs(rng, 1, T, 1, dk, dv, neg_eig=True)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    g = oracle.bwd(q, k, v, la, b, w, S0, dO, dST)
    cuts = [0, 8, 16, 23]
    segs = [slice(a, e) for a, e in zip(cuts[:-1], cuts[1:])]
    cut = lambda x, sl: np.ascontiguousarray(x[:, sl])  # noqa: E731
    M, N = [], []
    for sl in segs:
        zero_v = np.zeros(cut(q, sl).shape)  # value width dk: columns of the identity start state
        _, Ms = oracle.fwd(cut(q, sl), cut(k, sl), zero_v, cut(la, sl), cut(b, sl), np.ones(zero_v.shape),
                           np.eye(dk)[None, None])
        _, Ns = oracle.fwd(cut(q, sl), cut(k, sl), cut(v, sl), cut(la, sl), cut(b, sl), cut(w, sl), None)
        M.append(Ms[0, 0])
        N.append(Ns[0, 0])
    starts = [S0[0, 0]]
    for s in range(len(segs)):
        starts.append(M[s] @ starts[s] + N[s])
    np.testing.assert_allclose(starts[-1], ST[0, 0], atol=1e-12)
    for s, sl in enumerate(segs):
        os_, _ = oracle.fwd(cut(q, sl), cut(k, sl), cut(v, sl), cut(la, sl), cut(b, sl), cut(w, sl),
                            starts[s][None, None])
        np.testing.assert_allclose(os_, o[:, sl], atol=1e-12)
    # backward: offsets from zero end-gradient, combined with the forward's transfers transposed
    dN = []
    for s, sl in enumerate(segs):
        gs = oracle.bwd(cut(q, sl), cut(k, sl), cut(v, sl), cut(la, sl), cut(b, sl), cut(w, sl),
                        starts[s][None, None], cut(dO, sl), None)
        dN.append(gs["dS0"][0, 0])
    ends = [None] * len(segs)
    ends[-1] = dST[0, 0]
    for s in range(len(segs) - 1, 0, -1):
        ends[s - 1] = M[s].T @ ends[s] + dN[s]
    np.testing.assert_allclose(M[0].T @ ends[0] + dN[0], g["dS0"][0, 0], atol=1e-12)
    for s, sl in enumerate(segs):
        gs = oracle.bwd(cut(q, sl), cut(k, sl), cut(v, sl), cut(la, sl), cut(b, sl), cut(w, sl),
                        starts[s][None, None], cut(dO, sl), ends[s][None, None])
        for name in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"):
            np.testing.assert_allclose(gs[name], g[name][:, sl], atol=1e-11, err_msg=name)


# --- packed variable-length batches ------------------------------------------------------------

def test_pin_varlen_equal_lengths_is_the_batch():
    """N sequences of one length L packed back to back are the batch [N, L] of the unpacked oracle:
    pins the offsets and the per-sequence state bookkeeping of fwd_varlen / bwd_varlen."""
    rng = RNG(14)
    N, L, H, dk, dv = 3, 7, 2, 4, 3
    q, k, v, la, b, w, S0 = _rand_inputs(rng, N, L, H, dk, dv, neg_eig=True)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    pack = lambda x: x.reshape(N * L, *x.shape[2:])  # noqa: E731
    cu = np.arange(N + 1) * L
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    op, STp = oracle.fwd_varlen(*(pack(x) for x in (q, k, v, la, b, w)), cu, S0)
    np.testing.assert_array_equal(op, pack(o))
    np.testing.assert_array_equal(STp, ST)
    g = oracle.bwd(q, k, v, la, b, w, S0, dO, dST)
    gp = oracle.bwd_varlen(*(pack(x) for x in (q, k, v, la, b, w)), cu, S0, pack(dO), dST)
    for name in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"):
        np.testing.assert_array_equal(gp[name], pack(g[name]))
    np.testing.assert_array_equal(gp["dS0"], g["dS0"])


def test_pin_varlen_state_reset():
    """The state restarts at every boundary (review, Appendix C.6): changing one sequence's inputs
    changes none of the other sequences' outputs or gradients; an empty sequence passes its state (and
    its state gradient) through; one sequence over the whole axis is the unpacked oracle."""
    rng = RNG(15)
    T, H, dk, dv = 20, 1, 3, 2
    q, k, v, la, b, w, _ = _rand_inputs(rng, 1, T, H, dk, dv, s0=False)
    q, k, v, la, b, w = (x[0] for x in (q, k, v, la, b, w))
    cu = np.array([0, 6, 6, 13, 20])
    S0 = rng.standard_normal((4, H, dk, dv))
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    o, ST = oracle.fwd_varlen(q, k, v, la, b, w, cu, S0)
    g = oracle.bwd_varlen(q, k, v, la, b, w, cu, S0, dO, dST)
    k2 = k.copy()
    k2[6:13] = rng.standard_normal((7, H, dk))  # only sequence 2 changes
    o2, ST2 = oracle.fwd_varlen(q, k2, v, la, b, w, cu, S0)
    g2 = oracle.bwd_varlen(q, k2, v, la, b, w, cu, S0, dO, dST)
    for sl in (slice(0, 6), slice(13, 20)):
        np.testing.assert_array_equal(o2[sl], o[sl])
        for name in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"):
            np.testing.assert_array_equal(g2[name][sl], g[name][sl])
    assert _rel(o2[6:13], o[6:13]) > 1e-3
    np.testing.assert_array_equal(ST[1], S0[1])
    np.testing.assert_array_equal(g["dS0"][1], dST[1])
    o1, ST1 = oracle.fwd_varlen(q, k, v, la, b, w, np.array([0, T]), S0[:1])
    of, STf = oracle.fwd(q[None], k[None], v[None], la[None], b[None], w[None], S0[:1])
    np.testing.assert_array_equal(o1, of[0])
    np.testing.assert_array_equal(ST1, STf)


# --- gate and normalisation prologue ------------------------------------------------------------

def test_pin_prologue_closed_forms():
    """Values fixed by the definitions of Eqs. 11-12 and the L2 normalisation, at points where the
    functions have closed forms: softplus(0) = ln 2, softplus(ln(e - 1)) = 1, softplus(z) -> z for
    large z; sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, twice that in the negative-eigenvalue variant;
    ||q|| = 1 along x_q; a zero vector stays zero."""
    H, dk, dv = 2, 4, 3
    a = np.array([[0.0, np.log(0.1), 1.0, -2.0], [0.5, 0.0, 0.0, 0.0]])
    delta = np.zeros((H, dk))
    xf = np.zeros((1, 3, H, dk))
    xf[0, 1] = np.log(np.e - 1.0)
    xf[0, 2] = 40.0
    xq = np.zeros((1, 3, H, dk))
    xq[0, 0, 0] = [3.0, 0.0, 4.0, 0.0]
    xq[0, 1, 1] = [1.0, 1.0, 1.0, 1.0]
    xb = np.zeros((1, 3, H, dk))
    xb[0, 1] = np.log(3.0)
    xw = np.zeros((1, 3, H, dv))
    for neg in (False, True):
        o = oracle.prologue_fwd(xq, xq, xf, xb, xw, a, delta, neg_eig=neg)
        np.testing.assert_allclose(o["log_alpha"][0, 0], -np.exp(a) * np.log(2.0), rtol=1e-15)
        np.testing.assert_allclose(o["log_alpha"][0, 1], -np.exp(a), rtol=1e-15)
        np.testing.assert_allclose(o["log_alpha"][0, 2], -np.exp(a) * 40.0, rtol=1e-15)
        s = 2.0 if neg else 1.0
        np.testing.assert_allclose(o["b"][0, 0], s * 0.5, rtol=1e-15)
        np.testing.assert_allclose(o["b"][0, 1], s * 0.75, rtol=1e-15)
        np.testing.assert_allclose(o["w"][0, 0], 0.5, rtol=1e-15)
        np.testing.assert_allclose(o["q"][0, 0, 0], [0.6, 0.0, 0.8, 0.0], rtol=1e-15)
        np.testing.assert_allclose(o["q"][0, 1, 1], [0.5, 0.5, 0.5, 0.5], rtol=1e-15)
        assert np.all(o["q"][0, 2] == 0.0)


def test_pin_prologue_finite_differences():
    """Every gradient of L = sum(q.Rq + k.Rk + log_alpha.Rg + b.Rb + w.Rw) with respect to every
    input (the five pre-activations, a and delta) matches central differences (h = 1e-6)."""
    rng = RNG(16)
    B, T, H, dk, dv = 2, 3, 2, 4, 3
    x = {n: rng.standard_normal((B, T, H, dk)) for n in ("xq", "xk", "xf", "xb")}
    x["xw"] = rng.standard_normal((B, T, H, dv))
    x["a"] = np.log(0.1) + 0.3 * rng.standard_normal((H, dk))
    x["delta"] = 0.5 * rng.standard_normal((H, dk))
    R = {n: rng.standard_normal(x["xq"].shape) for n in ("q", "k", "log_alpha", "b")}
    R["w"] = rng.standard_normal(x["xw"].shape)
    for neg in (False, True):
        def loss():
            o = oracle.prologue_fwd(**x, neg_eig=neg)
            return sum(float(np.sum(o[n] * R[n])) for n in R)
        g = oracle.prologue_bwd(**x, dq=R["q"], dk=R["k"], dlog_alpha=R["log_alpha"], db=R["b"], dw=R["w"],
                                neg_eig=neg)
        names = {"xq": "dxq", "xk": "dxk", "xf": "dxf", "xb": "dxb", "xw": "dxw", "a": "da", "delta": "ddelta"}
        h = 1e-6
        for name, arr in x.items():
            num = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                saved = arr[idx]
                arr[idx] = saved + h
                lp = loss()
                arr[idx] = saved - h
                lm = loss()
                arr[idx] = saved
                num[idx] = (lp - lm) / (2 * h)
            assert _rel(g[names[name]], num) < 1e-7, (name, neg, _rel(g[names[name]], num))


# --- grouped value heads ------------------------------------------------------------------------

def test_pin_gva_group_of_one_and_identical_members():
    """G = 1 is the plain mixer; value heads of one group that get the same v, w and initial state give
    the same outputs, and their key-side gradients add up: G identical members give G times the
    key-side gradient of one (the chain rule of a tensor used G times)."""
    rng = RNG(17)
    B, T, H, dk, dv, G = 1, 9, 2, 4, 3, 3
    q, k, v1, la, b, w1, S1 = _rand_inputs(rng, B, T, H, dk, dv, neg_eig=True)
    o1, ST1 = oracle.fwd(q, k, v1, la, b, w1, S1)
    og, STg = oracle.fwd_gva(q, k, v1, la, b, w1, S1)
    np.testing.assert_array_equal(og, o1)
    np.testing.assert_array_equal(STg, ST1)
    rep = lambda x: np.repeat(x, G, axis=2)  # noqa: E731  (token tensors: head axis 2)
    reps = lambda x: np.repeat(x, G, axis=1)  # noqa: E731  (states: head axis 1)
    o3, ST3 = oracle.fwd_gva(q, k, rep(v1), la, b, rep(w1), reps(S1))
    for r in range(G):
        np.testing.assert_array_equal(o3[:, :, r::G], o1)
        np.testing.assert_array_equal(ST3[:, r::G], ST1)
    dO1 = rng.standard_normal(v1.shape)
    dS1 = rng.standard_normal(S1.shape)
    g1 = oracle.bwd(q, k, v1, la, b, w1, S1, dO1, dS1)
    g3 = oracle.bwd_gva(q, k, rep(v1), la, b, rep(w1), reps(S1), rep(dO1), reps(dS1))
    for name in ("dq", "dk", "dlog_alpha", "db"):
        np.testing.assert_allclose(g3[name], G * g1[name], rtol=1e-12, atol=1e-14)
    for name in ("dv", "dw"):
        for r in range(G):
            np.testing.assert_allclose(g3[name][:, :, r::G], g1[name], rtol=1e-12, atol=1e-14)


def test_pin_gva_finite_differences():
    """Every gradient of L = <o, dO> + <S_T, dS_T> for grouped value heads (H = 1 key head, Hv = 2)
    matches central differences, the key-side ones included (h = 1e-6)."""
    rng = RNG(18)
    B, T, H, Hv, dk, dv = 1, 5, 1, 2, 3, 2
    q, k, _, la, b, _, _ = _rand_inputs(rng, B, T, H, dk, dv, neg_eig=True)
    v = rng.standard_normal((B, T, Hv, dv))
    w = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv, dv))))
    S0 = 0.5 * rng.standard_normal((B, Hv, dk, dv))
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    g = oracle.bwd_gva(q, k, v, la, b, w, S0, dO, dST)
    args = {"q": q, "k": k, "v": v, "la": la, "b": b, "w": w, "S0": S0}
    names = {"q": "dq", "k": "dk", "v": "dv", "la": "dlog_alpha", "b": "db", "w": "dw", "S0": "dS0"}

    def loss():
        o, ST = oracle.fwd_gva(args["q"], args["k"], args["v"], args["la"], args["b"], args["w"], args["S0"])
        return float(np.sum(o * dO) + np.sum(ST * dST))
    h = 1e-6
    for name, arr in args.items():
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            saved = arr[idx]
            arr[idx] = saved + h
            lp = loss()
            arr[idx] = saved - h
            lm = loss()
            arr[idx] = saved
            num[idx] = (lp - lm) / (2 * h)
        assert _rel(g[names[name]], num) < 1e-7, (name, _rel(g[names[name]], num))
