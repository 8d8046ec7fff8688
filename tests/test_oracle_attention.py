"""Pins for the fp64 attention oracle (CPU only).

Each pin checks the oracle against something other than itself: scalar
brute-force loops, torch's fp64 CPU SDPA and autograd, central finite
differences, closed forms and invariances the definition implies, and the
hand-worked fixture in ``tests/golden/``.  ``test_planted_mistakes`` plants
plausible mistakes in a copy of the oracle and checks that some pin fails
for each one.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import attention_ref as ar

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------------------
# independent implementations used as pins

def brute_fwd(q, k, v, scale, causal):
    """Scalar loops with math.exp; one head; q, k, v nested lists."""
    n, d, dv = len(q), len(q[0]), len(v[0])
    o, lse = [], []
    for i in range(n):
        keys = [j for j in range(len(k)) if (not causal or j <= i)]
        s = [scale * sum(q[i][t] * k[j][t] for t in range(d)) for j in keys]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        tot = sum(e)
        o.append([sum(e[a] * v[j][c] for a, j in enumerate(keys)) / tot for c in range(dv)])
        lse.append(m + math.log(tot))
    return np.array(o), np.array(lse)


def torch_sdpa(q, k, v, scale, causal):
    t = [torch.tensor(x, dtype=torch.float64) for x in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(
        t[0], t[1], t[2], is_causal=causal, scale=scale).numpy()


def torch_grads(q, k, v, do, scale, causal):
    t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v)]
    o = torch.nn.functional.scaled_dot_product_attention(
        t[0], t[1], t[2], is_causal=causal, scale=scale)
    (o * torch.tensor(do, dtype=torch.float64)).sum().backward()
    return [x.grad.numpy() for x in t]


# ---------------------------------------------------------------------------
# pins, written against callables so that planted mistakes can be run through them

def pin_brute_force(fwd, bwd):
    for seed, (n, d, causal) in enumerate([(1, 1, False), (2, 3, True), (5, 4, False),
                                           (8, 3, True), (7, 2, False), (8, 4, True)]):
        q, k, v = rand((1, 1, n, d), seed), rand((1, 1, n, d), seed + 50), rand((1, 1, n, d), seed + 99)
        sc = 0.7
        o, lse = fwd(q, k, v, sc, causal)
        ob, lb = brute_fwd(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), sc, causal)
        np.testing.assert_allclose(o[0, 0], ob, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[0, 0], lb, rtol=1e-12, atol=1e-12)


def pin_torch_sdpa(fwd, bwd):
    for causal in (False, True):
        q, k, v = rand((2, 3, 37, 16), 1), rand((2, 3, 37, 16), 2), rand((2, 3, 37, 16), 3)
        sc = 1 / math.sqrt(16)
        o, lse = fwd(q, k, v, sc, causal)
        np.testing.assert_allclose(o, torch_sdpa(q, k, v, sc, causal), rtol=1e-11, atol=1e-12)
        s = sc * np.einsum("bhid,bhjd->bhij", q, k)
        if causal:
            s = np.where(np.tril(np.ones((37, 37), bool)), s, -np.inf)
        np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=-1), rtol=1e-12, atol=1e-12)


def pin_golden(fwd, bwd):
    env = {"log": math.log}
    vals = {}
    with open(os.path.join(GOLDEN, "attn_tiny_handworked.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, expr = line.split("=", 1)
            vals[key.strip()] = np.array(eval(expr, env), dtype=np.float64)
    q, k, v = (vals[n][None, None] for n in ("q", "k", "v"))
    for causal, tag in ((False, "noncausal"), (True, "causal")):
        o, lse = fwd(q, k, v, 1.0, causal)
        np.testing.assert_allclose(o[0, 0], vals[f"o_{tag}"], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(lse[0, 0], vals[f"l_{tag}"], rtol=1e-13, atol=1e-13)


def pin_closed_forms(fwd, bwd):
    n, d = 11, 8
    q, k, v = rand((1, 2, n, d), 7), rand((1, 2, n, d), 8), rand((1, 2, n, d), 9)
    # N = 1: O = V, L = S_00
    o, lse = fwd(q[:, :, :1], k[:, :, :1], v[:, :, :1], 0.3, False)
    np.testing.assert_allclose(o, v[:, :, :1], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, 0.3 * np.sum(q[:, :, :1] * k[:, :, :1], -1), rtol=1e-13, atol=1e-13)
    # scale = 0: O = mean(V), L = ln N; causal: prefix means, L_i = ln(i + 1)
    o, lse = fwd(q, k, v, 0.0, False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(2, keepdims=True), o.shape), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.full(lse.shape, math.log(n)), rtol=1e-13)
    o, lse = fwd(q, k, v, 0.0, True)
    prefix = np.cumsum(v, axis=2) / np.arange(1, n + 1)[None, None, :, None]
    np.testing.assert_allclose(o, prefix, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, n + 1)), lse.shape), rtol=1e-13)
    # identical keys: every score of a row equal -> mean of V (causal: prefix mean)
    k_same = np.broadcast_to(k[:, :, :1], k.shape).copy()
    o, _ = fwd(q, k_same, v, 0.5, False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(2, keepdims=True), o.shape), rtol=1e-12, atol=1e-13)
    o, _ = fwd(q, k_same, v, 0.5, True)
    np.testing.assert_allclose(o, prefix, rtol=1e-12, atol=1e-13)
    # causal row 0 sees only key 0
    o, lse = fwd(q, k, v, 0.9, True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, 0], 0.9 * np.sum(q[:, :, 0] * k[:, :, 0], -1), rtol=1e-13, atol=1e-13)


def pin_invariances(fwd, bwd):
    n, d = 13, 6
    q, k, v = rand((1, 1, n, d), 11), rand((1, 1, n, d), 12), rand((1, 1, n, d), 13)
    sc = 0.4
    o, lse = fwd(q, k, v, sc, False)
    # permuting K and V together leaves the non-causal output unchanged
    perm = np.random.default_rng(5).permutation(n)
    o2, lse2 = fwd(q, k[:, :, perm], v[:, :, perm], sc, False)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12, atol=1e-13)
    # softmax shift invariance: K <- K + 1 u^T shifts every score of row i by scale * q_i . u
    u = rand((d,), 14)
    for causal in (False, True):
        o, lse = fwd(q, k, v, sc, causal)
        o3, lse3 = fwd(q, k + u[None, None, None, :], v, sc, causal)
        np.testing.assert_allclose(o3, o, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse3, lse + sc * (q @ u), rtol=1e-11, atol=1e-12)
    # large magnitudes (Q x 30) stay finite and agree with torch
    qb = q * 30.0
    for causal in (False, True):
        o, lse = fwd(qb, k, v, sc, causal)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
        np.testing.assert_allclose(o, torch_sdpa(qb, k, v, sc, causal), rtol=1e-10, atol=1e-11)


def pin_rows_sum_to_one(fwd, bwd):
    q, k, v = rand((1, 1, 9, 5), 21), rand((1, 1, 9, 5), 22), rand((1, 1, 9, 5), 23)
    for causal in (False, True):
        # with V = identity-like one-hot columns O recovers P; rows of P sum to 1
        eye = np.eye(9)[None, None]
        p, lse = fwd(q, k, eye, 0.8, causal)
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-13)
        assert np.all(p >= 0)
        if causal:
            assert np.all(np.triu(p[0, 0], 1) == 0)
        # P = exp(S - L): the logsumexp reproduces the probabilities
        s = 0.8 * q[0, 0] @ k[0, 0].T
        if causal:
            s = np.where(np.tril(np.ones((9, 9), bool)), s, -np.inf)
        np.testing.assert_allclose(np.exp(s - lse[0, 0][:, None]), p[0, 0], rtol=1e-12, atol=1e-14)


def pin_backward(fwd, bwd):
    # torch fp64 autograd
    for causal in (False, True):
        shp = (2, 2, 19, 8)
        q, k, v, do = (rand(shp, s) for s in (31, 32, 33, 34))
        r = bwd(q, k, v, do, 0.35, causal)
        gq, gk, gv = torch_grads(q, k, v, do, 0.35, causal)
        np.testing.assert_allclose(r.dq, gq, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(r.dk, gk, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(r.dv, gv, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(r.delta_from_p, r.delta_from_o, rtol=1e-11, atol=1e-12)
    # central finite differences of sum(O * dO) through the oracle's own forward
    for causal in (False, True):
        shp = (1, 1, 6, 3)
        q, k, v, do = (rand(shp, s) for s in (41, 42, 43, 44))
        sc = 0.6
        r = bwd(q, k, v, do, sc, causal)

        def loss(qq, kk, vv):
            return float(np.sum(fwd(qq, kk, vv, sc, causal)[0] * do))

        h = 1e-6
        for name, grad in (("q", r.dq), ("k", r.dk), ("v", r.dv)):
            num = np.zeros(shp)
            for idx in np.ndindex(*shp):
                args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
                args[name][idx] += h
                lp = loss(args["q"], args["k"], args["v"])
                args[name][idx] -= 2 * h
                lm = loss(args["q"], args["k"], args["v"])
                num[idx] = (lp - lm) / (2 * h)
            err = np.max(np.abs(num - grad)) / max(np.max(np.abs(grad)), 1e-30)
            assert err <= 1e-6, (name, err)


PINS = [pin_brute_force, pin_torch_sdpa, pin_golden, pin_closed_forms, pin_invariances,
        pin_rows_sum_to_one, pin_backward]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.attn_fwd_ref, oracle.attn_bwd_ref)


# ---------------------------------------------------------------------------
# the online recurrence, the algorithm the kernel follows

def test_online_softmax_matches_two_pass():
    rng = np.random.default_rng(3)
    for trial in range(40):
        n = int(rng.integers(1, 300))
        x = rng.standard_normal(n) * float(rng.choice([0.1, 1.0, 10.0, 80.0]))
        if trial % 5 == 0:
            x[rng.random(n) < 0.3] = -np.inf
            x[0] = 0.0
        cuts = np.sort(rng.choice(np.arange(1, n), size=min(n - 1, int(rng.integers(0, 8))), replace=False)) if n > 1 else []
        sizes = np.diff(np.concatenate([[0], cuts, [n]])).astype(int).tolist()
        m, ell, p = oracle.online_softmax_ref(x, sizes)
        np.testing.assert_allclose(p, scipy.special.softmax(x), rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(m + math.log(ell), scipy.special.logsumexp(x), rtol=1e-12, atol=1e-12)
        assert m == np.max(x)


def test_online_attention_matches_definition():
    rng = np.random.default_rng(4)
    for causal in (False, True):
        for n, sizes in ((7, [7]), (20, [3, 5, 12]), (33, [16, 16, 1]), (40, [1] * 40)):
            q, k, v = (rng.standard_normal((n, 8)) for _ in range(3))
            o, lse = oracle.attn_fwd_online_ref(q, k, v, 0.5, causal, sizes)
            o_ref, l_ref = oracle.attn_fwd_ref(q[None, None], k[None, None], v[None, None], 0.5, causal)
            np.testing.assert_allclose(o, o_ref[0, 0], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse, l_ref[0, 0], rtol=1e-12, atol=1e-13)


def test_conditional_rescale_is_exact_and_bounded():
    """The reading of the conditional rescale (the running max kept until a
    block's max exceeds it by more than tau, log2 units; the stale max used
    for p, l, o and L alike): O and L equal the two-pass definition for
    tau = 0, 8 and 20 to fp64 rounding, p never exceeds 2^tau, and a larger
    tau moves the max less often on scores that grow along the key axis."""
    rng = np.random.default_rng(21)
    n, d = 160, 8
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    q[:, 0] = np.abs(q[:, 0]) + 1.0
    k[:, 0] += np.linspace(0.0, 12.0, n)          # scores grow with the key index
    sizes = [16] * 10
    for causal in (False, True):
        o_ref, l_ref = oracle.attn_fwd_ref(q[None, None], k[None, None], v[None, None], 0.9, causal)
        moves = {}
        for tau in (0.0, 8.0, 20.0):
            st = {}
            o, lse = oracle.attn_fwd_online_ref(q, k, v, 0.9, causal, sizes, tau_log2=tau, stats=st)
            np.testing.assert_allclose(o, o_ref[0, 0], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(lse, l_ref[0, 0], rtol=1e-12, atol=1e-12)
            assert st["p_max"] <= 2.0 ** tau * (1 + 1e-12)
            moves[tau] = st["rescales"]
        assert moves[8.0] < moves[0.0] and moves[20.0] <= moves[8.0]
        assert moves[20.0] >= n                   # every row sets its max at least once


def test_accepts_bf16_torch_exactly():
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(1, 1, 5, 4, generator=g).to(torch.bfloat16) for _ in range(3))
    o, _ = oracle.attn_fwd_ref(q, k, v, 0.5, False)
    o2, _ = oracle.attn_fwd_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), 0.5, False)
    assert np.array_equal(o, o2)


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin

def _mut_fwd(kind):
    def fwd(q, k, v, scale, causal):
        q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
        B, H, N, _ = q.shape
        o = np.zeros(q.shape[:3] + (v.shape[-1],))
        lse = np.zeros((B, H, N))
        for b in range(B):
            for h in range(H):
                sc = 1.0 if kind == "no_scale" else scale
                s = sc * (q[b, h] @ k[b, h].T)
                if kind == "transposed":
                    s = s.T
                if causal:
                    mask = ar.causal_mask(N, N)
                    if kind == "mask_off_by_one":
                        mask = np.tril(np.ones((N, N), bool), -1)   # j < i
                    if kind == "mask_upper":
                        mask = mask.T
                    s = np.where(mask, s, -np.inf)
                m = s.max(1)
                e = np.exp(s - m[:, None])
                ell = e.sum(1)
                if kind == "no_normalise":
                    ell = np.ones_like(ell)
                o[b, h] = (e / ell[:, None]) @ v[b, h]
                lse[b, h] = (np.log(ell) if kind == "lse_no_max" else m + np.log(ell))
        return o, lse
    return fwd


def _mut_bwd(kind):
    def bwd(q, k, v, do, scale, causal):
        r = oracle.attn_bwd_ref(q, k, v, do, scale, causal)
        if kind == "dk_no_scale":
            return r._replace(dk=r.dk / scale)
        if kind == "ds_sign":
            # dS = P * (dP + D): recompute with the sign flipped
            q_, k_, v_, do_ = (np.asarray(x, np.float64) for x in (q, k, v, do))
            dq = np.zeros_like(q_)
            for b in range(q_.shape[0]):
                for h in range(q_.shape[1]):
                    s = ar.scores_ref(q_[b, h], k_[b, h], scale, causal)
                    p = ar.softmax_ref(s)
                    dp = do_[b, h] @ v_[b, h].T
                    ds = p * (dp + np.sum(p * dp, 1, keepdims=True))
                    dq[b, h] = scale * ds @ k_[b, h]
            return r._replace(dq=dq)
        if kind == "dv_untransposed":
            q_, k_, v_, do_ = (np.asarray(x, np.float64) for x in (q, k, v, do))
            dv = np.zeros_like(v_)
            for b in range(q_.shape[0]):
                for h in range(q_.shape[1]):
                    p = ar.softmax_ref(ar.scores_ref(q_[b, h], k_[b, h], scale, causal))
                    dv[b, h] = p @ do_[b, h]
            return r._replace(dv=dv)
        return r
    return bwd


FWD_MUTANTS = ["no_scale", "transposed", "mask_off_by_one", "mask_upper", "no_normalise", "lse_no_max"]
BWD_MUTANTS = ["dk_no_scale", "ds_sign", "dv_untransposed"]


@pytest.mark.parametrize("kind", FWD_MUTANTS + BWD_MUTANTS)
def test_planted_mistakes(kind):
    fwd = _mut_fwd(kind) if kind in FWD_MUTANTS else oracle.attn_fwd_ref
    bwd = _mut_bwd(kind) if kind in BWD_MUTANTS else oracle.attn_bwd_ref
    caught = []
    for pin in PINS:
        try:
            pin(fwd, bwd)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {kind!r} passed every pin"


def test_rows_oracle_matches_full_definition():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((1, 1, 50, 8)) for _ in range(3))
    rows = [0, 1, 17, 49]
    for causal in (False, True):
        o, lse = oracle.attn_fwd_ref(q, k, v, 0.6, causal)
        o_r, l_r = oracle.attn_fwd_rows_ref(q[0, 0], k[0, 0], v[0, 0], 0.6, causal, rows)
        np.testing.assert_allclose(o_r, o[0, 0, rows], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(l_r, lse[0, 0, rows], rtol=1e-12, atol=1e-13)
        ob = [brute_fwd(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), 0.6, causal)]
        np.testing.assert_allclose(o_r, ob[0][0][rows], rtol=1e-12, atol=1e-12)
