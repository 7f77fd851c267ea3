"""Checks that pin the fp64 oracle to facts outside itself.

Each ``pin_*`` function takes a loaded oracle build (``oracle.OracleLib``) and
raises ``AssertionError`` when the build disagrees with what the pages and the
mathematics fix:

* closed forms of the logistic function and its derivative (gist.science
  summary, section 2.A; paper.rainbus.top summary, core method: sigma' =
  sigma (1 - sigma) <= 1/4);
* the hand-worked examples in ``tests/golden/worked_examples.json``;
* special cases that reduce to library routines (torch fp64 matmul/sigmoid and
  torch autograd on tiny inputs);
* closed-form special cases (alpha = 0, a single valid key);
* invariants (padding never changes results, padded rows are zero, linearity in
  V, permutation equivariance, the two bilinearity identities of the gradients);
* central finite differences of the oracle's own (pinned) forward;
* a per-sample bias (paperlayer.ai summary, section 3: b = -log(n)) and its
  gradient db against torch autograd, the alpha = 0 closed form and a finite
  difference;
* rectangular problems (a query slice against all keys, Lq != Lk) against
  torch autograd and against the square problem they embed in.

``tests/test_oracle_pins.py`` runs them on the real oracle and
``tests/test_oracle_mutants.py`` shows that builds with one plausible mistake
planted each fail at least one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "worked_examples.json")


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return (g.standard_normal(shape) * scale).astype(np.float32)


def _case(seed, Z=2, L=7, H=2, D=4, nq=(7, 4), nk=(5, 7), scale=1.0):
    q = _rand((Z, L, H, D), seed, scale)
    k = _rand((Z, L, H, D), seed + 1, scale)
    v = _rand((Z, L, H, D), seed + 2)
    do = _rand((Z, L, H, D), seed + 3)
    return q, k, v, do, np.asarray(nq, np.int32), np.asarray(nk, np.int32)


def _close(a, b, rtol, atol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    err = np.abs(a - b)
    tol = atol + rtol * np.abs(b)
    if not np.all(err <= tol):
        idx = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: max violation at {idx}: got {a[idx]!r}, want {b[idx]!r}")


def _sigma_tanh(x: float) -> float:
    """sigma through the tanh identity sigma(x) = (tanh(x/2) + 1) / 2, the form the
    kernel pages evaluate (paper.rainbus.top summary, method step (3))."""
    return 0.5 * (math.tanh(0.5 * x) + 1.0)


# ---------------------------------------------------------------- sigma


def pin_sigmoid_closed_forms(orc):
    xs = list(np.linspace(-40.0, 40.0, 801)) + [0.0, math.log(3.0), -math.log(3.0)]
    for x in xs:
        s = orc.sigmoid(x)
        if abs(s - _sigma_tanh(x)) > 4.5e-16:
            raise AssertionError(f"sigma({x}) = {s} disagrees with the tanh identity")
        if abs(s + orc.sigmoid(-x) - 1.0) > 4.5e-16:
            raise AssertionError(f"sigma({x}) + sigma({-x}) != 1")
    if orc.sigmoid(0.0) != 0.5:
        raise AssertionError("sigma(0) != 1/2")
    if abs(orc.sigmoid(math.log(3.0)) - 0.75) > 1e-16 or abs(orc.sigmoid(-math.log(3.0)) - 0.25) > 1e-16:
        raise AssertionError("sigma(+-ln 3) != 3/4, 1/4")
    # far tail: sigma(x) ~ e^x, relative accuracy is kept (no cancellation)
    for x in (-50.0, -300.0, -700.0):
        if abs(orc.sigmoid(x) / math.exp(x) - 1.0) > 1e-12:
            raise AssertionError(f"sigma({x}) lost relative accuracy in the tail")


def pin_sigmoid_derivative(orc):
    best = 0.0
    for x in np.linspace(-30.0, 30.0, 601):
        g = orc.sigmoid_grad(x)
        if g > 0.25 + 1e-17 or g < 0.0:
            raise AssertionError(f"sigma'({x}) = {g} outside [0, 1/4]")
        # closed form through tanh: sigma' = (1 - tanh^2(x/2)) / 4
        t = math.tanh(0.5 * x)
        if abs(g - 0.25 * (1.0 - t * t)) > 4.5e-16:
            raise AssertionError(f"sigma'({x}) disagrees with (1 - tanh^2(x/2))/4")
        h = 1e-5
        fd = (orc.sigmoid(x + h) - orc.sigmoid(x - h)) / (2 * h)
        if abs(fd - g) > 1e-9:
            raise AssertionError(f"sigma'({x}) disagrees with the finite difference of sigma")
        best = max(best, g)
    if orc.sigmoid_grad(0.0) != 0.25:
        raise AssertionError("sigma'(0) != 1/4 (the bound is attained at 0)")


# ---------------------------------------------------------------- golden


def pin_golden_examples(orc):
    with open(GOLDEN) as f:
        data = json.load(f)
    ln3 = math.log(3.0)
    for ex in data["examples"]:
        L, D = ex["L"], ex["D"]
        shp = (1, L, 1, D)
        q = np.asarray(ex["q"], np.float32).reshape(shp)
        k = np.asarray(ex["k"], np.float32).reshape(shp)
        v = np.asarray(ex["v"], np.float32).reshape(shp)
        do = np.asarray(ex["dout"], np.float32).reshape(shp)
        bias = ex["bias_over_ln3"] * ln3 if "bias_over_ln3" in ex else ex["bias"]
        nq, nk = [ex["n_q"]], [ex["n_k"]]
        o = orc.fwd(q, k, v, nq, nk, ln3, bias)
        dq, dk, dv = orc.bwd(q, k, v, do, nq, nk, ln3, bias)
        _close(o.reshape(L, D), ex["o"], 1e-13, 1e-13, ex["name"] + " O")
        _close(dq.reshape(L, D), np.asarray(ex["dq_over_ln3"]) * ln3, 1e-13, 1e-13, ex["name"] + " dQ")
        _close(dk.reshape(L, D), np.asarray(ex["dk_over_ln3"]) * ln3, 1e-13, 1e-13, ex["name"] + " dK")
        _close(dv.reshape(L, D), ex["dv"], 1e-13, 1e-13, ex["name"] + " dV")


# ---------------------------------------------------------------- library routes


def _torch_forward(q, k, v, nq, nk, alpha, bias):
    """torch fp64 route: per (z, h) slice the valid rows and use matmul + sigmoid."""
    Z, L, H, D = q.shape
    out = torch.zeros((Z, L, H, D), dtype=torch.float64)
    for z in range(Z):
        for h in range(H):
            Q = torch.from_numpy(q[z, : nq[z], h].astype(np.float64))
            K = torch.from_numpy(k[z, : nk[z], h].astype(np.float64))
            V = torch.from_numpy(v[z, : nk[z], h].astype(np.float64))
            out[z, : nq[z], h] = torch.sigmoid(alpha * Q @ K.T + bias) @ V
    return out.numpy()


def pin_forward_library_route(orc):
    for seed, kw in [(10, {}), (20, dict(Z=1, L=9, H=3, D=5, nq=(9,), nk=(9,))),
                     (30, dict(Z=3, L=6, H=1, D=2, nq=(0, 6, 3), nk=(6, 1, 2))),
                     (40, dict(Z=2, L=5, H=2, D=3, nq=(5, 2), nk=(3, 5), scale=4.0))]:
        q, k, v, do, nq, nk = _case(seed, **kw)
        alpha, bias = 0.37, -1.3
        got = orc.fwd(q, k, v, nq, nk, alpha, bias)
        want = _torch_forward(q, k, v, nq, nk, alpha, bias)
        _close(got, want, 1e-12, 1e-13, f"forward vs torch fp64 (seed {seed})")


def pin_backward_autograd_route(orc):
    for seed, kw in [(50, {}), (60, dict(Z=1, L=6, H=2, D=3, nq=(4,), nk=(6,))),
                     (70, dict(Z=2, L=5, H=1, D=4, nq=(5, 0), nk=(2, 5), scale=3.0))]:
        q, k, v, do, nq, nk = _case(seed, **kw)
        alpha, bias = 0.41, -0.8
        Z, L, H, D = q.shape
        tq, tk, tv = (torch.tensor(a.astype(np.float64), requires_grad=True) for a in (q, k, v))
        tdo = torch.from_numpy(do.astype(np.float64))
        kmask = torch.zeros((Z, L), dtype=torch.float64)
        qmask = torch.zeros((Z, L), dtype=torch.float64)
        for z in range(Z):
            kmask[z, : nk[z]] = 1.0
            qmask[z, : nq[z]] = 1.0
        # [Z, H, L, L] scores; padded keys weigh 0, padded query rows are zeroed
        s = alpha * torch.einsum("zihd,zjhd->zhij", tq, tk) + bias
        p = torch.sigmoid(s) * kmask[:, None, None, :]
        o = torch.einsum("zhij,zjhd->zihd", p, tv) * qmask[:, :, None, None]
        (o * tdo).sum().backward()
        dq, dk, dv = orc.bwd(q, k, v, do, nq, nk, alpha, bias)
        _close(orc.fwd(q, k, v, nq, nk, alpha, bias), o.detach().numpy(), 1e-12, 1e-13,
               f"forward vs autograd graph (seed {seed})")
        _close(dq, tq.grad.numpy(), 1e-11, 1e-12, f"dQ vs torch autograd (seed {seed})")
        _close(dk, tk.grad.numpy(), 1e-11, 1e-12, f"dK vs torch autograd (seed {seed})")
        _close(dv, tv.grad.numpy(), 1e-11, 1e-12, f"dV vs torch autograd (seed {seed})")


# ---------------------------------------------------------------- closed-form cases


def pin_alpha_zero(orc):
    q, k, v, do, nq, nk = _case(80)
    bias = -0.9
    o = orc.fwd(q, k, v, nq, nk, 0.0, bias)
    dq, dk, dv = orc.bwd(q, k, v, do, nq, nk, 0.0, bias)
    s = _sigma_tanh(bias)
    Z, L, H, D = q.shape
    for z in range(Z):
        vsum = v[z, : nk[z]].astype(np.float64).sum(axis=0)       # [H, D]
        dosum = do[z, : nq[z]].astype(np.float64).sum(axis=0)     # [H, D]
        for i in range(L):
            want = s * vsum if i < nq[z] else np.zeros_like(vsum)
            _close(o[z, i], want, 1e-13, 1e-13, "alpha=0: O_i = sigma(b) sum_j V_j")
        for j in range(L):
            want = s * dosum if j < nk[z] else np.zeros_like(dosum)
            _close(dv[z, j], want, 1e-13, 1e-13, "alpha=0: dV_j = sigma(b) sum_i dO_i")
    _close(dq, np.zeros_like(dq), 0, 0, "alpha=0: dQ = 0")
    _close(dk, np.zeros_like(dk), 0, 0, "alpha=0: dK = 0")


def pin_single_valid_key(orc):
    q, k, v, do, nq, nk = _case(90, Z=1, L=6, H=2, D=3, nq=(6,), nk=(1,))
    alpha, bias = 0.7, 0.2
    o = orc.fwd(q, k, v, nq, nk, alpha, bias)
    for h in range(2):
        for i in range(6):
            x = alpha * float(np.dot(q[0, i, h].astype(np.float64), k[0, 0, h].astype(np.float64))) + bias
            _close(o[0, i, h], _sigma_tanh(x) * v[0, 0, h].astype(np.float64), 1e-13, 1e-14,
                   "one valid key: O_i = sigma(x_i0) V_0")


# ---------------------------------------------------------------- invariants


def pin_padding_invariance(orc):
    q, k, v, do, nq, nk = _case(100, Z=2, L=8, H=2, D=3, nq=(5, 8), nk=(6, 3))
    alpha, bias = 0.5, -1.0
    base = (orc.fwd(q, k, v, nq, nk, alpha, bias),) + orc.bwd(q, k, v, do, nq, nk, alpha, bias)
    g = np.random.default_rng(7)
    q2, k2, v2, do2 = q.copy(), k.copy(), v.copy(), do.copy()
    for z in range(2):
        q2[z, nq[z]:] = g.uniform(-1e3, 1e3, q2[z, nq[z]:].shape)
        do2[z, nq[z]:] = g.uniform(-1e3, 1e3, do2[z, nq[z]:].shape)
        k2[z, nk[z]:] = g.uniform(-1e3, 1e3, k2[z, nk[z]:].shape)
        v2[z, nk[z]:] = g.uniform(-1e3, 1e3, v2[z, nk[z]:].shape)
    new = (orc.fwd(q2, k2, v2, nq, nk, alpha, bias),) + orc.bwd(q2, k2, v2, do2, nq, nk, alpha, bias)
    for name, a, b in zip(("O", "dQ", "dK", "dV"), base, new):
        _close(b, a, 0, 0, f"padding contents changed {name}")
    o, dq, dk, dv = base
    for z in range(2):
        for name, t, n in (("O", o, nq[z]), ("dQ", dq, nq[z]), ("dK", dk, nk[z]), ("dV", dv, nk[z])):
            if np.any(t[z, n:] != 0.0):
                raise AssertionError(f"padded rows of {name} are not exactly zero")


def pin_linearity_in_v(orc):
    q, k, v, do, nq, nk = _case(110)
    # values on a 1/64 grid so that 2 V - 3 V2 is exact in fp32
    v = (np.round(v * 64.0) / 64.0).astype(np.float32)
    v2 = (np.round(_rand(v.shape, 111) * 64.0) / 64.0).astype(np.float32)
    alpha, bias = 0.6, -0.4
    o1 = orc.fwd(q, k, v, nq, nk, alpha, bias)
    o2 = orc.fwd(q, k, v2, nq, nk, alpha, bias)
    o3 = orc.fwd(q, k, (2.0 * v - 3.0 * v2).astype(np.float32), nq, nk, alpha, bias)
    _close(o3, 2.0 * o1 - 3.0 * o2, 1e-12, 1e-12, "O is linear in V")


def pin_permutation_equivariance(orc):
    q, k, v, do, nq, nk = _case(120, Z=1, L=7, H=2, D=3, nq=(7,), nk=(6,))
    alpha, bias = 0.8, -0.3
    o = orc.fwd(q, k, v, nq, nk, alpha, bias)
    perm = np.random.default_rng(3).permutation(6)
    k2, v2 = k.copy(), v.copy()
    k2[0, :6] = k[0, perm]
    v2[0, :6] = v[0, perm]
    _close(orc.fwd(q, k2, v2, nq, nk, alpha, bias), o, 1e-13, 1e-14,
           "O invariant under a joint permutation of valid keys")
    qperm = np.random.default_rng(4).permutation(7)
    q3 = q[:, qperm].copy()
    _close(orc.fwd(q3, k, v, nq, nk, alpha, bias), o[:, qperm], 1e-13, 1e-14,
           "O equivariant under a permutation of query rows")


def pin_gradient_identities(orc):
    q, k, v, do, nq, nk = _case(130, scale=2.0)
    alpha, bias = 0.45, -1.1
    o = orc.fwd(q, k, v, nq, nk, alpha, bias)
    dq, dk, dv = orc.bwd(q, k, v, do, nq, nk, alpha, bias)
    f64 = lambda a: a.astype(np.float64)
    lhs, rhs = np.sum(f64(do) * o), np.sum(dv * f64(v))
    # <dO, O> = <dV, V>: O is linear in V (padded dO rows do not contribute to O)
    mask_q = np.zeros(q.shape[:2], bool)
    for z in range(q.shape[0]):
        mask_q[z, : nq[z]] = True
    lhs = np.sum((f64(do) * o)[mask_q])
    if abs(lhs - rhs) > 1e-11 * max(1.0, abs(lhs)):
        raise AssertionError(f"<dO,O> = {lhs} != <dV,V> = {rhs}")
    # <dQ, Q> = <dK, K>: the scores are bilinear in Q and K
    a, b = np.sum(dq * f64(q)), np.sum(dk * f64(k))
    if abs(a - b) > 1e-11 * max(1.0, abs(a)):
        raise AssertionError(f"<dQ,Q> = {a} != <dK,K> = {b}")


def pin_finite_differences(orc):
    q, k, v, do, nq, nk = _case(140, Z=1, L=5, H=2, D=3, nq=(4,), nk=(3,))
    alpha, bias = 0.9, -0.6
    dq, dk, dv = orc.bwd(q, k, v, do, nq, nk, alpha, bias)
    do64 = do.astype(np.float64)

    def loss(qq, kk, vv):
        return float(np.sum(orc.fwd(qq, kk, vv, nq, nk, alpha, bias) * do64))

    h = np.float32(2.0 ** -10)
    for name, grad, which in (("dQ", dq, 0), ("dK", dk, 1), ("dV", dv, 2)):
        for idx in np.ndindex(q.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            step = float(args_p[which][idx]) - float(args_m[which][idx])
            fd = (loss(*args_p) - loss(*args_m)) / step
            if abs(fd - grad[idx]) > 1e-6 * max(1.0, abs(grad[idx])):
                raise AssertionError(f"{name}{idx}: oracle {grad[idx]} vs finite difference {fd}")


def pin_bf16_widening_and_rows(orc):
    # values exactly representable in bf16: the bf16 and fp32 routes must agree bit for bit
    q, k, v, do, nq, nk = _case(150)
    tq, tk, tv, tdo = (torch.from_numpy(a).to(torch.bfloat16) for a in (q, k, v, do))
    fq, fk, fv, fdo = (t.float().numpy() for t in (tq, tk, tv, tdo))
    alpha, bias = 0.3, -0.5
    a = orc.fwd(tq, tk, tv, nq, nk, alpha, bias)
    b = orc.fwd(fq, fk, fv, nq, nk, alpha, bias)
    _close(a, b, 0, 0, "bf16 inputs widen exactly")
    ga = orc.bwd(tq, tk, tv, tdo, nq, nk, alpha, bias)
    gb = orc.bwd(fq, fk, fv, fdo, nq, nk, alpha, bias)
    for x, y in zip(ga, gb):
        _close(x, y, 0, 0, "bf16 gradients widen exactly")
    # a scattered row subset returns the same rows as the full evaluation
    Z, L, H, D = q.shape
    items = np.array([[1, 1, 3], [0, 0, 6], [1, 0, 0], [0, 1, 2]], np.int64)
    rows = orc.fwd_rows(fq, fk, fv, nq, nk, alpha, bias, items)
    for t, (z, h, i) in enumerate(items):
        _close(rows[t], b[z, i, h], 0, 0, "row subset indexing")


# ---------------------------------------------------------------- per-sample bias, db


def pin_per_sample_bias_autograd(orc):
    """Per-sample bias b_z (paperlayer.ai summary, section 3: b = -log(n) per
    sequence) and its gradient db_z = sum dS, against torch fp64 autograd with b
    as a leaf tensor."""
    for seed, kw in [(160, {}), (170, dict(Z=3, L=6, H=2, D=3, nq=(6, 0, 3), nk=(4, 6, 6))),
                     (180, dict(Z=2, L=5, H=3, D=4, nq=(5, 2), nk=(2, 5), scale=3.0))]:
        q, k, v, do, nq, nk = _case(seed, **kw)
        Z, L, H, D = q.shape
        alpha = 0.45
        bz = -np.log(np.maximum(nk, 1).astype(np.float64)) + 0.1 * np.arange(Z)
        tq, tk, tv = (torch.tensor(a.astype(np.float64), requires_grad=True) for a in (q, k, v))
        tb = torch.tensor(bz, requires_grad=True)
        tdo = torch.from_numpy(do.astype(np.float64))
        kmask = torch.zeros((Z, L), dtype=torch.float64)
        qmask = torch.zeros((Z, L), dtype=torch.float64)
        for z in range(Z):
            kmask[z, : nk[z]] = 1.0
            qmask[z, : nq[z]] = 1.0
        s = alpha * torch.einsum("zihd,zjhd->zhij", tq, tk) + tb[:, None, None, None]
        p = torch.sigmoid(s) * kmask[:, None, None, :]
        o = torch.einsum("zhij,zjhd->zihd", p, tv) * qmask[:, :, None, None]
        (o * tdo).sum().backward()
        _close(orc.fwd(q, k, v, nq, nk, alpha, bz), o.detach().numpy(), 1e-12, 1e-13,
               f"forward with per-sample bias vs torch (seed {seed})")
        dq, dk, dv = orc.bwd(q, k, v, do, nq, nk, alpha, bz)
        _close(dq, tq.grad.numpy(), 1e-11, 1e-12, f"dQ with per-sample bias (seed {seed})")
        _close(dk, tk.grad.numpy(), 1e-11, 1e-12, f"dK with per-sample bias (seed {seed})")
        _close(dv, tv.grad.numpy(), 1e-11, 1e-12, f"dV with per-sample bias (seed {seed})")
        _close(orc.dbias(q, k, v, do, nq, nk, alpha, bz), tb.grad.numpy(), 1e-11, 1e-12,
               f"db vs torch autograd (seed {seed})")


def pin_per_sample_bias_slices(orc):
    """A per-sample bias equals running each sample alone with its scalar bias."""
    q, k, v, do, nq, nk = _case(190, Z=3, L=6, H=2, D=3, nq=(6, 3, 1), nk=(5, 6, 2))
    alpha, bz = 0.6, np.array([-1.2, 0.4, -2.5])
    o = orc.fwd(q, k, v, nq, nk, alpha, bz)
    g = orc.bwd(q, k, v, do, nq, nk, alpha, bz)
    db = orc.dbias(q, k, v, do, nq, nk, alpha, bz)
    for z in range(3):
        sl = slice(z, z + 1)
        args = (q[sl], k[sl], v[sl])
        lens = (nq[sl], nk[sl], alpha, float(bz[z]))
        _close(o[sl], orc.fwd(*args, *lens), 0, 0, "per-sample bias: forward slice")
        for x, y in zip(g, orc.bwd(*args, do[sl], *lens)):
            _close(x[sl], y, 0, 0, "per-sample bias: gradient slice")
        _close(db[z], orc.dbias(*args, do[sl], *lens)[0], 0, 0, "per-sample bias: db slice")


def pin_dbias_alpha_zero(orc):
    """alpha = 0: every valid score is b_z, so dS_ij = sigma'(b_z) dO_i.V_j and
    db_z = sigma'(b_z) sum_h (sum_{i<n_q} dO_i) . (sum_{j<n_k} V_j)."""
    q, k, v, do, nq, nk = _case(200, Z=2, L=7, H=3, D=4, nq=(7, 3), nk=(2, 7))
    bz = np.array([-0.7, 1.1])
    db = orc.dbias(q, k, v, do, nq, nk, 0.0, bz)
    for z in range(2):
        s = _sigma_tanh(bz[z])
        dosum = do[z, : nq[z]].astype(np.float64).sum(axis=0)   # [H, D]
        vsum = v[z, : nk[z]].astype(np.float64).sum(axis=0)     # [H, D]
        _close(db[z], s * (1 - s) * float(np.sum(dosum * vsum)), 1e-12, 1e-13,
               "alpha=0: db closed form")


def pin_dbias_finite_difference(orc):
    """db_z against a central difference of sum(O * dO) in b_z."""
    q, k, v, do, nq, nk = _case(210, Z=2, L=6, H=2, D=3, nq=(5, 6), nk=(6, 3))
    alpha, bz = 0.8, np.array([-1.5, -0.4])
    db = orc.dbias(q, k, v, do, nq, nk, alpha, bz)
    do64 = do.astype(np.float64)
    h = 2.0 ** -12
    for z in range(2):
        bp, bm = bz.copy(), bz.copy()
        bp[z] += h
        bm[z] -= h
        fd = (np.sum(orc.fwd(q, k, v, nq, nk, alpha, bp) * do64) -
              np.sum(orc.fwd(q, k, v, nq, nk, alpha, bm) * do64)) / (2 * h)
        if abs(fd - db[z]) > 1e-7 * max(1.0, abs(db[z])):
            raise AssertionError(f"db[{z}]: oracle {db[z]} vs finite difference {fd}")


# ---------------------------------------------------------------- rectangular (Lq != Lk)


def _rect_case(seed, Z=2, Lq=4, Lk=7, H=2, D=3, nq=(4, 2), nk=(7, 5), scale=1.0):
    q = _rand((Z, Lq, H, D), seed, scale)
    k = _rand((Z, Lk, H, D), seed + 1, scale)
    v = _rand((Z, Lk, H, D), seed + 2)
    do = _rand((Z, Lq, H, D), seed + 3)
    return q, k, v, do, np.asarray(nq, np.int32), np.asarray(nk, np.int32)


def pin_rectangular_autograd(orc):
    """A query slice of length Lq against Lk keys (the context-parallel shape)
    against torch fp64 autograd with the same masks."""
    for seed, kw in [(220, {}), (230, dict(Z=1, Lq=6, Lk=3, H=3, D=4, nq=(5,), nk=(3,))),
                     (240, dict(Z=3, Lq=2, Lk=9, H=1, D=2, nq=(2, 0, 1), nk=(9, 4, 0)))]:
        q, k, v, do, nq, nk = _rect_case(seed, **kw)
        Z, Lq, H, D = q.shape
        Lk = k.shape[1]
        alpha, bias = 0.52, -0.9
        tq, tk, tv = (torch.tensor(a.astype(np.float64), requires_grad=True) for a in (q, k, v))
        tdo = torch.from_numpy(do.astype(np.float64))
        kmask = torch.zeros((Z, Lk), dtype=torch.float64)
        qmask = torch.zeros((Z, Lq), dtype=torch.float64)
        for z in range(Z):
            kmask[z, : nk[z]] = 1.0
            qmask[z, : nq[z]] = 1.0
        sc = alpha * torch.einsum("zihd,zjhd->zhij", tq, tk) + bias
        pr = torch.sigmoid(sc) * kmask[:, None, None, :]
        o = torch.einsum("zhij,zjhd->zihd", pr, tv) * qmask[:, :, None, None]
        (o * tdo).sum().backward()
        _close(orc.fwd(q, k, v, nq, nk, alpha, bias), o.detach().numpy(), 1e-12, 1e-13,
               f"rectangular forward vs torch (seed {seed})")
        dq, dk, dv = orc.bwd(q, k, v, do, nq, nk, alpha, bias)
        _close(dq, tq.grad.numpy(), 1e-11, 1e-12, f"rectangular dQ (seed {seed})")
        _close(dk, tk.grad.numpy(), 1e-11, 1e-12, f"rectangular dK (seed {seed})")
        _close(dv, tv.grad.numpy(), 1e-11, 1e-12, f"rectangular dV (seed {seed})")


def pin_rectangular_embedding(orc):
    """A rectangular problem equals the square one whose Q and dO are padded with
    extra rows beyond n_q (they are padding, so they change nothing)."""
    q, k, v, do, nq, nk = _rect_case(250, Z=2, Lq=3, Lk=6, H=2, D=3, nq=(3, 2), nk=(6, 4))
    alpha, bias = 0.7, -0.4
    Lq, Lk = q.shape[1], k.shape[1]
    pad = lambda a: np.concatenate([a, _rand((2, Lk - Lq) + a.shape[2:], 260)], axis=1)
    qs, dos = pad(q), pad(do)
    o_r = orc.fwd(q, k, v, nq, nk, alpha, bias)
    o_s = orc.fwd(qs, k, v, nq, nk, alpha, bias)
    _close(o_r, o_s[:, :Lq], 0, 0, "rectangular O = square O rows")
    g_r = orc.bwd(q, k, v, do, nq, nk, alpha, bias)
    g_s = orc.bwd(qs, k, v, dos, nq, nk, alpha, bias)
    _close(g_r[0], g_s[0][:, :Lq], 0, 0, "rectangular dQ = square dQ rows")
    _close(g_r[1], g_s[1], 0, 0, "rectangular dK = square dK")
    _close(g_r[2], g_s[2], 0, 0, "rectangular dV = square dV")


ALL_PINS = [
    pin_sigmoid_closed_forms,
    pin_sigmoid_derivative,
    pin_golden_examples,
    pin_forward_library_route,
    pin_backward_autograd_route,
    pin_alpha_zero,
    pin_single_valid_key,
    pin_padding_invariance,
    pin_linearity_in_v,
    pin_permutation_equivariance,
    pin_gradient_identities,
    pin_finite_differences,
    pin_bf16_widening_and_rows,
    pin_per_sample_bias_autograd,
    pin_per_sample_bias_slices,
    pin_dbias_alpha_zero,
    pin_dbias_finite_difference,
    pin_rectangular_autograd,
    pin_rectangular_embedding,
]
