"""GPU parity of the per-sample bias path (sigattn_fwd_bias / sigattn_bwd_bias)
and of the bias gradient db_z = sum over heads and valid (i, j) of dS_ij,
against the fp64 oracle on the same seeded inputs.

db tolerance: each term dS_ij = sigma'(x_ij) dP_ij carries the relative error
of the kernel's sigma' (dP comes from exact bf16 products summed in fp32), so
|db - ref| <= tol * sum |dS_ij|: tol = 2e-3 for the EXP form (sigma' = u g^2,
relative error <= 7e-4) and 3e-2 for the TANH form (1 - t^2 inherits the
~1.4% relative error of tanh.approx in the left tail, design reading R1); the
fp32 path uses 1e-4."""
import math

import numpy as np
import pytest
import torch

import oracle
from padding_aware_sigmoid_b200 import workloads
from tests import _compare as C

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("padding_aware_sigmoid_b200")

DB_TOL = {"tanh": 3e-2, "exp": 2e-3, "fp32": 1e-4}


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _mode(name):
    return sa.SIGMOID_TANH if name == "tanh" else sa.SIGMOID_EXP


def _inputs(Z, L, H, D, nq, nk, seed, dtype="bf16"):
    q, k, v, do = workloads.random_tensors(Z, L, H, D, seed, dtype)
    nq = np.asarray(nq, np.int32)
    nk = np.asarray(nk, np.int32)
    # the pages' b = -log(n), per sample, plus an offset so the samples differ
    bz = (-np.log(np.maximum(nk, 1)) + 0.25 * np.arange(Z)).astype(np.float32)
    return q, k, v, do, nq, nk, bz


def _abs_ds_sum(q, k, v, do, nq, nk, alpha, bz):
    """sum |dS| per sample in fp64 (scales the db tolerance; not a reference value)."""
    Z, L, H, D = q.shape
    out = np.zeros(Z)
    for z in range(Z):
        a, b = int(nq[z]), int(nk[z])
        if a == 0 or b == 0:
            continue
        for h in range(H):
            Q = q[z, :a, h].double()
            K = k[z, :b, h].double()
            V = v[z, :b, h].double()
            dO = do[z, :a, h].double()
            P = torch.sigmoid(alpha * Q @ K.T + float(bz[z]))
            out[z] += float((P * (1 - P) * (dO @ V.T)).abs().sum())
    return out


def _run(q, k, v, do, nq, nk, alpha, bz, dev):
    g = [t.to(dev) for t in (q, k, v, do)]
    nqd = torch.as_tensor(nq, device=dev)
    nkd = torch.as_tensor(nk, device=dev)
    bd = torch.as_tensor(bz, device=dev)
    o = sa.fwd_bias(g[0], g[1], g[2], nqd, nkd, alpha, bd)
    dq, dk, dv, db = sa.bwd_bias(*g, nqd, nkd, alpha, bd)
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    return o, dq, dk, dv, db


def _check_full(q, k, v, do, nq, nk, alpha, bz, outs, dtype, tol_db):
    o, dq, dk, dv, db = outs
    ref = oracle.fwd(q, k, v, nq, nk, alpha, bz)
    rdq, rdk, rdv = oracle.bwd(q, k, v, do, nq, nk, alpha, bz)
    for name, got, want in (("O", o, ref), ("dQ", dq, rdq), ("dK", dk, rdk), ("dV", dv, rdv)):
        g = got.float().cpu().numpy()
        if np.any(want != 0):
            C.assert_close(g, want, dtype, name + " (per-sample bias)")
        else:
            assert np.all(g == 0.0)
    rdb = oracle.dbias(q, k, v, do, nq, nk, alpha, bz)
    scale = _abs_ds_sum(q, k, v, do, nq, nk, alpha, bz)
    err = np.abs(db.cpu().numpy().astype(np.float64) - rdb)
    assert np.all(err <= tol_db * scale + 1e-30), (err, scale, rdb)
    return err / np.maximum(scale, 1e-30)


SMALL = [
    # Z, L, H, D, n_q, n_k
    (2, 256, 2, 64, (256, 77), (256, 77)),
    (2, 384, 3, 128, (300, 129), (129, 384)),
    (3, 200, 2, 64, (200, 1, 0), (127, 200, 5)),
    (2, 520, 2, 128, (513, 128), (520, 255)),
]


@pytest.mark.parametrize("mode", ["tanh", "exp"])
@pytest.mark.parametrize("Z,L,H,D,nq,nk", SMALL)
def test_bias_small_full(Z, L, H, D, nq, nk, mode):
    dev = _dev()
    q, k, v, do, nq, nk, bz = _inputs(Z, L, H, D, nq, nk, seed=3000 + L + D)
    alpha = 1.0 / math.sqrt(D)
    old = sa.get_sigmoid_mode()
    sa.set_sigmoid_mode(_mode(mode))
    try:
        outs = _run(q, k, v, do, nq, nk, alpha, bz, dev)
    finally:
        sa.set_sigmoid_mode(old)
    _check_full(q, k, v, do, nq, nk, alpha, bz, outs, "bf16", DB_TOL[mode])


@pytest.mark.parametrize("Z", [12, 70])
def test_dbias_persistent_many_tiles(Z):
    """At D = 64 the backward blocks walk the tiles with work (length-ranked up to
    64 samples, index order above) and an idle warp writes the rows and the db
    partials of the tiles without work: many tiles per block, empty samples,
    every output row and db per sample against the oracle."""
    dev = _dev()
    g = np.random.default_rng(Z)
    L, H = (1024, 2) if Z < 64 else (384, 1)   # 192 and 210 tiles for 148 blocks
    nq = g.integers(0, L + 1, size=Z)
    nk = g.integers(0, L + 1, size=Z)
    nq[::9], nk[1::11], nq[2], nk[2] = 0, 0, L, L
    q, k, v, do, nq, nk, bz = _inputs(Z, L, H, 64, nq, nk, seed=3300 + Z)
    outs = _run(q, k, v, do, nq, nk, 1.0 / 8.0, bz, dev)
    _check_full(q, k, v, do, nq, nk, 1.0 / 8.0, bz, outs, "bf16", DB_TOL["tanh"])


def test_bias_fp32_full():
    dev = _dev()
    q, k, v, do, nq, nk, bz = _inputs(2, 300, 2, 128, (300, 129), (45, 300), seed=3100,
                                      dtype="fp32")
    outs = _run(q, k, v, do, nq, nk, 1.0 / math.sqrt(128), bz, dev)
    _check_full(q, k, v, do, nq, nk, 1.0 / math.sqrt(128), bz, outs, "fp32", DB_TOL["fp32"])


@pytest.mark.parametrize("mode", ["tanh", "exp"])
def test_dbias_medium(mode):
    """db over several full tiles, ragged tails and an empty sample."""
    dev = _dev()
    q, k, v, do, nq, nk, bz = _inputs(3, 1000, 2, 128, (1000, 731, 0), (1000, 259, 600),
                                      seed=3200)
    alpha = 1.0 / math.sqrt(128)
    old = sa.get_sigmoid_mode()
    sa.set_sigmoid_mode(_mode(mode))
    try:
        outs = _run(q, k, v, do, nq, nk, alpha, bz, dev)
    finally:
        sa.set_sigmoid_mode(old)
    rel = _check_full(q, k, v, do, nq, nk, alpha, bz, outs, "bf16", DB_TOL[mode])
    print(f"db {mode}: |err| / sum|dS| per sample = {rel}")
    assert outs[4][2].item() == 0.0   # n_q = 0: no gradient


def test_dbias_workload2():
    """Workload 2 (Z=8, H=12, L=2048, D=64, lengths U[256, 2048]) with b_z = -ln n_z: db
    for every sample against the oracle, plus sampled rows of O, dQ, dK, dV."""
    dev = _dev()
    w = workloads.WORKLOADS[2]
    inp = workloads.make_inputs(w)
    nq, nk = inp["seqlens_q"], inp["seqlens_k"]
    bz = (-np.log(nk.astype(np.float64))).astype(np.float32)
    outs = _run(inp["q"], inp["k"], inp["v"], inp["dout"], nq, nk, w.alpha, bz, dev)
    o, dq, dk, dv, db = outs
    items_q = C.sample_items(w.Z, w.L, w.H, nq, 64, seed=5)
    items_k = C.sample_items(w.Z, w.L, w.H, nk, 64, seed=6)
    args = (inp["q"], inp["k"], inp["v"])
    ro = oracle.fwd_rows(*args, nq, nk, w.alpha, bz, items_q)
    rdq = oracle.dq_rows(*args, inp["dout"], nq, nk, w.alpha, bz, items_q)
    rdk, rdv = oracle.dkdv_rows(*args, inp["dout"], nq, nk, w.alpha, bz, items_k)
    for name, t, ref, items, n in (("O", o, ro, items_q, nq), ("dQ", dq, rdq, items_q, nq),
                                   ("dK", dk, rdk, items_k, nk), ("dV", dv, rdv, items_k, nk)):
        got = C.gather_rows(t, items)
        valid = C.valid_row_mask(items, n)
        assert np.all(got[~valid] == 0.0)
        C.assert_close(got[valid], ref[valid], "bf16", name)
    rdb = oracle.dbias(*args, inp["dout"], nq, nk, w.alpha, bz)
    scale = _abs_ds_sum(inp["q"], inp["k"], inp["v"], inp["dout"], nq, nk, w.alpha, bz)
    err = np.abs(db.cpu().numpy().astype(np.float64) - rdb)
    assert np.all(err <= DB_TOL["tanh"] * scale)


def test_constant_bias_array_matches_scalar_path():
    """A bias array holding one value everywhere runs the same kernels as the
    scalar bias: outputs are bit-identical."""
    dev = _dev()
    Z, L, H, D = 2, 384, 2, 128
    q, k, v, do = (t.to(dev) for t in workloads.random_tensors(Z, L, H, D, 3300, "bf16"))
    n = torch.tensor([384, 200], dtype=torch.int32, device=dev)
    alpha, b = 1.0 / math.sqrt(D), -math.log(L)
    bd = torch.full((Z,), b, dtype=torch.float32, device=dev)
    assert torch.equal(sa.fwd(q, k, v, n, n, alpha, b), sa.fwd_bias(q, k, v, n, n, alpha, bd))
    ref = sa.bwd(q, k, v, do, n, n, alpha, b)
    got = sa.bwd_bias(q, k, v, do, n, n, alpha, bd, want_dbias=False)
    for a, c in zip(ref, got[:3]):
        assert torch.equal(a, c)
    assert got[3] is None


def test_dbias_is_deterministic_and_additive_over_samples():
    """Full-size workload 4 (Z=4, L=16384, D=128, 25% padding) with b_z = -ln n_z:
    db is bit-identical across calls and equal, per sample, to running that
    sample alone (the partials of a sample do not depend on the others)."""
    dev = _dev()
    w = workloads.WORKLOADS[4]
    n = np.asarray(workloads.lengths(w), np.int32)
    g = torch.Generator(device=dev).manual_seed(11)
    q, k, v, do = (torch.randn((w.Z, w.L, w.H, w.D), generator=g, device=dev).to(torch.bfloat16)
                   for _ in range(4))
    nd = torch.as_tensor(n, device=dev)
    bd = torch.as_tensor(-np.log(n.astype(np.float64)), dtype=torch.float32, device=dev)
    db1 = sa.bwd_bias(q, k, v, do, nd, nd, w.alpha, bd)[3].clone()
    db2 = sa.bwd_bias(q, k, v, do, nd, nd, w.alpha, bd)[3].clone()
    assert torch.equal(db1, db2)
    for z in (0, 3):
        sl = slice(z, z + 1)
        one = sa.bwd_bias(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(),
                          do[sl].contiguous(), nd[sl].contiguous(), nd[sl].contiguous(), w.alpha,
                          bd[sl].contiguous())[3]
        assert torch.equal(one, db1[sl])
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    assert torch.isfinite(db1).all()


@pytest.mark.parametrize("index", [4])
def test_bias_workload_sampled(index):
    """Full-size padded workload with the pages' b_z = -ln n_z: sampled rows of
    O, dQ, dK, dV against the oracle."""
    dev = _dev()
    w = workloads.WORKLOADS[index]
    inp = workloads.make_inputs(w)
    nq, nk = inp["seqlens_q"], inp["seqlens_k"]
    bz = (-np.log(nk.astype(np.float64))).astype(np.float32)
    g = [inp[n].to(dev) for n in ("q", "k", "v", "dout")]
    nqd, nkd = torch.as_tensor(nq, device=dev), torch.as_tensor(nk, device=dev)
    bd = torch.as_tensor(bz, device=dev)
    o = sa.fwd_bias(g[0], g[1], g[2], nqd, nkd, w.alpha, bd)
    dq, dk, dv, _ = sa.bwd_bias(*g, nqd, nkd, w.alpha, bd, want_dbias=False)
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    items_q = C.sample_items(w.Z, w.L, w.H, nq, 32, seed=7)
    items_k = C.sample_items(w.Z, w.L, w.H, nk, 32, seed=8)
    args = (inp["q"], inp["k"], inp["v"])
    ro = oracle.fwd_rows(*args, nq, nk, w.alpha, bz, items_q)
    rdq = oracle.dq_rows(*args, inp["dout"], nq, nk, w.alpha, bz, items_q)
    rdk, rdv = oracle.dkdv_rows(*args, inp["dout"], nq, nk, w.alpha, bz, items_k)
    for name, t, ref, items, n in (("O", o, ro, items_q, nq), ("dQ", dq, rdq, items_q, nq),
                                   ("dK", dk, rdk, items_k, nk), ("dV", dv, rdv, items_k, nk)):
        got = C.gather_rows(t, items)
        valid = C.valid_row_mask(items, n)
        assert np.all(got[~valid] == 0.0)
        C.assert_close(got[valid], ref[valid], "bf16", name)


def test_autograd_learnable_and_per_sample_bias():
    """The module's bias options through autograd: a learnable scalar b gets
    sum_z db_z, and per-sample b_z = -ln n_k(z) matches the oracle."""
    dev = _dev()
    Z, L, H, D = 2, 256, 2, 64
    q, k, v, do, nq, nk, _ = _inputs(Z, L, H, D, (256, 100), (256, 100), seed=3400)
    alpha = 1.0 / math.sqrt(D)
    nqd, nkd = torch.as_tensor(nq, device=dev), torch.as_tensor(nk, device=dev)
    # learnable scalar
    mod = sa.SigmoidAttention(bias=-1.5, learnable_bias=True).to(dev)
    tq, tk, tv = (t.to(dev).clone().requires_grad_(True) for t in (q, k, v))
    o = mod(tq, tk, tv, nqd, nkd)
    o.backward(do.to(dev))
    torch.cuda.synchronize()
    bz = np.full(Z, -1.5, np.float32)
    rdb = oracle.dbias(q, k, v, do, nq, nk, alpha, bz).sum()
    scale = _abs_ds_sum(q, k, v, do, nq, nk, alpha, bz).sum()
    assert abs(mod.b.grad.item() - rdb) <= DB_TOL["tanh"] * scale
    rdq, rdk, rdv = oracle.bwd(q, k, v, do, nq, nk, alpha, bz)
    C.assert_close(tq.grad.float().cpu().numpy(), rdq, "bf16", "dQ (learnable bias)")
    C.assert_close(tv.grad.float().cpu().numpy(), rdv, "bf16", "dV (learnable bias)")
    # per-sample -ln n_k
    mod2 = sa.SigmoidAttention(per_sample_bias=True)
    o2 = mod2(q.to(dev), k.to(dev), v.to(dev), nqd, nkd)
    torch.cuda.synchronize()
    bz2 = (-np.log(nk.astype(np.float64))).astype(np.float32)
    C.assert_close(o2.float().cpu().numpy(), oracle.fwd(q, k, v, nq, nk, alpha, bz2), "bf16",
                   "O (per-sample -ln n)")


def test_log_length_bias_matches_minus_ln_n():
    """The library's b_z = -ln n_z, against numpy in fp64 rounded to fp32; n <= 1 gives 0."""
    dev = _dev()
    n = np.array([0, 1, 2, 3, 77, 128, 2048, 16384, 65536, 1 << 30], np.int32)
    got = sa.log_length_bias(torch.as_tensor(n, device=dev)).cpu().numpy()
    want = np.where(n > 1, -np.log(np.maximum(n, 1).astype(np.float64)), 0.0)
    assert got.dtype == np.float32
    assert np.all(np.abs(got - want) <= 2e-7 * np.maximum(np.abs(want), 1.0))
    assert got[0] == 0.0 and got[1] == 0.0


def test_learnable_bias_optimiser_built_before_first_call_updates_it():
    """The learnable bias exists from construction, so an optimiser built before
    the first call holds it and a step moves it by -lr * db."""
    dev = _dev()
    Z, L, H, D = 2, 256, 2, 64
    q, k, v, do, nq, nk, _ = _inputs(Z, L, H, D, (256, 100), (256, 100), seed=3401)
    mod = sa.SigmoidAttention(learnable_bias=True, max_len=L).to(dev)
    assert abs(mod.b.item() + math.log(L)) < 1e-6
    opt = torch.optim.SGD(mod.parameters(), lr=0.01)
    b0 = mod.b.item()
    o = mod(q.to(dev), k.to(dev), v.to(dev), torch.as_tensor(nq, device=dev),
            torch.as_tensor(nk, device=dev))
    o.backward(do.to(dev))
    g = mod.b.grad.item()
    opt.step()
    assert g != 0.0
    assert abs(mod.b.item() - (b0 - 0.01 * g)) <= 1e-6 * max(1.0, abs(b0))
