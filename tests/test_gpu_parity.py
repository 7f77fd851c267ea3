"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Small shapes are compared element by element over every
row; the full-size workloads are compared on sampled rows (boundary rows plus
random ones), which the oracle computes one by one."""
import math

import numpy as np
import pytest
import torch

import oracle
from padding_aware_sigmoid_b200 import workloads
from tests import _compare as C

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("padding_aware_sigmoid_b200")


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _to(d, dev):
    out = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    out["nq_dev"] = torch.as_tensor(d["seqlens_q"], dtype=torch.int32, device=dev)
    out["nk_dev"] = torch.as_tensor(d["seqlens_k"], dtype=torch.int32, device=dev)
    return out


def _case(Z, L, H, D, nq, nk, seed, dtype="bf16", scale=1.0):
    q, k, v, do = workloads.random_tensors(Z, L, H, D, seed, dtype, scale)
    return dict(q=q, k=k, v=v, dout=do, seqlens_q=np.asarray(nq, np.int32),
                seqlens_k=np.asarray(nk, np.int32), alpha=1.0 / math.sqrt(D), bias=-math.log(L))


def _run(inp, dev):
    g = _to(inp, dev)
    o = sa.fwd(g["q"], g["k"], g["v"], g["nq_dev"], g["nk_dev"], g["alpha"], g["bias"])
    dq, dk, dv = sa.bwd(g["q"], g["k"], g["v"], g["dout"], g["nq_dev"], g["nk_dev"], g["alpha"],
                        g["bias"])
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    return o, dq, dk, dv


def _check_full(inp, outs, dtype):
    """Element-wise comparison over every row; padded rows must be exactly zero."""
    o, dq, dk, dv = (t.float().cpu().numpy() for t in outs)
    args = (inp["q"], inp["k"], inp["v"])
    ro = oracle.fwd(*args, inp["seqlens_q"], inp["seqlens_k"], inp["alpha"], inp["bias"])
    rdq, rdk, rdv = oracle.bwd(*args, inp["dout"], inp["seqlens_q"], inp["seqlens_k"],
                               inp["alpha"], inp["bias"])
    Z = o.shape[0]
    for name, got, ref, lens in (("O", o, ro, inp["seqlens_q"]), ("dQ", dq, rdq, inp["seqlens_q"]),
                                 ("dK", dk, rdk, inp["seqlens_k"]), ("dV", dv, rdv, inp["seqlens_k"])):
        for z in range(Z):
            n = int(lens[z])
            assert np.all(got[z, n:] == 0.0), f"{name}: padded rows of sample {z} not exactly zero"
        if np.any(ref != 0):
            C.assert_close(got, ref, dtype, name)
        else:
            assert np.all(got == 0.0), f"{name}: expected all zeros"


SMALL = [
    # Z, L, H, D, n_q, n_k
    (1, 128, 1, 64, (128,), (128,)),
    (1, 128, 1, 128, (128,), (128,)),
    (2, 256, 2, 64, (256, 77), (256, 77)),
    (2, 384, 3, 128, (300, 129), (129, 384)),
    (3, 200, 2, 64, (200, 1, 0), (127, 200, 5)),
    (2, 520, 2, 128, (513, 128), (520, 255)),
    (1, 1000, 2, 64, (999,), (1000,)),
    (2, 640, 1, 128, (0, 640), (640, 0)),
    # lengths out of order, ties and empty samples: the kernels start samples by
    # decreasing length, so grid position and sample index differ here
    (6, 384, 2, 128, (100, 384, 0, 300, 384, 1), (384, 100, 200, 0, 383, 2)),
    (5, 256, 2, 64, (17, 256, 256, 129, 3), (256, 5, 256, 100, 256)),
]


@pytest.mark.parametrize("mode", ["tanh", "exp"])
@pytest.mark.parametrize("Z,L,H,D,nq,nk", SMALL)
def test_bf16_small_full(Z, L, H, D, nq, nk, mode):
    dev = _dev()
    inp = _case(Z, L, H, D, nq, nk, seed=1000 + L + D)
    old = sa.get_sigmoid_mode()
    sa.set_sigmoid_mode(sa.SIGMOID_TANH if mode == "tanh" else sa.SIGMOID_EXP)
    try:
        outs = _run(inp, dev)
    finally:
        sa.set_sigmoid_mode(old)
    _check_full(inp, outs, "bf16")


@pytest.mark.parametrize("Z,L,H,D,nq,nk", [(2, 128, 2, 64, (128, 77), (128, 77)),
                                           (2, 300, 2, 128, (300, 129), (45, 300))])
def test_fp32_small_full(Z, L, H, D, nq, nk):
    dev = _dev()
    inp = _case(Z, L, H, D, nq, nk, seed=2000 + L, dtype="fp32")
    _check_full(inp, _run(inp, dev), "fp32")


def test_workload1_fp32_full():
    dev = _dev()
    w = workloads.WORKLOADS[1]
    inp = workloads.make_inputs(w)
    _check_full(inp, _run(inp, dev), "fp32")


def _check_sampled(inp, outs, per_sample, seed):
    o, dq, dk, dv = outs
    Z, L, H, D = (int(s) for s in inp["q"].shape)
    items_q = C.sample_items(Z, L, H, inp["seqlens_q"], per_sample, seed)
    items_k = C.sample_items(Z, L, H, inp["seqlens_k"], per_sample, seed + 1)
    args = (inp["q"], inp["k"], inp["v"])
    lens = (inp["seqlens_q"], inp["seqlens_k"], inp["alpha"], inp["bias"])
    ro = oracle.fwd_rows(*args, *lens, items_q)
    rdq = oracle.dq_rows(*args, inp["dout"], *lens, items_q)
    rdk, rdv = oracle.dkdv_rows(*args, inp["dout"], *lens, items_k)
    report = {}
    for name, t, ref, items, n in (("O", o, ro, items_q, inp["seqlens_q"]),
                                   ("dQ", dq, rdq, items_q, inp["seqlens_q"]),
                                   ("dK", dk, rdk, items_k, inp["seqlens_k"]),
                                   ("dV", dv, rdv, items_k, inp["seqlens_k"])):
        got = C.gather_rows(t, items)
        valid = C.valid_row_mask(items, n)
        assert np.all(got[~valid] == 0.0), f"{name}: a padded row is not exactly zero"
        report[name] = C.assert_close(got[valid], ref[valid], "bf16", name)
    return report


@pytest.mark.parametrize("mode", ["tanh", "exp"])
@pytest.mark.parametrize("index", [2, 3, 4, 5])
def test_workload_sampled(index, mode):
    """Full-size workloads, both in-register sigma forms, forward and backward."""
    dev = _dev()
    w = workloads.WORKLOADS[index]
    inp = workloads.make_inputs(w)
    old = sa.get_sigmoid_mode()
    sa.set_sigmoid_mode(sa.SIGMOID_TANH if mode == "tanh" else sa.SIGMOID_EXP)
    try:
        outs = _run(inp, dev)
    finally:
        sa.set_sigmoid_mode(old)
    per = 48 if w.L >= 8192 else 96
    rep = _check_sampled(inp, outs, per, seed=index)
    print(f"workload {index} ({w.name}), sigma {mode}: max-abs/max|ref| / L1 rel:",
          {k: ("%.2e/%.2e" % v) for k, v in rep.items()})


def test_padding_contents_never_matter():
    """Finite garbage (|x| <= 1e3) in every padded position leaves all outputs bit-identical."""
    dev = _dev()
    Z, L, H, D = 2, 384, 2, 128
    nq, nk = (300, 200), (250, 384)
    inp = _case(Z, L, H, D, nq, nk, seed=77)
    base = _run(inp, dev)
    g = torch.Generator().manual_seed(5)
    inp2 = dict(inp)
    for key, lens in (("q", nq), ("dout", nq), ("k", nk), ("v", nk)):
        t = inp[key].clone()
        for z in range(Z):
            n = lens[z]
            t[z, n:] = ((torch.rand(t[z, n:].shape, generator=g) * 2 - 1) * 1e3).to(t.dtype)
        inp2[key] = t
    new = _run(inp2, dev)
    for a, b in zip(base, new):
        assert torch.equal(a, b)


def test_no_write_outside_outputs():
    """Outputs are views into larger buffers filled with a sentinel; the sentinel
    before and after each output must survive."""
    dev = _dev()
    Z, L, H, D = 2, 200, 2, 64
    inp = _case(Z, L, H, D, (200, 100), (150, 200), seed=9)
    g = _to(inp, dev)
    n = Z * L * H * D
    pad = 4096
    bufs = [torch.full((n + 2 * pad,), -7.0, dtype=torch.bfloat16, device=dev) for _ in range(4)]
    views = [b[pad:pad + n].view(Z, L, H, D) for b in bufs]
    sa.fwd(g["q"], g["k"], g["v"], g["nq_dev"], g["nk_dev"], g["alpha"], g["bias"], out=views[0])
    sa.bwd(g["q"], g["k"], g["v"], g["dout"], g["nq_dev"], g["nk_dev"], g["alpha"], g["bias"],
           dq=views[1], dk=views[2], dv=views[3])
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.all(b[:pad] == -7.0) and torch.all(b[pad + n:] == -7.0)


def test_out_of_range_lengths_are_clamped_and_flagged():
    dev = _dev()
    Z, L, H, D = 2, 256, 1, 64
    inp = _case(Z, L, H, D, (300, -5), (256, 999), seed=11)
    g = _to(inp, dev)
    o = sa.fwd(g["q"], g["k"], g["v"], g["nq_dev"], g["nk_dev"], g["alpha"], g["bias"])
    torch.cuda.synchronize()
    assert sa.last_device_status() == 8  # SIGATTN_ERR_SEQLEN_RANGE
    clamped = dict(inp, seqlens_q=np.asarray([256, 0], np.int32),
                   seqlens_k=np.asarray([256, 256], np.int32))
    ref = oracle.fwd(clamped["q"], clamped["k"], clamped["v"], clamped["seqlens_q"],
                     clamped["seqlens_k"], inp["alpha"], inp["bias"])
    got = o.float().cpu().numpy()
    assert np.all(got[1] == 0.0)
    C.assert_close(got[0], ref[0], "bf16", "O (clamped lengths)")


def test_bounded_wait_timeout_is_reported():
    """A wait that nothing signals gives up after its limit, records
    SIGATTN_ERR_TIMEOUT and leaves the context usable."""
    dev = _dev()
    assert sa.last_device_status() == 0
    sa.selftest_wait_timeout(50_000_000)  # 50 ms
    torch.cuda.synchronize()
    assert sa.last_device_status() == 7
    inp = _case(1, 128, 1, 64, (128,), (128,), seed=3)
    _check_full(inp, _run(inp, dev), "bf16")


def test_argument_errors():
    dev = _dev()
    x = torch.zeros((1, 128, 1, 96), dtype=torch.bfloat16, device=dev)
    n = torch.full((1,), 128, dtype=torch.int32, device=dev)
    with pytest.raises(sa.SigattnError) as e:
        sa.fwd(x, x, x, n, n, 1.0, 0.0)
    assert e.value.code == 2
    y = torch.zeros((1, 128, 1, 64), dtype=torch.float16, device=dev)
    with pytest.raises(TypeError):
        sa.fwd(y, y, y, n, n, 1.0, 0.0)
    z = torch.zeros((0, 128, 1, 64), dtype=torch.bfloat16, device=dev)
    nz = torch.zeros((0,), dtype=torch.int32, device=dev)
    assert sa.fwd(z, z, z, nz, nz, 1.0, 0.0).shape == z.shape


def test_autograd_module_matches_oracle():
    dev = _dev()
    inp = _case(2, 256, 2, 64, (256, 100), (256, 100), seed=21)
    g = _to(inp, dev)
    q, k, v = (g[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    mod = sa.SigmoidAttention()
    o = mod(q, k, v, g["nq_dev"], g["nk_dev"])
    o.backward(g["dout"])
    torch.cuda.synchronize()
    _check_full(inp, (o.detach(), q.grad, k.grad, v.grad), "bf16")



@pytest.mark.parametrize("mode", ["tanh", "exp"])
@pytest.mark.parametrize("D", [64, 128])
def test_long_sequence_sampled(D, mode):
    """L = 65536 (4x the headline length) with one full and one ragged sample:
    sampled rows of every output against the oracle (the deepest key loops and
    the most negative bias, b = -ln 65536, where the tanh form's left-tail error
    is largest)."""
    dev = _dev()
    Z, L, H = 2, 65536, 1
    n = (65536, 40001)
    inp = _case(Z, L, H, D, n, n, seed=4000 + D)
    old = sa.get_sigmoid_mode()
    sa.set_sigmoid_mode(sa.SIGMOID_TANH if mode == "tanh" else sa.SIGMOID_EXP)
    try:
        outs = _run(inp, dev)
    finally:
        sa.set_sigmoid_mode(old)
    rep = _check_sampled(inp, outs, 12, seed=40 + D)
    print(f"L=65536 D={D} sigma {mode}: max-abs/max|ref| / L1 rel:",
          {k: ("%.2e/%.2e" % v) for k, v in rep.items()})


def test_tanh_margin_at_32k():
    """The tanh form's error grows with L (b = -ln L pushes the scores into the
    left tail, where 0.5 + 0.5 tanh cancels).  At L = 32768, D = 128, with one
    full and one ragged sample, sampled rows of every output must pass the bf16
    bar in tanh mode; the test prints the margin left to the L1 bar."""
    dev = _dev()
    Z, L, H, D = 2, 32768, 1, 128
    n = (32768, 20001)
    inp = _case(Z, L, H, D, n, n, seed=4300)
    old = sa.get_sigmoid_mode()
    sa.set_sigmoid_mode(sa.SIGMOID_TANH)
    try:
        outs = _run(inp, dev)
    finally:
        sa.set_sigmoid_mode(old)
    rep = _check_sampled(inp, outs, 12, seed=43)
    worst = max(v[1] for v in rep.values())
    print(f"L=32768 D=128 sigma tanh: max-abs/max|ref| / L1 rel:",
          {k: ("%.2e/%.2e" % v) for k, v in rep.items()},
          f"worst L1 {worst:.2e} = {100 * worst / C.BF16_L1_REL:.0f}% of the bar")


@pytest.mark.parametrize("Z,L,H,D,dtype", [(3, 384, 2, 128, "bf16"), (4, 256, 2, 64, "bf16"),
                                           (3, 200, 1, 64, "fp32"),
                                           (9, 130, 2, 64, "bf16"),
                                           # samples split into head groups of 2, 2, 1 and 2, 2
                                           (1, 16384, 5, 128, "bf16"), (1, 8192, 4, 128, "fp32")])
def test_host_buffer_pipeline_matches_device_path(Z, L, H, D, dtype):
    """sigattn_fwd_bwd_host (pinned host buffers cut into (sample, head group)
    units of at least 8 MB per tensor, copies overlapped with compute, three
    device slots reused) returns exactly what the device calls return on the
    same data."""
    dev = _dev()
    nq = tuple(int(x) for x in np.linspace(L, L // 3, Z).astype(int))
    nk = tuple(int(x) for x in np.linspace(L // 2, L, Z).astype(int))
    inp = _case(Z, L, H, D, nq, nk, seed=6000 + L, dtype=dtype)
    hosts = [inp[n].contiguous().pin_memory() for n in ("q", "k", "v", "dout")]
    outs = sa.fwd_bwd_host(*hosts, inp["seqlens_q"], inp["seqlens_k"], inp["alpha"], inp["bias"])
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    ref = _run(inp, dev)
    for name, a, b in zip(("O", "dQ", "dK", "dV"), outs, ref):
        assert torch.equal(a, b.cpu()), name


def _random_case(seed):
    """A seeded random problem: 1-90 samples (ranked by length or in index
    order), 1-6 heads, a padded length that is rarely a multiple of 128, and
    lengths that include 0, 1 and L; small enough for the oracle to check every
    row in about a second."""
    g = np.random.default_rng(seed)
    D = int(g.choice([64, 128]))
    Z = int(g.choice([1, 2, 3, 5, 8, 17, 40, 64, 65, 90]))
    H = int(g.integers(1, 7))
    budget = 2.5e7 / (Z * H)                    # valid (query, key) pairs at most
    L = int(min(1200, max(60, np.sqrt(budget) * g.uniform(0.5, 1.5))))
    nq = g.integers(0, L + 1, size=Z)
    nk = g.integers(0, L + 1, size=Z)
    for arr in (nq, nk):
        arr[g.integers(0, Z)] = L
        if Z > 2:
            arr[g.integers(0, Z)] = 0
            arr[g.integers(0, Z)] = 1
    mode = "tanh" if g.integers(0, 2) == 0 else "exp"
    return Z, L, H, D, nq, nk, mode


@pytest.mark.parametrize("seed", range(16))
def test_random_shapes_full(seed):
    """Seeded random shapes and lengths (both head dimensions, both sigma forms,
    more and fewer than 64 samples): every output row against the oracle."""
    dev = _dev()
    Z, L, H, D, nq, nk, mode = _random_case(9000 + seed)
    inp = _case(Z, L, H, D, nq, nk, seed=9100 + seed)
    old = sa.get_sigmoid_mode()
    sa.set_sigmoid_mode(sa.SIGMOID_TANH if mode == "tanh" else sa.SIGMOID_EXP)
    try:
        outs = _run(inp, dev)
    finally:
        sa.set_sigmoid_mode(old)
    _check_full(inp, outs, "bf16")


@pytest.mark.parametrize("Z,H,L", [(12, 24, 768), (100, 4, 1024)])
def test_persistent_many_items_per_block(Z, H, L):
    """Head dimension 64 runs the forward and both backward passes as one
    persistent block per SM: with 12 samples the blocks walk several
    length-ranked items each (one- and two-tile items mixed in the forward),
    with 100 samples they walk the index-ordered grid and skip tiles without
    work, which an idle warp zero-fills.  Every output row against the oracle."""
    dev = _dev()
    g = np.random.default_rng(Z + L)
    nq = g.integers(0, L + 1, size=Z)
    nk = g.integers(0, L + 1, size=Z)
    nq[::9], nk[1::11] = 0, 0
    nq[2], nk[2] = L, L
    inp = _case(Z, L, H, 64, nq, nk, seed=8500 + Z)
    _check_full(inp, _run(inp, dev), "bf16")


@pytest.mark.parametrize("Z", [40, 70])
def test_many_samples_launch_order(Z):
    """Up to 64 samples the kernels rank them by length with two samples per
    lane (Z = 40 uses both); above 64 they keep the index order (Z = 70).  Lengths
    are shuffled, with ties and empty samples; every output must still match."""
    dev = _dev()
    L, H, D = 256, 1, 64
    g = np.random.default_rng(Z)
    nq = g.integers(0, L + 1, size=Z)
    nk = g.integers(0, L + 1, size=Z)
    nq[::7], nk[::5], nk[3] = 0, L, nk[4]
    inp = _case(Z, L, H, D, nq, nk, seed=8000 + Z)
    _check_full(inp, _run(inp, dev), "bf16")
