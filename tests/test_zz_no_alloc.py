"""The scratch-free forward (sigattn_fwd_noalloc) against the regular forward.

Some callers cannot allocate device memory when they call attention: code
inside a framework whose caching allocator owns the device memory, or a
service that reserves its memory at start-up and forbids allocation later.
For them the library offers a forward that keeps its scratch (the lengths and
the kernel's status word) in a fixed array of its own device memory and takes
the lengths on the host.  Both entry points run the same kernel on the same
data, so this test requires the results to be equal bit for bit, on two calls
in a row with different shapes and lengths (the second call must not see the
first one's lengths), and once more with the lengths in pinned host memory
that is overwritten as soon as the call returns.  It lives in a file that
pytest collects last, so a failure here never hides another test's result."""
import math

import numpy as np
import pytest
import torch

from padding_aware_sigmoid_b200 import workloads
from tests import _compare as C

pytestmark = pytest.mark.gpu
sa = pytest.importorskip("padding_aware_sigmoid_b200")


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _inputs(Z, L, H, D, seed, dev):
    q, k, v, _ = workloads.random_tensors(Z, L, H, D, seed, "bf16")
    return q.to(dev), k.to(dev), v.to(dev)


def test_noalloc_forward_matches_regular_forward_twice():
    dev = _dev()
    calls = [
        (2, 384, 2, 128, np.array([384, 200], np.int32), np.array([300, 384], np.int32), 1),
        (3, 256, 2, 64, np.array([77, 256, 0], np.int32), np.array([256, 5, 129], np.int32), 2),
    ]
    for Z, L, H, D, nq, nk, seed in calls:
        q, k, v = _inputs(Z, L, H, D, seed, dev)
        alpha, bias = 1.0 / math.sqrt(D), -math.log(L)
        ref = sa.fwd(q, k, v, torch.as_tensor(nq, device=dev), torch.as_tensor(nk, device=dev),
                     alpha, bias)
        out = torch.full_like(q, 7.0)
        got = sa.fwd_noalloc(q, k, v, nq, nk, alpha, bias, out=out)
        torch.cuda.synchronize()
        assert got.data_ptr() == out.data_ptr()
        assert torch.equal(got, ref), "no-alloc forward differs from the regular forward"
        g = got.float().cpu().numpy()
        for z in range(Z):
            assert np.all(g[z, nq[z]:] == 0.0), "padded query rows must be exactly zero"


def test_noalloc_forward_lengths_in_pinned_memory_reused_at_once():
    dev = _dev()
    Z, L, H, D = 600, 128, 1, 64     # more samples than one length launch carries
    q, k, v = _inputs(Z, L, H, D, 3, dev)
    n = np.random.default_rng(3).integers(0, L + 1, size=Z).astype(np.int32)
    pq = torch.from_numpy(n.copy()).pin_memory()
    pk = torch.from_numpy(n[::-1].copy()).pin_memory()
    alpha, bias = 1.0 / math.sqrt(D), -math.log(L)
    ref = sa.fwd(q, k, v, pq.to(dev), pk.to(dev), alpha, bias)
    lib = sa.load_library()
    out = torch.empty_like(q)
    code = lib.sigattn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   pq.data_ptr(), pk.data_ptr(), Z, L, H, D, alpha, bias, 0,
                                   torch.cuda.current_stream(dev).cuda_stream)
    assert code == 0
    pq.fill_(L)   # the call has returned: the library must not read these any more
    pk.fill_(0)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_noalloc_forward_rejects_oversized_batch_and_bad_lengths():
    dev = _dev()
    Z = sa.NOALLOC_MAX_Z + 1
    x = torch.zeros((Z, 1, 1, 64), dtype=torch.bfloat16, device=dev)
    n = np.ones(Z, np.int32)
    with pytest.raises(sa.SigattnError) as e:
        sa.fwd_noalloc(x, x, x, n, n, 1.0, 0.0)
    assert e.value.code == 9   # SIGATTN_ERR_TOO_LARGE
    y = torch.zeros((1, 128, 1, 64), dtype=torch.bfloat16, device=dev)
    with pytest.raises(sa.SigattnError) as e:
        sa.fwd_noalloc(y, y, y, np.array([129], np.int32), np.array([1], np.int32), 1.0, 0.0)
    assert e.value.code == 8   # SIGATTN_ERR_SEQLEN_RANGE
