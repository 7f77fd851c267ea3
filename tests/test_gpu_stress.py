"""GPU stress: the kernels' hand-offs under varied timing.  The same ragged
batches run many times on two streams at once (so that blocks of different
launches share the GPU and every wait sees other latencies), and every result
must equal, bit for bit, the one a single call on one stream gives, with no
device status set (a barrier phase missed under some timing ends in the
bounded-wait timeout).  It varies timing; it cannot force the rarest
interleavings, so a race can still pass it."""
import math

import numpy as np
import pytest
import torch

from padding_aware_sigmoid_b200 import workloads

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("padding_aware_sigmoid_b200")

CASES = [
    # Z, L, H, D, n (n_q = n_k)
    (6, 640, 3, 64, (640, 1, 0, 129, 511, 384)),
    (5, 512, 2, 128, (512, 300, 128, 0, 257)),
]


@pytest.mark.parametrize("Z,L,H,D,n", CASES)
def test_repeated_calls_on_two_streams_match_one_call(Z, L, H, D, n):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in workloads.random_tensors(Z, L, H, D, 4242 + D, "bf16"))
    nd = torch.as_tensor(np.asarray(n, np.int32), device=dev)
    alpha, bias = 1.0 / math.sqrt(D), -math.log(L)
    assert sa.last_device_status() == 0
    ref_o = sa.fwd(q, k, v, nd, nd, alpha, bias)
    ref = sa.bwd(q, k, v, do, nd, nd, alpha, bias)
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0

    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    outs = [None, None]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream(dev))
    for it in range(24):
        for si, s in enumerate(streams):
            with torch.cuda.stream(s):
                o = sa.fwd(q, k, v, nd, nd, alpha, bias)
                outs[si] = (o,) + tuple(sa.bwd(q, k, v, do, nd, nd, alpha, bias))
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    for got in outs:
        for name, a, b in zip(("O", "dQ", "dK", "dV"), got, (ref_o,) + tuple(ref)):
            assert torch.equal(a, b), name
