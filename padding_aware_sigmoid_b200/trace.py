"""Timeline of one steady-state CTA, read from the diagnostic build.

    python -m padding_aware_sigmoid_b200.build --trace        # libsigattn_trace.so
    python -m padding_aware_sigmoid_b200.trace dkdv [--D 128] [--L 8192] [--H 37]

In the diagnostic build the CTA at grid position (gridDim.x / 2, 0, 0) records
clock64() at its roles' waits and hand-offs (role 0: loads, role 1: MMA issue,
roles 2 and 3: the two sigma warpgroups; the events of each role are numbered in
the kernel source).  This runs one kernel on a full-length batch of one sample,
reads the record back and prints, per role and event, the mean period over steps
10-50 and each event's mean offset from event 0 of the same step.  GPU only.
"""
from __future__ import annotations

import argparse
import ctypes
import math
import os

ROLES, STEPS, EVENTS = 4, 256, 8   # kTraceRoles, kTraceSteps, kTraceEvents


def _load_trace_library():
    import padding_aware_sigmoid_b200 as sa
    from padding_aware_sigmoid_b200 import build
    if not os.path.exists(build.TRACE_OUT):
        raise SystemExit("libsigattn_trace.so is not built: python -m "
                         "padding_aware_sigmoid_b200.build --trace")
    sa._LIB_PATH = build.TRACE_OUT
    lib = sa.load_library()
    lib.sigattn_trace_dump.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.sigattn_trace_dump.restype = ctypes.c_int
    return sa, lib


def record(kernel: str, D: int, L: int, H: int):
    """Runs `kernel` ('fwd', 'dq' or 'dkdv') once after three warm-up launches and
    returns the trace as an int64 array [role][step][event] (0 = not recorded)."""
    import numpy as np
    import torch
    sa, lib = _load_trace_library()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    q, k, v, do = (torch.randn((1, L, H, D), generator=g, device=dev).to(torch.bfloat16)
                   for _ in range(4))
    n = torch.full((1,), L, dtype=torch.int32, device=dev)
    alpha, bias = 1.0 / math.sqrt(D), -math.log(L)
    run = {"fwd": lambda: sa.fwd(q, k, v, n, n, alpha, bias),
           "dq": lambda: sa.bwd_dq(q, k, v, do, n, n, alpha, bias),
           "dkdv": lambda: sa.bwd_dkdv(q, k, v, do, n, n, alpha, bias)}[kernel]
    buf = np.zeros(ROLES * STEPS * EVENTS, np.uint64)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    if lib.sigattn_trace_dump(buf.ctypes.data, buf.size) != buf.size:   # clears the record
        raise RuntimeError("sigattn_trace_dump failed")
    run()
    torch.cuda.synchronize()
    if lib.sigattn_trace_dump(buf.ctypes.data, buf.size) != buf.size:
        raise RuntimeError("sigattn_trace_dump failed")
    if sa.last_device_status() != 0:
        raise RuntimeError("device status word set")
    return buf.reshape(ROLES, STEPS, EVENTS).astype(np.int64)


def summarise(t, first: int = 10, last: int = 50) -> str:
    """Mean period per role and event over steps [first, last), and each event's
    mean offset from event 0 of the same step (roles whose event 0 was recorded)."""
    import numpy as np
    lines = ["mean period (clk) per role, events 0..7, steps %d-%d:" % (first, last)]
    for r in range(ROLES):
        cells = []
        for e in range(EVENTS):
            x = t[r, first:last, e]
            x = x[x > 0]
            cells.append("%6.0f" % np.diff(x).mean() if len(x) > 2 else "     -")
        lines.append("  role %d: %s" % (r, " ".join(cells)))
    lines.append("mean offset (clk) from event 0 of the same step:")
    for r in range(ROLES):
        seg = t[r, first:last]
        if not (seg[:, 0] > 0).all():
            continue
        cells = []
        for e in range(EVENTS):
            col = seg[:, e]
            cells.append("%6d" % int(np.mean(col - seg[:, 0])) if (col > 0).all() else "     -")
        lines.append("  role %d: %s" % (r, " ".join(cells)))
    return "\n".join(lines)


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("kernel", choices=("fwd", "dq", "dkdv"))
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--L", type=int, default=8192)
    ap.add_argument("--H", type=int, default=37)
    a = ap.parse_args(argv)
    print("%s, Z=1 H=%d L=%d D=%d, full lengths" % (a.kernel, a.H, a.L, a.D))
    print(summarise(record(a.kernel, a.D, a.L, a.H)))


if __name__ == "__main__":
    main()
