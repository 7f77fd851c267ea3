"""CPU checks of the C ABI: the library builds, loads, and exports exactly the
entry points include/sigattn.h declares; host-side argument validation works
without a GPU; the product path has no CPU fallback and never touches the
oracle."""
import ctypes
import os
import re
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sigattn.h")
PKG = os.path.join(ROOT, "padding_aware_sigmoid_b200")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sigattn_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from padding_aware_sigmoid_b200 import build
    if not os.path.exists(build.OUT):
        if shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"):
            pytest.skip("nvcc unavailable and library not built")
        build.build()
    import padding_aware_sigmoid_b200 as sa
    return sa.load_library()


def test_header_declares_the_boundary():
    names = _declared()
    assert "sigattn_fwd" in names and "sigattn_bwd" in names
    import padding_aware_sigmoid_b200 as sa
    assert sorted(sa.EXPORTS) == names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), f"{name} not exported by libsigattn.so"


def test_status_strings_and_version(lib):
    import padding_aware_sigmoid_b200 as sa
    for code, name in sa.STATUS_NAMES.items():
        assert sa.status_string(code) == name
    assert sa.version() >= 100


def test_host_validation_needs_no_gpu(lib):
    vp = ctypes.c_void_p
    dummy = vp(16)
    # unsupported head dim is rejected before any device call
    assert lib.sigattn_fwd(dummy, dummy, dummy, dummy, dummy, dummy, 1, 128, 1, 96, 1.0, 0.0, 0,
                           None) == 2
    # negative sizes and null pointers
    assert lib.sigattn_fwd(dummy, dummy, dummy, dummy, dummy, dummy, -1, 128, 1, 64, 1.0, 0.0, 0,
                           None) == 1
    assert lib.sigattn_fwd(None, dummy, dummy, dummy, dummy, dummy, 1, 128, 1, 64, 1.0, 0.0, 0,
                           None) == 1
    assert lib.sigattn_bwd(dummy, dummy, dummy, dummy, dummy, dummy, None, dummy, dummy, 1, 128, 1,
                           64, 1.0, 0.0, 0, None) == 1
    # unknown dtype
    assert lib.sigattn_fwd(dummy, dummy, dummy, dummy, dummy, dummy, 1, 128, 1, 64, 1.0, 0.0, 7,
                           None) == 3
    # misaligned base pointer
    odd = vp(16 + 2)
    assert lib.sigattn_fwd(odd, dummy, dummy, dummy, dummy, dummy, 1, 128, 1, 64, 1.0, 0.0, 0,
                           None) == 5
    # empty problems are a no-op
    assert lib.sigattn_fwd(dummy, dummy, dummy, dummy, dummy, dummy, 0, 128, 1, 64, 1.0, 0.0, 0,
                           None) == 0
    # sigmoid mode switch
    assert lib.sigattn_set_sigmoid_mode(5) == 1
    old = lib.sigattn_get_sigmoid_mode()
    assert lib.sigattn_set_sigmoid_mode(0) == 0 and lib.sigattn_get_sigmoid_mode() == 0
    assert lib.sigattn_set_sigmoid_mode(old) == 0
    assert lib.sigattn_set_wait_timeout_ns(0) == 1
    # below 1 ms the bound would also cut short the waits for in-flight loads
    assert lib.sigattn_set_wait_timeout_ns(999_999) == 1


def test_bias_entry_points_host_validation(lib):
    import padding_aware_sigmoid_b200 as sa
    vp = ctypes.c_void_p
    dummy = vp(16)
    # workspace: one float per dQ work unit (bf16: 128-row query tile x head; fp32: row x head)
    assert sa.dbias_workspace_bytes(2, 300, 3, __import__("torch").bfloat16) == 2 * 3 * 3 * 4
    assert sa.dbias_workspace_bytes(2, 300, 3, __import__("torch").float32) == 2 * 300 * 3 * 4
    assert lib.sigattn_dbias_workspace_bytes(0, 128, 1, 0) == 0
    # a null bias array is rejected before any device call
    assert lib.sigattn_fwd_bias(dummy, dummy, dummy, dummy, dummy, dummy, 1, 128, 1, 64, 1.0,
                                None, 0, None) == 1
    assert lib.sigattn_bwd_bias(dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                128, 1, 64, 1.0, None, None, None, 0, 0, None) == 1
    # dbias requested without a large enough, aligned workspace
    need = lib.sigattn_dbias_workspace_bytes(1, 128, 1, 0)
    assert lib.sigattn_bwd_bias(dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                128, 1, 64, 1.0, dummy, dummy, None, need, 0, None) == 1
    assert lib.sigattn_bwd_bias(dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                128, 1, 64, 1.0, dummy, dummy, dummy, need - 4, 0, None) == 1
    assert lib.sigattn_bwd_bias(dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                128, 1, 64, 1.0, dummy, dummy, vp(16 + 2), need, 0, None) == 1
    # empty problems are a no-op
    assert lib.sigattn_fwd_bias(dummy, dummy, dummy, dummy, dummy, dummy, 0, 128, 1, 64, 1.0,
                                None, 0, None) == 0


def test_rect_entry_points_host_validation(lib):
    vp = ctypes.c_void_p
    dummy = vp(16)
    # exactly one of Lq, Lk zero is rejected; both zero is an empty problem
    assert lib.sigattn_fwd_rect(dummy, dummy, dummy, dummy, dummy, dummy, 1, 128, 0, 1, 64, 1.0,
                                0.0, 0, None) == 1
    assert lib.sigattn_bwd_rect(dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1,
                                0, 128, 1, 64, 1.0, 0.0, 0, None) == 1
    assert lib.sigattn_fwd_rect(dummy, dummy, dummy, dummy, dummy, dummy, 1, 0, 0, 1, 64, 1.0,
                                0.0, 0, None) == 0
    assert lib.sigattn_fwd_rect(dummy, dummy, dummy, dummy, dummy, dummy, 1, 128, 256, 1, 96,
                                1.0, 0.0, 0, None) == 2


def test_no_cpu_fallback(lib):
    import torch
    import padding_aware_sigmoid_b200 as sa
    x = torch.zeros((1, 128, 1, 64), dtype=torch.bfloat16)
    n = torch.full((1,), 128, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        sa.fwd(x, x, x, n, n, 1.0, 0.0)


def test_product_path_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "sigattn_oracle" not in text, f


def test_launch_order_is_a_stable_descending_sort(lib):
    """The kernels start samples by decreasing work (ties by index); the host
    entry point applies the same rule, so it is checked here without a GPU."""
    import numpy as np
    import padding_aware_sigmoid_b200 as sa
    assert sa.launch_order([5, 9, 9, 0, 7]) == [1, 2, 4, 0, 3]
    assert sa.launch_order([]) == []
    assert sa.launch_order([3, 3, 3]) == [0, 1, 2]
    g = np.random.default_rng(3)
    for Z in (1, 2, 7, 64, 384):
        w = g.integers(0, 40, size=Z).astype(np.int32)
        want = np.argsort(-w.astype(np.int64), kind="stable").tolist()
        got = sa.launch_order(w)
        assert got == want
        assert sorted(got) == list(range(Z))
    assert lib.sigattn_launch_order(None, 3, None) == 1
    assert lib.sigattn_launch_order(None, -1, None) == 1
    assert lib.sigattn_launch_order(None, 0, None) == 0


def test_host_pipeline_units_from_workspace_size(lib):
    """The host-buffer call cuts a batch into about 16 (sample, head group) units
    of at least 8 MB per tensor, groups as even as the heads allow; its
    workspace is three unit slots of eight tensors plus 256 bytes per slot, so
    the size shows the heads per unit."""
    import math
    import torch
    import padding_aware_sigmoid_b200 as sa

    def heads_per_unit(Z, L, H, D, es):
        chunks = min(H, -(-16 // Z))
        hpu = -(-H // chunks)
        per_head = L * D * es
        hpu = max(hpu, min(H, -(-(8 << 20) // per_head)))
        chunks = -(-H // hpu)
        return -(-H // chunks)

    cases = [((2, 16384, 16, 128), torch.bfloat16, 2), ((4, 16384, 16, 128), torch.bfloat16, 4),
             ((8, 2048, 12, 64), torch.bfloat16, 12), ((4, 8192, 12, 64), torch.bfloat16, 6),
             ((1, 16384, 5, 128), torch.bfloat16, 2), ((1, 8192, 4, 128), torch.float32, 2),
             ((3, 384, 2, 128), torch.bfloat16, 2)]
    for (Z, L, H, D), dt, want in cases:
        es = 4 if dt == torch.float32 else 2
        assert heads_per_unit(Z, L, H, D, es) == want
        assert sa.fwd_bwd_host_workspace_bytes(Z, L, H, D, dt) == 3 * 8 * L * want * D * es + 3 * 256
    assert lib.sigattn_fwd_bwd_host_workspace_bytes(0, 128, 1, 64, 0) == 0
    assert lib.sigattn_fwd_bwd_host_workspace_bytes(1, 128, 1, 96, 0) == 0
