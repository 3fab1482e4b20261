"""CPU-side checks of the C ABI library: it builds for sm_100a, loads, exports
every entry point the header declares, and rejects bad arguments on the host
before touching any device (no GPU is needed for any of this)."""
import ctypes
import os
import subprocess

import pytest

from sparse_convolution_pruned_b200 import build as svbuild
from sparse_convolution_pruned_b200 import svconv as sv


@pytest.fixture(scope="module")
def L():
    svbuild.build()
    return sv.lib()


def test_library_exports_every_declared_symbol(L):
    declared = sv.declared_symbols()
    assert len(declared) >= 11
    out = subprocess.run(["nm", "-D", "--defined-only", sv.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared:
        assert name in exported, name
        assert hasattr(L, name)


def test_version_and_status_strings(L):
    assert sv.svconv_version() == 100
    assert sv.status_str(0) == "ok"
    assert "NULL" in sv.status_str(-1)
    assert "wait" in sv.status_str(sv.STATUS_TIMEOUT)


def test_host_validation_runs_before_any_device_call(L):
    P = ctypes.c_void_p
    fake = P(0x1000)
    # negative sizes
    assert L.svconv_fwd(sv.BF16, fake, fake, -1, 64, 64, fake, None, fake, None) == -2
    assert L.svconv_build_index(fake, fake, -1, 4, 4, 0, fake, None, None, None) == -2
    assert L.svconv_build_index(fake, fake, 1, 200, 200, 0, fake, None, None, None) == -2  # H*W > 16384
    # empty problems are no-ops
    assert L.svconv_fwd(sv.BF16, None, None, 0, 64, 64, None, None, None, None) == 0
    assert L.svconv_bwd_data(sv.BF16, None, None, 0, 64, 64, None, None, None) == 0
    # NULL pointers
    assert L.svconv_fwd(sv.BF16, None, fake, 10, 64, 64, fake, None, fake, None) == -1
    assert L.svconv_bwd_data(sv.BF16, fake, None, 10, 64, 64, fake, fake, None) == -1
    # adapter: channel counts must be multiples of 64
    assert L.svconv_adapter_fwd(fake, fake, fake, 4, 10, 1000, 256, fake, fake, None, fake, 2, 64, fake, 1 << 20,
                                None, None) == -3
    # workspace sizes (pure host arithmetic for fp32)
    # fp32: one split per 16 tokens (at most 128), each split 9 C_in + 1 rows of C_out floats
    assert sv.svconv_bwd_weight_workspace_size(sv.F32, 128, 16, 16) == 8 * (9 * 16 + 1) * 16 * 4
    assert sv.svconv_bwd_weight_workspace_size(sv.F32, 100000, 16, 16) == 128 * (9 * 16 + 1) * 16 * 4
    # the cross-attention partials: one slot per 128 rows of the largest group (at most 444 over
    # all groups), A records of 10 x 32 floats per slot
    assert sv.svconv_xattn_workspace_size(3, 600, 2) == 3 * 5 * 2 * 10 * 32 * 4
    assert sv.svconv_xattn_workspace_size(1, 282624, 1) == 444 * 10 * 32 * 4
    assert sv.svconv_xattn_workspace_size(4, 10 ** 7, 1) == 4 * 111 * 10 * 32 * 4
    # e4m3 forward: channel counts are checked before any device call
    assert L.svconv_fwd(sv.E4M3, fake, fake, 10, 64, 256, fake, None, fake, None) == -3
    assert sv.svconv_bwd_weight_workspace_size(sv.F32, 0, 16, 16) == 0
    assert sv.svconv_adapter_workspace_size(256, 100) == 2 * 128 * 256 * 2


def test_no_device_means_cuda_error_not_crash(L):
    """Without a GPU the first device query fails and the call reports it."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    fake = ctypes.c_void_p(0x1000)
    rc = L.svconv_fwd(sv.BF16, fake, fake, 10, 64, 64, fake, None, fake, None)
    assert rc in (-6, -7)


def test_product_never_imports_oracle():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "sparse_convolution_pruned_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "svconv_oracle" not in text, f


def test_epilogue_gelu_erf_constants_meet_the_published_bound():
    """The GELU epilogue evaluates erf by Abramowitz and Stegun, Handbook of Mathematical
    Functions, formula 7.1.28 (|error| <= 3e-7).  Read the six coefficients out of the CUDA
    source and check, in float64, that the formula they define keeps that bound against
    math.erf: a mistyped constant in the kernel fails here without a GPU."""
    import math
    import re

    src = open(os.path.join(os.path.dirname(sv.LIB_PATH), "csrc", "svconv_tc.cu")).read()
    body = src[src.index("float gelu_erf(float x)"):]
    body = body[:body.index("\n}\n")]
    # the literals other than 1 and 1/2, in source order: 1/sqrt(2), then the Horner
    # coefficients a6, a5, a4, a3, a2, a1
    lits = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body) if float(v) not in (1.0, 0.5)]
    assert len(lits) == 7, lits
    inv_sqrt2, a6, a5, a4, a3, a2, a1 = lits
    assert abs(inv_sqrt2 - 1 / math.sqrt(2)) < 1e-15
    worst = 0.0
    for i in range(60001):
        z = i * 6.0 / 60000
        p = 1.0 + z * (a1 + z * (a2 + z * (a3 + z * (a4 + z * (a5 + z * a6)))))
        worst = max(worst, abs(1.0 - p ** -16 - math.erf(z)))
    assert worst <= 3e-7, worst
    # (the kernel raises p^-1 to the 16th power by four squarings)
    assert body.count("r8 * r8") == 1 and "r4 = r2 * r2" in body and "r8 = r4 * r4" in body
