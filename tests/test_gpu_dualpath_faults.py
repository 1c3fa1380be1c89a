"""The dual-path GEMM's abort path: its bounded waits run out on purpose
(needs a B200).

uno_dualpath_test_hooks (a test-only hook of the C ABI) shortens every wait of
the kernel to a few milliseconds and makes the TMA producers wait for a T-tile
flag value that no tile writes, so the adapter loads never start: the
producers give up, then the MMA issuers and the epilogue warps, each setting
its fault bit. The kernel must still exit normally (no hang, no fault: the
device synchronises), report the bits through uno_device_fault_flags, and
leave the context usable: with the hook off, the same call is correct (oracle)
and sets no bit. Both layouts run: the CTA pair (M > 256) and the swapped
one-CTA tiles (M <= 256). The failure is made on the host side (a flag value
nothing writes); nothing faults or traps on the device.
"""

import numpy as np
import pytest
import torch

import oracle
from lossless_decoding_b200.inputs import dualpath_inputs
from tests.parity import assert_dualpath_close, widen

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
WAIT_NS = 5_000_000        # 5 ms per wait while the hook is on
SKEW = 0x40000000          # T-flag value = the call's epoch + SKEW: never written


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    from lossless_decoding_b200 import api as A
    return A


def _call(api, d):
    return api.dualpath_linear(d.x.to(DEV), d.W.to(DEV), d.A.to(DEV), d.Bm.to(DEV), d.scale)


@pytest.mark.parametrize("M", [512, 64])
def test_waits_run_out_and_the_context_stays_usable(api, M):
    from lossless_decoding_b200._lib import lib
    d = dualpath_inputs(M=M, d_in=512, d_out=1024, r=32, alpha=64.0, dtype="bf16", seed=M)
    assert api.device_fault_flags(clear=True) == 0
    assert lib.uno_dualpath_test_hooks(WAIT_NS, SKEW) == 0
    try:
        _call(api, d)
        torch.cuda.synchronize()  # the kernel returned: no hang, no device fault
        flags = api.device_fault_flags(clear=True)
    finally:
        assert lib.uno_dualpath_test_hooks(0, 0) == 0
    assert flags & 1, f"the producers' T-flag waits did not report (flags {flags:#x})"
    # hook off: the same call is correct and sets nothing
    y_ar, y_dr = _call(api, d)
    torch.cuda.synchronize()
    assert api.device_fault_flags(clear=True) == 0
    ref_ar, ref_dr, _ = oracle.dualpath_linear(widen(d.x), widen(d.W), widen(d.A), widen(d.Bm),
                                               d.scale, round_t_to_bf16=True)
    assert_dualpath_close(y_ar, ref_ar)
    assert_dualpath_close(y_dr, ref_dr)
