"""The allocation-free verifier entry point matches the regular one (needs a B200).

uno_verify_block_noalloc serves callers that cannot allocate device memory
when they call (for example a plug-in whose host engine owns every byte of
device memory, or a path that cannot afford cudaMalloc's synchronisation):
its scratch is a fixed array inside the library. These tests call it through
the C ABI and compare it with uno_verify_block on the same inputs, on two
calls in a row, since every call reuses the same scratch array.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from lossless_decoding_b200.inputs import verify_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
PROB_ATOL = 1e-5  # the probability tolerance of the parity tests


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    from lossless_decoding_b200 import api
    from lossless_decoding_b200._lib import lib
    return api, lib


def _outputs(B, K):
    return (torch.full((B, K + 1), -9, dtype=torch.int32, device=DEV),
            torch.full((B,), -9, dtype=torch.int32, device=DEV),
            torch.full((B, K), -1.0, dtype=torch.float32, device=DEV),
            torch.full((B, K), -1.0, dtype=torch.float32, device=DEV),
            torch.full((B, 2 * K + 1), -1.0, dtype=torch.float32, device=DEV))


def _call_noalloc(lib, v, seed, step):
    B, K1, V = v.p_logits.shape
    K = K1 - 1
    out = _outputs(B, K)
    dt = 0 if v.p_logits.dtype == torch.bfloat16 else 1
    st = lib.uno_verify_block_noalloc(
        v.p_logits.data_ptr(), v.q_logits.data_ptr(), v.draft_tokens.data_ptr(), B, K, V, dt,
        ctypes.c_uint64(seed), ctypes.c_uint64(step), out[0].data_ptr(), out[1].data_ptr(),
        out[2].data_ptr(), out[3].data_ptr(), out[4].data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.uno_status_string(st).decode()
    return out


@pytest.mark.parametrize("B,K,V,dtype", [(64, 16, 151936, "bf16"), (5, 7, 4097, "f32")])
def test_noalloc_matches_regular_entry_point_twice(libs, B, K, V, dtype):
    api, lib = libs
    v = verify_inputs(B, K, V, dtype=dtype, dist="gumbel", sigma=1.0, seed=B + K, device=DEV)
    for call, (seed, step) in enumerate(((11, 0), (11, 1))):
        got = _call_noalloc(lib, v, seed, step)
        ref = api.verify_block(v.p_logits, v.q_logits, v.draft_tokens, seed, step,
                               want_probs=True, want_lse=True)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref.out_tokens), f"call {call}: tokens differ"
        assert torch.equal(got[1], ref.accepted_len), f"call {call}: accepted lengths differ"
        for g, r in ((got[2], ref.p_at_draft), (got[3], ref.q_at_draft)):
            assert (g - r).abs().max().item() < PROB_ATOL
        assert (got[4] - ref.row_lse).abs().max().item() < 1e-4
        assert int(got[1].min().item()) >= 0


def test_noalloc_rejects_problems_beyond_its_scratch(libs):
    _, lib = libs
    # B = 4096, K = 64 needs more than the 4 MiB of fixed scratch.
    fake = ctypes.c_void_p(1 << 20)
    st = lib.uno_verify_block_noalloc(fake, fake, fake, 4096, 64, 151936, 0, ctypes.c_uint64(0),
                                      ctypes.c_uint64(0), fake, fake, None, None, None, None)
    assert lib.uno_status_string(st).decode().startswith("UNO_ERR_SIZE")
    assert lib.uno_verify_workspace_bytes(4096, 64, 151936, 0) > (4 << 20)


def test_noalloc_call_allocates_no_device_memory(libs):
    """After a first call on the device (module load, symbol look-up), a call
    changes neither the device's free memory nor PyTorch's allocations."""
    _, lib = libs
    v = verify_inputs(8, 6, 3001, dtype="bf16", seed=3, device=DEV)
    out = _outputs(8, 6)

    def call(step):
        st = lib.uno_verify_block_noalloc(
            v.p_logits.data_ptr(), v.q_logits.data_ptr(), v.draft_tokens.data_ptr(), 8, 6, 3001,
            0, ctypes.c_uint64(5), ctypes.c_uint64(step), out[0].data_ptr(), out[1].data_ptr(),
            out[2].data_ptr(), out[3].data_ptr(), out[4].data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert st == 0, lib.uno_status_string(st).decode()

    call(0)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for step in range(1, 4):
        call(step)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert int(out[1].min().item()) >= 0

