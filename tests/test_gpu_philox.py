"""The device's Philox4x32-10 against the generator's published known answers
(needs a B200 and nvcc).

Two checks, both against tests/golden/philox_kat.json (Random123's
known-answer vectors for Philox4x32-10, Salmon et al., SC'11), not against
the oracle:
  * the library's device function (uno_device.cuh), compiled into a test-only
    kernel, returns the published words at every published counter and key;
  * through the C ABI, the verifier's accept test, its residual draw and the
    draft sampler decide as the all-zero vector's words 0, 1 and 2 dictate:
    sequence 0, position 0, step 0 under seed 0 is that counter and key.
"""

import ctypes
import json
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden", "philox_kat.json")


def _cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def _words(case, key):
    return [int(w, 16) for w in case[key]]


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    from lossless_decoding_b200 import api as A
    return A


@pytest.fixture(scope="module")
def philox_lib(api):
    out_dir = os.path.join(ROOT, "_build", "tests")
    os.makedirs(out_dir, exist_ok=True)
    so = os.path.join(out_dir, "libphilox_words.so")
    src = os.path.join(ROOT, "tests", "csrc", "philox_words.cu")
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared",
           "-I", os.path.join(ROOT, "lossless_decoding_b200", "csrc"),
           "-I", os.path.join(ROOT, "include"), src, "-o", so]
    subprocess.run(cmd, check=True)
    lib = ctypes.CDLL(so)
    lib.philox_words.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.philox_words.restype = ctypes.c_int
    return lib


def test_device_philox_reproduces_published_vectors(philox_lib):
    cases = _cases()
    inp = np.array([_words(c, "counter") + _words(c, "key") for c in cases], dtype=np.uint32)
    out = np.zeros((len(cases), 4), dtype=np.uint32)
    st = philox_lib.philox_words(inp.ctypes.data, out.ctypes.data, len(cases))
    assert st == 0, f"CUDA error {st}"
    for c, w in zip(cases, out):
        assert [f"{int(v):08x}" for v in w] == c["out"], c["name"]


def _u24(word: int) -> float:
    return (word >> 8) * 2.0**-24


def _zero_words():
    return _words(next(c for c in _cases() if c["name"] == "zeros"), "out")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_verifier_decides_by_the_published_words(api, dtype):
    w = _zero_words()
    u, u_draw = _u24(w[0]), _u24(w[1])
    # q_0 = (1, 0, 0): the draft x_0 = 0 has q = 1, so it is accepted iff u < p_0(0).
    # After a rejection the residual max(0, p_0 - q_0) = (0, p1, p2) gives token 1
    # iff u' * (p1 + p2) < p1.
    for a, s, n_want, tok_want in ((u + 0.02, 0.5, 1, None), (u - 0.02, u_draw + 0.02, 0, 1),
                                   (u - 0.02, u_draw - 0.02, 0, 2)):
        p0 = np.array([a, (1 - a) * s, (1 - a) * (1 - s)])
        p = torch.tensor(np.log(np.stack([p0, [1 / 3] * 3]))[None], dtype=dtype)
        q = torch.tensor([[[0.0, -np.inf, -np.inf]]], dtype=dtype)
        x = torch.zeros((1, 1), dtype=torch.int32)
        res = api.verify_block(p.to(DEV), q.to(DEV), x.to(DEV), seed=0, step=0)
        torch.cuda.synchronize()
        assert int(res.accepted_len.item()) == n_want
        if tok_want is not None:
            assert int(res.out_tokens[0, 0].item()) == tok_want


def test_draft_sampler_decides_by_the_published_words(api):
    u2 = _u24(_zero_words()[2])
    # row (q(0), 1 - q(0)): token 0 iff u2 * 1 < q(0)
    for q0, want in ((u2 + 0.02, 0), (u2 - 0.02, 1)):
        q = torch.tensor(np.log([[[q0, 1 - q0]]]), dtype=torch.float32)
        ids = api.sample_drafts(q.to(DEV), seed=0, step=0)
        torch.cuda.synchronize()
        assert int(ids.item()) == want
