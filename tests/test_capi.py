"""The C ABI library loads and exports every function include/uno.h declares.

Runs without a GPU: only host-side entry points and argument validation are
called (validation happens before any CUDA call, so bad arguments are
reported on any machine).
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "uno.h")


@pytest.fixture(scope="module")
def lib():
    from lossless_decoding_b200.build import build_library
    build_library()
    from lossless_decoding_b200._lib import lib as L
    return L


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(uno_[a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("uno_verify_block", "uno_dualpath_linear", "uno_verify_workspace_bytes",
                     "uno_dualpath_workspace_bytes", "uno_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(os.path.join(ROOT, "lossless_decoding_b200", "libuno.so"))
    for name in _declared_functions():
        assert hasattr(raw, name), name


def test_status_strings(lib):
    for code in range(-7, 1):
        s = lib.uno_status_string(code).decode()
        assert s.startswith("UNO_")
    assert lib.uno_status_string(-99).decode() == "UNO_ERR_UNKNOWN"
    assert lib.uno_version() >= 100


def test_workspace_sizes(lib):
    assert lib.uno_verify_workspace_bytes(64, 16, 151936, 0) > 0
    assert lib.uno_verify_workspace_bytes(-1, 16, 100, 0) == 0
    assert lib.uno_verify_workspace_bytes(1, 0, 100, 0) == 0
    assert lib.uno_verify_workspace_bytes(1, 257, 100, 0) == 0
    assert lib.uno_verify_workspace_bytes(1, 4, 100, 7) == 0
    assert lib.uno_dualpath_workspace_bytes(1024, 4096, 4096, 128, 0) >= 1024 * 128 * 2
    assert lib.uno_dualpath_workspace_bytes(16, 4096, 151936, 128, 0) > 0
    assert lib.uno_dualpath_workspace_bytes(16, 4100, 4096, 128, 0) == 0   # d_in % 8
    assert lib.uno_dualpath_workspace_bytes(16, 4096, 4096, 257, 0) == 0   # r > 256
    assert lib.uno_dualpath_workspace_bytes(16, 4096, 4096, 12, 0) == 0    # r % 8 (bf16)
    assert lib.uno_dualpath_workspace_bytes(16, 4096, 4096, 12, 1) > 0     # r % 4 (f32)


def test_argument_errors_need_no_gpu(lib):
    from lossless_decoding_b200._lib import STATUS
    fake = ctypes.c_void_p(4096)  # never dereferenced: validation fails first
    odd = ctypes.c_void_p(4096 + 2)
    u64 = ctypes.c_uint64
    # verify: dtype, size, null, alignment, workspace
    call = lib.uno_verify_block
    assert STATUS[call(fake, fake, fake, 1, 4, 10, 9, u64(0), u64(0), fake, fake, None, None,
                       None, fake, 1 << 20, None)] == "UNO_ERR_DTYPE"
    assert STATUS[call(fake, fake, fake, 1, 0, 10, 0, u64(0), u64(0), fake, fake, None, None,
                       None, fake, 1 << 20, None)] == "UNO_ERR_SIZE"
    assert STATUS[call(None, fake, fake, 1, 4, 10, 0, u64(0), u64(0), fake, fake, None, None,
                       None, fake, 1 << 20, None)] == "UNO_ERR_NULL"
    assert STATUS[call(odd, fake, fake, 1, 4, 10, 0, u64(0), u64(0), fake, fake, None, None,
                       None, fake, 1 << 20, None)] == "UNO_ERR_ALIGN"
    assert STATUS[call(fake, fake, fake, 1, 4, 10, 0, u64(0), u64(0), fake, fake, None, None,
                       None, fake, 8, None)] == "UNO_ERR_WORKSPACE"
    assert STATUS[call(fake, fake, fake, 1, 4, 10, 0, u64(0), u64(0), fake, fake, None, None,
                       None, None, 1 << 20, None)] == "UNO_ERR_WORKSPACE"
    # B = 0 is an empty, valid call
    assert call(None, None, None, 0, 4, 10, 0, u64(0), u64(0), None, None, None, None, None,
                None, 0, None) == 0
    # dual path
    dual = lib.uno_dualpath_linear
    assert STATUS[dual(fake, fake, fake, fake, 2.0, fake, fake, 16, 4096, 4096, 128, 5, fake,
                       1 << 30, None)] == "UNO_ERR_DTYPE"
    assert STATUS[dual(fake, fake, fake, fake, 2.0, fake, fake, 16, 4095, 4096, 128, 0, fake,
                       1 << 30, None)] == "UNO_ERR_SIZE"
    assert STATUS[dual(fake, fake, fake, fake, 2.0, None, None, 16, 4096, 4096, 128, 0, fake,
                       1 << 30, None)] == "UNO_ERR_NULL"
    assert STATUS[dual(fake, fake, None, fake, 2.0, fake, fake, 16, 4096, 4096, 128, 0, fake,
                       1 << 30, None)] == "UNO_ERR_NULL"
    assert STATUS[dual(fake, odd, fake, fake, 2.0, fake, fake, 16, 4096, 4096, 128, 0, fake,
                       1 << 30, None)] == "UNO_ERR_ALIGN"
    assert STATUS[dual(fake, fake, fake, fake, 2.0, fake, fake, 16, 4096, 4096, 128, 0, fake,
                       16, None)] == "UNO_ERR_WORKSPACE"
    assert dual(None, None, None, None, 2.0, None, None, 0, 4096, 4096, 128, 0, None, 0,
                None) == 0
    # grouped dual path
    grouped = lib.uno_dualpath_linear_grouped
    vp3 = ctypes.c_void_p * 3
    outs = (ctypes.c_int * 3)(4096, 1024, 1024)
    ptrs = vp3(fake, fake, fake)
    sc = (ctypes.c_float * 3)(2.0, 2.0, 2.0)
    assert STATUS[grouped(0, fake, ptrs, ptrs, ptrs, sc, None, ptrs, ptrs, 16, 4096, outs, 128, 0,
                          fake, 1 << 30, None)] == "UNO_ERR_SIZE"
    assert STATUS[grouped(5, fake, ptrs, ptrs, ptrs, sc, None, ptrs, ptrs, 16, 4096, outs, 128, 0,
                          fake, 1 << 30, None)] == "UNO_ERR_SIZE"
    mixed = vp3(fake, None, fake)  # y_draft for some projections only
    assert STATUS[grouped(3, fake, ptrs, ptrs, ptrs, sc, None, ptrs, mixed, 16, 4096, outs, 128, 0,
                          fake, 1 << 30, None)] == "UNO_ERR_NULL"
    bad = (ctypes.c_int * 3)(4096, 1020, 1024)  # d_out % 8
    assert STATUS[grouped(3, fake, ptrs, ptrs, ptrs, sc, None, ptrs, ptrs, 16, 4096, bad, 128, 0,
                          fake, 1 << 30, None)] == "UNO_ERR_SIZE"
    assert STATUS[grouped(3, fake, ptrs, ptrs, ptrs, None, None, ptrs, ptrs, 16, 4096, outs, 128, 0,
                          fake, 1 << 30, None)] == "UNO_ERR_NULL"
    # per-projection areas (T and its flags) plus one shared area for split partials
    need1 = lib.uno_dualpath_workspace_bytes(16, 4096, 4096, 128, 0)
    need3 = lib.uno_dualpath_grouped_workspace_bytes(3, 16, 4096, outs, 128, 0)
    need2 = lib.uno_dualpath_grouped_workspace_bytes(2, 16, 4096, outs, 128, 0)
    assert need1 < need2 < need3 < 3 * need1
    assert need3 - need2 == need2 - need1  # one more projection adds its own area
    assert lib.uno_dualpath_grouped_workspace_bytes(5, 16, 4096, outs, 128, 0) == 0
    assert STATUS[grouped(3, fake, ptrs, ptrs, ptrs, sc, None, ptrs, ptrs, 16, 4096, outs, 128, 0,
                          fake, need3 - 1, None)] == "UNO_ERR_WORKSPACE"
    assert grouped(3, None, ptrs, ptrs, ptrs, sc, None, ptrs, ptrs, 0, 4096, outs, 128, 0, None, 0,
                   None) == 0


def test_binding_refuses_cpu_tensors(lib):
    import torch
    from lossless_decoding_b200 import api
    p = torch.zeros(1, 3, 8)
    with pytest.raises(ValueError):
        api.verify_block(p, torch.zeros(1, 2, 8), torch.zeros(1, 2, dtype=torch.int32), 0, 0)
    x = torch.zeros(4, 8)
    with pytest.raises(ValueError):
        api.dualpath_linear(x, torch.zeros(8, 8), torch.zeros(8, 8), torch.zeros(8, 8), 1.0)


def test_tree_argument_errors_need_no_gpu(lib):
    from lossless_decoding_b200._lib import STATUS
    fake = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4096 + 2)
    u64 = ctypes.c_uint64
    assert lib.uno_tree_nodes(15, 16) == 1 + 15 * 16
    assert lib.uno_tree_nodes(0, 4) == 0 and lib.uno_tree_nodes(17, 4) == 0
    assert lib.uno_tree_nodes(4, 0) == 0 and lib.uno_tree_nodes(4, 65) == 0
    draft = lib.uno_tree_draft
    need = lib.uno_tree_draft_workspace_bytes(2, 15, 1000, 4)
    assert need > 0 and lib.uno_tree_draft_workspace_bytes(2, 17, 1000, 4) == 0
    assert lib.uno_tree_draft_workspace_bytes(2, 15, 1000, 17) == 0
    # small batches split each row over more CTAs: more partial lists
    assert lib.uno_tree_draft_workspace_bytes(1, 15, 151936, 4) > 15 * 4 * 8
    ok = (fake, 2, 15, 1000, 0, 4, 16, fake, fake, fake, fake, fake, fake, fake, need, None)

    def d(**kw):
        args = list(ok)
        for i, name in enumerate(("q", "B", "D", "V", "dtype", "top_k", "budget", "ids", "logq",
                                  "tok", "par", "dep", "n", "ws", "ws_bytes")):
            if name in kw:
                args[i] = kw[name]
        return STATUS[draft(*args)]

    assert d(dtype=3) == "UNO_ERR_DTYPE"
    assert d(D=0) == "UNO_ERR_SIZE" and d(D=17) == "UNO_ERR_SIZE"
    assert d(top_k=0) == "UNO_ERR_SIZE" and d(top_k=17) == "UNO_ERR_SIZE"
    assert d(budget=0) == "UNO_ERR_SIZE" and d(budget=65) == "UNO_ERR_SIZE"
    assert d(V=0) == "UNO_ERR_SIZE" and d(B=-1) == "UNO_ERR_SIZE"
    assert d(q=None) == "UNO_ERR_NULL" and d(n=None) == "UNO_ERR_NULL"
    odd1 = ctypes.c_void_p(4096 + 1)
    assert d(q=odd1) == "UNO_ERR_ALIGN" and d(logq=odd) == "UNO_ERR_ALIGN"
    assert d(ws=None) == "UNO_ERR_WORKSPACE" and d(ws_bytes=need - 1) == "UNO_ERR_WORKSPACE"
    assert d(ws=ctypes.c_void_p(4096 + 128)) == "UNO_ERR_WORKSPACE"  # not 256-byte aligned
    assert d(B=0, q=None, ids=None) == "UNO_OK"
    ver = lib.uno_tree_verify
    good = [fake, fake, fake, fake, fake, 2, 15, 16, 1000, 0, u64(0), u64(0), fake, fake, fake,
            None]

    def v(i, val):
        args = list(good)
        args[i] = val
        return STATUS[ver(*args)]

    assert v(9, 4) == "UNO_ERR_DTYPE"
    assert v(6, 0) == "UNO_ERR_SIZE" and v(7, 65) == "UNO_ERR_SIZE" and v(8, 0) == "UNO_ERR_SIZE"
    assert v(0, None) == "UNO_ERR_NULL" and v(12, None) == "UNO_ERR_NULL"
    assert v(0, odd1) == "UNO_ERR_ALIGN" and v(13, odd) == "UNO_ERR_ALIGN"
    assert v(5, 0) == "UNO_OK"


def test_head_argument_errors_need_no_gpu(lib):
    from lossless_decoding_b200._lib import STATUS
    fake = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4096 + 4)
    u64 = ctypes.c_uint64
    assert lib.uno_dualpath_stats_tiles(1088, 151936) == 594
    # swapped operands (M <= 256): one partial per CTA of the launch
    assert lib.uno_dualpath_stats_tiles(256, 151936) == 148
    assert lib.uno_dualpath_stats_tiles(17, 151936) == 148
    assert lib.uno_dualpath_stats_tiles(0, 151936) == 0
    assert lib.uno_dualpath_stats_tiles(17, 0) == 0
    st = lib.uno_dualpath_linear_stats
    # statistics of an output that is not written
    assert STATUS[st(fake, fake, fake, fake, 2.0, None, None, fake, fake, fake, 1088, 4096, 4096,
                     128, 0, fake, 1 << 30, None)] == "UNO_ERR_NULL"
    assert STATUS[st(fake, fake, fake, fake, 2.0, None, fake, fake, odd, fake, 1088, 4096, 4096,
                     128, 0, fake, 1 << 30, None)] == "UNO_ERR_ALIGN"
    vh = lib.uno_verify_block_head
    args = [fake, fake, fake, fake, 594, fake, 64, 16, 151936, 0, u64(0), u64(0), fake, fake,
            None, None, None, fake, 1 << 30, None]

    def v(i, val):
        a = list(args)
        a[i] = val
        return STATUS[vh(*a)]

    assert v(9, 7) == "UNO_ERR_DTYPE"
    assert v(4, 0) == "UNO_ERR_SIZE" and v(7, 0) == "UNO_ERR_SIZE"
    assert v(2, None) == "UNO_ERR_NULL" and v(5, None) == "UNO_ERR_NULL"
    assert v(2, odd) == "UNO_ERR_ALIGN"
    assert v(17, None) == "UNO_ERR_WORKSPACE" and v(18, 8) == "UNO_ERR_WORKSPACE"
    assert v(6, 0) == "UNO_OK"


def test_valid_calls_without_a_device_report_an_error(lib):
    """On a host with no CUDA device, a call whose arguments all pass the
    checks stops at the device check (UNO_ERR_CUDA or UNO_ERR_DEVICE): nothing
    is launched and no pointer is touched. Skipped where a GPU exists, since
    the fake pointers would then reach a launch."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    from lossless_decoding_b200._lib import STATUS
    fake = ctypes.c_void_p(1 << 20)  # 256-byte aligned, never dereferenced
    u64 = ctypes.c_uint64
    bad = {"UNO_ERR_CUDA", "UNO_ERR_DEVICE"}
    need_v = lib.uno_verify_workspace_bytes(2, 4, 1000, 0)
    assert STATUS[lib.uno_verify_block(fake, fake, fake, 2, 4, 1000, 0, u64(0), u64(0), fake,
                                       fake, None, None, None, fake, need_v, None)] in bad
    assert STATUS[lib.uno_verify_block_head(fake, fake, fake, fake, 4, fake, 2, 4, 1000, 0,
                                            u64(0), u64(0), fake, fake, None, None, None, fake,
                                            need_v, None)] in bad
    need_d = lib.uno_dualpath_workspace_bytes(512, 256, 512, 32, 0)
    assert STATUS[lib.uno_dualpath_linear(fake, fake, fake, fake, 2.0, fake, fake, 512, 256, 512,
                                          32, 0, fake, need_d, None)] in bad
    assert STATUS[lib.uno_dualpath_linear_stats(fake, fake, fake, fake, 2.0, None, fake, fake,
                                                fake, fake, 512, 256, 512, 32, 0, fake, need_d,
                                                None)] in bad
    need_s = lib.uno_dualpath_workspace_bytes(17, 256, 512, 32, 0)
    assert STATUS[lib.uno_dualpath_linear_stats(fake, fake, fake, fake, 2.0, None, fake, fake,
                                                fake, fake, 17, 256, 512, 32, 0, fake, need_s,
                                                None)] in bad
    assert STATUS[lib.uno_sample_drafts(fake, 2, 4, 1000, 0, u64(0), u64(0), fake, None)] in bad
    assert STATUS[lib.uno_sample_drafts_blocks(fake, 2, 4, 5, 1000, 0, u64(0), u64(0), fake,
                                               None)] in bad
    need_t = lib.uno_tree_draft_workspace_bytes(2, 3, 1000, 2)
    assert STATUS[lib.uno_tree_draft(fake, 2, 3, 1000, 0, 2, 2, fake, fake, fake, fake, fake,
                                     fake, fake, need_t, None)] in bad
    assert STATUS[lib.uno_tree_verify(fake, fake, fake, fake, fake, 2, 3, 2, 1000, 0, u64(0),
                                      u64(0), fake, fake, fake, None)] in bad


def test_sampler_argument_errors_need_no_gpu(lib):
    """uno_sample_drafts_blocks checks dtype, sizes (block_rows >= K), the empty
    batch, null pointers and alignment before it looks for a device."""
    from lossless_decoding_b200._lib import STATUS
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 1)
    u64 = ctypes.c_uint64

    def s(B, K, R, V, dt, q=fake, out=fake):
        return STATUS[lib.uno_sample_drafts_blocks(q, B, K, R, V, dt, u64(0), u64(0), out, None)]

    assert s(2, 4, 5, 1000, 7) == "UNO_ERR_DTYPE"
    assert s(2, 0, 5, 1000, 0) == "UNO_ERR_SIZE"
    assert s(2, 4, 3, 1000, 0) == "UNO_ERR_SIZE"      # fewer rows per block than drafts
    assert s(2, 4, 5000, 1000, 0) == "UNO_ERR_SIZE"   # block_rows above 4096
    assert s(2, 4, 5, 0, 0) == "UNO_ERR_SIZE"
    assert s(0, 4, 5, 1000, 0) == "UNO_OK"
    assert s(2, 4, 5, 1000, 0, q=None) == "UNO_ERR_NULL"
    assert s(2, 4, 5, 1000, 0, out=None) == "UNO_ERR_NULL"
    assert s(2, 4, 5, 1000, 0, q=odd) == "UNO_ERR_ALIGN"


def test_noalloc_checks_sizes_before_the_empty_batch(lib):
    # B = 0 is accepted only with valid K and V, as for uno_verify_block
    for K, V, want in ((4, 100, "UNO_OK"), (257, 100, "UNO_ERR_SIZE"), (4, 0, "UNO_ERR_SIZE")):
        st = lib.uno_verify_block_noalloc(None, None, None, 0, K, V, 0, ctypes.c_uint64(0),
                                          ctypes.c_uint64(0), None, None, None, None, None, None)
        assert lib.uno_status_string(st).decode().startswith(want)
        ref = lib.uno_verify_block(None, None, None, 0, K, V, 0, ctypes.c_uint64(0),
                                   ctypes.c_uint64(0), None, None, None, None, None, None, 0,
                                   None)
        assert ref == st
