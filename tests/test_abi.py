"""CPU: the C-ABI library loads, exports every declared symbol, and validates arguments on the
host before touching the GPU (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

from quantized_paged_kv_q4_b200 import build, kvattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvattn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kvattn.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KVATTN_API\s+[\w\s\*]+?\b(kvattn_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ("kvattn_decode", "kvattn_prefill_chunk", "kvattn_select_blocks", "kvattn_merge_lse",
                     "kvattn_stream_pages", "kvattn_quantize_append", "kvattn_block_summaries"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", kvattn.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(kvattn_\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)
    # nothing undeclared leaks out of the library
    assert exported <= set(declared_symbols())


def test_binding_covers_every_symbol():
    assert set(declared_symbols()) <= set(kvattn._SIGS)


def test_status_strings_and_page_sizes(lib):
    assert kvattn.status_string(0) == "ok"
    assert "page" in kvattn.status_string(kvattn.ERR_BAD_PAGE)
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_K, kvattn.FMT_Q8_0) == 34816
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_V, kvattn.FMT_Q4_0) == 18432
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_V, kvattn.FMT_Q8_0) == 34816
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_K, kvattn.FMT_Q4_0) == 18432
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_K, kvattn.FMT_Q5_1) == 24576
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_V, kvattn.FMT_Q5_1) == 0
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_K, kvattn.FMT_Q5_0) == 22528
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_V, kvattn.FMT_Q4_1) == 20480
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_V, kvattn.FMT_Q5_0) == 0
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_K, kvattn.FMT_Q4_1) == 0
    assert kvattn.kvattn_page_bytes(kvattn.ROLE_K, 5) == 0


def _desc(**kw):
    base = dict(n_kv_heads=4, n_q_heads=24, k_pool=16 * 1000, v_pool=16 * 5000, n_pages=64)
    base.update(kw)
    return kvattn.make_desc(**base)


def _status(fn, *args):
    return fn(*args)


def test_host_validation_rejects_bad_arguments(lib):
    L = lib
    d = _desc()
    by = ctypes.byref
    # null / misaligned pointers and bad shapes are refused before any CUDA call
    assert L.kvattn_decode(None, 16, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_INVALID_ARG
    assert L.kvattn_decode(by(d), None, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_INVALID_ARG
    assert L.kvattn_decode(by(d), 18, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_INVALID_ARG
    assert L.kvattn_decode(by(d), 16, 5, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_UNSUPPORTED_SHAPE
    bad = _desc()
    bad.head_dim = 128
    assert L.kvattn_decode(by(bad), 16, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_UNSUPPORTED_FORMAT
    # format pairs outside the supported set
    for kf, vf in (("q5_0", "q4_0"), ("q8_0", "q4_1"), ("q4_0", "q4_1"), ("q5_0", "q8_0")):
        bad = _desc(k_fmt=kf, v_fmt=vf)
        assert L.kvattn_decode(by(bad), 16, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == \
            kvattn.ERR_UNSUPPORTED_FORMAT, (kf, vf)
    bad = _desc(v_fmt="q5_1")
    assert L.kvattn_decode(by(bad), 16, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_UNSUPPORTED_FORMAT
    # Q4_0 / Q5_1 keys: decode and the summaries take them; chunked prefill takes every format
    # pair the descriptor accepts and refuses the rest
    for kf in ("q4_0", "q5_1"):
        kd = _desc(k_fmt=kf)
        assert L.kvattn_decode_workspace_size(by(kd), 1, 1024) == L.kvattn_decode_workspace_size(by(d), 1, 1024)
    for kf, vf, ok in (("q8_0", "q4_0", True), ("q4_0", "q4_0", True), ("q5_1", "q4_0", True),
                       ("q5_0", "q4_1", True), ("q8_0", "q8_0", True), ("q5_1", "q8_0", True),
                       ("q4_0", "q8_0", True), ("q5_0", "q4_0", False), ("q8_0", "q4_1", False)):
        kd = _desc(k_fmt=kf, v_fmt=vf)
        st = L.kvattn_prefill_chunk(by(kd), 16, 1, 16, 16, None, None, 1, 4096, 16, 16, 16, 1 << 20, None)
        assert (st != kvattn.ERR_UNSUPPORTED_FORMAT) if ok else (st == kvattn.ERR_UNSUPPORTED_FORMAT), (kf, vf, st)
    bad = _desc(n_q_heads=25)
    assert L.kvattn_decode(by(bad), 16, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_INVALID_ARG
    bad = _desc(k_pool=16 * 1000 + 8)
    assert L.kvattn_decode(by(bad), 16, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_INVALID_ARG
    # a workspace that is too small is refused
    need = L.kvattn_decode_workspace_size(by(d), 1, 1024)
    assert need > 0
    assert L.kvattn_decode(by(d), 16, 1, 16, 16, None, None, 1024, 16, 16, 256, need - 1, None) == \
        kvattn.ERR_WORKSPACE_TOO_SMALL
    assert L.kvattn_quantize_append(by(d), 16, 16, 1, 128 * 10, 16, 10, None) == kvattn.ERR_INVALID_ARG
    assert L.kvattn_merge_lse(16, 16, 1, 2, 6, 16, 16, None) == kvattn.ERR_INVALID_ARG
    assert L.kvattn_select_blocks(16, 16, 1, 6, 10, 10, 9, 4, 2, 16, 16, 16, 16, 100, 256, 10 ** 6, None) == \
        kvattn.ERR_INVALID_ARG
    assert L.kvattn_select_blocks(16, 16, 1, 6, 20000, 20000, 20000, 4, 2, 16, 16, 16, 16, 100, 256, 10 ** 9,
                                  None) == kvattn.ERR_UNSUPPORTED_SHAPE


def test_decode_workspace_plan(lib):
    d = _desc()
    # 148 SMs / 4 KV heads = 37 splits; 8 padded rows (6 query heads x 1 token)
    n_splits, rows = 37, 8
    want = ((4 * n_splits * rows * 4 + 255) // 256) * 256 + 4 * n_splits * rows * 256 * 4
    got = kvattn.kvattn_decode_workspace_size(d, 1, 1024)
    if got != want:
        pytest.skip("workspace planned for a different SM count on this machine")
    assert kvattn.kvattn_decode_workspace_size(d, 1, 1) == 0       # one page: no split, no workspace
    assert kvattn.kvattn_decode_workspace_size(d, 4, 1024) > got
    # an SM budget of 132 leaves 16 SMs free: 33 splits per KV head; a budget above the SM
    # count plans for every SM
    d.sm_budget = 132
    want_b = ((4 * 33 * rows * 4 + 255) // 256) * 256 + 4 * 33 * rows * 256 * 4
    assert kvattn.kvattn_decode_workspace_size(d, 1, 1024) == want_b
    d.sm_budget = 1000
    assert kvattn.kvattn_decode_workspace_size(d, 1, 1024) == got


def test_descriptor_budget_fields_checked(lib):
    L = lib
    by = ctypes.byref
    for field, value in (("sm_budget", -1), ("reserved", 1)):
        d = _desc()
        setattr(d, field, value)
        assert L.kvattn_decode(by(d), 16, 1, 16, 16, None, None, 1, 16, 16, None, 0, None) == kvattn.ERR_INVALID_ARG


def test_stream_plan_coalesces_runs(lib):
    assert kvattn.kvattn_stream_plan([], []) == []
    assert kvattn.kvattn_stream_plan([5], [0]) == [(0, 1)]
    host = [3, 4, 5, 9, 10, 11, 12, 2]
    dev = [0, 1, 2, 3, 4, 6, 7, 8]
    assert kvattn.kvattn_stream_plan(host, dev) == [(0, 3), (3, 2), (5, 2), (7, 1)]
    with pytest.raises(kvattn.KVAttnError):
        kvattn.kvattn_stream_pages(16, 64, 16, 64, 64, [1, -1], [0, 1], copy_stream=0)


def test_resident_update_validation(lib):
    f = kvattn.lib().kvattn_resident_update
    one = 16  # any non-null address: validation fails before anything is read
    args = [one, one, 8, 2, 100, 90, one, one, 16, one, 0, one, one, one, one, one, None]
    bad = [
        (2, 0),        # cap
        (3, 0),        # n_units
        (4, 0),        # n_blocks
        (5, 101),      # n_full > n_blocks
        (8, 0),        # n_slots
        (8, 16385),    # n_slots over the limit
        (10, -1),      # first_page
        (0, None),     # null selection
    ]
    for i, v in bad:
        a = list(args)
        a[i] = v
        assert f(*a) == kvattn.ERR_INVALID_ARG


def test_binding_refuses_host_tensors_for_device_arguments(lib):
    import torch

    d = _desc()
    q_cpu = torch.zeros((1, 24, 256))
    with pytest.raises(ValueError, match="CUDA tensor"):
        kvattn.kvattn_decode(d, q_cpu, 1, 16, 16, None, None, 1, 16, 16, None, 0, stream=0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kvattn.kvattn_hadamard(torch.zeros((2, 256)), stream=0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kvattn.make_desc(1, 6, torch.zeros(64, dtype=torch.uint8), 16, 1)
    # a host pool must be a host tensor
    with pytest.raises(ValueError, match="host"):
        kvattn._h(type("FakeCuda", (), {"is_cuda": True})())
    with pytest.raises(ValueError, match="contiguous"):
        kvattn._h(torch.zeros((4, 4)).t())
