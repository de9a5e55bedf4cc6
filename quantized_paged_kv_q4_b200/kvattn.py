"""Thin ctypes binding of libkvattn (include/kvattn.h).

Argument marshalling only: every computation runs in the CUDA library.  Pointer arguments
accept torch tensors (their data_ptr), plain integers (raw addresses) or None; a tensor must
be contiguous, on the GPU for device-memory arguments and on the host for the pinned host
pools (anything else raises ValueError before the library is called); stream
arguments accept torch.cuda.Stream objects, raw handles or None (the current torch
stream).  A nonzero status raises KVAttnError.  If libkvattn.so is missing the import of
any entry point fails loudly: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_int, c_int32, c_int64, c_size_t, c_uint16, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvattn.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_ARCH = -2
ERR_UNSUPPORTED_FORMAT = -3
ERR_BAD_PAGE = -4
ERR_WORKSPACE_TOO_SMALL = -5
ERR_CUDA = -6
ERR_TIMEOUT = -7
ERR_UNSUPPORTED_SHAPE = -8
ERR_NOT_INITIALIZED = -9

FMT_Q4_0 = 4
FMT_Q8_0 = 8
FMT_Q5_1 = 51
FMT_Q5_0 = 50
FMT_Q4_1 = 41
ROLE_K = 0
ROLE_V = 1
FMT = {"q4_0": FMT_Q4_0, "q8_0": FMT_Q8_0, "q5_1": FMT_Q5_1, "q5_0": FMT_Q5_0, "q4_1": FMT_Q4_1}


class KVAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class kvattn_kv_desc(ctypes.Structure):
    _fields_ = [
        ("n_kv_heads", c_int32), ("n_q_heads", c_int32), ("head_dim", c_int32), ("page_tokens", c_int32),
        ("k_fmt", c_int32), ("v_fmt", c_int32), ("k_pool", c_void_p), ("v_pool", c_void_p),
        ("k_page_stride", c_int64), ("v_page_stride", c_int64), ("n_pages", c_int64),
        ("sm_budget", c_int32), ("reserved", c_int32),
    ]


_SIGS = {
    "kvattn_init": (c_int, [c_int]),
    "kvattn_status_string": (ctypes.c_char_p, [c_int]),
    "kvattn_last_cuda_error": (c_int, []),
    "kvattn_device_error": (c_int, [c_void_p]),
    "kvattn_page_bytes": (c_int64, [c_int, c_int]),
    "kvattn_quantize_append": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_void_p, c_int, c_int32, c_void_p, c_int,
                                       c_void_p]),
    "kvattn_decode_workspace_size": (c_size_t, [POINTER(kvattn_kv_desc), c_int, c_int]),
    "kvattn_decode": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                              c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "kvattn_append_decode": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_void_p, c_int, c_int32, c_void_p, c_int,
                                     c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                     c_void_p, c_void_p, c_size_t, c_void_p]),
    "kvattn_decode_splits": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "kvattn_decode_merge_splits": (c_int, [POINTER(kvattn_kv_desc), c_int, c_int, c_void_p, c_void_p, c_void_p,
                                           c_size_t, c_void_p]),
    "kvattn_decode_noalloc": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_int, c_void_p, c_void_p, c_void_p]),
    "kvattn_merge_lse": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "kvattn_block_summaries": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_int, c_int, c_int, c_int, c_void_p,
                                       c_void_p]),
    "kvattn_select_workspace_size": (c_size_t, [c_int, c_int]),
    "kvattn_select_blocks": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "kvattn_prefill_workspace_size": (c_size_t, [POINTER(kvattn_kv_desc), c_int, c_int, c_int]),
    "kvattn_prefill_chunk": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_int, c_int, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "kvattn_prefill_chunk_f16": (c_int, [POINTER(kvattn_kv_desc), c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "kvattn_stream_pages": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_int,
                                    c_void_p, c_void_p, POINTER(c_int)]),
    "kvattn_gather_pages": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_int64, c_int64, c_int64, c_void_p,
                                    c_void_p, c_int, c_int, c_void_p]),
    "kvattn_scatter_pages": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_int64, c_int64, c_int64, c_void_p,
                                     c_void_p, c_int, c_int, c_void_p]),
    "kvattn_stream_plan": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int]),
    "kvattn_stream_wait": (c_int, [c_void_p, c_int]),
    "kvattn_hadamard": (c_int, [c_void_p, c_void_p, c_int64, c_void_p]),
    "kvattn_resident_update": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_int,
                                       c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p]),
}

_lib = None


def lib():
    """The loaded libkvattn.so (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with quantized_paged_kv_q4_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _d(x):
    """A device-memory argument: a contiguous CUDA tensor, a raw address (int) or None.  A CPU
    tensor is refused here: its address would reach a kernel as device memory."""
    if x is None or isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError(f"expected a CUDA tensor for a device-memory argument, got one on {x.device}")
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor (the library reads dense row-major arrays)")
    return x.data_ptr()


def _h(x):
    """A host-memory argument (pinned pools): a contiguous CPU tensor, a raw address or None."""
    if x is None or isinstance(x, int):
        return x
    if x.is_cuda:
        raise ValueError("expected a host (pinned CPU) tensor for a host-memory argument")
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor (the library reads dense row-major arrays)")
    return x.data_ptr()


def _s(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str) -> int:
    if status != OK:
        raise KVAttnError(status, what)
    return status


def status_string(status: int) -> str:
    return lib().kvattn_status_string(status).decode()


def make_desc(n_kv_heads, n_q_heads, k_pool, v_pool, n_pages, v_fmt="q4_0", k_page_stride=None,
              v_page_stride=None, head_dim=256, page_tokens=128, k_fmt="q8_0", sm_budget=0) -> kvattn_kv_desc:
    kf, vf = FMT[k_fmt] if isinstance(k_fmt, str) else k_fmt, FMT[v_fmt] if isinstance(v_fmt, str) else v_fmt
    return kvattn_kv_desc(n_kv_heads, n_q_heads, head_dim, page_tokens, kf, vf, _d(k_pool), _d(v_pool),
                          k_page_stride or kvattn_page_bytes(ROLE_K, kf), v_page_stride or kvattn_page_bytes(ROLE_V, vf),
                          n_pages, sm_budget, 0)


# ---------------------------------------------------------------- entry points
def kvattn_init(device: int = 0) -> None:
    _check(lib().kvattn_init(device), "kvattn_init")


def kvattn_last_cuda_error() -> int:
    return lib().kvattn_last_cuda_error()


def kvattn_device_error(stream=None) -> int:
    """Returns (and clears) the device error word; does not raise for BAD_PAGE/TIMEOUT."""
    st = lib().kvattn_device_error(_s(stream))
    if st in (ERR_CUDA, ERR_NOT_INITIALIZED):
        raise KVAttnError(st, "kvattn_device_error")
    return st


def kvattn_page_bytes(role: int, fmt: int) -> int:
    return lib().kvattn_page_bytes(role, fmt)


def kvattn_quantize_append(desc, k, v, n_tok, pos0, page_table, n_blocks, stream=None) -> None:
    _check(lib().kvattn_quantize_append(ctypes.byref(desc), _d(k), _d(v), n_tok, pos0, _d(page_table), n_blocks,
                                        _s(stream)), "kvattn_quantize_append")


def kvattn_decode_workspace_size(desc, n_q, max_pages) -> int:
    return lib().kvattn_decode_workspace_size(ctypes.byref(desc), n_q, max_pages)


def kvattn_decode(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse, ws, ws_bytes,
                  stream=None) -> None:
    _check(lib().kvattn_decode(ctypes.byref(desc), _d(q), n_q, _d(q_pos), _d(page_list), _d(page_logical),
                               _d(n_pages), max_pages, _d(out), _d(lse), _d(ws), ws_bytes, _s(stream)),
           "kvattn_decode")


def kvattn_append_decode(desc, k_new, v_new, n_new, pos0, page_table, n_blocks, q, n_q, q_pos, page_list,
                         page_logical, n_pages, max_pages, out, lse, ws, ws_bytes, stream=None) -> None:
    """kvattn_quantize_append of n_new tokens and kvattn_decode in one grid."""
    _check(lib().kvattn_append_decode(ctypes.byref(desc), _d(k_new), _d(v_new), n_new, pos0, _d(page_table), n_blocks,
                                      _d(q), n_q, _d(q_pos), _d(page_list), _d(page_logical), _d(n_pages), max_pages,
                                      _d(out), _d(lse), _d(ws), ws_bytes, _s(stream)), "kvattn_append_decode")


def kvattn_decode_splits(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse, ws, ws_bytes,
                         stream=None) -> None:
    """The split grid of kvattn_decode alone (partials into the workspace)."""
    _check(lib().kvattn_decode_splits(ctypes.byref(desc), _d(q), n_q, _d(q_pos), _d(page_list), _d(page_logical),
                                      _d(n_pages), max_pages, _d(out), _d(lse), _d(ws), ws_bytes, _s(stream)),
           "kvattn_decode_splits")


def kvattn_decode_merge_splits(desc, n_q, max_pages, out, lse, ws, ws_bytes, stream=None) -> None:
    """The merge grid of kvattn_decode alone (partials in the workspace -> out, lse)."""
    _check(lib().kvattn_decode_merge_splits(ctypes.byref(desc), n_q, max_pages, _d(out), _d(lse), _d(ws), ws_bytes,
                                            _s(stream)), "kvattn_decode_merge_splits")


def kvattn_decode_noalloc(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse,
                          stream=None) -> None:
    """kvattn_decode without a caller workspace (scratch in a fixed device array of the library)."""
    _check(lib().kvattn_decode_noalloc(ctypes.byref(desc), _d(q), n_q, _d(q_pos), _d(page_list), _d(page_logical),
                                       _d(n_pages), max_pages, _d(out), _d(lse), _s(stream)),
           "kvattn_decode_noalloc")


def kvattn_merge_lse(o_parts, lse_parts, n_parts, rows, dim, out, lse, stream=None) -> None:
    _check(lib().kvattn_merge_lse(_d(o_parts), _d(lse_parts), n_parts, rows, dim, _d(out), _d(lse), _s(stream)),
           "kvattn_merge_lse")


def kvattn_block_summaries(desc, page_table, n_units, n_blocks, block_begin, block_end, summaries,
                           stream=None) -> None:
    _check(lib().kvattn_block_summaries(ctypes.byref(desc), _d(page_table), n_units, n_blocks, block_begin,
                                        block_end, _d(summaries), _s(stream)), "kvattn_block_summaries")


def kvattn_select_workspace_size(n_units, n_blocks) -> int:
    return lib().kvattn_select_workspace_size(n_units, n_blocks)


def kvattn_select_blocks(summaries, q_group, n_units, group, n_blocks, n_full, n_total, budget, recent, page_table,
                         sel_logical, sel_phys, n_sel, cap, ws, ws_bytes, stream=None) -> None:
    _check(lib().kvattn_select_blocks(_d(summaries), _d(q_group), n_units, group, n_blocks, n_full, n_total, budget,
                                      recent, _d(page_table), _d(sel_logical), _d(sel_phys), _d(n_sel), cap, _d(ws),
                                      ws_bytes, _s(stream)), "kvattn_select_blocks")


def kvattn_prefill_workspace_size(desc, n_q, max_pages, kv_split_tokens) -> int:
    return lib().kvattn_prefill_workspace_size(ctypes.byref(desc), n_q, max_pages, kv_split_tokens)


def kvattn_prefill_chunk(desc, q_bf16, n_q, q_pos, page_list, page_logical, n_pages, max_pages, kv_split_tokens, out,
                         lse, ws, ws_bytes, stream=None) -> None:
    _check(lib().kvattn_prefill_chunk(ctypes.byref(desc), _d(q_bf16), n_q, _d(q_pos), _d(page_list),
                                      _d(page_logical), _d(n_pages), max_pages, kv_split_tokens, _d(out), _d(lse),
                                      _d(ws), ws_bytes, _s(stream)), "kvattn_prefill_chunk")


def kvattn_prefill_chunk_f16(desc, q_bf16, n_q, q_pos, page_list, page_logical, n_pages, max_pages, kv_split_tokens,
                             out, lse, ws, ws_bytes, stream=None) -> None:
    _check(lib().kvattn_prefill_chunk_f16(ctypes.byref(desc), _d(q_bf16), n_q, _d(q_pos), _d(page_list),
                                          _d(page_logical), _d(n_pages), max_pages, kv_split_tokens, _d(out), _d(lse),
                                          _d(ws), ws_bytes, _s(stream)), "kvattn_prefill_chunk_f16")


def kvattn_gather_pages(host_pool, host_stride, n_host_pages, dev_pool, dev_stride, n_slots, page_bytes, host_ids,
                        dev_slots, n, n_ctas=0, stream=None) -> None:
    """Host (pinned, mapped) -> device page copy driven by device-side page lists."""
    _check(lib().kvattn_gather_pages(_h(host_pool), host_stride, n_host_pages, _d(dev_pool), dev_stride, n_slots,
                                     page_bytes, _d(host_ids), _d(dev_slots), n, n_ctas, _s(stream)),
           "kvattn_gather_pages")


def kvattn_scatter_pages(host_pool, host_stride, n_host_pages, dev_pool, dev_stride, n_slots, page_bytes, host_ids,
                         dev_slots, n, n_ctas=0, stream=None) -> None:
    """Device -> host (pinned, mapped) page copy driven by device-side page lists."""
    _check(lib().kvattn_scatter_pages(_h(host_pool), host_stride, n_host_pages, _d(dev_pool), dev_stride, n_slots,
                                      page_bytes, _d(host_ids), _d(dev_slots), n, n_ctas, _s(stream)),
           "kvattn_scatter_pages")


def kvattn_hadamard(x, out=None, rows=None, stream=None):
    """out = x R over rows of 256 fp32 values (R = H_256 / 16); in place when out is None."""
    out = x if out is None else out
    n = rows if rows is not None else x.numel() // 256
    _check(lib().kvattn_hadamard(_d(x), _d(out), n, _s(stream)), "kvattn_hadamard")
    return out


def kvattn_resident_update(sel_logical, n_sel, cap, n_units, n_blocks, n_full, slot_of_block, block_of_slot,
                           n_slots, host_page_of_block, first_page, extra_page, page_list, copy_host, copy_dst,
                           n_copies, stream=None) -> None:
    """Resident-page reuse: update each unit's slot pool for its new selection and write the
    decode page list and the copy list of the misses (all device arrays)."""
    _check(lib().kvattn_resident_update(_d(sel_logical), _d(n_sel), cap, n_units, n_blocks, n_full,
                                        _d(slot_of_block), _d(block_of_slot), n_slots, _d(host_page_of_block),
                                        first_page, _d(extra_page), _d(page_list), _d(copy_host), _d(copy_dst),
                                        _d(n_copies), _s(stream)),
           "kvattn_resident_update")


def _host_i32(a):
    import numpy as np

    arr = np.ascontiguousarray(a, dtype=np.int32)
    return arr, arr.ctypes.data


def kvattn_stream_plan(host_ids, dev_slots):
    """Returns the list of (first index, length) copy runs kvattn_stream_pages would issue."""
    import numpy as np

    h, hp = _host_i32(host_ids)
    d, dp = _host_i32(dev_slots)
    n = int(h.size)
    first = np.zeros(max(n, 1), np.int32)
    length = np.zeros(max(n, 1), np.int32)
    runs = lib().kvattn_stream_plan(hp, dp, n, first.ctypes.data, length.ctypes.data, n)
    if runs < 0:
        raise KVAttnError(runs, "kvattn_stream_plan")
    return list(zip(first[:runs].tolist(), length[:runs].tolist()))


def _event_handle(event, stream=None):
    """The cudaEvent_t of a torch.cuda.Event (created on first record, so an unused one is
    recorded on `stream` once to bring it into existence) or a raw handle passed as int."""
    if isinstance(event, int):
        return event
    if event.cuda_event == 0:
        import torch

        event.record(stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.current_stream())
    return event.cuda_event


def kvattn_stream_pages(host_pool, host_stride, dev_pool, dev_stride, page_bytes, host_ids, dev_slots,
                        copy_stream=None, done=None) -> int:
    """host_ids / dev_slots are host sequences; returns the number of copies issued."""
    h, hp = _host_i32(host_ids)
    d, dp = _host_i32(dev_slots)
    n_copies = c_int(0)
    ev = None if done is None else _event_handle(done, copy_stream)
    _check(lib().kvattn_stream_pages(_h(host_pool), host_stride, _d(dev_pool), dev_stride, page_bytes, hp, dp,
                                     int(h.size), _s(copy_stream), ev, ctypes.byref(n_copies)),
           "kvattn_stream_pages")
    return n_copies.value


def kvattn_stream_wait(event, timeout_ms: int) -> int:
    """Returns OK or ERR_TIMEOUT; raises on other errors."""
    st = lib().kvattn_stream_wait(_event_handle(event), timeout_ms)
    if st not in (OK, ERR_TIMEOUT):
        raise KVAttnError(st, "kvattn_stream_wait")
    return st
