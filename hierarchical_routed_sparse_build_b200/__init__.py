"""Python binding of libhga (``include/hga.h``): routed attention on B200 (sm_100a).

Argument marshalling only. Every entry point has the name of the C call it
wraps, takes torch tensors that already live on the GPU (or raw device
addresses), passes their addresses and the current CUDA stream, and raises
``HgaError`` on a non-OK status. All arithmetic runs in the CUDA kernels of
``libhga.so``; there is no fallback: importing this package on a machine where
the library cannot be loaded raises ``ImportError``.

The method: "Hierarchical Global Attention (HGA)" (arXiv 2606.30709),
abstract: per-chunk key summaries pick chunks, per-group summaries inside them
pick groups, and exact softmax attention runs over the picked tokens, with the
first and last chunk always kept (HISA article, block-then-token filter).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "HgaError", "hga_params", "hga_kv", "make_params", "make_kv", "library_path",
    "hga_summary_bytes", "hga_build_summaries", "hga_max_routed_tokens", "hga_route",
    "hga_attend", "hga_decode", "hga_set_launch_option", "hga_get_device_error",
    "hga_status_string", "hga_route_blocks", "hga_prefill_attend", "hga_prefill_workspace_size",
    "hga_prefill", "hga_prefill_noalloc", "hga_append", "hga_route_blocks_growing",
    "hga_prefill_growing_workspace_size", "hga_prefill_growing", "hga_host_kv_pointer", "hga_decode_hisa", "hga_max_hisa_tokens",
    "hga_decode_workspace_size", "hga_decode_ws", "hga_decode_hisa_workspace_size", "hga_decode_hisa_ws",
    "HGA_OPT_CTAS_PER_HEAD", "HGA_OPT_DECODE_KERNEL",
    "HGA_OPT_TEST_EXPIRE_PREFILL_WAIT", "STATUS_NAMES",
    "EXPORTED",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libhga.so")

HGA_OK = 0
HGA_OPT_CTAS_PER_HEAD = 1
HGA_OPT_DECODE_KERNEL = 2
HGA_OPT_TEST_EXPIRE_PREFILL_WAIT = 4
STATUS_NAMES = {0: "HGA_OK", 1: "HGA_ERR_INVALID_ARG", 2: "HGA_ERR_UNSUPPORTED", 3: "HGA_ERR_CUDA",
                4: "HGA_ERR_DEVICE_FAULT", 5: "HGA_ERR_TIMEOUT"}
EXPORTED = ("hga_summary_bytes", "hga_build_summaries", "hga_max_routed_tokens", "hga_route",
            "hga_attend", "hga_decode", "hga_set_launch_option", "hga_get_device_error",
            "hga_status_string", "hga_route_blocks", "hga_prefill_attend", "hga_prefill_workspace_size",
            "hga_prefill", "hga_prefill_noalloc", "hga_append", "hga_route_blocks_growing",
            "hga_prefill_growing_workspace_size", "hga_prefill_growing", "hga_host_kv_pointer",
            "hga_decode_hisa", "hga_max_hisa_tokens", "hga_decode_workspace_size", "hga_decode_ws",
            "hga_decode_hisa_workspace_size", "hga_decode_hisa_ws")


class HgaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({_status_text(status)})")


class hga_params(ctypes.Structure):
    _fields_ = [("chunk", ctypes.c_int32), ("group", ctypes.c_int32), ("top_chunks", ctypes.c_int32),
                ("top_groups", ctypes.c_int32), ("scale", ctypes.c_float)]


class hga_kv(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("seq_lens", ctypes.c_void_p), ("batch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_len", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing; build it with "
                          "`python hierarchical_routed_sparse_build_b200/build.py`")
    L = ctypes.CDLL(_LIB_PATH)
    i32, vp, sz = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
    P, KV = ctypes.POINTER(hga_params), ctypes.POINTER(hga_kv)
    sig = {
        "hga_summary_bytes": ([KV, P, ctypes.POINTER(sz), ctypes.POINTER(sz)], i32),
        "hga_build_summaries": ([KV, P, vp, vp, vp], i32),
        "hga_max_routed_tokens": ([KV, P], i32),
        "hga_route": ([vp, i32, KV, vp, vp, P, vp, i32, vp, vp], i32),
        "hga_attend": ([vp, i32, KV, vp, i32, vp, P, vp, vp, vp], i32),
        "hga_decode": ([vp, i32, KV, vp, vp, P, vp, vp, vp, i32, vp, vp], i32),
        "hga_set_launch_option": ([i32, i32], i32),
        "hga_get_device_error": ([vp, ctypes.POINTER(i32)], i32),
        "hga_status_string": ([i32], ctypes.c_char_p),
        "hga_route_blocks": ([vp, i32, i32, i32, KV, i32, vp, vp, P, vp, i32, vp, vp], i32),
        "hga_prefill_attend": ([vp, i32, i32, i32, KV, i32, vp, i32, vp, P, vp, vp], i32),
        "hga_prefill_workspace_size": ([KV, i32, i32, i32, i32, P], sz),
        "hga_prefill": ([vp, i32, i32, i32, KV, i32, vp, vp, P, vp, vp, sz, vp], i32),
        "hga_append": ([KV, vp, vp, vp, P, vp, vp, vp], i32),
        "hga_route_blocks_growing": ([vp, i32, i32, i32, KV, i32, vp, vp, P, vp, i32, vp, vp], i32),
        "hga_prefill_growing_workspace_size": ([KV, i32, i32, i32, i32, P], sz),
        "hga_prefill_growing": ([vp, i32, i32, i32, KV, i32, vp, vp, P, vp, vp, sz, vp], i32),
        "hga_host_kv_pointer": ([vp, ctypes.POINTER(vp)], i32),
        "hga_decode_hisa": ([vp, i32, KV, vp, P, i32, vp, vp, vp, i32, vp, vp], i32),
        "hga_max_hisa_tokens": ([KV, P, i32], i32),
        "hga_prefill_noalloc": ([vp, i32, i32, i32, KV, i32, vp, vp, P, vp, vp], i32),
        "hga_decode_workspace_size": ([KV, i32, P], sz),
        "hga_decode_ws": ([vp, i32, KV, vp, vp, P, vp, vp, vp, i32, vp, vp, sz, vp], i32),
        "hga_decode_hisa_workspace_size": ([KV, P], sz),
        "hga_decode_hisa_ws": ([vp, i32, KV, vp, P, i32, vp, vp, vp, i32, vp, vp, sz, vp], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


_lib = _load()


def _status_text(status: int) -> str:
    return _lib.hga_status_string(int(status)).decode()


def hga_status_string(status: int) -> str:
    return _status_text(status)


def _check(status: int, where: str) -> None:
    if status != HGA_OK:
        raise HgaError(status, where)


def _addr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if not x.is_contiguous():
            raise ValueError("tensors passed to libhga must be contiguous")
        return x.data_ptr()
    raise TypeError(f"expected a torch.Tensor or a device address, got {type(x)}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_params(chunk: int, group: int, top_chunks: int, top_groups: int, scale: float = 0.0) -> hga_params:
    return hga_params(chunk, group, top_chunks, top_groups, scale)


def make_kv(k, v, seq_lens, *, n_kv_heads: int, head_dim: int, max_len: int, batch: int,
            page_table=None, page_size: int = 0, max_pages: int = 0, num_pages: int = 0) -> hga_kv:
    """Describe a K/V cache (see hga_kv in hga.h). The caller keeps the tensors alive."""
    return hga_kv(_addr(k), _addr(v), _addr(page_table), _addr(seq_lens), batch, n_kv_heads, head_dim,
                  max_len, page_size, max_pages, num_pages)


def hga_summary_bytes(kv: hga_kv, p: hga_params) -> tuple[int, int]:
    cb, gb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(_lib.hga_summary_bytes(ctypes.byref(kv), ctypes.byref(p), ctypes.byref(cb), ctypes.byref(gb)),
           "hga_summary_bytes")
    return cb.value, gb.value


def hga_build_summaries(kv: hga_kv, p: hga_params, chunk_sum, group_sum, stream=None) -> None:
    _check(_lib.hga_build_summaries(ctypes.byref(kv), ctypes.byref(p), _addr(chunk_sum), _addr(group_sum),
                                    _stream(stream)), "hga_build_summaries")


def hga_max_routed_tokens(kv: hga_kv, p: hga_params) -> int:
    n = _lib.hga_max_routed_tokens(ctypes.byref(kv), ctypes.byref(p))
    if n < 0:
        raise HgaError(1, "hga_max_routed_tokens")
    return n


def hga_route(q, n_q_heads: int, kv: hga_kv, chunk_sum, group_sum, p: hga_params, idx, idx_stride: int,
              n_idx, stream=None) -> None:
    _check(_lib.hga_route(_addr(q), n_q_heads, ctypes.byref(kv), _addr(chunk_sum), _addr(group_sum),
                          ctypes.byref(p), _addr(idx), idx_stride, _addr(n_idx), _stream(stream)), "hga_route")


def hga_attend(q, n_q_heads: int, kv: hga_kv, idx, idx_stride: int, n_idx, p: hga_params, out, lse=None,
               stream=None) -> None:
    _check(_lib.hga_attend(_addr(q), n_q_heads, ctypes.byref(kv), _addr(idx), idx_stride, _addr(n_idx),
                           ctypes.byref(p), _addr(out), _addr(lse), _stream(stream)), "hga_attend")


def hga_decode(q, n_q_heads: int, kv: hga_kv, chunk_sum, group_sum, p: hga_params, out, lse=None,
               idx=None, idx_stride: int = 0, n_idx=None, stream=None) -> None:
    _check(_lib.hga_decode(_addr(q), n_q_heads, ctypes.byref(kv), _addr(chunk_sum), _addr(group_sum),
                           ctypes.byref(p), _addr(out), _addr(lse), _addr(idx), idx_stride, _addr(n_idx),
                           _stream(stream)), "hga_decode")


def hga_decode_workspace_size(kv: hga_kv, n_q_heads: int, p: hga_params) -> int:
    n = _lib.hga_decode_workspace_size(ctypes.byref(kv), n_q_heads, ctypes.byref(p))
    if n == 0:
        raise HgaError(1, "hga_decode_workspace_size")
    return int(n)


def hga_decode_ws(q, n_q_heads: int, kv: hga_kv, chunk_sum, group_sum, p: hga_params, out, lse, idx,
                  idx_stride: int, n_idx, workspace, workspace_bytes: int, stream=None) -> None:
    _check(_lib.hga_decode_ws(_addr(q), n_q_heads, ctypes.byref(kv), _addr(chunk_sum), _addr(group_sum),
                              ctypes.byref(p), _addr(out), _addr(lse), _addr(idx), idx_stride, _addr(n_idx),
                              _addr(workspace), workspace_bytes, _stream(stream)), "hga_decode_ws")


def hga_route_blocks(q, n_q_heads: int, n_queries: int, block: int, kv: hga_kv, cache_len: int, chunk_sum,
                     group_sum, p: hga_params, idx, idx_stride: int, n_idx, stream=None) -> None:
    _check(_lib.hga_route_blocks(_addr(q), n_q_heads, n_queries, block, ctypes.byref(kv), cache_len,
                                 _addr(chunk_sum), _addr(group_sum), ctypes.byref(p), _addr(idx), idx_stride,
                                 _addr(n_idx), _stream(stream)), "hga_route_blocks")


def hga_prefill_attend(q, n_q_heads: int, n_queries: int, block: int, kv: hga_kv, cache_len: int, idx,
                       idx_stride: int, n_idx, p: hga_params, out, stream=None) -> None:
    _check(_lib.hga_prefill_attend(_addr(q), n_q_heads, n_queries, block, ctypes.byref(kv), cache_len, _addr(idx),
                                   idx_stride, _addr(n_idx), ctypes.byref(p), _addr(out), _stream(stream)),
           "hga_prefill_attend")


def hga_prefill_workspace_size(kv: hga_kv, n_q_heads: int, n_queries: int, block: int, cache_len: int,
                               p: hga_params) -> int:
    n = _lib.hga_prefill_workspace_size(ctypes.byref(kv), n_q_heads, n_queries, block, cache_len, ctypes.byref(p))
    if n == 0:
        raise HgaError(1, "hga_prefill_workspace_size")
    return n


def hga_prefill(q, n_q_heads: int, n_queries: int, block: int, kv: hga_kv, cache_len: int, chunk_sum, group_sum,
                p: hga_params, out, workspace, workspace_bytes: int, stream=None) -> None:
    _check(_lib.hga_prefill(_addr(q), n_q_heads, n_queries, block, ctypes.byref(kv), cache_len, _addr(chunk_sum),
                            _addr(group_sum), ctypes.byref(p), _addr(out), _addr(workspace), workspace_bytes,
                            _stream(stream)), "hga_prefill")


def hga_prefill_noalloc(q, n_q_heads: int, n_queries: int, block: int, kv: hga_kv, cache_len: int, chunk_sum,
                        group_sum, p: hga_params, out, stream=None) -> None:
    """hga_prefill without a workspace, for callers that cannot allocate device memory
    (the routed lists live in a 2 MiB array inside the library; see hga.h)."""
    _check(_lib.hga_prefill_noalloc(_addr(q), n_q_heads, n_queries, block, ctypes.byref(kv), cache_len,
                                    _addr(chunk_sum), _addr(group_sum), ctypes.byref(p), _addr(out),
                                    _stream(stream)), "hga_prefill_noalloc")


def hga_append(kv: hga_kv, seq_lens, k_new, v_new, p: hga_params, chunk_sum, group_sum, stream=None) -> None:
    """Append one token per sequence (k_new, v_new [B][Hkv][d] bf16) and refresh the completed chunk's
    summaries; seq_lens (kv's length array) grows by one on the device."""
    _check(_lib.hga_append(ctypes.byref(kv), _addr(seq_lens), _addr(k_new), _addr(v_new), ctypes.byref(p),
                           _addr(chunk_sum), _addr(group_sum), _stream(stream)), "hga_append")


def hga_route_blocks_growing(q, n_q_heads: int, n_queries: int, block: int, kv: hga_kv, cache_len: int,
                             chunk_sum, group_sum, p: hga_params, idx, idx_stride: int, n_idx, stream=None) -> None:
    _check(_lib.hga_route_blocks_growing(_addr(q), n_q_heads, n_queries, block, ctypes.byref(kv), cache_len,
                                         _addr(chunk_sum), _addr(group_sum), ctypes.byref(p), _addr(idx),
                                         idx_stride, _addr(n_idx), _stream(stream)), "hga_route_blocks_growing")


def hga_prefill_growing_workspace_size(kv: hga_kv, n_q_heads: int, n_queries: int, block: int, cache_len: int,
                                       p: hga_params) -> int:
    n = _lib.hga_prefill_growing_workspace_size(ctypes.byref(kv), n_q_heads, n_queries, block, cache_len,
                                                ctypes.byref(p))
    if n == 0:
        raise HgaError(1, "hga_prefill_growing_workspace_size")
    return n


def hga_prefill_growing(q, n_q_heads: int, n_queries: int, block: int, kv: hga_kv, cache_len: int, chunk_sum,
                        group_sum, p: hga_params, out, workspace, workspace_bytes: int, stream=None) -> None:
    _check(_lib.hga_prefill_growing(_addr(q), n_q_heads, n_queries, block, ctypes.byref(kv), cache_len,
                                    _addr(chunk_sum), _addr(group_sum), ctypes.byref(p), _addr(out),
                                    _addr(workspace), workspace_bytes, _stream(stream)), "hga_prefill_growing")


def hga_host_kv_pointer(host_tensor) -> int:
    """Device address of a pinned, mapped host buffer (a pinned CPU torch tensor or a raw address), for
    hga_kv.k / hga_kv.v of a host-resident cache."""
    dev = ctypes.c_void_p(0)
    _check(_lib.hga_host_kv_pointer(_addr(host_tensor), ctypes.byref(dev)), "hga_host_kv_pointer")
    return int(dev.value)


def hga_decode_hisa(q, n_q_heads: int, kv: hga_kv, chunk_sum, p: hga_params, top_tokens: int, out, lse=None,
                    idx=None, idx_stride: int = 0, n_idx=None, stream=None) -> None:
    """Block-then-token routed decode: top chunks by summary, then the top_tokens tokens inside them."""
    _check(_lib.hga_decode_hisa(_addr(q), n_q_heads, ctypes.byref(kv), _addr(chunk_sum), ctypes.byref(p),
                                top_tokens, _addr(out), _addr(lse), _addr(idx), idx_stride, _addr(n_idx),
                                _stream(stream)), "hga_decode_hisa")


def hga_decode_hisa_workspace_size(kv: hga_kv, p: hga_params) -> int:
    n = _lib.hga_decode_hisa_workspace_size(ctypes.byref(kv), ctypes.byref(p))
    if n == 0:
        raise HgaError(1, "hga_decode_hisa_workspace_size")
    return int(n)


def hga_decode_hisa_ws(q, n_q_heads: int, kv: hga_kv, chunk_sum, p: hga_params, top_tokens: int, out, workspace,
                       workspace_bytes: int, lse=None, idx=None, idx_stride: int = 0, n_idx=None,
                       stream=None) -> None:
    """hga_decode_hisa with a logits workspace: the kept tokens' K is read once."""
    _check(_lib.hga_decode_hisa_ws(_addr(q), n_q_heads, ctypes.byref(kv), _addr(chunk_sum), ctypes.byref(p),
                                   top_tokens, _addr(out), _addr(lse), _addr(idx), idx_stride, _addr(n_idx),
                                   _addr(workspace), workspace_bytes, _stream(stream)), "hga_decode_hisa_ws")


def hga_max_hisa_tokens(kv: hga_kv, p: hga_params, top_tokens: int) -> int:
    n = _lib.hga_max_hisa_tokens(ctypes.byref(kv), ctypes.byref(p), top_tokens)
    if n < 0:
        raise HgaError(1, "hga_max_hisa_tokens")
    return n


def hga_set_launch_option(option: int, value: int) -> None:
    _check(_lib.hga_set_launch_option(option, value), "hga_set_launch_option")


def hga_get_device_error(stream=None) -> tuple[int, int]:
    """(status, raw error bits); synchronises the stream and clears the word."""
    bits = ctypes.c_int32(0)
    st = _lib.hga_get_device_error(_stream(stream), ctypes.byref(bits))
    return st, bits.value
