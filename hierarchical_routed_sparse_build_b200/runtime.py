"""Device-side plumbing around the C ABI: torch-owned buffers for one K/V cache.

``RoutedCache`` keeps a K/V cache (contiguous or paged), its sequence lengths and
its summary buffers on the GPU, and forwards to the libhga calls. It allocates
with torch and performs no arithmetic of its own.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (hga_append, hga_attend, hga_build_summaries, hga_decode_hisa, hga_decode_hisa_workspace_size,
               hga_decode_hisa_ws, hga_decode_workspace_size, hga_decode_ws,
               hga_max_hisa_tokens, hga_max_routed_tokens, hga_route, hga_summary_bytes, make_kv, make_params)


def _dev_u16(a: np.ndarray, device) -> torch.Tensor:
    """bfloat16 bit patterns (numpy uint16) -> torch.bfloat16 on device, same bytes."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to(device=device, non_blocking=False).view(torch.bfloat16)


class RoutedCache:
    """One K/V cache with its routing summaries, resident in GPU memory.

    Contiguous: k, v are [B][Hkv][max_len][d]. Paged: k, v are a page pool
    [P][Hkv][page][d] with page_table [B][max_pages]. Arrays may be numpy uint16
    bfloat16 patterns (copied to the device) or bfloat16 CUDA tensors (used as is).
    """

    def __init__(self, k, v, seq_lens, *, chunk: int, group: int, top_chunks: int, top_groups: int,
                 n_q_heads: int, scale: float = 0.0, page_table=None, device="cuda"):
        self.device = torch.device(device)
        self.k = k if isinstance(k, torch.Tensor) else _dev_u16(k, self.device)
        self.v = v if isinstance(v, torch.Tensor) else _dev_u16(v, self.device)
        self.seq_lens = torch.as_tensor(np.asarray(seq_lens, dtype=np.int32)).to(self.device)
        self.paged = page_table is not None
        self.page_table = (torch.as_tensor(np.asarray(page_table, dtype=np.int32)).to(self.device)
                           if self.paged else None)
        if self.paged:
            n_pages, hkv, page, d = self.k.shape
            batch, max_pages = self.page_table.shape
            max_len = max_pages * page
        else:
            batch, hkv, max_len, d = self.k.shape
            n_pages, page, max_pages = 0, 0, 0
        self.batch, self.n_kv_heads, self.head_dim, self.max_len = batch, hkv, d, max_len
        self.n_q_heads = n_q_heads
        self.params = make_params(chunk, group, top_chunks, top_groups, scale)
        self.kv = make_kv(self.k, self.v, self.seq_lens, n_kv_heads=hkv, head_dim=d, max_len=max_len,
                          batch=batch, page_table=self.page_table, page_size=page, max_pages=max_pages,
                          num_pages=n_pages)
        cb, gb = hga_summary_bytes(self.kv, self.params)
        gpc = chunk // group
        if self.paged:
            self.chunk_sum = torch.zeros((n_pages, hkv, d), dtype=torch.bfloat16, device=self.device)
            self.group_sum = torch.zeros((n_pages, hkv, gpc, d), dtype=torch.bfloat16, device=self.device)
        else:
            nc = max_len // chunk
            self.chunk_sum = torch.zeros((batch, hkv, nc, d), dtype=torch.bfloat16, device=self.device)
            self.group_sum = torch.zeros((batch, hkv, nc, gpc, d), dtype=torch.bfloat16, device=self.device)
        assert self.chunk_sum.numel() * 2 == cb and self.group_sum.numel() * 2 == gb
        self.idx_stride = hga_max_routed_tokens(self.kv, self.params)
        # decode workspace (route lists and softmax partials of the balanced decode)
        with torch.cuda.device(self.device):
            self.ws_bytes = hga_decode_workspace_size(self.kv, n_q_heads, self.params)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)

    # -- buffers -----------------------------------------------------------------
    def q_tensor(self, q) -> torch.Tensor:
        return q if isinstance(q, torch.Tensor) else _dev_u16(q, self.device)

    def out_buffers(self, with_lse: bool = True):
        out = torch.empty((self.batch, self.n_q_heads, self.head_dim), dtype=torch.float32, device=self.device)
        lse = torch.empty((self.batch, self.n_q_heads), dtype=torch.float32, device=self.device) if with_lse else None
        return out, lse

    def idx_buffers(self):
        idx = torch.full((self.batch, self.n_kv_heads, self.idx_stride), -1, dtype=torch.int32, device=self.device)
        n_idx = torch.zeros((self.batch, self.n_kv_heads), dtype=torch.int32, device=self.device)
        return idx, n_idx

    # -- calls -------------------------------------------------------------------
    def build_summaries(self, stream=None) -> None:
        hga_build_summaries(self.kv, self.params, self.chunk_sum, self.group_sum, stream)

    def decode_hisa(self, q, top_tokens: int, out=None, lse=None, want_idx: bool = False, stream=None,
                    logits_workspace: bool = True):
        """Block-then-token routed decode (top chunks by summary, then the top_tokens tokens inside them).
        With logits_workspace (the default) the token step keeps its per-head logits in a workspace owned by
        this cache and the attention reads only V for the kept tokens (hga_decode_hisa_ws); without it the
        attention re-reads their K (hga_decode_hisa)."""
        q = self.q_tensor(q)
        if out is None:
            out, lse = self.out_buffers()
        idx = n_idx = None
        stride = 0
        if want_idx:
            stride = hga_max_hisa_tokens(self.kv, self.params, top_tokens)
            idx = torch.full((self.batch, self.n_kv_heads, max(stride, 1)), -1, dtype=torch.int32,
                             device=self.device)
            n_idx = torch.zeros((self.batch, self.n_kv_heads), dtype=torch.int32, device=self.device)
        if logits_workspace:
            if getattr(self, "hisa_workspace", None) is None:
                self.hisa_ws_bytes = hga_decode_hisa_workspace_size(self.kv, self.params)
                self.hisa_workspace = torch.empty(self.hisa_ws_bytes, dtype=torch.uint8, device=self.device)
            hga_decode_hisa_ws(q, self.n_q_heads, self.kv, self.chunk_sum, self.params, top_tokens, out,
                               self.hisa_workspace, self.hisa_ws_bytes, lse, idx,
                               max(stride, 1) if want_idx else 0, n_idx, stream)
        else:
            hga_decode_hisa(q, self.n_q_heads, self.kv, self.chunk_sum, self.params, top_tokens, out, lse, idx,
                            max(stride, 1) if want_idx else 0, n_idx, stream)
        return (out, lse, idx, n_idx) if want_idx else (out, lse)

    def append(self, k_new, v_new, stream=None) -> None:
        """One more token per sequence (k_new, v_new: [B][Hkv][d] bfloat16 on the device); the lengths grow on
        the device and a completed chunk's summaries are written (no host synchronisation: graph-capturable)."""
        hga_append(self.kv, self.seq_lens, k_new, v_new, self.params, self.chunk_sum, self.group_sum, stream)

    def route(self, q, idx=None, n_idx=None, stream=None):
        q = self.q_tensor(q)
        if idx is None:
            idx, n_idx = self.idx_buffers()
        hga_route(q, self.n_q_heads, self.kv, self.chunk_sum, self.group_sum, self.params, idx,
                  self.idx_stride, n_idx, stream)
        return idx, n_idx

    def attend(self, q, idx, n_idx, out=None, lse=None, stream=None):
        q = self.q_tensor(q)
        if out is None:
            out, lse = self.out_buffers()
        hga_attend(q, self.n_q_heads, self.kv, idx, idx.shape[-1], n_idx, self.params, out, lse, stream)
        return out, lse

    def decode(self, q, out=None, lse=None, idx=None, n_idx=None, want_idx: bool = False, stream=None):
        q = self.q_tensor(q)
        if out is None:
            out, lse = self.out_buffers()
        if want_idx and idx is None:
            idx, n_idx = self.idx_buffers()
        hga_decode_ws(q, self.n_q_heads, self.kv, self.chunk_sum, self.group_sum, self.params, out, lse,
                      idx, self.idx_stride if idx is not None else 0, n_idx, self.workspace, self.ws_bytes, stream)
        return (out, lse, idx, n_idx) if want_idx else (out, lse)
