"""Buffer ownership for one decode layer: the caller-side plumbing around the C ABI.

``LayerCache`` holds the per-layer retrieval metadata (page summaries, codes,
block means) next to the caller's K/V cache; ``DecodeStep`` owns the workspaces
and outputs of one decode step and runs append-encode -> select -> sparse
attention through the C ABI on one stream. PyTorch only allocates memory here;
every step of the path runs in the library's kernels.
"""
from __future__ import annotations

import math

import torch

from . import hhr


class LayerCache:
    """Retrieval metadata of one layer, laid out as include/hhr.h documents."""

    def __init__(self, d: hhr.Dims, device, hashing=True, block_means=False):
        n, G, P = d.n_phys_pages, d.n_kv_heads, d.page_size
        # Zero-filled, so that slots past a sequence's end have deterministic contents.
        sdt = torch.float16 if d.summary_fp16 else torch.float32
        self.page_minmax = (torch.zeros(n, G, 2, d.head_dim, dtype=sdt, device=device)
                            if hashing else None)
        self.codes = (torch.zeros(n, G, P, d.code_bits // 32, dtype=torch.int32, device=device)
                      if hashing else None)
        self.block_mean = (torch.zeros(n, G, d.head_dim, dtype=torch.float32, device=device)
                           if block_means else None)


class DecodeStep:
    """Workspaces and outputs of one decode step (hash mode) or one selection (indexer)."""

    def __init__(self, d: hhr.Dims, mode: int, m_pages: int, keep_div: int, top_k: int, device,
                 attention: bool = True, sink_pages: int = 0, local_pages: int = 0):
        self.d, self.mode, self.m_pages, self.keep_div, self.top_k = d, mode, m_pages, keep_div, top_k
        self.opts = hhr.make_opts(sink_pages, local_pages)  # forced pages (hash mode variant)
        rows = hhr.sel_rows(d) if mode == hhr.HHR_MODE_HASH else d.n_q_heads
        ws = hhr.hhr_select_workspace_bytes(d, mode, m_pages, keep_div, top_k)
        if ws == 0:
            raise ValueError("unsupported selection parameters")
        self.sel_ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.idx = torch.empty(d.batch, rows, top_k, dtype=torch.int32, device=device)
        self.count = torch.empty(d.batch, rows, dtype=torch.int32, device=device)
        self.m_max = hhr.hhr_kept_max(d, m_pages, keep_div)
        self.attention = attention and mode == hhr.HHR_MODE_HASH
        self.fused_ws = None
        if self.attention:
            aws = hhr.hhr_attn_workspace_bytes(d, top_k)
            self.attn_ws = torch.empty(aws, dtype=torch.uint8, device=device)
            self.out = torch.empty(d.batch, d.n_q_heads, d.head_dim, dtype=torch.float32,
                                   device=device)

    def encode(self, k_cache, page_table, start, n_new, max_new, R, W, cache: LayerCache,
               stream=None):
        hhr.hhr_encode_keys(self.d, k_cache, page_table, start, n_new, max_new, R, W,
                            cache.page_minmax, cache.codes, cache.block_mean, stream)

    def select(self, q, seq_len, page_table, cache: LayerCache, R=None, W=None, k_cache=None,
               q_pos=None, trace=None, stream=None):
        hhr.hhr_select(self.d, self.mode, q, seq_len, q_pos, page_table, R, W, cache.page_minmax,
                       cache.codes, cache.block_mean, k_cache, self.m_pages, self.keep_div,
                       self.top_k, self.idx, self.count, self.sel_ws, trace, stream, self.opts)

    def attend(self, q, k_cache, v_cache, page_table, seq_len, scale=None, stream=None):
        if scale is None:
            scale = 1.0 / math.sqrt(self.d.head_dim)
        hhr.hhr_sparse_attn(self.d, q, k_cache, v_cache, page_table, seq_len, self.idx,
                            self.count, self.top_k, scale, self.out, self.attn_ws, stream)

    def fused_step(self, q, k_cache, v_cache, page_table, seq_len, R, W, cache: LayerCache,
                   k_new=None, v_new=None, scale=None, stream=None):
        """One decode step through hhr_decode_step (the fused single-call path)."""
        if self.fused_ws is None:
            n = hhr.hhr_decode_step_workspace_bytes(self.d, self.m_pages, self.keep_div,
                                                    self.top_k)
            self.fused_ws = torch.empty(n, dtype=torch.uint8, device=self.idx.device)
        if scale is None:
            scale = 1.0 / math.sqrt(self.d.head_dim)
        hhr.hhr_decode_step(self.d, q, k_new, v_new, k_cache, v_cache, page_table, seq_len, R, W,
                            cache.page_minmax, cache.codes, self.m_pages, self.keep_div,
                            self.top_k, scale, self.idx, self.count, self.out, self.fused_ws,
                            stream, self.opts)
        return self.out

    def step(self, q, k_cache, v_cache, page_table, seq_len, R, W, cache: LayerCache,
             append_start, append_n, stream=None):
        """One HHR decode step: encode the appended key(s), select, attend."""
        self.encode(k_cache, page_table, append_start, append_n, 1, R, W, cache, stream)
        self.select(q, seq_len, page_table, cache, R=R, W=W, stream=stream)
        self.attend(q, k_cache, v_cache, page_table, seq_len, stream=stream)
        return self.out
