"""The allocation-free attention entry point (hhr_sparse_attn_noalloc).

Some callers cannot allocate device memory when they call the library: a runtime
with no device allocator of its own, code that runs while a memory pool is frozen,
or a plugin whose host forbids cudaMalloc. For them the library keeps the
attention's split-K scratch in a fixed 8 MiB device array. This test calls that
entry point through the C ABI twice in a row and compares each result with the
regular entry point (which takes a caller workspace), within the attention
tolerance used by the parity tests. It lives in its own file, collected last, and
passes both alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import hhr_synth as S
from hash_hierarchical_top_b200 import build, hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3


def _rel_err(a, b):
    a = a.double()
    b = b.double()
    den = b.abs().amax(dim=-1).clamp_min(1e-30)
    return float(((a - b).abs().amax(dim=-1) / den).max())


def _selected(wl, layer):
    inp = S.make_inputs(wl, device="cuda", layer=layer)
    d = hhr.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.page_size, inp["max_pages"],
                      inp["n_phys"])
    cache = LayerCache(d, "cuda")
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    zero = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    step.encode(inp["k_cache"], inp["page_table"], zero, inp["seq_len"],
                int(inp["seq_len"].max()), inp["R"], inp["W"], cache)
    step.select(inp["q"], inp["seq_len"], inp["page_table"], cache, R=inp["R"], W=inp["W"])
    return inp, d, step


def test_noalloc_matches_workspace_entry_point_twice():
    build.build()
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], batch=2, seq_lens=(9000, 6000), top_k=1000)
    for call, layer in enumerate((0, 1)):
        inp, d, step = _selected(wl, layer)
        scale = 1.0 / np.sqrt(128.0)
        step.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_len"],
                    scale)
        ref = step.out.clone()
        out = torch.full_like(ref, float("nan"))
        hhr.hhr_sparse_attn_noalloc(d, inp["q"], inp["k_cache"], inp["v_cache"],
                                    inp["page_table"], inp["seq_len"], step.idx, step.count,
                                    wl.top_k, scale, out)
        torch.cuda.synchronize()
        assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
        assert torch.isfinite(out).all(), f"call {call}: non-finite output"
        err = _rel_err(out, ref)
        assert err <= ATTN_TOL, f"call {call}: max relative error {err}"


def test_noalloc_rejects_sizes_beyond_the_array():
    build.build()
    L = hhr.lib()
    # Grow the batch (8 KV heads, 8-head groups, top_k 8192) until the split-K partials
    # no longer fit in the 8 MiB array.
    batch = 32
    while True:
        d = hhr.make_dims(batch, 64, 8, 32, 4096, 4096 * 32)
        if hhr.hhr_attn_workspace_bytes(d, 8192) > 8 * 1024 * 1024:
            break
        batch *= 2
        assert batch <= 65535
    p = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    st = L.hhr_sparse_attn_noalloc(ctypes.byref(d), p, p, p, p, p, p, p, 8192,
                                   ctypes.c_float(0.1), p, None)
    assert st == hhr.HHR_ERR_WORKSPACE
