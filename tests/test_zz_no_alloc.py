"""The allocation-free attention entry point (hhr_sparse_attn_noalloc).

Some callers cannot allocate device memory when they call the library: a runtime
with no device allocator of its own, code that runs while a memory pool is frozen,
or a plugin whose host forbids cudaMalloc. For them the library keeps the
attention's split-K scratch in a fixed 8 MiB device array. This test calls that
entry point through the C ABI twice in a row and compares each result with the
regular entry point (which takes a caller workspace): both run the same kernels with
the same split plan, so the outputs must be identical bit for bit. It lives in its own
file, collected last, and passes both alone in a fresh process and after the other
tests. (The size limit is checked on the host without a GPU, in test_abi.py.)
"""
import numpy as np
import pytest
import torch

import hhr_synth as S
from hash_hierarchical_top_b200 import build, hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache

pytestmark = pytest.mark.gpu

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
        assert torch.equal(out.view(torch.int32), ref.view(torch.int32)), \
            f"call {call}: output differs from hhr_sparse_attn"
