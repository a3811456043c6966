"""Device-side checks: bad page ids and token indices are skipped and reported, never a fault.

The out-of-range values below are caught by the kernels' own bounds checks (every
page id is compared with n_phys_pages and every token with seq_len before use).
"""
import numpy as np
import pytest
import torch

import hhr_synth as S
from hash_hierarchical_top_b200 import hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
from parity_helpers import dims_of

pytestmark = pytest.mark.gpu


def test_bad_page_id_is_flagged():
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(2000,), top_k=100)
    inp = S.make_inputs(wl, device="cuda")
    d = dims_of(wl, inp)
    cache = LayerCache(d, "cuda")
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    hhr.hhr_read_device_status()
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    step.encode(inp["k_cache"], inp["page_table"], z, inp["seq_len"], 2000, inp["R"], inp["W"],
                cache)
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    pt = inp["page_table"].clone()
    pt[0, 5] = d.n_phys_pages + 7
    step.select(inp["q"], inp["seq_len"], pt, cache, R=inp["R"], W=inp["W"])
    step.attend(inp["q"], inp["k_cache"], inp["v_cache"], pt, inp["seq_len"])
    st, bits = hhr.hhr_read_device_status()
    assert st == hhr.HHR_ERR_DEVICE_STATUS and bits & 1
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)   # cleared


def test_bad_token_index_is_flagged():
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(2000,), top_k=100)
    inp = S.make_inputs(wl, device="cuda")
    d = dims_of(wl, inp)
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    step.idx.copy_(torch.arange(100, dtype=torch.int32).repeat(1, 8, 1))
    step.idx[0, 3, 10] = 2000 + 5
    step.count.fill_(100)
    hhr.hhr_read_device_status()
    step.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_len"])
    st, bits = hhr.hhr_read_device_status()
    assert st == hhr.HHR_ERR_DEVICE_STATUS and bits & 2
    assert torch.isfinite(step.out).all()
