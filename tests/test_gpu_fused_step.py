"""hhr_decode_step (one fused call) against the separate calls it replaces: encode the newest
key, select, attend. Same kernels' arithmetic, so every output must be bit-identical."""
import numpy as np
import pytest
import torch

import hhr_synth as S
from hash_hierarchical_top_b200 import build, hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
from parity_helpers import check_hash_group, dims_of

pytestmark = pytest.mark.gpu


def _prefill(wl, inp, d, upto):
    """Encode positions [0, upto[b]) of every sequence; returns the cache."""
    cache = LayerCache(d, "cuda")
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda",
                     sink_pages=wl.sink_pages, local_pages=wl.local_pages)
    z = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    step.encode(inp["k_cache"], inp["page_table"], z, upto, int(upto.max()), inp["R"], inp["W"],
                cache)
    return cache


@pytest.mark.parametrize("f16", [0, 1])
@pytest.mark.parametrize("with_new_rows", [False, True])
def test_fused_step_equals_separate_calls(f16, with_new_rows):
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=5, ragged=(33, 6000), top_k=300)
    _fused_vs_separate(wl, f16, with_new_rows)


@pytest.mark.parametrize("heads", [(8, 1), (8, 8), (10, 2), (6, 2), (14, 2)])
def test_fused_step_group_shapes(heads):
    """Every group size has its own prologue instantiation: each must match."""
    hq, g = heads
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=3, ragged=(33, 4000), top_k=200,
                  n_q_heads=hq, n_kv_heads=g)
    _fused_vs_separate(wl, 1, True)


@pytest.mark.parametrize("bits", [64, 256])
@pytest.mark.parametrize("heads", [(32, 8), (8, 1), (14, 2)])
def test_fused_step_code_lengths(bits, heads):
    """64- and 256-bit codes: the prologue projects 2 words on ranks 0-1, or 2 words on
    every rank, and must match the separate encoder and query prep bit for bit."""
    hq, g = heads
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=3, ragged=(33, 4000), top_k=200,
                  n_q_heads=hq, n_kv_heads=g, code_bits=bits)
    _fused_vs_separate(wl, 1, True)


@pytest.mark.parametrize("bits", [64, 128])
def test_fused_step_flat(bits):
    """Flat hash top-k (every page kept): no page-bound kernel in either path."""
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=3, ragged=(33, 6000), top_k=300,
                  m_pages=4096, keep_div=0, code_bits=bits)
    _fused_vs_separate(wl, 1, True)


@pytest.mark.parametrize("forced", [(1, 2), (0, 3)])
def test_fused_step_forced_pages(forced):
    """Forced sink/local pages: the fused call equals the separate calls."""
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=4, ragged=(33, 6000), top_k=300,
                  sink_pages=forced[0], local_pages=forced[1])
    _fused_vs_separate(wl, 1, True)


def test_fused_step_many_rows():
    """192 top-m + Hamming CTAs (more than the SMs): the 512-thread instantiation."""
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=12, ragged=(33, 3000), top_k=200)
    _fused_vs_separate(wl, 1, True)


@pytest.mark.parametrize("heads", [(32, 8), (8, 1)])
def test_fused_step_per_head(heads):
    """One selection per query head: the fused call equals the separate calls."""
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=3, ragged=(33, 4000), top_k=200,
                  n_q_heads=heads[0], n_kv_heads=heads[1], select_per_head=True)
    _fused_vs_separate(wl, 1, True)


@pytest.mark.parametrize("case", ["groups", "f32", "forced", "per_head", "flat", "gs2",
                                  "short_seq"])
def test_fused_step_row_cluster(case):
    """Small batches run steps a2-a5 as one cluster of 16 or 8 CTAs per selection row (2
    kernels per call). With at most 8 attention splits per row in both plans (top-k <= 512),
    the fused call equals the separate calls bit for bit."""
    kw = dict(batch=1, ragged=(12000, 20000), top_k=512)
    f16 = 1
    if case == "f32":
        f16 = 0
    elif case == "forced":
        kw.update(sink_pages=1, local_pages=2)
    elif case == "per_head":
        kw.update(n_q_heads=8, n_kv_heads=1, select_per_head=True)
    elif case == "flat":
        kw.update(m_pages=4096, keep_div=0, ragged=(5000, 9000), top_k=512)
    elif case == "gs2":
        kw.update(batch=2, n_q_heads=8, n_kv_heads=4, top_k=448)
    elif case == "short_seq":
        kw.update(batch=4, n_q_heads=4, n_kv_heads=2, ragged=(33, 3000), top_k=300)
    wl = S.scaled(S.WORKLOADS["ragged_b32"], **kw)
    _fused_vs_separate(wl, f16, True, expect_kernels=2)


def _fused_vs_separate(wl, f16, with_new_rows, expect_kernels=None):
    build.build()
    inp = S.make_inputs(wl, device="cuda")
    d = dims_of(wl, inp, f16)
    if expect_kernels is not None:
        assert hhr.hhr_decode_step_kernels(d, wl.m_pages, wl.keep_div, wl.top_k) == expect_kernels
    lens = inp["seq_len"]
    G, P = wl.n_kv_heads, wl.page_size
    # The newest row of each sequence: remember it, and (for the k_new path) wipe it from
    # the caches so that only the fused call can put it back.
    t = (lens - 1).long()
    pt = inp["page_table"].long()
    phys = pt[torch.arange(wl.batch, device="cuda"), t // P]
    k_new = inp["k_cache"][phys, :, t % P].contiguous()
    v_new = inp["v_cache"][phys, :, t % P].contiguous()

    # Reference: separate calls.
    ref_cache = _prefill(wl, inp, d, lens - 1)
    ref = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda",
                     sink_pages=wl.sink_pages, local_pages=wl.local_pages)
    one = torch.ones(wl.batch, dtype=torch.int32, device="cuda")
    ref.step(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], lens, inp["R"],
             inp["W"], ref_cache, (lens - 1).to(torch.int32), one)

    # Fused.
    cache = _prefill(wl, inp, d, lens - 1)
    kc, vc = inp["k_cache"].clone(), inp["v_cache"].clone()
    if with_new_rows:
        kc[phys, :, t % P] = 0
        vc[phys, :, t % P] = 0
    fs = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda",
                     sink_pages=wl.sink_pages, local_pages=wl.local_pages)
    fs.fused_step(inp["q"], kc, vc, inp["page_table"], lens, inp["R"], inp["W"], cache,
                  k_new=k_new if with_new_rows else None, v_new=v_new if with_new_rows else None)
    torch.cuda.synchronize()
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    assert torch.equal(kc, inp["k_cache"]) and torch.equal(vc, inp["v_cache"])
    assert torch.equal(cache.codes, ref_cache.codes)
    assert torch.equal(cache.page_minmax, ref_cache.page_minmax)
    assert torch.equal(fs.count, ref.count)
    assert torch.equal(fs.idx, ref.idx)
    assert torch.equal(fs.out.view(torch.int32), ref.out.view(torch.int32))


@pytest.mark.parametrize("variant", ["hierarchical", "flat", "forced", "per_head"])
def test_fused_step_against_oracle(variant):
    """The fused call's outputs through the layered oracle checks (selection + attention)."""
    build.build()
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(7777,), top_k=700)
    if variant == "flat":
        wl = S.scaled(wl, m_pages=4096, keep_div=0)
    elif variant == "forced":
        wl = S.scaled(wl, sink_pages=2, local_pages=4)
    elif variant == "per_head":
        wl = S.scaled(wl, select_per_head=True)
    inp = S.make_inputs(wl, device="cuda")
    inp_np = S.to_numpy_inputs(inp)
    d = dims_of(wl, inp, 1)
    cache = _prefill(wl, inp, d, inp["seq_len"] - 1)
    fs = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda",
                     sink_pages=wl.sink_pages, local_pages=wl.local_pages)
    B, Hq = wl.batch, wl.n_q_heads
    tr = dict(q_rot=torch.empty(B, Hq, 128, device="cuda"),
              q_code=torch.empty(B, Hq, wl.code_bits // 32, dtype=torch.int32, device="cuda"))
    fs.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_len"],
                  inp["R"], inp["W"], cache)
    torch.cuda.synchronize()
    # Intermediates live in the fused workspace; recompute them with the select call to
    # feed the layered checks (the fused selection must equal it).
    sel = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda",
                     sink_pages=wl.sink_pages, local_pages=wl.local_pages)
    rows = hhr.sel_rows(d)
    bounds = torch.empty(B, rows, d.max_pages_per_seq, device="cuda")
    kept = torch.empty(B, rows, sel.m_max, dtype=torch.int32, device="cuda")
    kc = torch.empty(B, rows, dtype=torch.int32, device="cuda")
    trace = hhr.make_trace(q_rot=tr["q_rot"], q_code=tr["q_code"], bounds=bounds, kept=kept,
                           kept_count=kc)
    sel.select(inp["q"], inp["seq_len"], inp["page_table"], cache, R=inp["R"], W=inp["W"],
               trace=trace)
    torch.cuda.synchronize()
    assert torch.equal(sel.idx, fs.idx) and torch.equal(sel.count, fs.count)
    g_out = dict(idx=fs.idx.cpu().numpy(), count=fs.count.cpu().numpy(),
                 out=fs.out.cpu().numpy(), page_minmax=cache.page_minmax.float().cpu().numpy(),
                 summary_fp16=True, codes=cache.codes.cpu().numpy().view(np.uint32),
                 q_rot=tr["q_rot"].cpu().numpy(),
                 q_code=tr["q_code"].cpu().numpy().view(np.uint32),
                 bounds=bounds.cpu().numpy(), kept=kept.cpu().numpy(),
                 kept_count=kc.cpu().numpy())
    rep = {}
    for g in range(wl.n_kv_heads):
        check_hash_group(wl, inp_np, g_out, 0, g, rep)
