"""hhr_decode_step, the call the benchmark times, against the fp64 oracle on the full-size
configurations: Llama-3.1-8B shapes at 128K context and batch 8 (4096 pages of 32 keys per
sequence, keep 1/16, top-2048, 128-bit codes, f16 summaries), the same at batch 1 and at 32K
context (keep 1/8, top-3276; on the small-batch path, one cluster per selection row),
and the ragged batch of 32 sequences of 8K..128K keys in a permuted page pool (top-1024).

The cache is built as a serving loop holds it at a decode step: positions [0, n - 1) of every
sequence are prefilled with the bulk (tensor-core) encoder, and the newest key/value rows are
handed to hhr_decode_step, which writes them into the cache, encodes the key, selects and
attends. The fused call's selection must equal hhr_select's on the resulting cache bit for
bit; hhr_select's trace then feeds the layered oracle checks (codes, summaries, rotated
queries, bounds, kept pages, Hamming top-k, attention) of sampled (sequence, KV group) rows.
The oracle is run on a sample because it takes seconds per row at 128K keys.
"""
import numpy as np
import pytest
import torch

import hhr_synth as S
from hash_hierarchical_top_b200 import build, hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
from parity_helpers import check_hash_group, dims_of

pytestmark = pytest.mark.gpu


def _decode_step_outputs(wl, expect_kernels=None):
    build.build()
    inp = S.make_inputs(wl, device="cuda")
    d = dims_of(wl, inp, 1)
    B, P, Hq = wl.batch, wl.page_size, wl.n_q_heads
    lens = inp["seq_len"]
    t = (lens - 1).long()
    phys = inp["page_table"].long()[torch.arange(B, device="cuda"), t // P]
    k_new = inp["k_cache"][phys, :, t % P].clone()
    v_new = inp["v_cache"][phys, :, t % P].clone()
    # The newest rows are not in the cache yet: only the decode step can put them there.
    inp["k_cache"][phys, :, t % P] = 0
    inp["v_cache"][phys, :, t % P] = 0
    if expect_kernels is not None:
        assert hhr.hhr_decode_step_kernels(d, wl.m_pages, wl.keep_div, wl.top_k) == expect_kernels
    cache = LayerCache(d, "cuda")
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    prev = (lens - 1).to(torch.int32)
    step.encode(inp["k_cache"], inp["page_table"], z, prev, int(prev.max()), inp["R"], inp["W"],
                cache)
    step.out.fill_(float("nan"))
    step.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], lens, inp["R"],
                    inp["W"], cache, k_new=k_new, v_new=v_new)
    torch.cuda.synchronize()
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    assert torch.equal(inp["k_cache"][phys, :, t % P], k_new)
    assert torch.equal(inp["v_cache"][phys, :, t % P], v_new)
    assert torch.isfinite(step.out).all()
    # Intermediates for the layered checks: hhr_select on the cache the step left behind.
    sel = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    rows = hhr.sel_rows(d)
    tr = dict(q_rot=torch.empty(B, Hq, 128, device="cuda"),
              q_code=torch.empty(B, Hq, wl.code_bits // 32, dtype=torch.int32, device="cuda"),
              bounds=torch.empty(B, rows, d.max_pages_per_seq, device="cuda"),
              kept=torch.empty(B, rows, sel.m_max, dtype=torch.int32, device="cuda"),
              kept_count=torch.empty(B, rows, dtype=torch.int32, device="cuda"))
    sel.select(inp["q"], lens, inp["page_table"], cache, R=inp["R"], W=inp["W"],
               trace=hhr.make_trace(**tr))
    torch.cuda.synchronize()
    assert torch.equal(sel.count, step.count), "fused selection counts differ from hhr_select"
    assert torch.equal(sel.idx, step.idx), "fused selection differs from hhr_select"
    g_out = dict(idx=step.idx.cpu().numpy(), count=step.count.cpu().numpy(),
                 out=step.out.cpu().numpy(), page_minmax=cache.page_minmax.float().cpu().numpy(),
                 summary_fp16=True, codes=cache.codes.cpu().numpy().view(np.uint32),
                 q_rot=tr["q_rot"].cpu().numpy(), q_code=tr["q_code"].cpu().numpy().view(np.uint32),
                 bounds=tr["bounds"].cpu().numpy(), kept=tr["kept"].cpu().numpy(),
                 kept_count=tr["kept_count"].cpu().numpy())
    return inp, g_out


def test_decode_step_llama8b_128k_batch8():
    """Every one of the 8 sequences, each on its own KV group (groups 0..7), plus groups 7 and 0
    of the first and last sequences."""
    wl = S.WORKLOADS["llama8b_128k_b8"]
    inp, g_out = _decode_step_outputs(wl)
    assert np.all(g_out["count"] == wl.top_k)
    inp_np = S.to_numpy_inputs(inp)
    rep = {}
    for b, g in [(b, b) for b in range(8)] + [(0, 7), (7, 0)]:
        check_hash_group(wl, inp_np, g_out, b, g, rep)
    print(rep)


def test_decode_step_ragged_batch32():
    """The shortest and the longest sequence, and six others, each on two KV groups."""
    wl = S.WORKLOADS["ragged_b32"]
    inp, g_out = _decode_step_outputs(wl)
    inp_np = S.to_numpy_inputs(inp)
    lens = inp_np["seq_len"]
    order = np.argsort(lens, kind="stable")
    picks = [int(order[0]), int(order[-1])] + [int(order[i]) for i in (4, 9, 14, 19, 24, 28)]
    rep = {}
    for j, b in enumerate(picks):
        for g in (j % 8, (j + 5) % 8):
            check_hash_group(wl, inp_np, g_out, b, g, rep)
    print(rep)


def test_decode_step_llama8b_128k_batch1():
    """One sequence at 128K (32768 pages over its 8 KV groups: the kernel chain, not the
    row-cluster path). Every group."""
    wl = S.WORKLOADS["llama8b_128k_b1"]
    inp, g_out = _decode_step_outputs(wl, expect_kernels=4)
    assert np.all(g_out["count"] == wl.top_k)
    inp_np = S.to_numpy_inputs(inp)
    rep = {}
    for g in range(8):
        check_hash_group(wl, inp_np, g_out, 0, g, rep)
    print(rep)


def test_decode_step_llama8b_32k():
    """32K context, keep 1/8 (128 of 1024 pages), top-3276 over the 4096 kept keys; small-batch
    path. Groups 0, 3 and 7."""
    wl = S.WORKLOADS["llama8b_32k"]
    inp, g_out = _decode_step_outputs(wl, expect_kernels=2)
    inp_np = S.to_numpy_inputs(inp)
    rep = {}
    for g in (0, 3, 7):
        check_hash_group(wl, inp_np, g_out, 0, g, rep)
    print(rep)
