"""Edge cases of the CUDA path that the oracle comparisons do not reach on their own:
an empty selection under both attention split plans, and f16 page summaries that
saturate to -inf (a key channel below the f16 range) on a channel where the group's
folded query is exactly zero."""
import math

import numpy as np
import pytest
import torch

import hhr_synth as S
import oracle
from hash_hierarchical_top_b200 import build, hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
from parity_helpers import BOUND_TOL, dims_of

O = oracle.hhr_oracle
pytestmark = pytest.mark.gpu


def _splits(d, top_k):
    """Split count of the attention plan, read back from the workspace size:
    rows * splits * gs * (d + 2) floats, each part rounded up to 256 bytes."""
    rows = d.batch * hhr.sel_rows(d)
    gs = d.n_q_heads // hhr.sel_rows(d)
    ws = hhr.hhr_attn_workspace_bytes(d, top_k)
    for ns in range(1, 4097):
        a = -(-rows * ns * gs * d.head_dim * 4 // 256) * 256
        b = -(-rows * ns * gs * 2 * 4 // 256) * 256
        if a + b == ws:
            return ns
    raise AssertionError("no split count matches the workspace size")


@pytest.mark.parametrize("top_k,one_split", [(64, True), (1024, False)])
def test_empty_selection_gives_zero_output(top_k, one_split):
    """A row whose selection is empty must come out as exact zeros, whether its group is
    attended in one split (no merge after it) or in several (merged by the combine kernel);
    every other row is unchanged, bit for bit."""
    build.build()
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], batch=2, seq_lens=(3000, 2500), top_k=top_k)
    inp = S.make_inputs(wl, device="cuda")
    d = dims_of(wl, inp)
    assert (_splits(d, top_k) == 1) == one_split
    cache = LayerCache(d, "cuda")
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    z = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    step.encode(inp["k_cache"], inp["page_table"], z, inp["seq_len"],
                int(inp["seq_len"].max()), inp["R"], inp["W"], cache)
    step.select(inp["q"], inp["seq_len"], inp["page_table"], cache, R=inp["R"], W=inp["W"])
    step.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_len"])
    torch.cuda.synchronize()
    ref = step.out.clone()
    step.count[0, 3] = 0
    step.out.fill_(float("nan"))
    step.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_len"])
    torch.cuda.synchronize()
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    gs = wl.n_q_heads // wl.n_kv_heads
    empty = step.out[0, 3 * gs:4 * gs]
    assert torch.equal(empty, torch.zeros_like(empty))
    keep = torch.ones(wl.batch, wl.n_q_heads, dtype=torch.bool)
    keep[0, 3 * gs:4 * gs] = False
    assert torch.equal(step.out[keep].view(torch.int32), ref[keep].view(torch.int32))


def test_empty_sequence_in_fused_step():
    """A sequence with no keys in a fused decode step: count 0, indices -1, zero output."""
    build.build()
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], batch=2, seq_lens=(3000, 0), top_k=512)
    inp = S.make_inputs(wl, device="cuda")
    d = dims_of(wl, inp, 1)
    cache = LayerCache(d, "cuda")
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    z = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    n_prev = torch.clamp(inp["seq_len"] - 1, min=0).to(torch.int32)
    step.encode(inp["k_cache"], inp["page_table"], z, n_prev, int(n_prev.max()), inp["R"],
                inp["W"], cache)
    step.out.fill_(float("nan"))
    step.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"],
                    inp["seq_len"], inp["R"], inp["W"], cache)
    torch.cuda.synchronize()
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    assert torch.equal(step.count[1], torch.zeros_like(step.count[1]))
    assert bool((step.idx[1] == -1).all())
    assert torch.equal(step.out[1], torch.zeros_like(step.out[1]))
    kept = -(-(-(-3000 // wl.page_size)) // wl.keep_div)      # pages kept of the 3000 keys
    assert torch.isfinite(step.out[0]).all()
    assert bool((step.count[0] == min(wl.top_k, kept * wl.page_size)).all())


def _bf16_bits(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def test_saturated_f16_summary_with_zero_query_channel():
    """f16 summaries: a rotated key channel below -65504 saturates the page minimum to -inf.
    Where every query head of the group is >= 0 on that channel, the folded qneg is exactly
    0 and that channel contributes 0 to the bound (0 * kmin for every finite key), so the
    bound stays finite: it must equal the fold computed that way, within the bound
    tolerance, and dominate every true summed logit of its page."""
    build.build()
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(1000,), top_k=128, n_kv_heads=2,
                  n_q_heads=8, m_pages=4, keep_div=0)
    inp = S.make_inputs(wl, device="cuda")
    P, gs, g = wl.page_size, wl.n_q_heads // wl.n_kv_heads, 0
    # Group 0 rotates by the identity, so channel 0 of a key is its rotated channel 0.
    inp["R"][g] = torch.eye(128, device="cuda")
    pt = inp["page_table"][0].long()
    t_big = 77                               # logical key 77: page 2, slot 13
    phys = int(pt[t_big // P])
    inp["k_cache"][phys, g, t_big % P, 0] = _bf16_bits(-70000.0)
    q = inp["q"][0, g * gs:(g + 1) * gs].float()
    q[:, 0] = q[:, 0].abs() + 0.5            # every head > 0 on channel 0: qneg_0 = 0
    inp["q"][0, g * gs:(g + 1) * gs] = q.to(torch.bfloat16)
    d = dims_of(wl, inp, 1)
    cache = LayerCache(d, "cuda")
    step = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda")
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    step.encode(inp["k_cache"], inp["page_table"], z, inp["seq_len"], 1000, inp["R"], inp["W"],
                cache)
    rows = hhr.sel_rows(d)
    q_rot = torch.empty(1, wl.n_q_heads, 128, device="cuda")
    bounds = torch.empty(1, rows, d.max_pages_per_seq, device="cuda")
    trace = hhr.make_trace(q_rot=q_rot, bounds=bounds)
    step.select(inp["q"], inp["seq_len"], inp["page_table"], cache, R=inp["R"], W=inp["W"],
                trace=trace)
    step.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_len"])
    torch.cuda.synchronize()
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    mm = cache.page_minmax[phys, g].float().cpu().numpy()
    assert np.isneginf(mm[0, 0]), "the page minimum of channel 0 should saturate to -inf"
    n_pages = -(-1000 // P)
    beta = bounds[0, g, :n_pages].double().cpu().numpy()
    assert np.all(np.isfinite(beta)), "a bound is NaN or infinite"
    assert torch.isfinite(step.out).all()
    # The fold with 0 * (+-inf) taken as 0, in fp64 on the GPU's summaries and rotated queries.
    qr = q_rot[0, g * gs:(g + 1) * gs].double().cpu().numpy()
    qneg, qpos = np.minimum(qr, 0).sum(0), np.maximum(qr, 0).sum(0)
    assert qneg[0] == 0.0
    summ = cache.page_minmax[pt[:n_pages], g].double().cpu().numpy()   # [pages][2][d]

    def prod(a, k):
        return np.where(a == 0, 0.0, a * np.where(np.isfinite(k), k, 0.0)) + \
            np.where((a != 0) & ~np.isfinite(k), np.inf, 0.0)

    with np.errstate(invalid="ignore"):
        ref = (prod(qneg[None], summ[:, 0]) + prod(qpos[None], summ[:, 1])).sum(1)
        mag = np.where(np.isfinite(summ), np.abs(summ), 0.0).max(1)
        scale = (np.abs(qr)[:, None, :] * mag[None]).sum(axis=(0, 2))
    assert np.all(np.abs(beta - ref) <= BOUND_TOL * scale)
    # The bound invariant against the oracle's logits of the same keys.
    K = O.logical_rows(S.to_numpy_inputs({"k": inp["k_cache"]})["k"],
                       inp["page_table"][0].cpu().numpy(), g, 1000, P)
    Krot = O.rotate(inp["R"][g].double().cpu().numpy(), K)
    Q = O.bf16_to_f64(S.to_numpy_inputs({"q": inp["q"]})["q"][0, g * gs:(g + 1) * gs])
    Qrot = O.rotate(inp["R"][g].double().cpu().numpy(), Q)
    summed = (Krot @ Qrot.T).sum(axis=1)
    page_max = np.full(n_pages, -np.inf)
    np.maximum.at(page_max, np.arange(1000) // P, summed)
    assert np.all(beta >= page_max - 1e-5 * scale), "bound below a true logit"
