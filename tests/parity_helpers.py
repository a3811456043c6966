"""Shared machinery of the GPU parity tests: run the CUDA path through the C ABI and
compare every stage with the fp64 oracle, layer by layer.

Layered comparison: each stage is checked by feeding the GPU's output of the
previous stage into the oracle's next stage, so a legitimate near-tie upstream
cannot hide a bug downstream. Tolerances (written here, applied in tests):
  * codes: bit-exact except bits whose projection satisfies |p| < 1e-4 ||k||;
  * summaries / rotated queries / block means: fp32 vs fp64, |diff| <= 1e-5 (1 + max|ref|);
  * page bounds: |beta - beta_ref| <= 1e-3 * sum_{h,c} |q'_hc| max(|kmin_c|, |kmax_c|);
  * kept pages: identical to the oracle's top-m of the GPU's own fp32 bounds, and to
    the oracle's fp64 top-m wherever the margin at the cut exceeds the bound tolerance;
  * Hamming top-k indices and counts: bit-exact given the GPU's codes and kept pages;
  * attention: max_i |o_i - r_i| / max_i |r_i| <= 2e-3 per (sequence, head), with r the
    oracle on the GPU's selected set.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import hhr_synth as S
import oracle
from hash_hierarchical_top_b200 import hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache

O = oracle.hhr_oracle

ATTN_TOL = 2e-3
BOUND_TOL = 1e-3
FP32_TOL = 1e-5


def dims_of(wl, inp, summary_fp16=0):
    return hhr.make_dims(wl.batch, wl.n_queries if wl.mode == "indexer" else wl.n_q_heads,
                         wl.n_kv_heads, wl.page_size, inp["max_pages"], inp["n_phys"],
                         head_dim=wl.head_dim, code_bits=wl.code_bits,
                         summary_fp16=summary_fp16,
                         select_per_head=int(getattr(wl, "select_per_head", False)))


def run_gpu(wl, inp, bulk=True, trace=True, encode_chunks=None, summary_fp16=0):
    """Encode the whole cache, select and (hash mode) attend. Returns numpy results."""
    dev = inp["k_cache"].device
    d = dims_of(wl, inp, summary_fp16)
    hashing = wl.mode == "hash"
    mode = hhr.HHR_MODE_HASH if hashing else hhr.HHR_MODE_INDEXER
    cache = LayerCache(d, dev, hashing=hashing, block_means=not hashing)
    B = wl.batch
    lens = inp["seq_len"]
    if encode_chunks is None:
        start = torch.zeros(B, dtype=torch.int32, device=dev)
        step = DecodeStep(d, mode, wl.m_pages, wl.keep_div, wl.top_k, dev,
                          sink_pages=wl.sink_pages, local_pages=wl.local_pages)
        step.encode(inp["k_cache"], inp["page_table"], start, lens, int(lens.max()),
                    inp["R"] if hashing else None, inp["W"] if hashing else None, cache)
    else:
        # Append in pieces of at most `encode_chunks` keys, as a decode loop would.
        step = DecodeStep(d, mode, wl.m_pages, wl.keep_div, wl.top_k, dev,
                          sink_pages=wl.sink_pages, local_pages=wl.local_pages)
        done = torch.zeros(B, dtype=torch.int32, device=dev)
        while bool((done < lens).any()):
            n_new = torch.clamp(lens - done, max=encode_chunks).to(torch.int32)
            step.encode(inp["k_cache"], inp["page_table"], done, n_new, encode_chunks,
                        inp["R"] if hashing else None, inp["W"] if hashing else None, cache)
            done = (done + n_new).to(torch.int32)
    rows = hhr.sel_rows(d) if hashing else d.n_q_heads
    tr_t = dict(
        q_rot=torch.empty(B, d.n_q_heads, 128, dtype=torch.float32, device=dev) if hashing else None,
        q_code=(torch.empty(B, d.n_q_heads, d.code_bits // 32, dtype=torch.int32, device=dev)
                if hashing else None),
        bounds=torch.empty(B, rows, d.max_pages_per_seq, dtype=torch.float32, device=dev),
        kept=torch.empty(B, rows, step.m_max, dtype=torch.int32, device=dev),
        kept_count=torch.empty(B, rows, dtype=torch.int32, device=dev),
    )
    tr = hhr.make_trace(**tr_t) if trace else None
    step.select(inp["q"], lens, inp["page_table"], cache, R=inp["R"] if hashing else None,
                W=inp["W"] if hashing else None, k_cache=None if hashing else inp["k_cache"],
                q_pos=inp.get("q_pos"), trace=tr)
    if hashing:
        step.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], lens)
    torch.cuda.synchronize()
    st, bits = hhr.hhr_read_device_status()
    assert st == hhr.HHR_OK, f"device status bits {bits}"
    out = dict(idx=step.idx.cpu().numpy(), count=step.count.cpu().numpy(), m_max=step.m_max)
    if hashing:
        out["out"] = step.out.cpu().numpy()
        out["page_minmax"] = cache.page_minmax.float().cpu().numpy()
        out["summary_fp16"] = bool(summary_fp16)
        out["codes"] = cache.codes.cpu().numpy().view(np.uint32)
    else:
        out["block_mean"] = cache.block_mean.cpu().numpy()
    if trace:
        for k, v in tr_t.items():
            if v is not None:
                out[k] = v.cpu().numpy()
        if hashing:
            out["q_code"] = out["q_code"].view(np.uint32)
    return out


def gpu_codes_logical(g_out, pt_row, g, n, P):
    """GPU codes of one sequence/group in logical token order, [n][code words]."""
    n_pages = -(-n // P)
    c = g_out["codes"][np.asarray(pt_row[:n_pages], dtype=np.int64), g]  # [n_pages][P][CW]
    return c.reshape(n_pages * P, -1)[:n]


def check_hash_group(wl, inp_np, g_out, b, g, report):
    """Every layered check for one (sequence, group) of the HHR path."""
    P = wl.page_size
    gs = wl.n_q_heads // wl.n_kv_heads
    n = int(inp_np["seq_len"][b])
    n_pages = -(-n // P)
    pt = inp_np["page_table"][b]
    R, W = inp_np["R"][g], inp_np["W"][g]

    # a0: codes and summaries.
    enc = O.encode_group(inp_np["k_cache"], pt, g, n, P, R, W)
    gc = gpu_codes_logical(g_out, pt, g, n, P)
    diff = gc ^ enc["codes"]
    bad = 0
    CW = wl.code_bits // 32
    for w in range(CW):
        for bit in range(32):
            flips = ((diff[:, w] >> np.uint32(bit)) & 1).astype(bool)
            bad += int(np.count_nonzero(flips & ~enc["fragile"][:, 32 * w + bit]))
    assert bad == 0, f"{bad} non-fragile code bits differ (b={b}, g={g})"
    report["fragile_flips"] = report.get("fragile_flips", 0) + int(
        sum(bin(int(x)).count("1") for x in diff.ravel()))
    phys = np.asarray(pt[:n_pages], dtype=np.int64)
    gmm = g_out["page_minmax"][phys, g].astype(np.float64)     # [n_pages][2][d]
    for side, ref, got in ((0, enc["kmin"], gmm[:, 0]), (1, enc["kmax"], gmm[:, 1])):
        lim = FP32_TOL * (1 + np.abs(ref).max(axis=1, keepdims=True))
        if g_out.get("summary_fp16"):
            # f16 storage rounded outward: within one f16 step, and on the outer side.
            assert np.all(np.abs(got - ref) <= 2.0 ** -10 * np.abs(ref) + 6e-8 + lim)
            outward = (got <= ref + lim) if side == 0 else (got >= ref - lim)
            assert np.all(outward), f"f16 summary not rounded outward (b={b}, g={g})"
        else:
            assert np.all(np.abs(got - ref) <= lim), f"summary error (b={b}, g={g})"

    # a1: rotated queries and query codes.
    Qg = O.bf16_to_f64(inp_np["q"][b, g * gs:(g + 1) * gs])
    Qrot, qcodes, qfrag = O.query_prep(R, W, Qg)
    qr = g_out["q_rot"][b, g * gs:(g + 1) * gs].astype(np.float64)
    assert np.abs(qr - Qrot).max() <= FP32_TOL * (1 + np.abs(Qrot).max())
    gq = g_out["q_code"][b, g * gs:(g + 1) * gs]
    qd = gq ^ qcodes
    for h in range(gs):
        for w in range(CW):
            for bit in range(32):
                if (int(qd[h, w]) >> bit) & 1:
                    assert qfrag[h, 32 * w + bit], "non-fragile query code bit differs"

    # a2-a5 per selection row: the whole group, or each of its query heads on its own.
    def select_row(row, hs):
        qr_r, Qrot_r, Qg_r, gq_r = qr[hs], Qrot[hs], Qg[hs], gq[hs]
        # a2: bounds (oracle on the GPU's summaries) and kept pages.
        kmin_g, kmax_g = gmm[:, 0], gmm[:, 1]
        beta_ref = O.page_bounds(qr_r, kmin_g, kmax_g)
        beta_gpu = g_out["bounds"][b, row, :n_pages].astype(np.float64)
        scale = (np.abs(qr_r)[:, None, :] * np.maximum(np.abs(kmin_g), np.abs(kmax_g))[None]).sum(axis=(0, 2))
        assert np.all(np.abs(beta_gpu - beta_ref) <= BOUND_TOL * scale), "page bound out of tolerance"
        # Invariant at any size: the GPU's bound dominates every true summed logit of its page.
        Krot = O.rotate(R, O.logical_rows(inp_np["k_cache"], pt, g, n, P))
        summed = (Krot @ Qrot_r.T).sum(axis=1)
        page_max = np.full(n_pages, -np.inf)
        np.maximum.at(page_max, np.arange(n) // P, summed)
        assert np.all(beta_gpu >= page_max - 1e-5 * scale), "bound below a true logit"
        forced = O.forced_pages(n_pages, wl.sink_pages, wl.local_pages)
        m = max(O.kept_count(n_pages, wl.m_pages, wl.keep_div), len(forced))
        kc = int(g_out["kept_count"][b, row])
        assert kc == m
        kept_gpu = g_out["kept"][b, row, :kc]
        # Same-precision decision: the oracle's top-m of the GPU's own fp32 bounds.
        beta_gpu32 = g_out["bounds"][b, row, :n_pages]
        want = O.top_m_forced(beta_gpu32, m, forced) if len(forced) else O.top_m(beta_gpu32, m)
        assert np.array_equal(kept_gpu, want), "top-m differs"
        # Against the full fp64 oracle bounds (over the pages that are not forced): exact unless
        # the cut is within tolerance.
        beta_full = O.page_bounds(Qrot_r, enc["kmin"], enc["kmax"])
        rest = np.setdiff1d(np.arange(n_pages), forced)
        mr = m - len(forced)
        order = np.sort(beta_full[rest])[::-1]
        tol_cut = BOUND_TOL * float(scale.max())
        if 0 < mr < len(rest):
            margin = order[mr - 1] - order[mr]
            if margin > 2 * tol_cut:
                assert np.array_equal(kept_gpu, O.top_m_forced(beta_full, m, forced))
            else:
                report["near_tie_cuts"] = report.get("near_tie_cuts", 0) + 1
                sure_in = set(rest[beta_full[rest] > order[mr - 1] + 2 * tol_cut]) | set(forced)
                maybe = set(rest[beta_full[rest] >= order[mr - 1] - 2 * tol_cut]) | set(forced)
                assert sure_in <= set(kept_gpu) <= maybe
        else:
            assert np.array_equal(kept_gpu, O.top_m_forced(beta_full, m, forced))

        # a3 + a4: Hamming top-k on the GPU's codes and kept pages, bit-exact.
        cand = O.candidates_of(kept_gpu, n, P)
        delta = O.hamming(gq_r, gc[cand])
        if len(forced):
            S_ref = O.top_k_forced(delta, cand, min(wl.top_k, len(cand)), np.isin(cand // P, forced))
        else:
            S_ref = O.top_k_smallest(delta, cand, min(wl.top_k, len(cand)))
        cnt = int(g_out["count"][b, row])
        assert cnt == len(S_ref)
        assert np.array_equal(g_out["idx"][b, row, :cnt], S_ref), "Hamming top-k differs"
        assert np.all(g_out["idx"][b, row, cnt:] == -1)

        # a5: attention on the GPU's selected set.
        K = O.logical_rows(inp_np["k_cache"], pt, g, n, P)
        V = O.logical_rows(inp_np["v_cache"], pt, g, n, P)
        ref = O.sparse_attention(Qg_r, K[S_ref], V[S_ref], 1.0 / math.sqrt(wl.head_dim))
        got = g_out["out"][b, [g * gs + h for h in hs]].astype(np.float64)
        for j, h in enumerate(hs):
            den = max(np.abs(ref[j]).max(), 1e-30)
            rel = np.abs(got[j] - ref[j]).max() / den
            report["attn_max_rel"] = max(report.get("attn_max_rel", 0.0), float(rel))
            assert rel <= ATTN_TOL, f"attention rel err {rel} (b={b}, h={g * gs + h})"
        return dict(kept_oracle=O.top_m(beta_full, m), kept_gpu=kept_gpu, idx=S_ref)


    if getattr(wl, "select_per_head", False):
        return [select_row(g * gs + h, [h]) for h in range(gs)]
    return select_row(g, list(range(gs)))

def check_indexer_query(wl, inp_np, g_out, b, i, report):
    """Layered checks of the HISA indexer for one (sequence, chunk query)."""
    P = wl.page_size
    n = int(inp_np["seq_len"][b])
    pt = inp_np["page_table"][b]
    pos = int(inp_np["q_pos"][b, i])
    K = O.logical_rows(inp_np["k_cache"], pt, 0, n, P)
    mu = O.block_means(K, P)
    n_blk = -(-n // P)
    phys = np.asarray(pt[:n_blk], dtype=np.int64)
    gmu = g_out["block_mean"][phys, 0].astype(np.float64)
    assert np.all(np.abs(gmu - mu).max(axis=1) <= FP32_TOL * (1 + np.abs(mu).max(axis=1)))
    q = O.bf16_to_f64(inp_np["q"][b, i])
    n_elig = min(pos // P + 1, n_blk)
    s_ref = gmu[:n_elig] @ q
    s_gpu = g_out["bounds"][b, i, :n_blk].astype(np.float64)
    tol = FP32_TOL * np.linalg.norm(q) * np.linalg.norm(gmu, axis=1).max()
    assert np.all(np.abs(s_gpu[:n_elig] - s_ref) <= tol)
    assert np.all(np.isneginf(s_gpu[n_elig:]))
    m = min(wl.m_pages, n_elig)
    kc = int(g_out["kept_count"][b, i])
    assert kc == m
    kept_gpu = g_out["kept"][b, i, :kc]
    assert np.array_equal(kept_gpu, O.top_m(g_out["bounds"][b, i, :n_elig], m))
    # Token refinement on the GPU's kept blocks: exact set unless a near-tie at the cut.
    cand = O.candidates_of(kept_gpu, min(n, pos + 1), P)
    sigma = K[cand] @ q
    k_eff = min(wl.top_k, len(cand))
    cnt = int(g_out["count"][b, i])
    assert cnt == k_eff
    got = g_out["idx"][b, i, :cnt]
    assert np.all(np.diff(got) > 0)
    ref = O.top_k_largest(sigma, cand, k_eff)
    tol_t = 1e-5 * np.linalg.norm(q) * np.linalg.norm(K[cand], axis=1).max()
    if not np.array_equal(got, ref):
        srt = np.sort(sigma)[::-1]
        kth = srt[k_eff - 1]
        sure_in = set(cand[sigma > kth + tol_t].tolist())
        maybe = set(cand[sigma >= kth - tol_t].tolist())
        assert sure_in <= set(got.tolist()) <= maybe, "token top-k differs beyond the near-tie band"
        report["token_near_ties"] = report.get("token_near_ties", 0) + 1
    assert np.all(g_out["idx"][b, i, cnt:] == -1)
