#!/usr/bin/env python
"""Decode-step benchmark of the coarse-to-fine retrieval path on B200.

A step is one HHR decode step for a whole batch: append-encode the newest key of
every sequence (step a0), select (a1-a4: query prep, page bounds, top-m pages,
Hamming top-k) and GQA sparse attention (a5), all through the C ABI. Default
workload: Llama-3.1-8B shapes at 128K context, batch 8 (32 query / 8 KV heads,
d=128, pages of 32, keep 1/16 of the pages, top-2048, 128-bit codes).

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0). Multi-GPU runs are independent replicas (weak
scaling, no collective on the data path); the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode queries/s (all heads) at 128K ctx; select+attn HBM GB/s vs ~8 TB/s peak"
NOMINAL_HBM_GBS = 8000.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama8b_128k_b8")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling: override the workload's batch (same context per sequence)")
    ap.add_argument("--layers", type=int, default=0, help="layer caches rotated (0 = auto)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads (other_workloads field)")
    ap.add_argument("--no-quality", action="store_true",
                    help="skip the selection-quality figures (selection_quality field)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--summary", default="f16", choices=["f16", "f32"],
                    help="page-summary storage (f16 rounded outward, or f32)")
    ap.add_argument("--path", default="fused", choices=["fused", "calls"],
                    help="fused: hhr_decode_step; calls: encode + select + attention calls")
    ap.add_argument("--select-only", action="store_true",
                    help="profiling case: no V cache and no attention (step = encode + select)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def required_bytes(wl, lens, m_of, sbytes=4):
    """Algorithmic bytes of one step: summaries (unless every page is kept: a flat top-k
    needs no bounds) + kept-page codes + selected K/V rows, for every selection row (KV
    group, or query head with per-head selection, whose sets are read separately)."""
    G, P, d = wl.n_kv_heads, wl.page_size, wl.head_dim
    rows = wl.n_q_heads if wl.select_per_head else G
    summ = codes = kv = 0
    for n in lens:
        npg = -(-n // P)
        m = m_of(npg)
        cand = min(n, m * P)
        if m < npg:
            summ += G * npg * 2 * d * sbytes
        codes += rows * cand * (wl.code_bits // 8)
        kv += rows * min(wl.top_k, cand) * 2 * d * 2
    return summ, codes, kv


def dense_kv_bytes(wl, lens):
    """K and V bytes one dense (full-context) decode step reads: every key and value row of
    every KV group, for comparison with the step's required bytes."""
    return sum(lens) * wl.n_kv_heads * wl.head_dim * 2 * 2


def bound_kernel_bytes(wl, lens, sbytes=4):
    """Algorithmic bytes of one page-bound launch: per (page, group) the summary read
    (2 x 128 x sbytes) and the 4-byte bound write; per page its 4-byte page-table entry;
    per (sequence, group) the 1 KB folded query."""
    G = wl.n_kv_heads
    tot = 0
    for n in lens:
        npg = -(-n // wl.page_size)
        tot += npg * G * (2 * wl.head_dim * sbytes + 4) + npg * 4 + G * 2 * wl.head_dim * 4
    return tot


def step_kernel_bytes(wl, lens, m_of, sbytes=4):
    """Algorithmic bytes of each kernel of one fused step (the names of kernels_us):
    encode = the prologue (R_g and W_g once per group, the new K/V rows and the queries read;
    rotated queries and folded queries written); bound = bound_kernel_bytes; hamming = the
    bounds, the kept pages' page-table entries and codes read, the selected ids and cache
    rows written; attn = the selected rows' offsets, K and V read, the queries read and the
    outputs written; row = bound + hamming + attn (the small-batch kernel that does all three)."""
    G, Hq, d, P = wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.page_size
    rows = Hq if wl.select_per_head else G
    B = len(lens)
    enc = G * (d * d + wl.code_bits * d) * 4 + B * G * 2 * d * 2 + B * Hq * d * (2 + 4) \
        + B * G * 2 * d * 4
    ham = attn = 0
    for n in lens:
        npg = -(-n // P)
        m = m_of(npg)
        cand = min(n, m * P)
        k = min(wl.top_k, cand)
        ham += rows * (npg * 4 + m * 4 + cand * (wl.code_bits // 8) + k * 8)
        attn += rows * k * (4 + 2 * d * 2)
    attn += B * Hq * d * (2 + 4)
    bound = bound_kernel_bytes(wl, lens, sbytes)
    return {"encode": enc, "bound": bound, "hamming": ham, "attn": attn,
            "row": bound + ham + attn}


def kernel_table(kern_us, kbytes, peak_gbs):
    """Per kernel: bracketed time, algorithmic bytes, GB/s and its fraction of 8 TB/s and of
    the measured copy bandwidth (kernels without a byte figure get the time only)."""
    out = {}
    for name, us in kern_us.items():
        row = {"us": us}
        if name in kbytes and us > 0:
            gbs = kbytes[name] / (us * 1e-6) / 1e9
            row.update(algorithmic_bytes=kbytes[name], gbs=gbs, frac_of_8tbs=gbs / 8000.0,
                       frac_of_measured=gbs / peak_gbs)
        out[name] = row
    return out


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def _once(self):
        try:
            r = subprocess.run(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                "--format=csv,noheader,nounits", "-i", self.uuid],
                               capture_output=True, text=True, timeout=10)
            return r.stdout.strip().splitlines()
        except Exception:
            return []

    def start(self):
        self.lines += self._once()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.uuid], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
                self.lines += out.strip().splitlines()
            except Exception:
                self.proc.kill()
        self.lines += self._once()

    def summary(self):
        mhz, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(mhz)}


def traffic_from_profile(name, kernel_src_hash):
    """(DRAM bytes, algorithmic bytes) of the profiled launch from the committed ncu summary
    profiles/<name>, or None if the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for ln in f:
            if "=" in ln and not ln.startswith("#"):
                k, v = ln.split("=", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256") != kernel_src_hash:
        return None
    try:
        return float(vals["dram_bytes_per_full_launch"]), float(vals["algorithmic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def kernel_source_hash():
    """sha256 of the page-bound kernel's section of select.cuh (its step-a2 block)."""
    with open(os.path.join(ROOT, "hash_hierarchical_top_b200", "csrc", "select.cuh")) as fh:
        s = fh.read()
    mark = "// " + "-" * 76
    a = s.index(mark + " a2")
    b = s.index(mark, a + len(mark))
    return hashlib.sha256(s[a:b].encode()).hexdigest()


# ----------------------------------------------------------------------------- ranks
# One process per GPU under torchrun; the timing of a multi-GPU run is the slowest rank's.


def rank_env():
    """(world size, rank, local rank) from the torchrun environment; (1, 0, 0) without it."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x, world, device):
    """x (a duration) maximised over the ranks (every rank must call it, in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_step, steps, ms_max):
    """Whole-job units/s: each of `world` ranks processed `units_per_step` per step for `steps`
    steps, and the job took the slowest rank's `ms_max` milliseconds."""
    return world * units_per_step * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------- selection quality
# Measures how well the GPU path's selections match exact ones on the synthetic workloads
# (HHR page, Figure 4: recall of the true top-k; Figure 2: Hamming distance against logits;
# HISA page, Abstract: overlap of the hierarchical with the flat indexer's selection).


def recall_at_k(sel, true):
    """|sel ∩ true| / |true| for two 1-D index tensors (sel may hold -1 padding)."""
    import torch
    sel = sel[sel >= 0]
    if true.numel() == 0:
        return 1.0
    return float(torch.isin(true, sel).sum().item()) / true.numel()


def iou(a, b):
    """Intersection over union of two index sets (-1 padding ignored)."""
    import torch
    a, b = a[a >= 0], b[b >= 0]
    inter = int(torch.isin(a, b).sum().item())
    union = a.numel() + b.numel() - inter
    return 1.0 if union == 0 else inter / union


def mass_recall(logits, sel, scale):
    """Mean over rows of logits [H][n] of the softmax(scale * logits) mass on sel."""
    import torch
    p = torch.softmax(logits.double() * scale, dim=-1)
    sel = sel[sel >= 0]
    return float(p[:, sel].sum(dim=-1).mean().item())


def spearman(x, y):
    """Spearman rank correlation of two 1-D tensors (average ranks for ties)."""
    import torch

    def ranks(v):
        v = v.double()
        order = torch.argsort(v)
        r = torch.empty_like(v)
        r[order] = torch.arange(v.numel(), dtype=torch.float64, device=v.device)
        # average the ranks of equal values
        uniq, inv = torch.unique(v, return_inverse=True)
        sums = torch.zeros(uniq.numel(), dtype=torch.float64, device=v.device).index_add_(0, inv, r)
        cnt = torch.zeros(uniq.numel(), dtype=torch.float64, device=v.device).index_add_(
            0, inv, torch.ones_like(r))
        return (sums / cnt)[inv]

    rx, ry = ranks(x), ranks(y)
    rx, ry = rx - rx.mean(), ry - ry.mean()
    return float((rx * ry).sum().item() / ((rx.square().sum() * ry.square().sum()).sqrt().item()))


def popcount32(x):
    """Per-element popcount of an int32 tensor (bit-parallel sums; int64 result)."""
    x = x.to(__import__("torch").int64) & 0xFFFFFFFF
    x = x - ((x >> 1) & 0x55555555)
    x = (x & 0x33333333) + ((x >> 2) & 0x33333333)
    x = (x + (x >> 4)) & 0x0F0F0F0F
    return ((x * 0x01010101) & 0xFFFFFFFF) >> 24


def hhr_quality(wl, inp, dev, R, m_pages, keep_div, full=True, W=None, k_true=None, hot=None):
    """Encode layer inputs `inp` with rotation R (and projection W, default inp["W"], of
    wl.code_bits rows), select wl.top_k keys with the given page budget and score the
    selection against the exact group logits' top-k_true (default wl.top_k; see
    selection_quality). hot: {sequence: [planted hot pages of each KV group]}, for the share
    of them the page stage keeps."""
    import statistics
    import torch
    from hash_hierarchical_top_b200 import hhr
    from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
    W = inp["W"] if W is None else W
    CW = wl.code_bits // 32
    d = hhr.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.page_size, inp["max_pages"],
                      inp["n_phys"], summary_fp16=1, code_bits=wl.code_bits,
                      select_per_head=int(wl.select_per_head))
    cache = LayerCache(d, dev)
    zero = torch.zeros(wl.batch, dtype=torch.int32, device=dev)
    hhr.hhr_encode_keys(d, inp["k_cache"], inp["page_table"], zero, inp["seq_len"],
                        int(inp["seq_len"].max()), R, W, cache.page_minmax, cache.codes,
                        None)
    st = DecodeStep(d, hhr.HHR_MODE_HASH, m_pages, keep_div, wl.top_k, dev, attention=False,
                    sink_pages=wl.sink_pages, local_pages=wl.local_pages)
    B, G, gs, P = wl.batch, wl.n_kv_heads, wl.n_q_heads // wl.n_kv_heads, wl.page_size
    qcode = torch.empty(B, wl.n_q_heads, CW, dtype=torch.int32, device=dev)
    rows = hhr.sel_rows(d)
    kept = torch.empty(B, rows, st.m_max, dtype=torch.int32, device=dev)
    kcnt = torch.empty(B, rows, dtype=torch.int32, device=dev)
    st.select(inp["q"], inp["seq_len"], inp["page_table"], cache, R=R, W=W,
              trace=hhr.make_trace(q_code=qcode, kept=kept, kept_count=kcnt))
    torch.cuda.synchronize()
    rec, mass, page_rec, ham_rec, rho, hot_kept = [], [], [], [], [], []
    scale = 1.0 / math.sqrt(wl.head_dim)
    gen = torch.Generator(device=dev).manual_seed(0)
    for b in range(B):
        n = int(inp["seq_len"][b])
        npg = -(-n // P)
        pages = inp["page_table"][b, :npg].long()
        for g in range(G):
            K = inp["k_cache"][pages, g].reshape(npg * P, -1)[:n].float()
            lg = inp["q"][b, g * gs:(g + 1) * gs].float() @ K.T          # [gs][n]
            if wl.select_per_head:  # each head against its own logits' top-k
                for h in range(gs):
                    r = g * gs + h
                    true = torch.topk(lg[h], min(k_true or wl.top_k, n)).indices
                    sel = st.idx[b, r, :int(st.count[b, r])].long()
                    rec.append(recall_at_k(sel, true))
                    mass.append(mass_recall(lg[h:h + 1], sel, scale))
                    kp = kept[b, r, :int(kcnt[b, r])].long()
                    in_kept = torch.isin(true // P, kp)
                    page_rec.append(float(in_kept.float().mean().item()))
                    if bool(in_kept.any()):
                        ham_rec.append(recall_at_k(sel, true[in_kept]))
                continue
            grp = lg.sum(0)
            true = torch.topk(grp, min(k_true or wl.top_k, n)).indices
            sel = st.idx[b, g, :int(st.count[b, g])].long()
            rec.append(recall_at_k(sel, true))
            mass.append(mass_recall(lg, sel, scale))
            kp = kept[b, g, :int(kcnt[b, g])].long()
            in_kept = torch.isin(true // P, kp)
            page_rec.append(float(in_kept.float().mean().item()))
            if bool(in_kept.any()):
                ham_rec.append(recall_at_k(sel, true[in_kept]))
            if hot is not None:
                hp = torch.tensor(hot[b][g], device=dev, dtype=torch.long)
                hot_kept.append(float(torch.isin(hp, kp).float().mean().item()))
            if full:
                codes = cache.codes[pages, g].reshape(npg * P, CW)[:n]
                qc = qcode[b, g * gs:(g + 1) * gs]                        # [gs][CW]
                delta = popcount32(qc[:, None, :] ^ codes[None, :, :]).sum(dim=(0, 2))
                smp = torch.randint(0, n, (16384,), device=dev, generator=gen)
                rho.append(spearman(-delta[smp].double(), grp[smp].double()))
    res = {"recall_at_k": statistics.mean(rec), "recall_at_k_min": min(rec),
           "attention_mass_recall": statistics.mean(mass),
           "true_topk_in_kept_pages": statistics.mean(page_rec),
           "hamming_recall_within_kept_pages": statistics.mean(ham_rec) if ham_rec else None,
           "k": wl.top_k, "k_true": k_true or wl.top_k, "kept_pages": st.m_max,
           "rows": B * rows}
    if hot_kept:
        res["hot_pages_kept"] = statistics.mean(hot_kept)
    if full:
        res["spearman_minus_hamming_vs_logit"] = statistics.mean(rho)
        res["random_selection_mass"] = wl.top_k / float(inp["seq_len"].float().mean())
    del cache, st
    return res


def selection_quality(dev):
    """Recall, attention-mass recall and Hamming/logit correlation of the HHR selection on the
    128K batch-8 workload, and overlap of the HISA selection with the flat indexer's."""
    import statistics
    import torch
    import hhr_synth as S
    from hash_hierarchical_top_b200 import hhr
    from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
    out = {}
    # HHR: GPU selection (hhr_select on layer 0) against exact group logits.
    wl = S.WORKLOADS["llama8b_128k_b8"]
    inp = S.make_inputs(wl, device=dev, layer=0, with_values=False)
    out["hhr_llama8b_128k_b8"] = hhr_quality(wl, inp, dev, inp["R"], wl.m_pages, wl.keep_div)
    out["hhr_llama8b_128k_b8"]["true_set"] = ("top-k of the group-summed logits sum_h q_h . k_t "
                                              "(one selection per KV group)")
    # Stage variants and the page budget: bounds without the rotation (R = I, QUEST-style
    # page min/max of the raw keys), keep 1/8 and 1/32, and 64- and 256-bit codes.
    eye = torch.eye(wl.head_dim, device=dev).expand(wl.n_kv_heads, -1, -1).contiguous()
    sweep = {"quest_R_identity_keep_1/16": hhr_quality(wl, inp, dev, eye, 0, 16, full=False)}
    for kd in (8, 32):
        sweep[f"gkr_keep_1/{kd}"] = hhr_quality(wl, inp, dev, inp["R"], 0, kd, full=False)
    sweep["flat_all_4096_pages"] = hhr_quality(wl, inp, dev, inp["R"], 4096, 0, full=False)
    # Page stage only (every key of the 256 kept pages attended, no Hamming ranking), with
    # GKR bounds and with QUEST-style bounds; recall against the true top-2048.
    every = S.scaled(wl, top_k=256 * wl.page_size)
    sweep["gkr_only_keep_1/16_attend_kept_pages"] = hhr_quality(
        every, inp, dev, inp["R"], 0, 16, full=False, k_true=wl.top_k)
    sweep["quest_R_identity_keep_1/16_attend_kept_pages"] = hhr_quality(
        every, inp, dev, eye, 0, 16, full=False, k_true=wl.top_k)
    for k in (1024, 4096):
        sweep[f"gkr_keep_1/16_k{k}"] = hhr_quality(S.scaled(wl, top_k=k), inp, dev, inp["R"], 0,
                                                   16, full=False)
    sweep["per_query_head_keep_1/16"] = hhr_quality(
        S.scaled(wl, select_per_head=True), inp, dev, inp["R"], 0, 16, full=False)
    sweep["sink_1_local_2_pages_keep_1/16"] = hhr_quality(
        S.scaled(wl, sink_pages=1, local_pages=2), inp, dev, inp["R"], 0, 16, full=False)
    for bits in (64, 256):
        wb = S.scaled(wl, code_bits=bits)
        Wb = S.lhp_projection(wb, layer=0).to(dev)
        sweep[f"codes_{bits}_bit_keep_1/16"] = hhr_quality(wb, inp, dev, inp["R"], 0, 16,
                                                          full=False, W=Wb)
    out["hhr_variants_llama8b_128k_b8"] = sweep
    del inp
    # Flat hash top-k (every page kept, HATA-style) against the hierarchical selection at 32K.
    wl = S.WORKLOADS["llama8b_32k"]
    inp = S.make_inputs(wl, device=dev, layer=0, with_values=False)
    npg = -(-int(inp["seq_len"].max()) // wl.page_size)
    budget = f"{wl.m_pages}_pages" if wl.m_pages else f"keep_1/{wl.keep_div}"
    out["llama8b_32k_hierarchical_vs_flat"] = {
        f"hierarchical_{budget}": hhr_quality(wl, inp, dev, inp["R"], wl.m_pages, wl.keep_div,
                                              full=False),
        f"flat_all_{npg}_pages": hhr_quality(wl, inp, dev, inp["R"], npg, 0, full=False)}
    del inp
    # Planted page locality: the keys each query attends to cluster in a few pages (8 runs of 8
    # hot pages per KV group, 2048 hot keys); the same stages and budgets as above.
    wl = S.WORKLOADS["llama8b_128k_planted"]
    inp = S.make_inputs(wl, device=dev, layer=0, with_values=False)
    hot = {b: S.hot_pages(wl, b, int(inp["seq_len"][b]), 0) for b in range(wl.batch)}
    every = S.scaled(wl, top_k=256 * wl.page_size)
    out["hhr_planted_llama8b_128k_b2"] = {
        "gkr_keep_1/16": hhr_quality(wl, inp, dev, inp["R"], 0, 16, hot=hot),
        "quest_R_identity_keep_1/16": hhr_quality(wl, inp, dev, eye, 0, 16, full=False, hot=hot),
        "gkr_keep_1/32": hhr_quality(wl, inp, dev, inp["R"], 0, 32, full=False, hot=hot),
        "flat_all_4096_pages": hhr_quality(wl, inp, dev, inp["R"], 4096, 0, full=False),
        "gkr_only_keep_1/16_attend_kept_pages": hhr_quality(
            every, inp, dev, inp["R"], 0, 16, full=False, k_true=wl.top_k, hot=hot),
        "planted": f"{wl.hot_runs} runs of {wl.hot_run_pages} hot pages per KV group, keys "
                   f"shifted by {wl.hot_scale} sqrt(d) along the group's mean query direction"}
    del inp
    # HISA: hierarchical selection against the flat indexer's causal top-k over all keys.
    for name in ("hisa_128k_t1", "hisa_128k_t64", "hisa_128k_t1_planted"):
        wl = S.WORKLOADS[name]
        inp = S.make_inputs(wl, device=dev, layer=0, with_values=False)
        d = hhr.make_dims(wl.batch, wl.n_queries, 1, wl.page_size, inp["max_pages"], inp["n_phys"])
        cache = LayerCache(d, dev, hashing=False, block_means=True)
        zero = torch.zeros(wl.batch, dtype=torch.int32, device=dev)
        hhr.hhr_encode_keys(d, inp["k_cache"], inp["page_table"], zero, inp["seq_len"],
                            int(inp["seq_len"].max()), None, None, None, None, cache.block_mean)
        st = DecodeStep(d, hhr.HHR_MODE_INDEXER, wl.m_pages, 0, wl.top_k, dev, attention=False)
        st.select(inp["q"], inp["seq_len"], inp["page_table"], cache, k_cache=inp["k_cache"],
                  q_pos=inp["q_pos"])
        torch.cuda.synchronize()
        n = int(inp["seq_len"][0])
        P = wl.page_size
        npg = -(-n // P)
        pages = inp["page_table"][0, :npg].long()
        K = inp["k_cache"][pages, 0].reshape(npg * P, -1)[:n].float()
        ious = []
        for t in range(wl.n_queries):
            pos = int(inp["q_pos"][0, t])
            sc = inp["q"][0, t].float() @ K[:pos + 1].T
            flat = torch.topk(sc, min(wl.top_k, pos + 1)).indices
            ious.append(iou(st.idx[0, t, :int(st.count[0, t])].long(), flat))
        out[name] = {"iou_with_flat_indexer": statistics.mean(ious),
                     "iou_min": min(ious), "queries": wl.n_queries, "k": wl.top_k,
                     "kept_blocks": wl.m_pages}
        del inp, cache, st
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- other workloads

def measure_dense_attention(layers, wl, dev, stream, steps=200):
    """Dense decode attention over the whole cache with the library's own attention kernel
    (every key of every sequence selected: top_k = the context), graph-timed over the same
    layer caches as the step: the full attention the hierarchical step replaces."""
    import torch
    from hash_hierarchical_top_b200 import hhr
    B, G, Hq, d0 = wl.batch, wl.n_kv_heads, wl.n_q_heads, layers[0][1]
    L = len(layers)
    lens = layers[0][0]["seq_len"]
    n = int(lens.max())
    idx = torch.arange(n, dtype=torch.int32, device=dev).expand(B, G, n).contiguous()
    count = lens.to(torch.int32).view(B, 1).expand(B, G).contiguous()
    ws = torch.empty(hhr.hhr_attn_workspace_bytes(d0, n), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, wl.head_dim, device=dev)
    scale = 1.0 / math.sqrt(wl.head_dim)

    def run(l):
        inp, d = layers[l % L][0], layers[l % L][1]
        hhr.hhr_sparse_attn(d, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"],
                            inp["seq_len"], idx, count, n, scale, out, ws)

    for l in range(L):
        run(l)
    torch.cuda.synchronize()
    st_, bits = hhr.hhr_read_device_status()
    if st_ != hhr.HHR_OK or not bool(torch.isfinite(out).all()):
        raise RuntimeError(f"dense attention: device status {bits}")
    graphs = []
    for l in range(L):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            run(l)
        graphs.append(gr)
    for i in range(2 * L):
        graphs[i % L].replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        graphs[i % L].replay()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    kv = dense_kv_bytes(wl, [int(x) for x in lens.tolist()])
    del graphs
    return {"api": "hhr_sparse_attn with every key selected (top_k = context)",
            "us_per_step": ms * 1e3, "kv_bytes": kv, "achieved_gbs": kv / (ms / 1e3) / 1e9}


SECONDARY = ("llama8b_128k_b1", "ragged_b32", "llama8b_32k", "tiny_1h_4k", "hisa_128k_t1",
             "hisa_128k_t64", "llama8b_128k_b8_codes64", "llama8b_128k_b8_codes256",
             "llama8b_128k_b8_flat", "llama8b_128k_b8_sink1_local2", "llama8b_128k_b8_per_head")


def indexer_required_bytes(wl, lens):
    """Algorithmic bytes of one HISA selection: block means (512 B per block, read once per
    step) + the kept blocks' keys of every chunk query (256 B per key; the union of the
    queries' kept blocks would be the minimum, the per-query sum is what the kernel reads)."""
    d, P = wl.head_dim, wl.page_size
    tot = 0
    for n in lens:
        nblk = -(-n // P)
        tot += nblk * d * 4 + wl.n_queries * min(wl.m_pages, nblk) * P * d * 2
    return tot


def measure_secondary(name, dev, l2, f16, steps, stream, mem_cap):
    """Graph-replayed decode steps of another workload; returns its figures."""
    import torch
    import hhr_synth as S
    from hash_hierarchical_top_b200 import hhr
    from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
    wl = S.WORKLOADS[name]
    lens = S.seq_lens_of(wl)
    hashing = wl.mode == "hash"
    if hashing:
        m_of = (lambda npg: min(npg, -(-npg // wl.keep_div))) if wl.m_pages == 0 else (
            lambda npg: min(wl.m_pages, npg))
        req = sum(required_bytes(wl, lens, m_of, 2 if f16 else 4))
        queries = wl.batch
    else:
        req = indexer_required_bytes(wl, lens)
        queries = wl.batch * wl.n_queries
    # Layer caches for an L2-cold rotation (>= 4x L2 of required bytes), within a memory cap.
    per_layer = sum(lens) * wl.n_kv_heads * wl.head_dim * 2 * (2 if hashing else 1)
    L = max(2, min(-(-4 * l2 // req), max(2, mem_cap // max(per_layer, 1)), 64))
    layers, graphs = [], []
    for l in range(L):
        inp = S.make_inputs(wl, device=dev, layer=l, with_values=hashing)
        d = hhr.make_dims(wl.batch, wl.n_q_heads if hashing else wl.n_queries, wl.n_kv_heads,
                          wl.page_size, inp["max_pages"], inp["n_phys"],
                          summary_fp16=f16 if hashing else 0, code_bits=wl.code_bits,
                          select_per_head=int(wl.select_per_head))
        cache = LayerCache(d, dev, hashing=hashing, block_means=not hashing)
        zero = torch.zeros(wl.batch, dtype=torch.int32, device=dev)
        hhr.hhr_encode_keys(d, inp["k_cache"], inp["page_table"], zero, inp["seq_len"],
                            int(inp["seq_len"].max()), inp["R"] if hashing else None,
                            inp["W"] if hashing else None,
                            cache.page_minmax if hashing else None,
                            cache.codes if hashing else None,
                            None if hashing else cache.block_mean)
        mode = hhr.HHR_MODE_HASH if hashing else hhr.HHR_MODE_INDEXER
        st = DecodeStep(d, mode, wl.m_pages, wl.keep_div, wl.top_k, dev, attention=hashing,
                        sink_pages=wl.sink_pages, local_pages=wl.local_pages)
        if hashing:
            t = (inp["seq_len"] - 1).long()
            phys = inp["page_table"][torch.arange(wl.batch, device=dev), t // wl.page_size].long()
            kn = inp["k_cache"][phys, :, t % wl.page_size].contiguous()
            vn = inp["v_cache"][phys, :, t % wl.page_size].contiguous()

            def run(inp=inp, cache=cache, st=st, kn=kn, vn=vn):
                st.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"],
                              inp["seq_len"], inp["R"], inp["W"], cache, k_new=kn, v_new=vn)
        else:
            def run(inp=inp, cache=cache, st=st):
                st.select(inp["q"], inp["seq_len"], inp["page_table"], cache,
                          k_cache=inp["k_cache"], q_pos=inp["q_pos"])
        run()
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            run()
        layers.append((inp, cache, st))
        graphs.append(gr)
    for i in range(3 * L):
        graphs[i % L].replay()
    torch.cuda.synchronize()
    st_, bits = hhr.hhr_read_device_status()
    if st_ != hhr.HHR_OK:
        raise RuntimeError(f"{name}: device status {bits}")
    K = max(steps, 2 * L)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(K):
        graphs[i % L].replay()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / K
    peak, _ = measured_peaks()
    gbs = req / (ms / 1e3) / 1e9
    del graphs, layers
    torch.cuda.empty_cache()
    return {"api": "hhr_decode_step" if hashing else "hhr_select (indexer)",
            "queries_per_s": queries / (ms / 1e3), "us_per_step": ms * 1e3,
            "queries_per_step": queries, "required_bytes": req, "achieved_gbs": gbs,
            "frac_of_measured": gbs / peak, "layer_caches_rotated": L,
            "l2_cold": L * req >= 4 * l2}


# ----------------------------------------------------------------------------- oracle arm
# The fp64 oracle's decode step, timed on every host core: one spawned worker process per
# core (BLAS limited to one thread in each), all starting together after a barrier. The
# sample is sequence 0 of the workload: its pages, queries, R and W are written once to a
# temporary directory with the oracle's encoding of every KV group (untimed); worker w runs
# the decode step of group w % G over and over (append-encode the newest key into its page's
# summary and code, bounds, top-m, Hamming top-k, attention on the selected rows).


def oracle_group_step(O, a, enc, g):
    """The oracle's decode step for one KV group of the sample (arrays in ``a``)."""
    import numpy as np
    P, n, gs, d = a["P"], a["n"], a["gs"], a["d"]
    R, W = a["R"][g], a["W"][g]
    lp = (n - 1) // P
    page_keys = O.bf16_to_f64(a["k_cache"][lp, g, : n - lp * P])
    kmin, kmax = enc["kmin"].copy(), enc["kmax"].copy()
    pmin, pmax = O.page_summaries(O.rotate(R, page_keys), P)
    kmin[lp], kmax[lp] = pmin[0], pmax[0]
    codes = np.array(enc["codes"])
    codes[n - 1] = O.sign_codes(R, W, page_keys[-1:])[0]
    m = O.kept_count(-(-n // P), a["m_pages"], a["keep_div"])
    Qg = O.bf16_to_f64(a["q"][g * gs:(g + 1) * gs])
    r = O.select_group(Qg, R, W, kmin, kmax, codes, n, P, m, a["top_k"])
    idx = r["idx"]
    rows_k = O.bf16_to_f64(a["k_cache"][idx // P, g, idx % P])
    rows_v = O.bf16_to_f64(a["v_cache"][idx // P, g, idx % P])
    return O.sparse_attention(Qg, rows_k, rows_v, 1.0 / math.sqrt(d))


def _oracle_arrays(data_dir):
    import numpy as np
    meta = json.load(open(os.path.join(data_dir, "meta.json")))
    a = dict(meta)
    for k in ("k_cache", "v_cache", "q", "R", "W"):
        a[k] = np.load(os.path.join(data_dir, k + ".npy"), mmap_mode="r")
    return a


def oracle_sample(wl, inp, data_dir):
    """Write the oracle sample (sequence 0 of ``inp``) and every group's oracle encoding."""
    import numpy as np
    import torch
    import oracle
    O = oracle.hhr_oracle
    n = int(inp["seq_len"][0])
    P = wl.page_size
    npg = -(-n // P)
    phys = inp["page_table"][0, :npg].long()
    bits = lambda t: t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    np.save(os.path.join(data_dir, "k_cache.npy"), bits(inp["k_cache"][phys]))
    np.save(os.path.join(data_dir, "v_cache.npy"), bits(inp["v_cache"][phys]))
    np.save(os.path.join(data_dir, "q.npy"), bits(inp["q"][0]))
    np.save(os.path.join(data_dir, "R.npy"), inp["R"].cpu().numpy())
    np.save(os.path.join(data_dir, "W.npy"), inp["W"].cpu().numpy())
    meta = dict(n=n, P=P, gs=wl.n_q_heads // wl.n_kv_heads, d=wl.head_dim, G=wl.n_kv_heads,
                m_pages=wl.m_pages, keep_div=wl.keep_div, top_k=wl.top_k)
    json.dump(meta, open(os.path.join(data_dir, "meta.json"), "w"))
    a = _oracle_arrays(data_dir)
    local_pt = np.arange(npg, dtype=np.int32)
    for g in range(wl.n_kv_heads):
        e = O.encode_group(a["k_cache"], local_pt, g, n, P, a["R"][g], a["W"][g])
        np.savez(os.path.join(data_dir, f"enc{g}.npz"), kmin=e["kmin"], kmax=e["kmax"],
                 codes=e["codes"])


def _oracle_worker(wid, data_dir, seconds, steps, warmup, barrier, results):
    """One host core's share of the oracle timing (a spawned process)."""
    from threadpoolctl import threadpool_limits
    import numpy as np
    import oracle
    O = oracle.hhr_oracle
    with threadpool_limits(limits=1):
        a = _oracle_arrays(data_dir)
        g = wid % a["G"]
        e = np.load(os.path.join(data_dir, f"enc{g}.npz"))
        enc = dict(kmin=np.array(e["kmin"]), kmax=np.array(e["kmax"]), codes=np.array(e["codes"]))
        for _ in range(warmup):
            oracle_group_step(O, a, enc, g)
        barrier.wait(timeout=600)
        t0 = time.perf_counter()
        done = 0
        while True:
            oracle_group_step(O, a, enc, g)
            done += 1
            el = time.perf_counter() - t0
            if steps is not None and done >= steps:
                break
            if seconds is not None and el >= seconds:
                break
    results.put((wid, done, el))


def host_cores():
    return len(os.sched_getaffinity(0))


def run_oracle_timed(wl, inp, seconds=None, steps=None, warmup=1):
    """Time the oracle's decode step on every host core. Returns queries/s (a query = the
    G group steps of one sequence), the cores used, and the group steps and wall time."""
    import multiprocessing as mp
    import tempfile
    nw = host_cores()
    with tempfile.TemporaryDirectory(prefix="hhr_oracle_") as data_dir:
        oracle_sample(wl, inp, data_dir)
        ctx = mp.get_context("spawn")
        barrier = ctx.Barrier(nw + 1)
        results = ctx.Queue()
        env_keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
        saved = {k: os.environ.get(k) for k in env_keys}
        for k in env_keys:
            os.environ[k] = "1"
        try:
            procs = [ctx.Process(target=_oracle_worker,
                                 args=(w, data_dir, seconds, steps, warmup, barrier, results))
                     for w in range(nw)]
            for p in procs:
                p.start()
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        barrier.wait(timeout=600)
        got = [results.get(timeout=600 + (seconds or 0) + 60) for _ in range(nw)]
        for p in procs:
            p.join(timeout=60)
    done = sum(x[1] for x in got)
    wall = max(x[2] for x in got)
    return dict(value=done / wall / wl.n_kv_heads, cores=nw, group_steps=done, wall_s=wall,
                steps_per_core=min(x[1] for x in got))


def oracle_sample_text(wl, r):
    keys = wl.seq_lens[0] if wl.seq_lens else "ragged"
    return (f"the fp64 oracle's decode step of sequence 0 of {wl.name} ({keys} keys): "
            f"append-encode the newest key, bounds, top-m, "
            f"Hamming top-k, attention; one spawned process per host core ({r['cores']}, BLAS "
            f"1 thread each), process w on KV group w % {wl.n_kv_heads}; {r['group_steps']} "
            f"group steps in {r['wall_s']:.2f} s; a query = {wl.n_kv_heads} group steps")


def timing_events(n, stream):
    """n pairs of timing events, each recorded once so that the CUDA event exists
    (torch creates it lazily) before its handle is given to the library's hook. The stop
    event is recorded first: a pair that no launch records again keeps a negative span."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        b.record(stream)
        a.record(stream)
    stream.synchronize()
    return evs


# ----------------------------------------------------------------------------- main

def main():
    args = parse()
    import numpy as np
    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    import hhr_synth as S
    wl = S.WORKLOADS[args.workload]
    if args.batch > 0 and wl.ragged is None:
        wl = S.scaled(wl, batch=args.batch, seq_lens=(wl.seq_lens[0],) * args.batch)

    if args.impl == "reference":
        # The oracle arm: rank 0 alone runs it on the host cores.
        if rank != 0:
            return
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        inp = S.make_inputs(wl, device=dev, layer=0)
        r = run_oracle_timed(wl, inp, steps=args.steps, warmup=args.warmup)
        val = r["value"]
        line = {
            "metric": METRIC, "value": val, "unit": "queries/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["wall_s"] / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "batch": wl.batch, "context": wl.seq_lens[0],
                       "q_heads": wl.n_q_heads, "kv_heads": wl.n_kv_heads,
                       "page_size": wl.page_size,
                       "keep": f"1/{wl.keep_div}" if wl.keep_div else f"{wl.m_pages} pages",
                       "top_k": wl.top_k, "code_bits": wl.code_bits,
                       "step": f"every host core runs one group step of the sample "
                               f"({r['cores']} group steps = {r['cores'] / wl.n_kv_heads:g} "
                               f"queries)"},
            "cpu_baseline": {"value": val, "unit": "queries/s", "cores": r["cores"],
                             "kind": "oracle", "sample": oracle_sample_text(wl, r)},
            "e2e": {"value": val, "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return

    from hash_hierarchical_top_b200 import build, hhr
    from hash_hierarchical_top_b200.step import DecodeStep, LayerCache
    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    lens = S.seq_lens_of(wl)
    P = wl.page_size
    m_of = lambda npg: min(npg, -(-npg // wl.keep_div)) if wl.m_pages == 0 else min(wl.m_pages, npg)
    f16 = 1 if args.summary == "f16" else 0
    sbytes = 2 if f16 else 4
    summ_b, codes_b, kv_b = required_bytes(wl, lens, m_of, sbytes)
    req = summ_b + codes_b + kv_b
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    L = args.layers or max(2, math.ceil(4 * l2 / req))

    # Layer caches: inputs drawn on the device (seeded), cache encoded once (untimed).
    layers = []
    for l in range(L):
        inp = S.make_inputs(wl, device=dev, layer=l, with_values=not args.select_only)
        d = hhr.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, P, inp["max_pages"],
                          inp["n_phys"], summary_fp16=f16)
        cache = LayerCache(d, dev)
        zero = torch.zeros(wl.batch, dtype=torch.int32, device=dev)
        hhr.hhr_encode_keys(d, inp["k_cache"], inp["page_table"], zero, inp["seq_len"],
                            int(inp["seq_len"].max()), inp["R"], inp["W"], cache.page_minmax,
                            cache.codes, None)
        start = (inp["seq_len"] - 1).to(torch.int32)
        one = torch.ones(wl.batch, dtype=torch.int32, device=dev)
        if not args.select_only:
            # The newest K/V row of every sequence, as a decode step receives it from the
            # model ([B][G][d]); appending it rewrites the same cache slot every step.
            t = start.long()
            phys = inp["page_table"][torch.arange(wl.batch, device=dev), t // P].long()
            inp["k_new"] = inp["k_cache"][phys, :, t % P].contiguous()
            inp["v_new"] = inp["v_cache"][phys, :, t % P].contiguous()
        layers.append((inp, d, cache, start, one))
    d0 = layers[0][1]
    step = DecodeStep(d0, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, dev,
                      attention=not args.select_only)
    # All work runs on one non-default stream (graph capture needs one); the library
    # launches on torch's current stream.
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    def run(i):
        inp, d, cache, start, one = layers[i % L]
        if args.select_only:
            step.encode(inp["k_cache"], inp["page_table"], start, one, 1, inp["R"], inp["W"],
                        cache)
            step.select(inp["q"], inp["seq_len"], inp["page_table"], cache, R=inp["R"],
                        W=inp["W"])
            return
        if args.path == "fused":
            # Append the newest K/V rows (they equal the cached ones, so every step sees the
            # same cache), encode the key, select, attend: one hhr_decode_step call.
            step.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"],
                            inp["seq_len"], inp["R"], inp["W"], cache, k_new=inp["k_new"],
                            v_new=inp["v_new"])
            return
        step.step(inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_len"],
                  inp["R"], inp["W"], cache, start, one)

    fused = args.path == "fused" and not args.select_only
    # Small batches: hhr_decode_step runs steps a2-a5 as one cluster per selection row.
    row_path = fused and hhr.hhr_decode_step_kernels(d0, wl.m_pages, wl.keep_div, wl.top_k) == 2
    if args.select_only:
        names = ("encode", "qprep", "bound", "hamming")
    elif row_path:
        names = ("encode", "row")
    elif args.path == "fused":
        names = ("encode", "bound", "hamming", "attn", "combine")
    else:
        names = ("encode", "qprep", "bound", "hamming", "attn", "combine")
    for i in range(3):  # eager warm-up: sets kernel attributes outside any capture
        run(i)
    torch.cuda.synchronize()
    st, bits = hhr.hhr_read_device_status()
    if st != hhr.HHR_OK:
        raise RuntimeError(f"device status {bits}")

    # Each decode step is one CUDA graph replay (one launch from the host). NG graphs cycle
    # over the L layer caches; graph j carries its own event pair around the dominant kernel
    # (the page bounds, or the row clusters on the small-batch path), so the last NG replays
    # of the timed region give its duration.
    rk = "row" if row_path else "bound"
    NG = L * max(1, 48 // L)
    ev_b = timing_events(NG, stream)
    graphs = []
    for j in range(NG):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            hhr.hhr_profile_next(rk, ev_b[j][0], ev_b[j][1])
            run(j)
        graphs.append(gr)
    # The same steps without the event nodes (which sit between kernels and cut the
    # programmatic-launch overlap): all timed replays but the last NG use these.
    plain = []
    for l in range(L):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            run(l)
        plain.append(gr)
    # Per-kernel breakdown graphs (events around every kernel), one per layer.
    ev_k = {name: timing_events(L, stream) for name in names}
    kgraphs = []
    for l in range(L):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for name in names:
                hhr.hhr_profile_next(name, ev_k[name][l][0], ev_k[name][l][1])
            run(l)
            for name in names:  # drop pairs of kernels this configuration did not launch
                hhr.hhr_profile_next(name, None, None)
        kgraphs.append(gr)
    torch.cuda.synchronize()

    for i in range(max(args.warmup, 3)):
        graphs[i % NG].replay()
    torch.cuda.synchronize()
    st, bits = hhr.hhr_read_device_status()
    if st != hhr.HHR_OK:
        raise RuntimeError(f"device status {bits}")

    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = Clocks(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    # The last nbr replays (about 1/16 of them, at least one per layer cache, at most NG)
    # carry the page-bound kernel's events; the rest replay the plain graphs.
    nbr = min(NG, K, max(L, (K // 16) // L * L))
    used = []
    for i in range(K):
        j = i - (K - nbr)
        if j >= 0:  # same layer rotation; each bracketed graph replays once
            used.append((j // L) * L + i % L)
            graphs[used[-1]].replay()
        else:
            plain[i % L].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    if world > 1:
        dist.barrier()
    ms_total = t0.elapsed_time(t1)
    # The bracketed replays of the timed region hold the page-bound kernel's events.
    bound_ms = [ev_b[u][0].elapsed_time(ev_b[u][1]) for u in used]
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / K
    value = job_throughput(world, wl.batch, K, ms_total)

    # Per-kernel averages: replays of the breakdown graphs, read after each replay.
    kern = {name: [] for name in names}
    for r in range(30):
        kgraphs[r % L].replay()
        torch.cuda.synchronize()
        for name in names:
            a_, b_ = ev_k[name][r % L]
            kern[name].append(a_.elapsed_time(b_) * 1e3)
    # Launches per step: every kernel of the breakdown that ran (an unlaunched kernel's
    # events are the two pre-recorded ones, stop before start: a negative span).
    kern = {k: statistics.mean(v) for k, v in kern.items() if min(v) > 0}
    kernels_per_step = len(kern)

    # End to end through the public API with host buffers: every step copies its query and
    # newest K/V rows from pinned host memory and reads its output back to pinned host memory.
    # The steps rotate over the same L layer caches as the device-timed loop (so the e2e
    # figure is as L2-cold as `value`), and consecutive steps are pipelined as a serving loop
    # would: a step's input copy runs on a copy stream while the previous step computes, its
    # output copy while the next step computes (device inputs and outputs double-buffered);
    # E_STEPS = 2 L steps are captured per graph, so only the first input and the last output
    # copy of a replay are exposed.
    e2e = None
    if not args.no_e2e and not args.select_only:
        E_STEPS = 2 * L
        Bq, G = wl.batch, wl.n_kv_heads
        nq = Bq * wl.n_q_heads * wl.head_dim
        nkv = Bq * G * wl.head_dim
        # Per layer one pinned host buffer [query | newest K rows | newest V rows] (bf16).
        host_in = []
        for l in range(L):
            inp_l = layers[l][0]
            h = torch.empty(nq + 2 * nkv, dtype=torch.bfloat16)
            h[:nq] = inp_l["q"].reshape(-1).cpu()
            h[nq:nq + nkv] = inp_l["k_new"].reshape(-1).cpu()
            h[nq + nkv:] = inp_l["v_new"].reshape(-1).cpu()
            host_in.append(h.pin_memory())
        dev_in = [torch.empty(nq + 2 * nkv, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        out_host = [torch.empty(Bq, wl.n_q_heads, wl.head_dim, dtype=torch.float32).pin_memory()
                    for _ in range(2)]
        steps = [step, DecodeStep(d0, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, dev)]
        # Each layer's output, for the check of the host copies below.
        ref_out = []
        for l in range(L):
            plain[l].replay()
            torch.cuda.synchronize()
            ref_out.append(step.out.cpu())
        cs = torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(E_STEPS)]
        ev_done = [torch.cuda.Event() for _ in range(E_STEPS)]
        ev_fork, ev_join = torch.cuda.Event(), torch.cuda.Event()

        def e2e_steps():
            ev_fork.record(stream)
            cs.wait_event(ev_fork)

            def copy_in(i):
                with torch.cuda.stream(cs):
                    dev_in[i % 2].copy_(host_in[i % L], non_blocking=True)
                    ev_in[i].record(cs)

            copy_in(0)
            copy_in(1)
            for i in range(E_STEPS):
                sl = i % 2
                inp, d, cache, start, one = layers[i % L]
                stream.wait_event(ev_in[i])
                x = dev_in[sl]
                steps[sl].fused_step(x[:nq].view(Bq, wl.n_q_heads, wl.head_dim), inp["k_cache"],
                                     inp["v_cache"], inp["page_table"], inp["seq_len"], inp["R"],
                                     inp["W"], cache, k_new=x[nq:nq + nkv].view(Bq, G, wl.head_dim),
                                     v_new=x[nq + nkv:].view(Bq, G, wl.head_dim))
                ev_done[i].record(stream)
                with torch.cuda.stream(cs):
                    cs.wait_event(ev_done[i])
                    out_host[sl].copy_(steps[sl].out, non_blocking=True)
                if i + 2 < E_STEPS:
                    copy_in(i + 2)
            ev_join.record(cs)
            stream.wait_event(ev_join)

        e2e_steps()
        torch.cuda.synchronize()
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge, stream=stream):
            e2e_steps()
        for _ in range(3):
            ge.replay()
        torch.cuda.synchronize()
        Ke = max(8, min(K, 5000) // E_STEPS)
        a, bev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(Ke):
            ge.replay()
        bev.record(stream)
        torch.cuda.synchronize()
        ms_e = max_over_ranks(a.elapsed_time(bev), world, dev)
        # Host slot s holds the output of the last step run in it: step E_STEPS - 2 + s.
        for sl in range(2):
            want = ref_out[(E_STEPS - 2 + sl) % L]
            if not torch.equal(out_host[sl], want):
                raise RuntimeError("pipelined e2e: host output differs from the device step output")
        e2e = {"value": job_throughput(world, Bq, Ke * E_STEPS, ms_e), "unit": "queries/s",
               "h2d_bytes_per_step": host_in[0].numel() * 2,
               "d2h_bytes_per_step": out_host[0].numel() * 4, "steps": Ke * E_STEPS,
               "how": f"graph replays of {E_STEPS} pipelined steps rotating over the {L} layer "
                      "caches of the device-timed loop; each step: one H2D copy of its pinned "
                      "[query | newest K | newest V] buffer (overlapping the previous step), "
                      "hhr_decode_step (which appends the rows), one D2H copy of its output "
                      "(overlapping the next step)"}

    # Bulk (prefill) encoding of one layer's whole cache on the tensor-core encoder.
    prefill = None
    if not args.select_only:
        inp, d, cache, start, one = layers[0]
        zero = torch.zeros(wl.batch, dtype=torch.int32, device=dev)
        maxn = int(inp["seq_len"].max())

        def prefill_once():
            hhr.hhr_encode_keys(d, inp["k_cache"], inp["page_table"], zero, inp["seq_len"], maxn,
                                inp["R"], inp["W"], cache.page_minmax, cache.codes, None)
        for _ in range(2):
            prefill_once()
        torch.cuda.synchronize()
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        pa.record(stream)
        for _ in range(reps):
            prefill_once()
        pb.record(stream)
        torch.cuda.synchronize()
        p_ms = pa.elapsed_time(pb) / reps
        rows = sum(lens) * wl.n_kv_heads
        # The method's own work per key-group row: k' = R k and W k' (two 128 x 128 products,
        # 2 flops per multiply-add); the kernel issues three bf16 split products of [R; W R].
        flops_method = rows * 2 * 128 * 128 * 2
        flops_issued = rows * 256 * 128 * 2 * 3
        mp = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
            os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
        tpk = float(mp.get("bf16_tflops", 1590.0))
        t_method = flops_method / (p_ms / 1e3) / 1e12
        t_issued = flops_issued / (p_ms / 1e3) / 1e12
        prefill = {"kernel": "encode_tc_kernel (tcgen05)", "keys": sum(lens),
                   "key_group_rows": rows, "ms": p_ms, "keys_per_s": sum(lens) / (p_ms / 1e3),
                   "tflops_method": t_method, "frac_method": t_method / tpk,
                   "tflops_issued_3split": t_issued, "frac_issued_3split": t_issued / tpk,
                   "peak_tflops": tpk,
                   "peak_source": "measured bf16 dense (burst)" if mp else "fallback"}

    peak, peak_kind = measured_peaks()
    kbytes = step_kernel_bytes(wl, lens, m_of, sbytes)
    bound_bytes = kbytes[rk]
    bound_avg_ms = statistics.mean(bound_ms)
    achieved = bound_bytes / (bound_avg_ms / 1e3) / 1e9
    # DRAM bytes of the profiled launch, scaled to this launch's algorithmic bytes (the
    # kernel's traffic grows in proportion to the pages and rows it reads).
    rk_name = "row_cluster" if row_path else f"page_bound_{args.summary}"
    prof = traffic_from_profile(f"{rk_name}_kernel_{wl.name}.txt", kernel_source_hash())
    traffic = prof[0] * bound_bytes / prof[1] if prof is not None else None
    step_gbs = req / (ms_step / 1e3) / 1e9

    # The other workloads (tiny single head, 32K, 128K at batch 1, the HISA indexer and the
    # ragged batch), each graph-timed on its own layer caches; single-GPU default runs only.
    other = None
    if (rank == 0 and world == 1 and not args.no_secondary and fused and args.batch == 0
            and args.workload == "llama8b_128k_b8"):
        other = {w: measure_secondary(w, dev, l2, f16, 2000, stream, 24 << 30) for w in SECONDARY}
    dense = None
    if (rank == 0 and world == 1 and not args.no_secondary and fused and args.batch == 0
            and args.workload == "llama8b_128k_b8"):
        try:
            dense = measure_dense_attention(layers, wl, dev, stream)
            dense["hhr_step_speedup"] = dense["us_per_step"] / (ms_step * 1e3)
        except Exception as exc:  # context only: never fail the run over it
            dense = {"error": f"{type(exc).__name__}: {exc}"}
    quality = None
    if (rank == 0 and world == 1 and not args.no_quality and fused and args.batch == 0
            and args.workload == "llama8b_128k_b8"):
        quality = selection_quality(dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.select_only:
        r = run_oracle_timed(wl, layers[0][0], seconds=args.cpu_seconds)
        cpu = {"value": r["value"], "unit": "queries/s", "cores": r["cores"], "kind": "oracle",
               "sample": oracle_sample_text(wl, r) + f"; {args.cpu_seconds:.0f} s per core"}

    if rank == 0:
        ck = clocks.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "context": lens[0],
                       "q_heads": wl.n_q_heads, "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim,
                       "page_size": P,
                       "keep": f"1/{wl.keep_div}" if wl.keep_div else f"{wl.m_pages} pages",
                       "top_k": wl.top_k,
                       "code_bits": wl.code_bits, "layer_caches_rotated": L,
                       "summaries": args.summary,
                       "l2": f"inputs larger than L2: steps rotate over {L} layer caches, "
                             f"{L * req / 1e6:.0f} MB of required bytes per cycle vs "
                             f"{l2 / 1e6:.0f} MB L2",
                       "parallelism": f"replicas x{world}",
                       "api": "hhr_decode_step" if args.path == "fused" else
                              "hhr_encode_keys + hhr_select + hhr_sparse_attn",
                       "timing": f"CUDA-graph replay per step, CUDA events on the stream; the "
                                 f"last {nbr} of {K} replays carry event nodes around the "
                                 f"{'row-cluster' if row_path else 'page-bound'} kernel (its "
                                 f"duration for the roofline)"},
            "roofline": {"bound": "hbm", "kernel": f"{rk_name}_kernel",
                         "scope": "the dominant kernel alone (its CUDA-event duration in "
                                  "bracketed replays); the whole step's fraction is step_hbm",
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind,
                         "traffic": traffic, "algorithmic_bytes": bound_bytes,
                         "avg_launch_us": bound_avg_ms * 1e3,
                         "step_frac_of_measured": step_gbs / peak},
            "step_hbm": {"required_bytes": req, "summaries": summ_b, "codes": codes_b,
                         "kv_rows": kv_b, "achieved_gbs": step_gbs,
                         "frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS,
                         "frac_of_measured": step_gbs / peak,
                         "dense_kv_bytes": dense_kv_bytes(wl, lens),
                         "dense_over_required": dense_kv_bytes(wl, lens) / req},
            "kernels_us": kern,
            "kernels": kernel_table(kern, kbytes, peak),
            "prefill_encode": prefill,
            "other_workloads": other,
            "dense_attention": dense,
            "selection_quality": quality,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": ck,
            "gpu_launches": kernels_per_step * K,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
