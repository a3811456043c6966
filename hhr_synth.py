"""Seeded synthetic workloads for the decode-time coarse-to-fine retrieval path.

This module only draws inputs: query, paged K/V cache, page table, sequence
lengths, the head-wise orthogonal rotation R and the hash projection W. It holds
none of the method's arithmetic (no rotation, bound, code, distance, selection or
attention step), so both the CPU oracle and the CUDA path can take their inputs
from here without sharing any computation.

Shapes follow the Llama-3.1-8B layout printed in the HHR appendix (Table 3:
32 attention heads, 8 KV heads, hidden 4096, so head_dim 128, max context
131072). The HHR pages evaluate on LongBench / RULER / NIAH with trained models;
none of that is available here, so seeded Gaussian caches with magnitude-outlier
channels (the motivation of HHR Figure 3) and a slowly drifting per-page key mean
stand in for real activations.

Randomness comes from ``torch.Generator`` on the requested device. The same seed
gives different numbers on CPU and on CUDA; every consumer uses one device per
workload instance and hands the resulting arrays to both sides.

Layouts (all row-major, "phys" = physical page index into a shared pool):
  k_cache, v_cache : bf16 [n_phys][G][P][d]
  q                : bf16 [B][Hq][d]   (hash mode)  or [B][T][d] (indexer mode)
  R                : f32  [G][d][d]    orthogonal, applied as x' = R x
  W                : f32  [G][bits][d] hash projection, applied to x'
  page_table       : i32  [B][max_pages]  logical page -> physical page
  seq_len          : i32  [B]
  q_pos            : i32  [B][T] absolute positions of chunk queries (indexer)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int                 # seed family
    mode: str                   # "hash" or "indexer"
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    page_size: int
    code_bits: int
    seq_lens: tuple             # per sequence, or () for ragged (drawn at generation)
    m_pages: int                # >0: absolute kept pages (clipped to n_b)
    keep_div: int               # >0: kept pages = ceil(n_b / keep_div)
    top_k: int
    n_outlier: int
    outlier_scale: float
    drift_sigma: float          # AR(1) innovation std of the per-page key mean (0 = none)
    drift_rho: float = 0.99
    n_queries: int = 1          # indexer: chunk length T
    n_needles: int = 0
    needle_scale: float = 4.0
    ragged: Optional[tuple] = None   # (lo, hi) inclusive bounds of per-sequence lengths
    permute_pages: bool = False      # page table = random permutation of the pool
    sink_pages: int = 0              # selection variant: forced first pages of a sequence
    local_pages: int = 0             # selection variant: forced last pages of a sequence
    select_per_head: bool = False    # selection variant: one selection per query head
    # Planted page locality (quality workloads only): per sequence and KV group, hot_runs runs
    # of hot_run_pages consecutive logical pages whose keys are shifted by
    # hot_scale * sqrt(head_dim) along the group's mean query direction, so that the keys a
    # query attends to cluster in a few pages, as relevant context does in real attention.
    hot_runs: int = 0
    hot_run_pages: int = 0
    hot_scale: float = 0.0

    @property
    def group_size(self):
        return self.n_q_heads // self.n_kv_heads


def _wl(**kw):
    return Workload(**kw)


WORKLOADS = {
    # Tiny single-head decode: 64 pages of 64 keys, keep 16, top-256.
    "tiny_1h_4k": _wl(name="tiny_1h_4k", cfg_id=1, mode="hash", batch=1, n_q_heads=1,
                      n_kv_heads=1, head_dim=128, page_size=64, code_bits=128,
                      seq_lens=(4096,), m_pages=16, keep_div=0, top_k=256,
                      n_outlier=4, outlier_scale=8.0, drift_sigma=0.0),
    # Llama-3.1-8B decode layer at 32K: 1024 pages of 32, keep 1/8, top 10% of context.
    "llama8b_32k": _wl(name="llama8b_32k", cfg_id=2, mode="hash", batch=1, n_q_heads=32,
                       n_kv_heads=8, head_dim=128, page_size=32, code_bits=128,
                       seq_lens=(32768,), m_pages=0, keep_div=8, top_k=3276,
                       n_outlier=6, outlier_scale=10.0, drift_sigma=0.1),
    # Same shapes at 128K: 4096 pages of 32, keep 1/16, top-2048; batch 1 and 8.
    "llama8b_128k_b1": _wl(name="llama8b_128k_b1", cfg_id=3, mode="hash", batch=1,
                           n_q_heads=32, n_kv_heads=8, head_dim=128, page_size=32,
                           code_bits=128, seq_lens=(131072,), m_pages=0, keep_div=16,
                           top_k=2048, n_outlier=6, outlier_scale=10.0, drift_sigma=0.1),
    "llama8b_128k_b8": _wl(name="llama8b_128k_b8", cfg_id=3, mode="hash", batch=8,
                           n_q_heads=32, n_kv_heads=8, head_dim=128, page_size=32,
                           code_bits=128, seq_lens=(131072,) * 8, m_pages=0, keep_div=16,
                           top_k=2048, n_outlier=6, outlier_scale=10.0, drift_sigma=0.1),
    # HISA indexer variant: one indexer head, 128-key blocks, keep 64 blocks, top-2048.
    "hisa_128k_t1": _wl(name="hisa_128k_t1", cfg_id=4, mode="indexer", batch=1,
                        n_q_heads=1, n_kv_heads=1, head_dim=128, page_size=128,
                        code_bits=128, seq_lens=(131072,), m_pages=64, keep_div=0,
                        top_k=2048, n_outlier=0, outlier_scale=1.0, drift_sigma=0.0,
                        n_queries=1, n_needles=32),
    "hisa_128k_t64": _wl(name="hisa_128k_t64", cfg_id=4, mode="indexer", batch=1,
                         n_q_heads=1, n_kv_heads=1, head_dim=128, page_size=128,
                         code_bits=128, seq_lens=(131072,), m_pages=64, keep_div=0,
                         top_k=2048, n_outlier=0, outlier_scale=1.0, drift_sigma=0.0,
                         n_queries=64, n_needles=32),
    # Ragged serving batch: 32 sequences of 8K..128K keys in a permuted shared page pool.
    "ragged_b32": _wl(name="ragged_b32", cfg_id=5, mode="hash", batch=32, n_q_heads=32,
                      n_kv_heads=8, head_dim=128, page_size=32, code_bits=128, seq_lens=(),
                      m_pages=0, keep_div=16, top_k=1024, n_outlier=6, outlier_scale=10.0,
                      drift_sigma=0.1, ragged=(8192, 131072), permute_pages=True),
}


# Variants of the 128K batch-8 decode (same keys, queries and rotations): a flat hash top-k
# (every page kept), forced sink and local pages, and codes of 64 or 256 bits (W has 64 or
# 256 rows).
WORKLOADS["llama8b_128k_b8_flat"] = dataclasses.replace(
    WORKLOADS["llama8b_128k_b8"], name="llama8b_128k_b8_flat", m_pages=4096, keep_div=0)
WORKLOADS["llama8b_128k_b8_sink1_local2"] = dataclasses.replace(
    WORKLOADS["llama8b_128k_b8"], name="llama8b_128k_b8_sink1_local2", sink_pages=1,
    local_pages=2)
WORKLOADS["llama8b_128k_b8_per_head"] = dataclasses.replace(
    WORKLOADS["llama8b_128k_b8"], name="llama8b_128k_b8_per_head", select_per_head=True)
for _bits in (64, 256):
    _n = f"llama8b_128k_b8_codes{_bits}"
    WORKLOADS[_n] = dataclasses.replace(WORKLOADS["llama8b_128k_b8"], name=_n, code_bits=_bits)

# Quality workloads with planted page locality (selection_quality only): the 128K decode at
# batch 2 with 8 runs of 8 hot pages per KV group (2048 hot keys, as many as the top-k), and
# the HISA single query with 4 runs of 4 hot 128-key blocks (2048 hot keys).
WORKLOADS["llama8b_128k_planted"] = dataclasses.replace(
    WORKLOADS["llama8b_128k_b8"], name="llama8b_128k_planted", cfg_id=6, batch=2,
    seq_lens=(131072,) * 2, hot_runs=8, hot_run_pages=8, hot_scale=2.5)
WORKLOADS["hisa_128k_t1_planted"] = dataclasses.replace(
    WORKLOADS["hisa_128k_t1"], name="hisa_128k_t1_planted", cfg_id=7, n_needles=0,
    hot_runs=4, hot_run_pages=4, hot_scale=0.5)


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of ``wl`` with some fields replaced (e.g. shorter contexts for parity tests)."""
    return dataclasses.replace(wl, **changes)


# Seed streams: key = 1000*cfg_id + j, j as below, plus the sequence index and layer.
J_KEYS, J_VALUES, J_QUERIES, J_R, J_W, J_OUTLIER, J_DRIFT, J_LAYOUT, J_NEEDLE, J_HOT = range(10)


def _gen(device, wl, j, *extra):
    # Mix the stream id into one 63-bit seed (odd multipliers; plain integer hashing).
    s = 1000 * wl.cfg_id + j
    for e in extra:
        s = (s * 0x9E3779B1 + 0x85EBCA77 * (e + 1)) % (1 << 62)
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def seq_lens_of(wl: Workload) -> list:
    if wl.ragged is None:
        return list(wl.seq_lens)
    lo, hi = wl.ragged
    g = _gen("cpu", wl, J_LAYOUT, 0)
    return [int(x) for x in torch.randint(lo, hi + 1, (wl.batch,), generator=g)]


def make_inputs(wl: Workload, device="cpu", layer: int = 0, with_values: bool = True):
    """Draw every input of one decode step of ``wl`` on ``device``.

    Returns a dict of torch tensors (see the module docstring for layouts) plus
    python ints ``n_phys`` and ``max_pages``.
    """
    B, G, Hq, d, P = wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.page_size
    lens = seq_lens_of(wl)
    npages = [-(-n // P) for n in lens]
    max_pages = max(npages)
    n_phys = sum(npages)

    # Page table: sequence b owns npages[b] distinct physical pages of the pool.
    page_table = torch.full((B, max_pages), -1, dtype=torch.int32)
    if wl.permute_pages:
        perm = torch.randperm(n_phys, generator=_gen("cpu", wl, J_LAYOUT, 1 + layer))
    else:
        perm = torch.arange(n_phys)
    off = 0
    for b in range(B):
        page_table[b, : npages[b]] = perm[off: off + npages[b]].to(torch.int32)
        off += npages[b]

    # Outlier channels: a seeded set per KV group, shared by q, k and v of that group.
    scale = torch.ones(G, d)
    if wl.n_outlier > 0:
        go = _gen("cpu", wl, J_OUTLIER, layer)
        for g in range(G):
            ch = torch.randperm(d, generator=go)[: wl.n_outlier]
            scale[g, ch] = wl.outlier_scale
    scale = scale.to(device)

    k_cache = torch.zeros(n_phys, G, P, d, dtype=torch.bfloat16, device=device)
    v_cache = torch.zeros_like(k_cache) if with_values else None
    T = wl.n_queries if wl.mode == "indexer" else Hq

    # Queries first: needles (indexer) are aligned with the chunk's mean query.
    gq = _gen(device, wl, J_QUERIES, layer)
    q = torch.randn(B, T, d, generator=gq, device=device)
    if wl.mode == "hash":
        q = q * scale.repeat_interleave(wl.group_size, dim=0)[None]
    q_bf = q.to(torch.bfloat16)

    for b in range(B):
        n = lens[b]
        gk = _gen(device, wl, J_KEYS, b, layer)
        k = torch.randn(G, n, d, generator=gk, device=device) * scale[:, None, :]
        if wl.drift_sigma > 0:
            # AR(1) walk over logical pages, mu_{p+1} = rho*mu_p + eps_p: a slowly drifting
            # per-page key mean that stays bounded at any context length. Drawn on the CPU.
            gd = _gen("cpu", wl, J_DRIFT, b, layer)
            eps = torch.randn(npages[b], G, d, generator=gd, dtype=torch.float64) * wl.drift_sigma
            mu = torch.empty_like(eps)
            acc = torch.zeros(G, d, dtype=torch.float64)
            for p in range(npages[b]):
                acc = wl.drift_rho * acc + eps[p]
                mu[p] = acc
            mu = mu.to(torch.float32).to(device).permute(1, 0, 2)
            k = k + mu.repeat_interleave(P, dim=1)[:, :n]
        if wl.n_needles > 0:
            gn = _gen("cpu", wl, J_NEEDLE, b, layer)
            pos = torch.randperm(n, generator=gn)[: wl.n_needles].to(device)
            u = q[b].float().mean(0)
            u = u / u.norm()
            k[:, pos, :] = (wl.needle_scale * math.sqrt(d) * u)[None, None, :]
        if wl.hot_runs > 0:
            k = k + _hot_shift(wl, q[b], b, n, layer, device)
        _scatter(k_cache, page_table[b].to(device), k.to(torch.bfloat16), P)
        del k
        if with_values:
            gv = _gen(device, wl, J_VALUES, b, layer)
            v = torch.randn(G, n, d, generator=gv, device=device) * scale[:, None, :]
            _scatter(v_cache, page_table[b].to(device), v.to(torch.bfloat16), P)
            del v

    gR = _gen("cpu", wl, J_R, layer)
    R = torch.empty(G, d, d, dtype=torch.float32)
    for g in range(G):
        a = torch.randn(d, d, generator=gR, dtype=torch.float64)
        Qm, Rr = torch.linalg.qr(a)
        # Fix the column signs so the factorisation is unique.
        Qm = Qm * torch.sign(torch.diagonal(Rr))[None, :]
        R[g] = Qm.to(torch.float32)
    W = lhp_projection(wl, layer)

    out = dict(
        k_cache=k_cache, v_cache=v_cache, q=q_bf,
        R=R.to(device), W=W.to(device),
        page_table=page_table.to(device),
        seq_len=torch.tensor(lens, dtype=torch.int32, device=device),
        n_phys=n_phys, max_pages=max_pages,
    )
    if wl.mode == "indexer":
        qp = torch.tensor([[lens[b] - T + i for i in range(T)] for b in range(B)],
                          dtype=torch.int32)
        out["q_pos"] = qp.to(device)
    return out


def hot_pages(wl: Workload, b: int, n: int, layer: int = 0) -> list:
    """The planted hot logical pages of sequence b (n keys), per KV group: hot_runs runs of
    hot_run_pages consecutive pages, at distinct run-aligned starts drawn from the sequence's
    hot stream."""
    npg = -(-n // wl.page_size)
    slots = max(npg // wl.hot_run_pages, 1)
    gh = _gen("cpu", wl, J_HOT, b, layer)
    out = []
    for _ in range(wl.n_kv_heads):
        starts = torch.randperm(slots, generator=gh)[: wl.hot_runs] * wl.hot_run_pages
        pages = sorted(int(s0) + i for s0 in starts for i in range(wl.hot_run_pages)
                       if int(s0) + i < npg)
        out.append(pages)
    return out


def _hot_shift(wl: Workload, qb: torch.Tensor, b: int, n: int, layer: int, device):
    """Key shift [G][n][d] of the planted hot pages of sequence b: hot_scale * sqrt(d) times
    the unit mean query direction of each KV group (its query heads, or the chunk queries of
    the one indexer head)."""
    G, d, P = wl.n_kv_heads, wl.head_dim, wl.page_size
    per = qb.shape[0] // G
    shift = torch.zeros(G, n, d, device=device)
    for g, pages in enumerate(hot_pages(wl, b, n, layer)):
        u = qb[g * per:(g + 1) * per].float().mean(0)
        u = u / u.norm()
        for p in pages:
            shift[g, p * P: min((p + 1) * P, n)] = wl.hot_scale * math.sqrt(d) * u
    return shift


def lhp_projection(wl: Workload, layer: int = 0) -> torch.Tensor:
    """The projection W [G][code_bits][d] (float32, CPU) of a layer: N(0, 1) entries drawn
    group by group from the layer's W stream, the same draws make_inputs uses."""
    gW = _gen("cpu", wl, J_W, layer)
    W = torch.empty(wl.n_kv_heads, wl.code_bits, wl.head_dim, dtype=torch.float32)
    for g in range(wl.n_kv_heads):
        W[g] = torch.randn(wl.code_bits, wl.head_dim, generator=gW)
    return W


def _scatter(cache, pt_row, k, P):
    """Place logical keys k [G][n][d] into their physical pages (zero tail)."""
    G, n, d = k.shape
    npg = -(-n // P)
    pad = npg * P - n
    if pad:
        k = torch.cat([k, torch.zeros(G, pad, d, dtype=k.dtype, device=k.device)], dim=1)
    k = k.view(G, npg, P, d).permute(1, 0, 2, 3)
    cache[pt_row[:npg].long()] = k


def to_numpy_inputs(inp: dict) -> dict:
    """Host numpy copies; bf16 arrays become their raw uint16 bit patterns."""
    import numpy as np
    out = {}
    for key, v in inp.items():
        if isinstance(v, torch.Tensor):
            v = v.detach().cpu()
            if v.dtype == torch.bfloat16:
                out[key] = v.view(torch.int16).numpy().view(np.uint16)
            else:
                out[key] = v.numpy()
        else:
            out[key] = v
    return out
