"""Plain fp64 CPU oracle of coarse-to-fine key retrieval for top-k sparse attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only the test suite, the package's smoke check and the benchmark's CPU-baseline
leg use it. It shares no code, table or helper with the CUDA path.

It follows, step by step and in fp64, the two retrieval schemes of the pages:

* HHR (page "HHR: Hierarchical Hash Retrieval for Efficient LLM Generation",
  Abstract): Geometry-Aware Key Routing (GKR) rotates keys with a head-wise
  orthogonal R_h and prunes pages by page-level logit bounds; Learned Hash
  Projection (LHP) then ranks the keys of the surviving pages by the Hamming
  distance between binary codes of a head-wise projection; attention runs over
  the selected keys only.
* HISA (page "HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse
  Attention", Abstract): a block-level coarse filter scores pooled block
  representatives, then the original token indexer runs inside the kept blocks
  and a token top-k is taken.

The pages give prose only. Where they are silent, the reading taken here is the
plainest one and is listed in the design notes (rotation as x' = R x, hashing in
the rotated space, bit j = [projection_j > 0] packed LSB-first, one selection per
KV group with scores summed over the group's query heads, ties to the lower
index, kept pages m = ceil(n / keep_div), partial pages use valid keys only).

Inputs are the raw arrays of ``hhr_synth`` converted to numpy: bf16 arrays as
uint16 bit patterns (widened exactly), R and W as float32 (widened exactly).
"""
from __future__ import annotations

import math

import numpy as np


# --------------------------------------------------------------------------- inputs

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def logical_rows(cache_bits, page_table_row, g, n, P):
    """Rows 0..n-1 of KV group g of one sequence, gathered through its page table.

    cache_bits: uint16 [n_phys][G][P][d]; returns float64 [n][d].
    """
    n_pages = -(-n // P)
    phys = np.asarray(page_table_row[:n_pages], dtype=np.int64)
    rows = cache_bits[phys, g]                       # [n_pages][P][d]
    rows = rows.reshape(n_pages * P, -1)[:n]
    return bf16_to_f64(rows)


def kept_count(n_units, m_units, keep_div):
    """Kept pages (or blocks): m given absolutely (m>0), else ceil(n/keep_div); clipped to n."""
    if m_units > 0:
        return min(m_units, n_units)
    return min(n_units, -(-n_units // keep_div))


# --------------------------------------------------------------------------- step a0 / a1
# GKR rotation and LHP sign codes (HHR page, Abstract: "encoding queries and keys into
# binary codes"; Figure 2 caption: a projection followed by sign(.); Table 4: 128-bit codes).

def rotate(R_g, X):
    """x' = R_g x for every row x of X (float64)."""
    return X @ np.asarray(R_g, dtype=np.float64).T


def projections(W_g, Xrot):
    """p = W_g x' for every row x' (float64), shape [n][bits]."""
    return Xrot @ np.asarray(W_g, dtype=np.float64).T


def pack_sign_bits(proj):
    """Code words: bit j of the code is [p_j > 0], stored in word j//32 at bit j%32."""
    n, bits = proj.shape
    words = np.zeros((n, bits // 32), dtype=np.uint32)
    positive = proj > 0
    for j in range(bits):
        words[:, j // 32] |= positive[:, j].astype(np.uint32) << np.uint32(j % 32)
    return words


def sign_codes(R_g, W_g, X):
    """Codes of the raw rows X: sign bits of W_g R_g x, packed."""
    return pack_sign_bits(projections(W_g, rotate(R_g, X)))


def fragile_mask(proj, X, rel=1e-4):
    """Bits whose projection is too close to zero to be fixed by the code tolerance:
    |proj_j| < rel * ||x|| for each row x of X. Boolean [n][bits]."""
    nrm = np.linalg.norm(np.asarray(X, dtype=np.float64), axis=1, keepdims=True)
    return np.abs(proj) < rel * nrm


def fragile_bits(R_g, W_g, X, rel=1e-4):
    """fragile_mask of the projections W_g R_g x of the rows of X."""
    return fragile_mask(projections(W_g, rotate(R_g, X)), X, rel)


def page_summaries(Krot, P):
    """Per page, per channel min and max of the rotated keys over the page's valid keys.

    Krot: float64 [n][d] (logical order). Returns (kmin, kmax), each [n_pages][d].
    """
    n, d = Krot.shape
    n_pages = -(-n // P)
    kmin = np.empty((n_pages, d))
    kmax = np.empty((n_pages, d))
    for p in range(n_pages):
        rows = Krot[p * P: min(n, (p + 1) * P)]
        kmin[p] = rows.min(axis=0)
        kmax[p] = rows.max(axis=0)
    return kmin, kmax


def block_means(K, P):
    """HISA pooled block representative: mean of the block's valid (raw) keys, [n_blk][d]."""
    n, d = K.shape
    n_blk = -(-n // P)
    mu = np.empty((n_blk, d))
    for i in range(n_blk):
        mu[i] = K[i * P: min(n, (i + 1) * P)].mean(axis=0)
    return mu


def encode_group(k_bits, page_table_row, g, n, P, R_g, W_g):
    """Step a0 for one sequence and KV group: summaries of every page and codes of every key.

    Returns dict(kmin, kmax [n_pages][d], codes uint32 [n][bits/32], fragile [n][bits]).
    """
    K = logical_rows(k_bits, page_table_row, g, n, P)
    Krot = rotate(R_g, K)
    kmin, kmax = page_summaries(Krot, P)
    proj = projections(W_g, Krot)
    return dict(kmin=kmin, kmax=kmax, codes=pack_sign_bits(proj), fragile=fragile_mask(proj, K))


def query_prep(R_g, W_g, Qg):
    """Step a1: rotated queries q'_h = R_g q_h and their codes, for the heads of one group."""
    Qrot = rotate(R_g, Qg)
    proj = projections(W_g, Qrot)
    return Qrot, pack_sign_bits(proj), fragile_mask(proj, Qg)


# --------------------------------------------------------------------------- step a2
# GKR page-level logit bound and pruning (HHR page, Abstract: "derive more discriminative
# page-level logit bounds, enabling effective pruning of low-logit keys").

def page_bounds(Qrot, kmin, kmax):
    """beta_p = sum over the group's heads h and channels d of max(q'_hd*kmin_pd, q'_hd*kmax_pd).

    An upper bound on sum_h q'_h . k'_t for every valid key t of page p.
    """
    lo = Qrot[:, None, :] * kmin[None, :, :]          # [h][p][d]
    hi = Qrot[:, None, :] * kmax[None, :, :]
    return np.maximum(lo, hi).sum(axis=(0, 2))


def top_m(scores, m):
    """Indices of the m largest scores, ties to the lower index; returned ascending."""
    order = np.lexsort((np.arange(len(scores)), -np.asarray(scores)))
    return np.sort(order[:m])


# --------------------------------------------------------------------------- step a3 / a4
# LHP Hamming ranking (HHR page, Abstract: "using Hamming distance for key selection";
# HATA page, Abstract: hash codes give the relative qk score order for top-k attention).

def hamming(qcodes, codes):
    """delta_t = sum over the group's heads of popcount(qcode_h XOR code_t). [n]"""
    x = codes[None, :, :] ^ qcodes[:, None, :]       # [h][n][W]
    return np.bitwise_count(x).astype(np.int64).sum(axis=(0, 2))


def top_k_smallest(dist, tok, k):
    """The k candidates with the smallest (dist, token) pairs, returned as tokens ascending."""
    order = np.lexsort((tok, dist))
    return np.sort(np.asarray(tok)[order[:k]])


def top_k_largest(score, tok, k):
    """The k candidates with the largest score, ties to the lower token, tokens ascending."""
    order = np.lexsort((tok, -np.asarray(score)))
    return np.sort(np.asarray(tok)[order[:k]])


def candidates_of(kept_pages, n, P):
    """Logical tokens of the kept pages that exist (t < n), in ascending order."""
    t = (np.asarray(kept_pages, dtype=np.int64)[:, None] * P + np.arange(P)[None, :]).ravel()
    return t[t < n]


# --------------------------------------------------------------------------- forced pages
# Variant: sink and local-window pages. Neither HHR nor HISA forces any page; the HHR page's
# MagicPIG baseline attends to sink tokens and a local window (HHR appendix, baseline
# settings). Reading taken: the first `sink` and the last `local` logical pages of a sequence
# are always kept, inside the page budget (which grows only when it is smaller than the forced
# set), and their keys are selected ahead of the Hamming ranking, in token order.

def forced_pages(n_pages, sink, local):
    """Logical pages [0, sink) and [n_pages - local, n_pages), ascending."""
    p = np.arange(n_pages)
    return p[(p < sink) | (p >= n_pages - local)]


def top_m_forced(scores, m, forced):
    """The forced pages plus the m' - |forced| largest other scores (ties to the lower index),
    m' = max(m, |forced|); returned ascending. No forced pages: top_m."""
    forced = np.asarray(forced, dtype=np.int64)
    rest = np.setdiff1d(np.arange(len(scores)), forced)
    m_eff = max(m, len(forced))
    pick = rest[top_m(np.asarray(scores)[rest], m_eff - len(forced))]
    return np.sort(np.concatenate([forced, pick]))


def top_k_forced(dist, tok, k, is_forced):
    """k candidates: the forced ones first (in token order), then the smallest (dist, token)
    pairs of the rest; returned as tokens ascending. No forced candidates: top_k_smallest."""
    primary = np.where(np.asarray(is_forced, dtype=bool), -1, np.asarray(dist, dtype=np.int64))
    order = np.lexsort((tok, primary))
    return np.sort(np.asarray(tok)[order[:k]])


# --------------------------------------------------------------------------- step a5
# Attention over the selected subset only (HISA page, Abstract: "computing attention only
# over the selected subset"; GQA layout from HHR appendix Table 3: 32 heads, 8 KV heads).

def sparse_attention(Qg, Ksel, Vsel, scale):
    """o_h = sum_t softmax_t(scale * q_h . k_t) v_t over the selected rows, per head h."""
    if Ksel.shape[0] == 0:
        return np.zeros((Qg.shape[0], Vsel.shape[1]))
    logits = (Qg @ Ksel.T) * scale                   # [h][k]
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return (e @ Vsel) / e.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------- composites

def select_group(Qg, R_g, W_g, kmin, kmax, codes, n, P, m, k, sink=0, local=0):
    """Steps a1-a4 for one (sequence, KV group) in the HHR order: bound, prune, Hamming, top-k.

    codes are indexed by logical token; sink/local: forced pages (variant, see forced_pages).
    Returns a dict of every intermediate.
    """
    Qrot, qcodes, qfragile = query_prep(R_g, W_g, Qg)
    beta = page_bounds(Qrot, kmin, kmax)
    forced = forced_pages(len(beta), sink, local)
    if len(forced):
        kept = top_m_forced(beta, m, forced)
    else:
        kept = top_m(beta, m)
    cand = candidates_of(kept, n, P)
    delta = hamming(qcodes, codes[cand])
    if len(forced):
        S = top_k_forced(delta, cand, min(k, len(cand)), np.isin(cand // P, forced))
    else:
        S = top_k_smallest(delta, cand, min(k, len(cand)))
    return dict(q_rot=Qrot, qcodes=qcodes, qfragile=qfragile, bounds=beta, kept=kept,
                cand=cand, delta=delta, idx=S)


def decode_step_hash(inp, *, P, m_pages, keep_div, top_k, scale=None, groups=None, sink=0,
                     local=0, per_head=False):
    """Whole HHR decode step (a0-a5) for every (sequence, KV group), or for ``groups`` only;
    sink/local: forced pages (variant). per_head (variant): one selection per query head
    instead of per KV group -- head h of group g scores the group's summaries and codes
    with its own query alone and attends its own selection; the result for (b, g) is then
    a list of per-head dicts.

    inp: numpy dict from hhr_synth.to_numpy_inputs. Returns {(b, g): dict}.
    """
    k_bits, v_bits, q_bits = inp["k_cache"], inp["v_cache"], inp["q"]
    R, W, pt, lens = inp["R"], inp["W"], inp["page_table"], inp["seq_len"]
    B, Hq, d = q_bits.shape
    G = k_bits.shape[1]
    gs = Hq // G
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = {}
    for b in range(B):
        n = int(lens[b])
        n_pages = -(-n // P)
        m = kept_count(n_pages, m_pages, keep_div)
        for g in range(G):
            if groups is not None and (b, g) not in groups:
                continue
            enc = encode_group(k_bits, pt[b], g, n, P, R[g], W[g])
            Qg = bf16_to_f64(q_bits[b, g * gs:(g + 1) * gs])
            K = logical_rows(k_bits, pt[b], g, n, P)
            V = logical_rows(v_bits, pt[b], g, n, P)
            m_eff = max(m, len(forced_pages(n_pages, sink, local)))
            heads = [Qg[h:h + 1] for h in range(gs)] if per_head else [Qg]
            res = []
            for Qs in heads:
                r = select_group(Qs, R[g], W[g], enc["kmin"], enc["kmax"], enc["codes"], n, P,
                                 m, top_k, sink, local)
                r["out"] = sparse_attention(Qs, K[r["idx"]], V[r["idx"]], scale)
                r.update(enc)
                r["m"] = m_eff
                res.append(r)
            out[(b, g)] = res if per_head else res[0]
    return out


def indexer_select_one(q, pos, K, mu, n, P, m_blocks, k):
    """HISA for one query at absolute position pos (steps a1', a3, a4 of the indexer variant).

    Blocks whose start is <= pos are eligible; the m_blocks best by q . mu (ties to the
    lower block) are kept; inside them, tokens t <= pos (and t < n) are scored exactly by
    q . k_t and the top-k by (score desc, token asc) is returned ascending.
    """
    n_elig = min(pos // P + 1, -(-n // P))
    sblk = mu[:n_elig] @ q
    kept = top_m(sblk, min(m_blocks, n_elig))
    cand = candidates_of(kept, min(n, pos + 1), P)
    sigma = K[cand] @ q
    S = top_k_largest(sigma, cand, min(k, len(cand)))
    return dict(block_scores=sblk, kept=kept, cand=cand, sigma=sigma, idx=S)


def decode_step_indexer(inp, *, P, m_blocks, top_k, queries=None):
    """HISA indexer selection for every sequence and chunk query (or those in ``queries``).

    Single indexer head: k_cache is [n_phys][1][P][d], q is [B][T][d], q_pos [B][T].
    Returns {(b, i): dict}.
    """
    k_bits, q_bits, pt, lens = inp["k_cache"], inp["q"], inp["page_table"], inp["seq_len"]
    qpos = inp["q_pos"]
    B, T, d = q_bits.shape
    out = {}
    for b in range(B):
        n = int(lens[b])
        K = logical_rows(k_bits, pt[b], 0, n, P)
        mu = block_means(K, P)
        for i in range(T):
            if queries is not None and (b, i) not in queries:
                continue
            q = bf16_to_f64(q_bits[b, i])
            r = indexer_select_one(q, int(qpos[b, i]), K, mu, n, P, m_blocks, top_k)
            r["block_means"] = mu
            out[(b, i)] = r
    return out
