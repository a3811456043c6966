"""Plant plausible mistakes in the oracle (on the CPU) and require a pin to catch each.

This shows the pins are strong enough: a dropped term, a wrong sign or index, a
transposed operand or a wrong tie rule in any step fails at least one check.
"""
import numpy as np
import pytest

import oracle
from oracle_pins import ALL_CHECKS

O = oracle.hhr_oracle
_orig = {name: getattr(O, name) for name in dir(O) if not name.startswith("__")}


def _rotate_transposed(R, X):
    return X @ np.asarray(R, dtype=np.float64)


def _bounds_min(Qrot, kmin, kmax):
    return np.minimum(Qrot[:, None, :] * kmin[None], Qrot[:, None, :] * kmax[None]).sum(axis=(0, 2))


def _bounds_one_head(Qrot, kmin, kmax):
    return _orig["page_bounds"](Qrot[:1], kmin, kmax)


def _hamming_one_head(qcodes, codes):
    return _orig["hamming"](qcodes[:1], codes)


def _topk_ties_high(dist, tok, k):
    order = np.lexsort((-np.asarray(tok), dist))
    return np.sort(np.asarray(tok)[order[:k]])


def _topm_ties_high(scores, m):
    order = np.lexsort((-np.arange(len(scores)), -np.asarray(scores)))
    return np.sort(order[:m])


def _pack_msb_first(proj):
    n, bits = proj.shape
    words = np.zeros((n, bits // 32), dtype=np.uint32)
    for j in range(bits):
        words[:, j // 32] |= (proj[:, j] > 0).astype(np.uint32) << np.uint32(31 - j % 32)
    return words


def _attn_no_scale(Qg, Ksel, Vsel, scale):
    return _orig["sparse_attention"](Qg, Ksel, Vsel, 1.0)


def _attn_wrong_sign(Qg, Ksel, Vsel, scale):
    return _orig["sparse_attention"](Qg, Ksel, Vsel, -scale)


def _summaries_unrotated_order(Krot, P):
    # Off-by-one page boundary: pages start one key late.
    n, d = Krot.shape
    return _orig["page_summaries"](np.concatenate([Krot[:1], Krot])[:n], P)


def _block_sum(K, P):
    return _orig["block_means"](K, P) * P


def _indexer_eligible_late(q, pos, K, mu, n, P, m_blocks, k):
    return _orig["indexer_select_one"](q, pos + P, K, mu, n, P, m_blocks, k)


def _kept_floor(n_units, m_units, keep_div):
    if m_units > 0:
        return min(m_units, n_units)
    return max(1, n_units // keep_div)


def _cands_include_tail(kept, n, P):
    t = (np.asarray(kept, dtype=np.int64)[:, None] * P + np.arange(P)[None, :]).ravel()
    return t[t <= n]


def _topk_largest_ascending(score, tok, k):
    order = np.lexsort((tok, np.asarray(score)))
    return np.sort(np.asarray(tok)[order[:k]])


def _forced_local_one_early(n_pages, sink, local):
    p = np.arange(n_pages)
    return p[(p < sink) | (p >= n_pages - local - 1)]


def _forced_budget_fixed(scores, m, forced):
    forced = np.asarray(forced, dtype=np.int64)
    rest = np.setdiff1d(np.arange(len(scores)), forced)
    pick = rest[_orig["top_m"](np.asarray(scores)[rest], max(m - len(forced), 0))]
    return np.sort(np.concatenate([forced, pick]))[:m]


def _forced_keys_not_first(dist, tok, k, is_forced):
    return _orig["top_k_smallest"](dist, tok, k)


def _per_head_uses_group(inp, *, P, m_pages, keep_div, top_k, scale=None, groups=None, sink=0,
                         local=0, per_head=False):
    res = _orig["decode_step_hash"](inp, P=P, m_pages=m_pages, keep_div=keep_div, top_k=top_k,
                                    scale=scale, groups=groups, sink=sink, local=local)
    if not per_head:
        return res
    gs = inp["q"].shape[1] // inp["k_cache"].shape[1]
    return {key: [r] * gs for key, r in res.items()}


def _query_prep_unrotated_codes(R_g, W_g, Qg):
    Qrot = _orig["rotate"](R_g, Qg)
    proj = _orig["projections"](W_g, np.asarray(Qg, dtype=np.float64))  # hashes q, not q'
    nrm = np.linalg.norm(Qg, axis=1, keepdims=True)
    return Qrot, _orig["pack_sign_bits"](proj), np.abs(proj) < 1e-4 * nrm


def _projections_transposed(W_g, Xrot):
    # W applied transposed (possible only where W is square; elsewhere the shapes refuse).
    W = np.asarray(W_g, dtype=np.float64)
    return Xrot @ W if W.shape[0] == W.shape[1] else Xrot @ W.T


def _logical_rows_ignore_table(cache_bits, page_table_row, g, n, P):
    return _orig["logical_rows"](cache_bits, np.arange(len(page_table_row)), g, n, P)


def _summaries_swapped(Krot, P):
    kmin, kmax = _orig["page_summaries"](Krot, P)
    return kmax, kmin


def _indexer_pos_early(q, pos, K, mu, n, P, m_blocks, k):
    return _orig["indexer_select_one"](q, max(pos - 1, 0), K, mu, n, P, m_blocks, k)


def _bf16_wrong_shift(bits):
    u32 = bits.astype(np.uint32) << np.uint32(15)
    return u32.view(np.float32).astype(np.float64)


def _fragile_everything(proj, X, rel=1e-4):
    return np.ones(np.shape(proj), dtype=bool)


def _fragile_wrong_scale(proj, X, rel=1e-4):
    return _orig["fragile_mask"](proj, X, rel * 100)


MUTATIONS = {
    "rotate_transposed": ("rotate", _rotate_transposed),
    "bound_min_not_max": ("page_bounds", _bounds_min),
    "bound_drops_heads": ("page_bounds", _bounds_one_head),
    "hamming_drops_heads": ("hamming", _hamming_one_head),
    "topk_ties_to_higher": ("top_k_smallest", _topk_ties_high),
    "topm_ties_to_higher": ("top_m", _topm_ties_high),
    "pack_msb_first": ("pack_sign_bits", _pack_msb_first),
    "attention_no_scale": ("sparse_attention", _attn_no_scale),
    "attention_wrong_sign": ("sparse_attention", _attn_wrong_sign),
    "summaries_page_shift": ("page_summaries", _summaries_unrotated_order),
    "block_sum_not_mean": ("block_means", _block_sum),
    "indexer_causal_off": ("indexer_select_one", _indexer_eligible_late),
    "kept_floor": ("kept_count", _kept_floor),
    "candidates_past_end": ("candidates_of", _cands_include_tail),
    "indexer_smallest_scores": ("top_k_largest", _topk_largest_ascending),
    "forced_local_one_early": ("forced_pages", _forced_local_one_early),
    "forced_budget_not_grown": ("top_m_forced", _forced_budget_fixed),
    "forced_keys_not_first": ("top_k_forced", _forced_keys_not_first),
    "per_head_uses_group": ("decode_step_hash", _per_head_uses_group),
    "query_codes_unrotated": ("query_prep", _query_prep_unrotated_codes),
    "projections_transposed": ("projections", _projections_transposed),
    "page_table_ignored": ("logical_rows", _logical_rows_ignore_table),
    "summaries_min_max_swapped": ("page_summaries", _summaries_swapped),
    "indexer_causal_one_early": ("indexer_select_one", _indexer_pos_early),
    "bf16_wrong_shift": ("bf16_to_f64", _bf16_wrong_shift),
    "fragile_everything": ("fragile_mask", _fragile_everything),
    "fragile_wrong_scale": ("fragile_mask", _fragile_wrong_scale),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(O)
        except (AssertionError, IndexError, ValueError):
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
