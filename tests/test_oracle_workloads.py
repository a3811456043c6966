"""The oracle on the seeded workloads themselves (CPU only): invariants at workload scale."""
import numpy as np

import hhr_synth as S
import oracle

O = oracle.hhr_oracle


def test_tiny_workload_invariants():
    wl = S.WORKLOADS["tiny_1h_4k"]
    inp = S.to_numpy_inputs(S.make_inputs(wl))
    res = O.decode_step_hash(inp, P=wl.page_size, m_pages=wl.m_pages, keep_div=wl.keep_div,
                             top_k=wl.top_k)
    r = res[(0, 0)]
    n, P = int(inp["seq_len"][0]), wl.page_size
    K = O.logical_rows(inp["k_cache"], inp["page_table"][0], 0, n, P)
    Q = O.bf16_to_f64(inp["q"][0])
    logits = (O.rotate(inp["R"][0], Q) @ O.rotate(inp["R"][0], K).T).sum(axis=0)
    per_page_max = logits.reshape(-1, P).max(axis=1)
    assert np.all(r["bounds"] >= per_page_max - 1e-9 * np.abs(per_page_max).max())
    assert len(r["kept"]) == wl.m_pages and len(r["idx"]) == wl.top_k
    assert set((r["idx"] // P).tolist()) <= set(r["kept"].tolist())
    assert np.all(np.diff(r["idx"]) > 0)
    # Pruning keeps pages whose bound is at least that of every pruned page.
    pruned = np.setdiff1d(np.arange(n // P), r["kept"])
    assert r["bounds"][r["kept"]].min() >= r["bounds"][pruned].max()


def test_hisa_needles_are_selected():
    wl = S.scaled(S.WORKLOADS["hisa_128k_t1"], seq_lens=(32768,), m_pages=64, top_k=512)
    inp = S.to_numpy_inputs(S.make_inputs(wl, with_values=False))
    r = O.decode_step_indexer(inp, P=wl.page_size, m_blocks=wl.m_pages, top_k=wl.top_k)[(0, 0)]
    K = O.logical_rows(inp["k_cache"], inp["page_table"][0], 0, 32768, wl.page_size)
    norms = np.linalg.norm(K, axis=1)
    needles = np.nonzero(norms > 2.5 * np.sqrt(128))[0]
    assert len(needles) == wl.n_needles
    assert set(needles.tolist()) <= set(r["idx"].tolist())


def test_ragged_layout_is_a_partition():
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=5, ragged=(50, 700))
    inp = S.to_numpy_inputs(S.make_inputs(wl, with_values=False))
    pt, lens = inp["page_table"], inp["seq_len"]
    used = np.concatenate([pt[b, : -(-int(lens[b]) // wl.page_size)] for b in range(5)])
    assert sorted(used.tolist()) == list(range(inp["n_phys"]))
