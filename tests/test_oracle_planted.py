"""The method on data with the structure it relies on (HHR page, Abstract: page-level bounds
prune the pages, Hamming ranking picks the keys): with planted hot pages whose keys lie along
the group's mean query, the oracle's page stage keeps the hot pages and its selection is
mostly hot keys; on the same keys without the planted shift it is not. CPU only."""
import numpy as np

import hhr_synth as S
import oracle

O = oracle.hhr_oracle


def _wl(hot_runs):
    return S.scaled(S.WORKLOADS["llama8b_128k_planted"], batch=1, seq_lens=(8192,),
                    n_q_heads=8, n_kv_heads=2, hot_runs=hot_runs, hot_run_pages=4, top_k=256)


def _run(wl):
    inp = S.to_numpy_inputs(S.make_inputs(wl, device="cpu"))
    res = O.decode_step_hash(inp, P=wl.page_size, m_pages=wl.m_pages, keep_div=wl.keep_div,
                             top_k=wl.top_k)
    return inp, res


def test_planted_hot_pages_are_kept_and_selected():
    wl = _wl(2)  # 8 hot pages of 256 per group, 256 hot keys = top_k
    inp, res = _run(wl)
    hot = S.hot_pages(wl, 0, 8192)
    for g in range(wl.n_kv_heads):
        r = res[(0, g)]
        kept = set(int(p) for p in r["kept"])
        assert len(kept & set(hot[g])) >= 7, (g, sorted(kept & set(hot[g])))
        hot_keys = np.isin(np.asarray(r["idx"]) // wl.page_size, hot[g])
        assert hot_keys.mean() >= 0.75, hot_keys.mean()


def test_without_planting_the_same_pages_are_not_special():
    wl = _wl(2)
    cold = S.scaled(wl, hot_runs=0)
    _, res = _run(cold)
    hot = S.hot_pages(wl, 0, 8192)  # the pages the planted workload would shift
    for g in range(wl.n_kv_heads):
        r = res[(0, g)]
        kept = set(int(p) for p in r["kept"])
        assert len(kept & set(hot[g])) <= 3
