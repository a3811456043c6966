"""The planted page-locality workloads of the quality harness: hot pages come in runs of
consecutive pages, and only their keys are shifted, along the KV group's mean query direction."""
import math

import torch

import hhr_synth as S


def _small(**kw):
    base = S.scaled(S.WORKLOADS["llama8b_128k_planted"], batch=1, seq_lens=(3000,),
                    hot_runs=3, hot_run_pages=4, hot_scale=2.5)
    return S.scaled(base, **kw)


def test_hot_pages_are_runs():
    wl = _small()
    n = 3000
    npg = -(-n // wl.page_size)
    for pages in S.hot_pages(wl, 0, n):
        assert len(pages) == len(set(pages)) == wl.hot_runs * wl.hot_run_pages
        assert all(0 <= p < npg for p in pages)
        runs = {p // wl.hot_run_pages for p in pages}
        assert len(runs) == wl.hot_runs
        for r in runs:
            assert all(r * wl.hot_run_pages + i in pages for i in range(wl.hot_run_pages))


def test_only_hot_keys_move_along_the_mean_query():
    wl = _small()
    cold = S.scaled(wl, hot_runs=0)
    a = S.make_inputs(wl, with_values=False)
    b = S.make_inputs(cold, with_values=False)
    assert torch.equal(a["q"], b["q"])
    P, gs, d = wl.page_size, wl.group_size, wl.head_dim
    pt = a["page_table"][0].long()
    hot = S.hot_pages(wl, 0, 3000)
    for g in (0, 5):
        ka = a["k_cache"][pt, g].reshape(-1, d)[:3000].float()
        kb = b["k_cache"][pt, g].reshape(-1, d)[:3000].float()
        is_hot = torch.zeros(3000, dtype=torch.bool)
        for p in hot[g]:
            is_hot[p * P:(p + 1) * P] = True
        assert torch.equal(ka[~is_hot], kb[~is_hot])
        diff = (ka - kb)[is_hot].mean(0)
        # The group's mean query direction, from the bf16 queries both sides share (the
        # generator uses the fp32 draws; their bf16 rounding moves the direction by < 1e-2).
        u = a["q"][0, g * gs:(g + 1) * gs].float().mean(0)
        u = u / u.norm()
        assert abs(diff.norm().item() - wl.hot_scale * math.sqrt(d)) < 0.05 * wl.hot_scale * math.sqrt(d)
        assert torch.dot(diff / diff.norm(), u).item() > 0.99
