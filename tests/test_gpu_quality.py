"""The GPU selections on data with planted page locality (hhr_synth.hot_pages: runs of hot
pages whose keys lie along the group's mean query): the HHR page stage keeps the hot pages and
the Hamming top-k is mostly their keys (HHR page, Abstract); the HISA block filter keeps the
hot blocks and its token top-k matches the flat indexer's (HISA page, Abstract). These are
properties of the method on such data, checked beside the oracle parity tests."""
import numpy as np
import pytest
import torch

import hhr_synth as S
from hash_hierarchical_top_b200 import build, hhr
from hash_hierarchical_top_b200.step import DecodeStep, LayerCache

pytestmark = pytest.mark.gpu


def test_hhr_keeps_planted_hot_pages():
    build.build()
    wl = S.scaled(S.WORKLOADS["llama8b_128k_planted"], batch=1, seq_lens=(32768,), hot_runs=4,
                  top_k=1024)  # 32 hot pages (1024 keys) per KV group, 64 of 1024 pages kept
    inp = S.make_inputs(wl, device="cuda", with_values=False)
    d = hhr.make_dims(1, wl.n_q_heads, wl.n_kv_heads, wl.page_size, inp["max_pages"],
                      inp["n_phys"], summary_fp16=1)
    cache = LayerCache(d, "cuda")
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    hhr.hhr_encode_keys(d, inp["k_cache"], inp["page_table"], zero, inp["seq_len"],
                        int(inp["seq_len"].max()), inp["R"], inp["W"], cache.page_minmax,
                        cache.codes, None)
    st = DecodeStep(d, hhr.HHR_MODE_HASH, wl.m_pages, wl.keep_div, wl.top_k, "cuda",
                    attention=False)
    kept = torch.empty(1, wl.n_kv_heads, st.m_max, dtype=torch.int32, device="cuda")
    kcnt = torch.empty(1, wl.n_kv_heads, dtype=torch.int32, device="cuda")
    st.select(inp["q"], inp["seq_len"], inp["page_table"], cache, R=inp["R"], W=inp["W"],
              trace=hhr.make_trace(kept=kept, kept_count=kcnt))
    torch.cuda.synchronize()
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    hot = S.hot_pages(wl, 0, 32768)
    for g in range(wl.n_kv_heads):
        kp = set(kept[0, g, :int(kcnt[0, g])].tolist())
        assert len(kp & set(hot[g])) >= 0.95 * len(hot[g]), g
        sel = st.idx[0, g, :int(st.count[0, g])].cpu().numpy()
        assert np.isin(sel // wl.page_size, hot[g]).mean() >= 0.75, g


def test_hisa_finds_planted_hot_blocks():
    build.build()
    wl = S.WORKLOADS["hisa_128k_t1_planted"]
    inp = S.make_inputs(wl, device="cuda", with_values=False)
    d = hhr.make_dims(1, wl.n_queries, 1, wl.page_size, inp["max_pages"], inp["n_phys"])
    cache = LayerCache(d, "cuda", hashing=False, block_means=True)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    hhr.hhr_encode_keys(d, inp["k_cache"], inp["page_table"], zero, inp["seq_len"],
                        int(inp["seq_len"].max()), None, None, None, None, cache.block_mean)
    st = DecodeStep(d, hhr.HHR_MODE_INDEXER, wl.m_pages, 0, wl.top_k, "cuda", attention=False)
    kept = torch.empty(1, 1, st.m_max, dtype=torch.int32, device="cuda")
    kcnt = torch.empty(1, 1, dtype=torch.int32, device="cuda")
    st.select(inp["q"], inp["seq_len"], inp["page_table"], cache, k_cache=inp["k_cache"],
              q_pos=inp["q_pos"], trace=hhr.make_trace(kept=kept, kept_count=kcnt))
    torch.cuda.synchronize()
    assert hhr.hhr_read_device_status() == (hhr.HHR_OK, 0)
    n = int(inp["seq_len"][0])
    hot = S.hot_pages(wl, 0, n)[0]
    assert set(hot) <= set(kept[0, 0, :int(kcnt[0, 0])].tolist())
    P = wl.page_size
    npg = -(-n // P)
    K = inp["k_cache"][inp["page_table"][0, :npg].long(), 0].reshape(npg * P, -1)[:n].float()
    pos = int(inp["q_pos"][0, 0])
    flat = set(torch.topk(inp["q"][0, 0].float() @ K[:pos + 1].T, wl.top_k).indices.tolist())
    sel = set(st.idx[0, 0, :int(st.count[0, 0])].tolist())
    assert len(sel & flat) / len(sel | flat) >= 0.9
