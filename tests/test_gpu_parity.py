"""GPU parity: the CUDA path through the C ABI against the fp64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import hhr_synth as S
from parity_helpers import check_hash_group, check_indexer_query, run_gpu

pytestmark = pytest.mark.gpu


def _inputs(wl, with_values=True):
    inp = S.make_inputs(wl, device="cuda", with_values=with_values)
    return inp, S.to_numpy_inputs(inp)


def _check_all_groups(wl, inp_np, g_out, groups=None):
    report = {}
    B = wl.batch
    for b in range(B):
        for g in range(wl.n_kv_heads):
            if groups is None or (b, g) in groups:
                check_hash_group(wl, inp_np, g_out, b, g, report)
    return report


@pytest.fixture(scope="module", autouse=True)
def _built():
    from hash_hierarchical_top_b200 import build
    build.build()


F16 = pytest.mark.parametrize("f16", [0, 1], ids=["f32sum", "f16sum"])


@F16
def test_tiny_single_head(f16):
    wl = S.WORKLOADS["tiny_1h_4k"]
    inp, inp_np = _inputs(wl)
    rep = _check_all_groups(wl, inp_np, run_gpu(wl, inp, summary_fp16=f16))
    print(rep)


@F16
def test_llama_32k_full(f16):
    wl = S.WORKLOADS["llama8b_32k"]
    inp, inp_np = _inputs(wl)
    rep = _check_all_groups(wl, inp_np, run_gpu(wl, inp, summary_fp16=f16))
    print(rep)


@F16
def test_llama_32k_appended_in_pieces(f16):
    """Bulk encoding (tensor cores) and appends in pieces of 37 keys (pages filled across
    calls, per-page encoder) both match the oracle and each other."""
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(5000,), top_k=400)
    inp, inp_np = _inputs(wl)
    a = run_gpu(wl, inp, summary_fp16=f16)          # bulk: the tensor-core encoder
    c = run_gpu(wl, inp, encode_chunks=37, summary_fp16=f16)  # appends: per-page encoder
    # Both paths against the oracle (codes exact outside fragile bits, summaries within
    # tolerance, selection and attention layered checks).
    _check_all_groups(wl, inp_np, a)
    _check_all_groups(wl, inp_np, c)
    # And against each other: codes differ in at most a handful of (fragile) bits.
    diff = np.bitwise_count(a["codes"][:157] ^ c["codes"][:157]).sum()
    assert diff <= 16, diff


@F16
def test_llama_128k_sampled_groups(f16):
    """Full 128K context, batch 1: every group's selection and attention, oracle on 3 groups."""
    wl = S.WORKLOADS["llama8b_128k_b1"]
    inp, inp_np = _inputs(wl)
    out = run_gpu(wl, inp, summary_fp16=f16)
    assert np.all(out["count"] == wl.top_k)
    _check_all_groups(wl, inp_np, out, groups={(0, 0), (0, 3), (0, 7)})


@F16
def test_ragged_small(f16):
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=6, ragged=(1, 5000))
    inp, inp_np = _inputs(wl)
    _check_all_groups(wl, inp_np, run_gpu(wl, inp, summary_fp16=f16))


def test_ragged_full_sampled():
    wl = S.WORKLOADS["ragged_b32"]
    inp, inp_np = _inputs(wl)
    out = run_gpu(wl, inp, summary_fp16=1)
    lens = inp_np["seq_len"]
    short = int(np.argmin(lens))
    longest = int(np.argmax(lens))
    _check_all_groups(wl, inp_np, out, groups={(short, 0), (short, 5), (longest, 2), (7, 6)})


@pytest.mark.parametrize("case", [
    dict(seq_lens=(17,), page_size=32, m_pages=0, keep_div=16, top_k=1024),   # one partial page
    dict(seq_lens=(300,), page_size=32, m_pages=64, keep_div=0, top_k=5),     # keep all pages
    dict(seq_lens=(1000,), page_size=1, m_pages=40, keep_div=0, top_k=40),    # P = 1
    dict(seq_lens=(3000,), page_size=256, m_pages=3, keep_div=0, top_k=700),  # P max, k_eff < k
    dict(seq_lens=(2048,), page_size=32, m_pages=0, keep_div=4, top_k=1),     # k = 1
])
@F16
def test_edge_cases(case, f16):
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], **case)
    inp, inp_np = _inputs(wl)
    _check_all_groups(wl, inp_np, run_gpu(wl, inp, summary_fp16=f16))


@pytest.mark.parametrize("heads", [(8, 1), (8, 8), (6, 2), (10, 2)])
def test_group_shapes(heads):
    hq, g = heads
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], n_q_heads=hq, n_kv_heads=g, seq_lens=(3000, 1234),
                  batch=2, top_k=300)
    inp, inp_np = _inputs(wl)
    _check_all_groups(wl, inp_np, run_gpu(wl, inp))


@pytest.mark.parametrize("bits", [64, 256])
@pytest.mark.parametrize("heads", [(32, 8), (8, 1), (6, 2)])
def test_code_lengths(bits, heads):
    """64- and 256-bit codes (their own encoder, query-prep and Hamming instantiations; the
    256-bit Hamming stage runs 512 threads): every layered check, for a whole-sequence
    append and for appends in pieces of 37 keys."""
    hq, g = heads
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], code_bits=bits, n_q_heads=hq, n_kv_heads=g,
                  seq_lens=(5000, 2345), batch=2, top_k=400)
    inp, inp_np = _inputs(wl)
    a = run_gpu(wl, inp, summary_fp16=1)
    assert a["codes"].shape[-1] == bits // 32 and a["q_code"].shape[-1] == bits // 32
    _check_all_groups(wl, inp_np, a)
    c = run_gpu(wl, inp, encode_chunks=37)
    _check_all_groups(wl, inp_np, c)
    assert np.bitwise_count(a["codes"] ^ c["codes"]).sum() <= 16


@pytest.mark.parametrize("bits", [64, 256])
def test_code_lengths_128k_sampled(bits):
    """Full 128K context with 64- and 256-bit codes: 65536 candidates per group."""
    wl = S.scaled(S.WORKLOADS["llama8b_128k_b1"], code_bits=bits)
    inp, inp_np = _inputs(wl)
    out = run_gpu(wl, inp, summary_fp16=1)
    assert np.all(out["count"] == wl.top_k)
    _check_all_groups(wl, inp_np, out, groups={(0, 1), (0, 6)})


@pytest.mark.parametrize("bits", [128, 256])
def test_flat_hash_topk_128k(bits):
    """Flat hash top-k (every page kept, HATA-style) at 128K: 131072 candidates per group."""
    wl = S.scaled(S.WORKLOADS["llama8b_128k_b1"], m_pages=4096, keep_div=0, code_bits=bits)
    inp, inp_np = _inputs(wl)
    out = run_gpu(wl, inp, summary_fp16=1)
    assert np.all(out["count"] == wl.top_k)
    assert np.all(out["kept_count"] == 4096)
    _check_all_groups(wl, inp_np, out, groups={(0, 2), (0, 5)})


@pytest.mark.parametrize("forced", [(1, 2), (4, 0), (0, 8), (3, 3)])
def test_forced_sink_local_pages(forced):
    """Forced sink/local pages (variant): kept inside the budget, their keys selected first.
    Short sequences (n = 300: 10 pages, keep 1/16 = 1) grow the budget to the forced set;
    (3, 3) on 2 pages forces every page."""
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(5000, 300, 40), batch=3, top_k=400,
                  keep_div=16, sink_pages=forced[0], local_pages=forced[1])
    inp, inp_np = _inputs(wl)
    out = run_gpu(wl, inp, summary_fp16=1)
    _check_all_groups(wl, inp_np, out)
    # Every key of a forced page is selected while top_k leaves room for them.
    P = wl.page_size
    for b, n in enumerate(wl.seq_lens):
        npg = -(-n // P)
        fk = [t for t in range(n) if t // P < forced[0] or t // P >= npg - forced[1]]
        if len(fk) <= wl.top_k:
            for g in range(wl.n_kv_heads):
                assert set(fk) <= set(out["idx"][b, g, :out["count"][b, g]].tolist())


@pytest.mark.parametrize("bits", [64, 128])
def test_many_rows_two_ctas_per_sm(bits):
    """More (sequence, group) rows than SMs: the top-m + Hamming kernel runs 512 threads per
    CTA, two CTAs per SM. 12 sequences x 8 groups x 2 ranks = 192 CTAs."""
    wl = S.scaled(S.WORKLOADS["ragged_b32"], batch=12, ragged=(33, 3000), top_k=200,
                  code_bits=bits)
    inp, inp_np = _inputs(wl)
    _check_all_groups(wl, inp_np, run_gpu(wl, inp, summary_fp16=1))


@pytest.mark.parametrize("heads", [(32, 8), (8, 1), (6, 2)])
def test_per_query_head_selection(heads):
    """One selection per query head (variant): bounds, Hamming top-k and attention of every
    head on its own, each against the oracle."""
    hq, g = heads
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], n_q_heads=hq, n_kv_heads=g, seq_lens=(3000, 1234),
                  batch=2, top_k=300, select_per_head=True)
    inp, inp_np = _inputs(wl)
    out = run_gpu(wl, inp, summary_fp16=1)
    assert out["idx"].shape[1] == hq
    _check_all_groups(wl, inp_np, out)


@pytest.mark.parametrize("case", [
    dict(select_per_head=True, sink_pages=1, local_pages=2, code_bits=64),
    dict(select_per_head=True, m_pages=4096, keep_div=0, code_bits=256),
    dict(m_pages=4096, keep_div=0, sink_pages=2, local_pages=1, code_bits=256),
], ids=["per_head+forced+64", "per_head+flat+256", "flat+forced+256"])
def test_variant_combinations(case):
    """Variants together: per-head rows with forced pages or a flat top-k, across code
    lengths; every row against the oracle."""
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(3000, 700), batch=2, top_k=300, **case)
    inp, inp_np = _inputs(wl)
    _check_all_groups(wl, inp_np, run_gpu(wl, inp, summary_fp16=1))


def test_bulk_encoder_partial_start():
    """Tensor-core bulk append starting mid-page (merge with stored summaries)."""
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(20000, 13001), batch=2, top_k=500)
    inp, inp_np = _inputs(wl)
    out = run_gpu(wl, inp, encode_chunks=6007, summary_fp16=1)
    _check_all_groups(wl, inp_np, out)


def test_deterministic():
    wl = S.scaled(S.WORKLOADS["llama8b_32k"], seq_lens=(9000,), top_k=900)
    inp, _ = _inputs(wl)
    a, b = run_gpu(wl, inp), run_gpu(wl, inp)
    for key in ("idx", "count", "codes", "page_minmax", "bounds", "kept"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(a["out"].view(np.uint32), b["out"].view(np.uint32))


def test_indexer_decode_small():
    wl = S.scaled(S.WORKLOADS["hisa_128k_t1"], seq_lens=(20000,), m_pages=16, top_k=700)
    inp, inp_np = _inputs(wl, with_values=False)
    out = run_gpu(wl, inp)
    rep = {}
    check_indexer_query(wl, inp_np, out, 0, 0, rep)


def test_indexer_chunk_small():
    wl = S.scaled(S.WORKLOADS["hisa_128k_t64"], seq_lens=(9000,), m_pages=8, top_k=300,
                  n_queries=20)
    inp, inp_np = _inputs(wl, with_values=False)
    out = run_gpu(wl, inp)
    rep = {}
    for i in range(20):
        check_indexer_query(wl, inp_np, out, 0, i, rep)


def test_indexer_128k_full():
    for name in ("hisa_128k_t1", "hisa_128k_t64"):
        wl = S.WORKLOADS[name]
        inp, inp_np = _inputs(wl, with_values=False)
        out = run_gpu(wl, inp)
        rep = {}
        for i in sorted({0, wl.n_queries // 2, wl.n_queries - 1}):
            check_indexer_query(wl, inp_np, out, 0, i, rep)
        if wl.n_queries == 1:
            # Sanity (not parity): the planted needles are all selected.
            n = int(inp_np["seq_len"][0])
            K = S_logical_norms(inp_np, wl, n)
            needles = np.nonzero(K > 2.5 * np.sqrt(128))[0]
            assert set(needles.tolist()) <= set(out["idx"][0, 0].tolist())


def S_logical_norms(inp_np, wl, n):
    import oracle
    K = oracle.hhr_oracle.logical_rows(inp_np["k_cache"], inp_np["page_table"][0], 0, n,
                                       wl.page_size)
    return np.linalg.norm(K, axis=1)
