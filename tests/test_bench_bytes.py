"""The bench's algorithmic byte counts (the roofline numerators) against closed forms of the
128K batch-8 workload and its variants, on the CPU."""
import bench
import hhr_synth as S

KEEP_16 = lambda npg: min(npg, -(-npg // 16))  # keep 1/16 of the pages (ceil)
ALL = lambda npg: npg


def test_headline_step_bytes():
    # 8 sequences x 8 KV groups x 4096 pages: f16 summaries 512 B per (page, group); 256 kept
    # pages x 32 keys x 16-byte codes; 2048 selected K and V rows of 256 B each.
    wl = S.WORKLOADS["llama8b_128k_b8"]
    summ, codes, kv = bench.required_bytes(wl, [131072] * 8, KEEP_16, 2)
    assert summ == 8 * 8 * 4096 * 2 * 128 * 2 == 134217728
    assert codes == 8 * 8 * 256 * 32 * 16 == 8388608
    assert kv == 8 * 8 * 2048 * 2 * 128 * 2 == 67108864
    assert summ + codes + kv == 209715200


def test_variant_step_bytes():
    base = S.WORKLOADS["llama8b_128k_b8"]
    # Flat: every page kept, so no bounds (no summaries) but every key's code.
    summ, codes, kv = bench.required_bytes(S.WORKLOADS["llama8b_128k_b8_flat"], [131072] * 8, ALL,
                                           2)
    assert (summ, codes, kv) == (0, 8 * 8 * 131072 * 16, 67108864)
    # Per query head: summaries once per group, codes and rows once per head.
    summ, codes, kv = bench.required_bytes(S.WORKLOADS["llama8b_128k_b8_per_head"],
                                           [131072] * 8, KEEP_16, 2)
    assert (summ, codes, kv) == (134217728, 8 * 32 * 8192 * 16, 8 * 32 * 2048 * 512)
    # Code lengths scale only the code bytes.
    for bits in (64, 256):
        wl = S.WORKLOADS[f"llama8b_128k_b8_codes{bits}"]
        _, codes, _ = bench.required_bytes(wl, [131072] * 8, KEEP_16, 2)
        assert codes == 8 * 8 * 8192 * bits // 8
    # Fewer candidates than k: the selected rows are the candidates.
    _, _, kv = bench.required_bytes(base, [1000], KEEP_16, 2)
    assert kv == 8 * min(2048, 2 * 32) * 512


def test_bound_kernel_bytes():
    # Per (page, group): 512 B of f16 summary + a 4-byte bound; per page a 4-byte page-table
    # entry; per (sequence, group) the 1 KB folded query.
    wl = S.WORKLOADS["llama8b_128k_b8"]
    got = bench.bound_kernel_bytes(wl, [131072] * 8, 2)
    assert got == 8 * (4096 * 8 * 516 + 4096 * 4 + 8 * 1024) == 135462912


def test_indexer_bytes():
    # 1024 blocks of 128 keys: 512 B block means each; T queries x 64 kept blocks x 128 keys x
    # 256 B.
    for name, T in (("hisa_128k_t1", 1), ("hisa_128k_t64", 64)):
        wl = S.WORKLOADS[name]
        assert bench.indexer_required_bytes(wl, [131072]) == 1024 * 512 + T * 64 * 128 * 256


def test_step_kernel_bytes_and_table():
    wl = S.WORKLOADS["llama8b_128k_b8"]
    kb = bench.step_kernel_bytes(wl, [131072] * 8, KEEP_16, 2)
    assert kb["bound"] == 135462912
    # Attention: 8 x 8 groups x 2048 rows x (4-byte offset + 256 B K + 256 B V), plus 8 x 32
    # queries read (bf16) and written (f32).
    assert kb["attn"] == 8 * 8 * 2048 * 516 + 8 * 32 * 128 * 6
    # Hamming: 4096 bounds + 256 page-table entries + 8192 codes of 16 B + 2048 x 8 B out.
    assert kb["hamming"] == 8 * 8 * (4096 * 4 + 256 * 4 + 8192 * 16 + 2048 * 8)
    assert kb["encode"] == 8 * (128 * 128 * 2) * 4 + 8 * 8 * 512 + 8 * 32 * 128 * 6 + 8 * 8 * 1024
    t = bench.kernel_table({"bound": 25.0, "attn": 20.0, "combine": 2.0}, kb, 6548.0)
    assert t["combine"] == {"us": 2.0}
    assert abs(t["bound"]["gbs"] - 135462912 / 25e-6 / 1e9) < 1e-9
    assert abs(t["bound"]["frac_of_measured"] - t["bound"]["gbs"] / 6548.0) < 1e-12
    assert abs(t["attn"]["frac_of_8tbs"] - t["attn"]["gbs"] / 8000.0) < 1e-12


def test_dense_kv_bytes():
    """A dense step at 128K reads every K and V row of the 8 KV groups: 537 MB per sequence,
    20.5x the hierarchical step's required bytes with f16 summaries."""
    wl = S.WORKLOADS["llama8b_128k_b8"]
    dense = bench.dense_kv_bytes(wl, [131072] * 8)
    assert dense == 8 * 131072 * 8 * 128 * 2 * 2
    req = sum(bench.required_bytes(wl, [131072] * 8, KEEP_16, 2))
    assert abs(dense / req - 20.48) < 0.01
