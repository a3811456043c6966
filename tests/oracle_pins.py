"""Pins of the fp64 oracle against things other than itself.

Each ``check_*`` takes the oracle module ``O`` and raises AssertionError on a
violation. They are run on the real oracle (test_oracle_pins.py) and on copies
with a planted mistake (test_oracle_mutations.py), which must fail at least one.

Pins used (the pages print no worked numbers, so these are invariants, closed
forms, brute force on tiny inputs and special cases that reduce to a library
routine):
  * the page bound dominates every true logit of its page (HHR, Abstract: page-level
    logit bounds used for pruning);
  * page size 1 makes the bound equal the logit, so top-m becomes an exact top-m;
  * an orthogonal R leaves logits unchanged, R = I leaves summaries = raw min/max;
  * codes and Hamming distances recomputed by brute force from the definition
    (explicit sums, a bool list, mismatches counted without popcount);
  * top-k equals a full stable sort of (distance, token);
  * k = all keys and m = all pages gives dense softmax attention (library SDPA);
  * HISA: block size 1 makes block scores the token scores; keeping all blocks
    gives the flat indexer top-k; the causal rule by brute force;
  * forced sink/local pages: closed forms of the forced set, the kept set as the best
    subset by brute force over all subsets that hold the forced pages, and the token
    top-k decomposed into the forced keys plus a plain top-k of the others.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers

def rand_bf16_bits(rng, shape, scale=1.0):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def orthogonal(rng, d):
    q, r = np.linalg.qr(rng.standard_normal((d, d)))
    return (q * np.sign(np.diag(r))[None, :]).astype(np.float32)


def bf(bits):
    """bf16 bits -> python floats by explicit bit arithmetic (independent of the oracle)."""
    out = []
    for b in np.asarray(bits).ravel().tolist():
        sign = -1.0 if b & 0x8000 else 1.0
        e = (b >> 7) & 0xFF
        f = b & 0x7F
        if e == 0:
            v = sign * f * 2.0 ** (-133)
        else:
            v = sign * (1.0 + f / 128.0) * 2.0 ** (e - 127)
        out.append(v)
    return np.array(out).reshape(np.asarray(bits).shape)


def brute_rotate(R, x):
    d = len(x)
    return [math.fsum(float(R[i][j]) * x[j] for j in range(d)) for i in range(d)]


def brute_code_bits(R, W, x):
    """List of bools [ (W R x)_j > 0 ] by explicit sums."""
    xr = brute_rotate(R, x)
    return [math.fsum(float(W[j][i]) * xr[i] for i in range(len(xr))) > 0
            for j in range(len(W))]


def words_to_bits(words, bits):
    """Unpack LSB-first code words by integer arithmetic (no shifts on numpy arrays)."""
    val = 0
    for w_i, w in enumerate(np.asarray(words).tolist()):
        val += int(w) * (2 ** (32 * w_i))
    return [(val // (2 ** j)) % 2 == 1 for j in range(bits)]


def tiny_cache(rng, n, P, G, d, n_phys_extra=3):
    """A small paged cache with a shuffled page table (one sequence)."""
    n_pages = -(-n // P)
    n_phys = n_pages + n_phys_extra
    k = rand_bf16_bits(rng, (n_phys, G, P, d))
    v = rand_bf16_bits(rng, (n_phys, G, P, d))
    pt = rng.permutation(n_phys)[:n_pages].astype(np.int32)
    return k, v, pt


def brute_logical(cache, pt, g, n, P):
    rows = []
    for t in range(n):
        rows.append(bf(cache[pt[t // P], g, t % P]))
    return np.array(rows)


# ----------------------------------------------------------------------------- pins

def check_bound_invariant(O, seed=0):
    rng = np.random.default_rng(seed)
    for (n, P, gs, d) in [(77, 8, 4, 16), (64, 16, 1, 32), (130, 32, 2, 128)]:
        k, v, pt = tiny_cache(rng, n, P, 1, d)
        R = orthogonal(rng, d)
        Q = bf(rand_bf16_bits(rng, (gs, d), 2.0))
        K = O.logical_rows(k, pt, 0, n, P)
        Krot = O.rotate(R, K)
        Qrot = O.rotate(R, Q)
        kmin, kmax = O.page_summaries(Krot, P)
        beta = O.page_bounds(Qrot, kmin, kmax)
        Kb = brute_logical(k, pt, 0, n, P)
        Kbr = np.array([brute_rotate(R, list(r)) for r in Kb])
        Qbr = np.array([brute_rotate(R, list(r)) for r in Q])
        for t in range(n):
            s = math.fsum(float(Qbr[h] @ Kbr[t]) for h in range(gs))
            scale = sum(float(np.abs(Qbr[h]) @ np.abs(Kbr[t])) for h in range(gs))
            assert beta[t // P] >= s - 1e-12 * scale, (n, P, t)
        # The bound is attained by a key when the page holds exactly that key.
        assert len(beta) == -(-n // P)


def check_page_size_one(O, seed=1):
    """P = 1: the bound of a page is the summed logit of its only key; top-m is exact."""
    rng = np.random.default_rng(seed)
    n, gs, d, m = 40, 4, 16, 7
    k, v, pt = tiny_cache(rng, n, 1, 1, d)
    R = orthogonal(rng, d)
    Q = bf(rand_bf16_bits(rng, (gs, d)))
    K = O.logical_rows(k, pt, 0, n, 1)
    kmin, kmax = O.page_summaries(O.rotate(R, K), 1)
    beta = O.page_bounds(O.rotate(R, Q), kmin, kmax)
    Kb = brute_logical(k, pt, 0, n, 1)
    Qr = [brute_rotate(R, list(q)) for q in Q]
    Kr = [brute_rotate(R, list(x)) for x in Kb]
    logit = [math.fsum(Qr[h][i] * Kr[t][i] for h in range(gs) for i in range(d))
             for t in range(n)]
    for t in range(n):
        assert abs(beta[t] - logit[t]) <= 1e-11 * (1 + abs(logit[t])), t
    want = sorted(t for _, t in sorted(((-logit[t], t) for t in range(n)))[:m])
    assert list(O.top_m(beta, m)) == want


def check_rotation_preserves_logits(O, seed=2):
    rng = np.random.default_rng(seed)
    d = 128
    R = orthogonal(rng, d)
    X = bf(rand_bf16_bits(rng, (9, d), 3.0))
    Y = bf(rand_bf16_bits(rng, (5, d), 3.0))
    Xr, Yr = O.rotate(R, X), O.rotate(R, Y)
    for i in range(9):
        for j in range(5):
            raw = math.fsum(X[i, c] * Y[j, c] for c in range(d))
            rot = float(Xr[i] @ Yr[j])
            # R is fp32 and orthogonal to ~1e-7: logits agree to that level.
            assert abs(raw - rot) <= 1e-6 * np.linalg.norm(X[i]) * np.linalg.norm(Y[j])
    # A non-orthogonal stand-in must change them: the check is sensitive.
    assert not np.allclose(O.rotate(R * 1.01, X) @ O.rotate(R * 1.01, Y).T, X @ Y.T)


def check_identity_rotation_summaries(O, seed=3):
    rng = np.random.default_rng(seed)
    n, P, d, G = 45, 8, 12, 2
    k, v, pt = tiny_cache(rng, n, P, G, d)
    for g in range(G):
        K = O.logical_rows(k, pt, g, n, P)
        kmin, kmax = O.page_summaries(O.rotate(np.eye(d, dtype=np.float32), K), P)
        Kb = brute_logical(k, pt, g, n, P)
        for p in range(-(-n // P)):
            rows = [list(Kb[t]) for t in range(p * P, min(n, (p + 1) * P))]
            for c in range(d):
                assert kmin[p, c] == min(r[c] for r in rows)
                assert kmax[p, c] == max(r[c] for r in rows)


def check_codes_bruteforce(O, seed=4):
    rng = np.random.default_rng(seed)
    n, P, d, bits, gs = 20, 4, 16, 64, 3
    k, v, pt = tiny_cache(rng, n, P, 1, d)
    R = orthogonal(rng, d)
    W = rng.standard_normal((bits, d)).astype(np.float32)
    enc = O.encode_group(k, pt, 0, n, P, R, W)
    Kb = brute_logical(k, pt, 0, n, P)
    kbits = [brute_code_bits(R, W, list(x)) for x in Kb]
    for t in range(n):
        assert words_to_bits(enc["codes"][t], bits) == kbits[t], t
    Q = bf(rand_bf16_bits(rng, (gs, d)))
    _, qcodes, _ = O.query_prep(R, W, Q)
    qbits = [brute_code_bits(R, W, list(q)) for q in Q]
    for h in range(gs):
        assert words_to_bits(qcodes[h], bits) == qbits[h]
    dist = O.hamming(qcodes, enc["codes"])
    for t in range(n):
        mism = sum(1 for h in range(gs) for j in range(bits) if qbits[h][j] != kbits[t][j])
        assert dist[t] == mism, t
    # A square, non-symmetric projection (bits = d = 32): row j of W makes bit j.
    d2 = 32
    k2, _, pt2 = tiny_cache(rng, n, P, 1, d2)
    R2 = orthogonal(rng, d2)
    W2 = rng.standard_normal((d2, d2)).astype(np.float32)
    enc2 = O.encode_group(k2, pt2, 0, n, P, R2, W2)
    Kb2 = brute_logical(k2, pt2, 0, n, P)
    for t in range(n):
        assert words_to_bits(enc2["codes"][t], d2) == brute_code_bits(R2, W2, list(Kb2[t])), t


def check_fragile_bits(O, seed=14):
    """Fragile code bits (the only ones a GPU code may flip) are exactly those whose
    projection lies within 1e-4 ||x|| of zero, by explicit sums; on Gaussian data they are
    rare, and a bit placed on a zero projection is always fragile."""
    rng = np.random.default_rng(seed)
    d, bits, n = 16, 64, 40
    R = orthogonal(rng, d)
    W = rng.standard_normal((bits, d)).astype(np.float32)
    X = bf(rand_bf16_bits(rng, (n, d)))
    # Plant exact zeros: x orthogonal to the rotated row j of W (x = R^T v, v ⟂ W_j).
    Wj = W[3].astype(np.float64)
    v = rng.standard_normal(d)
    v -= (v @ Wj) / (Wj @ Wj) * Wj
    X[0] = R.astype(np.float64).T @ v
    fr = O.fragile_bits(R, W, X)
    for t in range(n):
        xr = brute_rotate(R, list(X[t]))
        nrm = math.sqrt(math.fsum(c * c for c in X[t]))
        for j in range(bits):
            p = math.fsum(float(W[j][i]) * xr[i] for i in range(d))
            if abs(abs(p) - 1e-4 * nrm) > 1e-12 * nrm:  # away from the cut itself
                assert bool(fr[t, j]) == (abs(p) < 1e-4 * nrm), (t, j)
    assert fr[0, 3]
    assert fr.mean() < 0.01
    # The masks the encoder and the query preparation return are the same rule.
    _, qmask = O.query_prep(R, W, X)[1:]
    assert np.array_equal(qmask, fr)
    P = 8
    kc, _, pt = tiny_cache(rng, n, P, 1, d)
    enc = O.encode_group(kc, pt, 0, n, P, R, W)
    Kb = brute_logical(kc, pt, 0, n, P)
    for t in range(n):
        xr = brute_rotate(R, list(Kb[t]))
        nrm = math.sqrt(math.fsum(c * c for c in Kb[t]))
        for j in range(bits):
            p = math.fsum(float(W[j][i]) * xr[i] for i in range(d))
            if abs(abs(p) - 1e-4 * nrm) > 1e-12 * nrm:
                assert bool(enc["fragile"][t, j]) == (abs(p) < 1e-4 * nrm), (t, j)


def check_codes_identity_projection(O, seed=5):
    """W = I: the code is the sign pattern of the rotated key itself."""
    rng = np.random.default_rng(seed)
    d = 128
    R = orthogonal(rng, d)
    X = bf(rand_bf16_bits(rng, (6, d)))
    codes = O.sign_codes(R, np.eye(d, dtype=np.float32), X)
    for i in range(6):
        xr = brute_rotate(R, list(X[i]))
        assert words_to_bits(codes[i], d) == [c > 0 for c in xr]
    # Hamming distance basics: d(x, x) = 0, symmetric, triangle inequality.
    h = lambda a, b: int(O.hamming(codes[a:a + 1], codes[b:b + 1])[0])
    for a in range(6):
        assert h(a, a) == 0
        for b in range(6):
            assert h(a, b) == h(b, a)
            for c in range(6):
                assert h(a, c) <= h(a, b) + h(b, c)


def check_topk_bruteforce(O, seed=6):
    rng = np.random.default_rng(seed)
    for trial in range(20):
        n = int(rng.integers(1, 200))
        tok = np.sort(rng.choice(5000, size=n, replace=False))
        dist = rng.integers(0, 6, size=n)          # heavy ties
        k = int(rng.integers(1, n + 1))
        want = sorted(t for _, t in sorted(zip(dist.tolist(), tok.tolist()))[:k])
        assert list(O.top_k_smallest(dist, tok, k)) == want
        score = rng.integers(-3, 3, size=n).astype(np.float64)
        want = sorted(t for _, t in sorted(zip((-score).tolist(), tok.tolist()))[:k])
        assert list(O.top_k_largest(score, tok, k)) == want
        want_m = sorted(i for _, i in sorted(zip((-score).tolist(), range(n)))[:k])
        assert list(O.top_m(score, k)) == want_m
    # All-equal distances give the first k candidates.
    tok = np.arange(10, 60)
    assert list(O.top_k_smallest(np.zeros(50, dtype=np.int64), tok, 7)) == list(range(10, 17))


def check_kept_count(O):
    assert O.kept_count(4096, 0, 16) == 256
    assert O.kept_count(1024, 0, 8) == 128
    assert O.kept_count(257, 0, 16) == 17
    assert O.kept_count(1, 0, 16) == 1
    assert O.kept_count(10, 64, 0) == 10
    assert O.kept_count(64, 16, 0) == 16


def check_flat_hash_topk(O, seed=7):
    """m = all pages: the selection is the flat Hamming top-k over every key (HATA form)."""
    rng = np.random.default_rng(seed)
    n, P, d, gs, bits, k = 50, 8, 32, 2, 64, 13
    kc, vc, pt = tiny_cache(rng, n, P, 1, d)
    R = orthogonal(rng, d)
    W = rng.standard_normal((bits, d)).astype(np.float32)
    enc = O.encode_group(kc, pt, 0, n, P, R, W)
    Q = bf(rand_bf16_bits(rng, (gs, d)))
    r = O.select_group(Q, R, W, enc["kmin"], enc["kmax"], enc["codes"], n, P, -(-n // P), k)
    Kb = brute_logical(kc, pt, 0, n, P)
    kbits = [brute_code_bits(R, W, list(x)) for x in Kb]
    qbits = [brute_code_bits(R, W, list(q)) for q in Q]
    dist = [sum(qbits[h][j] != kbits[t][j] for h in range(gs) for j in range(bits))
            for t in range(n)]
    want = sorted(t for _, t in sorted(zip(dist, range(n)))[:k])
    assert list(r["idx"]) == want


def check_dense_attention(O, seed=8):
    """k = all keys and m = all pages: the output is dense softmax attention (torch SDPA)."""
    rng = np.random.default_rng(seed)
    n, P, d, G, gs, bits = 70, 16, 32, 2, 2, 32
    kc, vc, pt = tiny_cache(rng, n, P, G, d)
    Hq = G * gs
    q = rand_bf16_bits(rng, (1, Hq, d))
    inp = dict(k_cache=kc, v_cache=vc, q=q, page_table=pt[None, :],
               seq_len=np.array([n], dtype=np.int32),
               R=np.stack([orthogonal(rng, d) for _ in range(G)]),
               W=rng.standard_normal((G, bits, d)).astype(np.float32))
    res = O.decode_step_hash(inp, P=P, m_pages=10 ** 6, keep_div=0, top_k=10 ** 6)
    for g in range(G):
        Kb = torch.tensor(brute_logical(kc, pt, g, n, P))
        Vb = torch.tensor(brute_logical(vc, pt, g, n, P))
        Qg = torch.tensor(bf(q[0, g * gs:(g + 1) * gs]))
        ref = torch.nn.functional.scaled_dot_product_attention(
            Qg[None, :, None, :], Kb[None, None].expand(1, gs, n, d),
            Vb[None, None].expand(1, gs, n, d))[0, :, 0, :].numpy()
        assert list(res[(0, g)]["idx"]) == list(range(n))
        np.testing.assert_allclose(res[(0, g)]["out"], ref, rtol=1e-12, atol=1e-12)


def check_single_key_attention(O, seed=9):
    rng = np.random.default_rng(seed)
    d = 16
    Q = bf(rand_bf16_bits(rng, (4, d), 5.0))
    K = bf(rand_bf16_bits(rng, (1, d)))
    V = bf(rand_bf16_bits(rng, (1, d)))
    out = O.sparse_attention(Q, K, V, 0.3)
    assert np.array_equal(out, np.repeat(V, 4, axis=0))


def check_hand_example(O):
    """A worked example computed by hand from the definitions (tests/golden/hand_d4.json)."""
    with open(os.path.join(GOLDEN, "hand_d4.json")) as f:
        ex = json.load(f)
    K = np.array(ex["keys"], dtype=np.float64)
    q = np.array([ex["query"]], dtype=np.float64)
    I = np.eye(4, dtype=np.float32)
    kmin, kmax = O.page_summaries(O.rotate(I, K), 2)
    assert kmin.tolist() == [ex["kmin"]] and kmax.tolist() == [ex["kmax"]]
    assert float(O.page_bounds(O.rotate(I, q), kmin, kmax)[0]) == ex["bound"]
    out = O.sparse_attention(q, K, np.array(ex["values"], dtype=np.float64), ex["scale"])
    np.testing.assert_allclose(out[0], ex["out"], rtol=1e-12, atol=1e-15)


def check_hisa_block_size_one(O, seed=10):
    """Block size 1: block scores are token scores and the selection is a full sort."""
    rng = np.random.default_rng(seed)
    n, d, k = 60, 16, 9
    kc, vc, pt = tiny_cache(rng, n, 1, 1, d)
    q = bf(rand_bf16_bits(rng, (d,)))
    K = O.logical_rows(kc, pt, 0, n, 1)
    mu = O.block_means(K, 1)
    r = O.indexer_select_one(q, n - 1, K, mu, n, 1, n, k)
    Kb = brute_logical(kc, pt, 0, n, 1)
    tok_score = [math.fsum(q[c] * Kb[t][c] for c in range(d)) for t in range(n)]
    np.testing.assert_allclose(r["block_scores"], tok_score, rtol=1e-13, atol=1e-13)
    want = sorted(t for _, t in sorted(zip([-s for s in tok_score], range(n)))[:k])
    assert list(r["idx"]) == want


def check_hisa_all_blocks_and_causal(O, seed=11):
    """Keeping every block gives the flat causal indexer; no token beyond pos is chosen."""
    rng = np.random.default_rng(seed)
    n, P, d, k = 200, 16, 16, 25
    kc, vc, pt = tiny_cache(rng, n, P, 1, d)
    K = O.logical_rows(kc, pt, 0, n, P)
    mu = O.block_means(K, P)
    Kb = brute_logical(kc, pt, 0, n, P)
    for pos in [0, 5, 15, 16, 100, 199]:
        q = bf(rand_bf16_bits(rng, (d,)))
        r = O.indexer_select_one(q, pos, K, mu, n, P, 10 ** 6, k)
        sc = [math.fsum(q[c] * Kb[t][c] for c in range(d)) for t in range(pos + 1)]
        want = sorted(t for _, t in sorted(zip([-s for s in sc], range(pos + 1)))[:k])
        assert list(r["idx"]) == want, pos
        # With few blocks kept, only eligible blocks appear and tokens stay causal.
        r2 = O.indexer_select_one(q, pos, K, mu, n, P, 2, k)
        assert all(b * P <= pos for b in r2["kept"])
        assert all(t <= pos for t in r2["idx"])
        # Block means by brute force.
        for b in range(-(-n // P)):
            rows = Kb[b * P: min(n, (b + 1) * P)]
            for c in range(d):
                assert abs(mu[b, c] - math.fsum(rows[:, c]) / len(rows)) <= 1e-15 * (
                    1 + abs(mu[b, c]))


def check_forced_pages(O, seed=12):
    """Forced sink/local pages: closed forms, subset brute force and decomposition."""
    import itertools
    assert list(O.forced_pages(10, 2, 3)) == [0, 1, 7, 8, 9]
    assert list(O.forced_pages(4, 3, 3)) == [0, 1, 2, 3]
    assert list(O.forced_pages(5, 0, 0)) == []
    assert list(O.forced_pages(5, 0, 1)) == [4]
    assert list(O.forced_pages(5, 1, 0)) == [0]
    assert list(O.forced_pages(1, 1, 1)) == [0]
    rng = np.random.default_rng(seed)
    # Kept set = the subset of size max(m, |forced|) that holds the forced pages and has the
    # largest score sum (distinct scores: unique), by enumeration.
    for trial in range(40):
        n = int(rng.integers(1, 9))
        sink, local = int(rng.integers(0, 3)), int(rng.integers(0, 3))
        m = int(rng.integers(1, n + 1))
        scores = rng.permutation(n).astype(np.float64) - 3.5
        forced = [p for p in range(n) if p < sink or p >= n - local]
        size = max(m, len(forced))
        best = max((c for c in itertools.combinations(range(n), size) if set(forced) <= set(c)),
                   key=lambda c: sum(scores[list(c)]))
        assert list(O.top_m_forced(scores, m, forced)) == list(best), (n, sink, local, m)
    # Equal scores: the forced pages, then the lowest other indices.
    assert list(O.top_m_forced(np.zeros(8), 4, [0, 7])) == [0, 1, 2, 7]
    assert list(O.top_m_forced(np.zeros(8), 4, [])) == [0, 1, 2, 3]
    # Token top-k: forced keys first in token order, the rest a plain top-k of the others.
    for trial in range(30):
        n = int(rng.integers(1, 120))
        tok = np.sort(rng.choice(3000, size=n, replace=False))
        dist = rng.integers(0, 5, size=n)
        isf = rng.random(n) < 0.3
        k = int(rng.integers(1, n + 1))
        ftok = sorted(tok[isf].tolist())
        if k <= len(ftok):
            want = ftok[:k]
        else:
            rest = sorted(zip(dist[~isf].tolist(), tok[~isf].tolist()))[:k - len(ftok)]
            want = sorted(ftok + [t for _, t in rest])
        assert list(O.top_k_forced(dist, tok, k, isf)) == want
    # Through the selection: the forced pages are kept and all their keys selected; the
    # other keys are the Hamming top-k (brute force) of the other kept pages' keys.
    n, P, d, gs, bits, k = 70, 8, 32, 2, 64, 30
    kc, vc, pt = tiny_cache(rng, n, P, 1, d)
    R = orthogonal(rng, d)
    W = rng.standard_normal((bits, d)).astype(np.float32)
    enc = O.encode_group(kc, pt, 0, n, P, R, W)
    Q = bf(rand_bf16_bits(rng, (gs, d)))
    r = O.select_group(Q, R, W, enc["kmin"], enc["kmax"], enc["codes"], n, P, 4, k, 1, 1)
    n_pages = -(-n // P)
    assert 0 in r["kept"] and n_pages - 1 in r["kept"] and len(r["kept"]) == 4
    forced_keys = [t for t in range(n) if t // P in (0, n_pages - 1)]
    assert set(forced_keys) <= set(r["idx"].tolist())
    Kb = brute_logical(kc, pt, 0, n, P)
    kbits = [brute_code_bits(R, W, list(x)) for x in Kb]
    qbits = [brute_code_bits(R, W, list(q)) for q in Q]
    others = [t for t in range(n) if t // P in r["kept"] and t not in forced_keys]
    dist = [sum(qbits[h][j] != kbits[t][j] for h in range(gs) for j in range(bits))
            for t in others]
    want = sorted(forced_keys + [t for _, t in sorted(zip(dist, others))[:k - len(forced_keys)]])
    assert list(r["idx"]) == want
    # Every page forced: the flat top-k of the forced keys in token order.
    r = O.select_group(Q, R, W, enc["kmin"], enc["kmax"], enc["codes"], n, P, 2, k, 9, 0)
    assert list(r["kept"]) == list(range(n_pages)) and list(r["idx"]) == list(range(k))


def check_per_head_selection(O, seed=13):
    """One selection per query head: identical heads reproduce the group selection (the
    group's bounds and distances are then gs times one head's), a group of one head is the
    group path, and with every page kept each head's set is its own brute-force Hamming
    top-k and its output its own dense attention over that set."""
    rng = np.random.default_rng(seed)
    n, P, d, G, gs, bits, k = 60, 8, 32, 1, 3, 64, 17
    kc, vc, pt = tiny_cache(rng, n, P, G, d)
    R = np.stack([orthogonal(rng, d) for _ in range(G)])
    W = rng.standard_normal((G, bits, d)).astype(np.float32)
    base = dict(k_cache=kc, v_cache=vc, page_table=pt[None, :],
                seq_len=np.array([n], dtype=np.int32), R=R, W=W)
    one = rand_bf16_bits(rng, (1, 1, d))
    same = dict(base, q=np.repeat(one, gs, axis=1))
    grp = O.decode_step_hash(same, P=P, m_pages=3, keep_div=0, top_k=k)[(0, 0)]
    per = O.decode_step_hash(same, P=P, m_pages=3, keep_div=0, top_k=k, per_head=True)[(0, 0)]
    assert len(per) == gs
    for r in per:
        assert list(r["kept"]) == list(grp["kept"]) and list(r["idx"]) == list(grp["idx"])
        np.testing.assert_allclose(r["out"][0], grp["out"][0], rtol=1e-12, atol=1e-12)
    solo = dict(base, q=one)
    a = O.decode_step_hash(solo, P=P, m_pages=3, keep_div=0, top_k=k)[(0, 0)]
    b = O.decode_step_hash(solo, P=P, m_pages=3, keep_div=0, top_k=k, per_head=True)[(0, 0)]
    assert list(a["idx"]) == list(b[0]["idx"])
    q = rand_bf16_bits(rng, (1, gs, d))
    per = O.decode_step_hash(dict(base, q=q), P=P, m_pages=10 ** 6, keep_div=0, top_k=k,
                             per_head=True)[(0, 0)]
    Kb = brute_logical(kc, pt, 0, n, P)
    Vb = brute_logical(vc, pt, 0, n, P)
    kbits = [brute_code_bits(R[0], W[0], list(x)) for x in Kb]
    sets = []
    for h in range(gs):
        qh = bf(q[0, h])
        qb = brute_code_bits(R[0], W[0], list(qh))
        dist = [sum(qb[j] != kbits[t][j] for j in range(bits)) for t in range(n)]
        want = sorted(t for _, t in sorted(zip(dist, range(n)))[:k])
        assert list(per[h]["idx"]) == want, h
        lg = [math.fsum(qh[c] * Kb[t][c] for c in range(d)) / math.sqrt(d) for t in want]
        mx = max(lg)
        w = [math.exp(x - mx) for x in lg]
        ref = [math.fsum(w[i] * Vb[t][c] for i, t in enumerate(want)) / math.fsum(w)
               for c in range(d)]
        np.testing.assert_allclose(per[h]["out"][0], ref, rtol=1e-10, atol=1e-12)
        sets.append(tuple(want))
    assert len(set(sets)) > 1  # distinct heads select differently on this input


ALL_CHECKS = [
    check_bound_invariant, check_page_size_one, check_rotation_preserves_logits,
    check_identity_rotation_summaries, check_codes_bruteforce,
    check_codes_identity_projection, check_topk_bruteforce, check_kept_count,
    check_flat_hash_topk, check_dense_attention, check_single_key_attention,
    check_hand_example, check_hisa_block_size_one, check_hisa_all_blocks_and_causal,
    check_forced_pages, check_per_head_selection, check_fragile_bits,
]
