"""The C ABI on the host (no GPU): the library loads, exports every declared symbol, and
host-side validation rejects bad arguments before any launch or CUDA call."""
import ctypes
import os
import re

import pytest

from hash_hierarchical_top_b200 import build, hhr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return hhr.lib()


def declared_functions():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(hhr_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
    assert sorted(hhr.EXPORTED) == names


def test_status_strings(L):
    assert hhr.status_string(0) == "HHR_OK"
    assert hhr.status_string(-4) == "HHR_ERR_WORKSPACE"
    assert hhr.status_string(12345) == "HHR_UNKNOWN_STATUS"


def _d(**kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, page_size=32, max_pages_per_seq=4096,
                n_phys_pages=4096)
    base.update(kw)
    return hhr.make_dims(**base)


def test_workspace_and_kept_sizes(L):
    d = _d()
    assert hhr.hhr_kept_max(d, 0, 16) == 256
    assert hhr.hhr_kept_max(d, 64, 0) == 64
    assert hhr.hhr_kept_max(_d(max_pages_per_seq=10), 64, 0) == 10
    ws = hhr.hhr_select_workspace_bytes(d, hhr.HHR_MODE_HASH, 0, 16, 2048)
    assert ws > 0 and ws % 256 == 0
    # bounds alone need B*G*max_pages floats
    assert ws >= 8 * 4096 * 4
    assert hhr.hhr_attn_workspace_bytes(d, 2048) % 256 == 0


@pytest.mark.parametrize("bad", [
    dict(head_dim=64), dict(code_bits=96), dict(code_bits=512), dict(code_bits=32),
    dict(n_q_heads=30), dict(n_q_heads=72),
    dict(page_size=0), dict(page_size=512), dict(batch=0), dict(max_pages_per_seq=40000),
])
def test_bad_dims_rejected(L, bad):
    d = _d(**bad)
    assert hhr.hhr_select_workspace_bytes(d, hhr.HHR_MODE_HASH, 0, 16, 2048) == 0
    st = L.hhr_select(ctypes.byref(d), 0, *([None] * 10), 0, 16, 2048, None, None, None, None, 0,
                      None, None)
    assert st in (hhr.HHR_ERR_INVALID_ARG, hhr.HHR_ERR_UNSUPPORTED)


@pytest.mark.parametrize("bits", [64, 128, 256])
@pytest.mark.parametrize("heads", [(32, 8), (8, 1)])
def test_flat_top_k_at_128k_accepted(L, bits, heads):
    # Every page of a 128K-key sequence kept (131072 candidates), for every code length.
    d = _d(code_bits=bits, n_q_heads=heads[0], n_kv_heads=heads[1])
    assert hhr.hhr_select_workspace_bytes(d, hhr.HHR_MODE_HASH, 4096, 0, 2048) > 0
    assert hhr.hhr_decode_step_workspace_bytes(d, 4096, 0, 2048) > 0


@pytest.mark.parametrize("bits", [64, 128, 256])
def test_code_lengths_accepted(L, bits):
    # 64-, 128- and 256-bit codes: the workspace holds B * Hq query codes of bits / 8 bytes.
    d = _d(code_bits=bits)
    ws = hhr.hhr_select_workspace_bytes(d, hhr.HHR_MODE_HASH, 0, 16, 2048)
    assert ws > 0
    assert hhr.hhr_decode_step_workspace_bytes(d, 0, 16, 2048) > 0
    base = hhr.hhr_select_workspace_bytes(_d(code_bits=64), hhr.HHR_MODE_HASH, 0, 16, 2048)
    q_code_64 = -(-d.batch * d.n_q_heads * 8 // 256) * 256
    q_code = -(-d.batch * d.n_q_heads * bits // 8 // 256) * 256
    assert ws - base == q_code - q_code_64


def test_select_opts_validated(L):
    """Forced sink/local pages: non-negative, within the page budget, hash mode only."""
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    args = [p] * 10
    d = _d()  # 4096 pages, keep 1/16 -> at most 256 kept pages

    def sel(dd, mode, m_pages, keep_div, opts):
        return L.hhr_select(ctypes.byref(dd), mode, *args, m_pages, keep_div, 2048,
                            ctypes.byref(opts), p, p, p, 1 << 30, None, None)

    assert sel(d, 0, 0, 16, hhr.SelectOpts(-1, 0)) == hhr.HHR_ERR_INVALID_ARG
    assert sel(d, 0, 0, 16, hhr.SelectOpts(0, -2)) == hhr.HHR_ERR_INVALID_ARG
    assert sel(d, 0, 0, 16, hhr.SelectOpts(200, 57)) == hhr.HHR_ERR_INVALID_ARG
    assert sel(d, 0, 64, 0, hhr.SelectOpts(60, 5)) == hhr.HHR_ERR_INVALID_ARG
    di = _d(n_q_heads=64, n_kv_heads=1, page_size=128, max_pages_per_seq=1024)
    assert sel(di, 1, 64, 0, hhr.SelectOpts(1, 0)) == hhr.HHR_ERR_UNSUPPORTED
    step = [p] * 11
    assert L.hhr_decode_step(ctypes.byref(d), *step, 0, 16, 2048,
                             ctypes.byref(hhr.SelectOpts(0, 300)), ctypes.c_float(0.1),
                             p, p, p, p, 1 << 30, None) == hhr.HHR_ERR_INVALID_ARG
    assert hhr.make_opts() is None
    o = hhr.make_opts(1, 2)
    assert (o.sink_pages, o.local_pages) == (1, 2)


def test_per_head_selection_sizes_and_validation(L):
    """select_per_head: rows per sequence become the query heads (workspaces grow with them);
    values other than 0/1, and the indexer mode, are rejected."""
    d0, d1 = _d(), _d(select_per_head=1)
    g = hhr.hhr_select_workspace_bytes(d0, hhr.HHR_MODE_HASH, 0, 16, 2048)
    h = hhr.hhr_select_workspace_bytes(d1, hhr.HHR_MODE_HASH, 0, 16, 2048)
    assert h > g > 0
    # bounds [B][rows][max_pages], kept [B][rows][m_max]: 4x the rows at 32 heads / 8 groups
    assert h - g >= (32 - 8) * (4096 + 256) * 4
    assert hhr.hhr_attn_workspace_bytes(d1, 2048) > 0  # 4x the rows, fewer splits per row
    assert hhr.hhr_decode_step_workspace_bytes(d1, 0, 16, 2048) > 0
    assert hhr.sel_rows(d0) == 8 and hhr.sel_rows(d1) == 32
    assert hhr.hhr_select_workspace_bytes(_d(select_per_head=2), hhr.HHR_MODE_HASH, 0, 16,
                                          2048) == 0
    di = _d(n_q_heads=64, n_kv_heads=1, page_size=128, max_pages_per_seq=1024, select_per_head=1)
    assert hhr.hhr_select_workspace_bytes(di, hhr.HHR_MODE_INDEXER, 64, 0, 2048) == 0
    # Selection rows are a grid dimension: at most 65535 query heads with per-head rows.
    big = _d(n_q_heads=8 * 10000, n_kv_heads=10000, select_per_head=1)
    assert hhr.hhr_select_workspace_bytes(big, hhr.HHR_MODE_HASH, 0, 16, 2048) == 0
    assert hhr.hhr_attn_workspace_bytes(big, 2048) == 0
    ok = _d(n_q_heads=8 * 8000, n_kv_heads=8000, select_per_head=1)
    assert hhr.hhr_attn_workspace_bytes(ok, 2048) > 0


def test_select_validation_order(L):
    d = _d()
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    args = [p] * 10
    # both m_pages and keep_div given
    assert L.hhr_select(ctypes.byref(d), 0, *args, 16, 16, 2048, None, p, p, p, 1 << 30, None,
                        None) == hhr.HHR_ERR_INVALID_ARG
    # top_k < 1
    assert L.hhr_select(ctypes.byref(d), 0, *args, 0, 16, 0, None, p, p, p, 1 << 30, None,
                        None) == hhr.HHR_ERR_INVALID_ARG
    # null query
    assert L.hhr_select(ctypes.byref(d), 0, None, *args[1:], 0, 16, 2048, None, p, p, p, 1 << 30, None,
                        None) == hhr.HHR_ERR_INVALID_ARG
    # workspace too small
    assert L.hhr_select(ctypes.byref(d), 0, *args, 0, 16, 2048, None, p, p, p, 16, None,
                        None) == hhr.HHR_ERR_WORKSPACE
    # too many candidates per row (m * P > 131072)
    assert L.hhr_select(ctypes.byref(_d(page_size=256)), 0, *args, 1024, 0, 2048, None, p, p, p,
                        1 << 30, None, None) == hhr.HHR_ERR_UNSUPPORTED
    # indexer mode needs a single KV head and m_pages
    assert L.hhr_select(ctypes.byref(d), 1, *args, 64, 0, 2048, None, p, p, p, 1 << 30, None,
                        None) == hhr.HHR_ERR_INVALID_ARG
    # unknown mode
    assert L.hhr_select(ctypes.byref(d), 7, *args, 0, 16, 2048, None, p, p, p, 1 << 30, None,
                        None) == hhr.HHR_ERR_INVALID_ARG


def test_encode_and_attn_validation(L):
    d = _d()
    p = ctypes.c_void_p(256)
    # codes without page_minmax
    assert L.hhr_encode_keys(ctypes.byref(d), p, p, p, p, 1, p, p, None, p, None,
                             None) == hhr.HHR_ERR_INVALID_ARG
    # neither hashing nor block means requested
    assert L.hhr_encode_keys(ctypes.byref(d), p, p, p, p, 1, None, None, None, None, None,
                             None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_encode_keys(ctypes.byref(d), p, p, p, p, -1, p, p, p, p, None,
                             None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_encode_keys(ctypes.byref(d), p, p, p, p, 0, p, p, p, p, None, None) == hhr.HHR_OK
    a = [p] * 7
    assert L.hhr_sparse_attn(ctypes.byref(d), *a, 2048, ctypes.c_float(0.1), p, p, 16,
                             None) == hhr.HHR_ERR_WORKSPACE
    assert L.hhr_sparse_attn(ctypes.byref(d), *a, 0, ctypes.c_float(0.1), p, p, 1 << 30,
                             None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_sparse_attn(ctypes.byref(d), *a, 2048, ctypes.c_float(float("nan")), p, p,
                             1 << 30, None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_sparse_attn(ctypes.byref(_d(n_q_heads=72)), *a, 2048, ctypes.c_float(0.1), p,
                             p, 1 << 30, None) == hhr.HHR_ERR_UNSUPPORTED


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(hhr, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(hhr, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        hhr.lib()


def test_misaligned_pointers_rejected(L):
    """Device buffers must start on a 16-byte boundary (checked before any launch)."""
    d = _d()
    p, bad = ctypes.c_void_p(256), ctypes.c_void_p(256 + 8)
    a = [p] * 7
    assert L.hhr_sparse_attn(ctypes.byref(d), bad, *a[1:], 2048, ctypes.c_float(0.1), p, p,
                             1 << 30, None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_encode_keys(ctypes.byref(d), bad, p, p, p, 1, p, p, p, p, None,
                             None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_encode_keys(ctypes.byref(d), p, p, p, p, 1, p, bad, p, p, None,
                             None) == hhr.HHR_ERR_INVALID_ARG
    step = [p, bad, bad, p, p, p, p, p, p, p, p]  # q, k_new, v_new, k/v cache, ..., codes
    assert L.hhr_decode_step(ctypes.byref(d), *step, 0, 16, 2048, None, ctypes.c_float(0.1),
                             p, p, p, p, 1 << 30, None) == hhr.HHR_ERR_INVALID_ARG
    step = [p] * 11
    step[7] = bad  # R
    assert L.hhr_decode_step(ctypes.byref(d), *step, 0, 16, 2048, None, ctypes.c_float(0.1),
                             p, p, p, p, 1 << 30, None) == hhr.HHR_ERR_INVALID_ARG


def test_noalloc_rejects_sizes_beyond_the_array(L):
    """hhr_sparse_attn_noalloc keeps its split-K partials in a fixed 8 MiB device array: a
    problem whose partials need more is refused with HHR_ERR_WORKSPACE, and bad arguments
    with HHR_ERR_INVALID_ARG, both before any CUDA call (null pointers here, so nothing
    could ever be dereferenced)."""
    batch = 32
    while True:
        d = hhr.make_dims(batch, 64, 8, 32, 4096, 4096 * 32)
        if hhr.hhr_attn_workspace_bytes(d, 8192) > 8 * 1024 * 1024:
            break
        batch *= 2
        assert batch <= 65535
    nul = [None] * 7
    st = L.hhr_sparse_attn_noalloc(ctypes.byref(d), *nul, 8192, ctypes.c_float(0.1), None, None)
    assert st == hhr.HHR_ERR_WORKSPACE
    small = _d(batch=2)
    assert hhr.hhr_attn_workspace_bytes(small, 1024) <= 8 * 1024 * 1024
    st = L.hhr_sparse_attn_noalloc(ctypes.byref(small), *nul, 1024, ctypes.c_float(0.1), None,
                                   None)
    assert st == hhr.HHR_ERR_INVALID_ARG
    st = L.hhr_sparse_attn_noalloc(ctypes.byref(small), *nul, 0, ctypes.c_float(0.1), None, None)
    assert st == hhr.HHR_ERR_INVALID_ARG


def test_decode_step_kernel_count_on_the_host(L):
    """hhr_decode_step_kernels validates like the decode step and, with no GPU to host the
    small-batch clusters, counts the kernel chain: prologue, bounds (none when every page is
    kept), top-m + Hamming, attention."""
    d = hhr.make_dims(8, 32, 8, 32, 4096, 8 * 4096, summary_fp16=1)
    assert hhr.hhr_decode_step_kernels(d, 0, 16, 2048) == 4
    assert hhr.hhr_decode_step_kernels(d, 4096, 0, 2048) == 3  # flat: no bound kernel
    with pytest.raises(hhr.HHRError):
        hhr.hhr_decode_step_kernels(d, 0, 0, 2048)  # neither m_pages nor keep_div
    with pytest.raises(hhr.HHRError):
        hhr.hhr_decode_step_kernels(d, 0, 16, 0)
