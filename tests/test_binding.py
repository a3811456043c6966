"""The Python binding's marshalling on the CPU: argument checks happen before any call into
the library, and error codes surface as exceptions with the library's status text."""
import pytest
import torch

from hash_hierarchical_top_b200 import hhr


def test_pointer_checks_reject_bad_arguments():
    assert hhr._p(None, hhr.I32, "x") is None
    with pytest.raises(TypeError):
        hhr._p([1, 2, 3], hhr.I32, "x")                      # not a tensor
    with pytest.raises(ValueError):
        hhr._p(torch.zeros(4, dtype=torch.int32), hhr.I32, "x")  # host memory


def test_status_errors_carry_the_status_text():
    err = hhr.HHRError("hhr_select", hhr.HHR_ERR_WORKSPACE)
    assert "hhr_select" in str(err)
    assert hhr.status_string(hhr.HHR_ERR_WORKSPACE) in str(err)
    hhr._check("hhr_select", hhr.HHR_OK)                      # no exception
    with pytest.raises(hhr.HHRError):
        hhr._check("hhr_select", hhr.HHR_ERR_INVALID_ARG)


def test_dims_and_options_layout():
    d = hhr.make_dims(2, 32, 8, 32, 4096, 9000, code_bits=256, summary_fp16=1, select_per_head=1)
    assert (d.batch, d.n_q_heads, d.n_kv_heads, d.head_dim, d.page_size) == (2, 32, 8, 128, 32)
    assert (d.code_bits, d.max_pages_per_seq, d.n_phys_pages) == (256, 4096, 9000)
    assert (d.summary_fp16, d.select_per_head) == (1, 1)
    assert hhr.sel_rows(d) == 32 and hhr.sel_rows(hhr.make_dims(2, 32, 8, 32, 4096, 9000)) == 8
    # The C structs: ten ints, two ints; the trace holds five pointers.
    import ctypes
    assert ctypes.sizeof(hhr.Dims) == 10 * 4
    assert ctypes.sizeof(hhr.SelectOpts) == 2 * 4
    assert ctypes.sizeof(hhr.Trace) == 5 * ctypes.sizeof(ctypes.c_void_p)
