"""Thin ctypes binding of the C ABI in include/hhr.h (argument marshalling only).

Every function has the C name and the C argument order; tensors are passed as
torch CUDA tensors (their device pointers) and the current torch stream is used
when ``stream`` is None. A non-zero status raises :class:`HHRError`. The shared
library must have been built (``python -m hash_hierarchical_top_b200.build``);
there is no fallback of any kind when it is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhhr.so")

HHR_OK = 0
HHR_ERR_INVALID_ARG = -1
HHR_ERR_UNSUPPORTED = -2
HHR_ERR_CUDA = -3
HHR_ERR_WORKSPACE = -4
HHR_ERR_DEVICE_STATUS = -6
HHR_MODE_HASH = 0
HHR_MODE_INDEXER = 1

EXPORTED = [
    "hhr_encode_keys", "hhr_kept_max", "hhr_select_workspace_bytes", "hhr_select",
    "hhr_attn_workspace_bytes", "hhr_sparse_attn", "hhr_read_device_status",
    "hhr_status_string", "hhr_profile_next", "hhr_last_cuda_error", "hhr_sparse_attn_noalloc",
    "hhr_decode_step_workspace_bytes", "hhr_decode_step", "hhr_decode_step_kernels",
]

KERNELS = ["encode", "qprep", "bound", "topm", "hamming", "block", "token", "token_topk", "attn",
           "combine", "row"]
KERNEL_ID = {name: i for i, name in enumerate(KERNELS)}


class HHRError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = f"{fn} failed: {status_string(status)} ({status})"
        if status == HHR_ERR_CUDA:
            msg += ": " + lib().hhr_last_cuda_error().decode()
        super().__init__(msg)


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "n_q_heads", "n_kv_heads", "head_dim", "page_size", "code_bits",
        "max_pages_per_seq", "n_phys_pages", "summary_fp16", "select_per_head")]


class SelectOpts(ctypes.Structure):
    """hhr_select_opts: forced sink and local-window pages (0 = none)."""
    _fields_ = [("sink_pages", ctypes.c_int), ("local_pages", ctypes.c_int)]


def make_opts(sink_pages=0, local_pages=0):
    """Options for hhr_select / hhr_decode_step, or None when nothing is forced."""
    if not sink_pages and not local_pages:
        return None
    return SelectOpts(int(sink_pages), int(local_pages))


class Trace(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q_rot", "q_code", "bounds", "kept", "kept_count")]


_lib = None


def lib():
    """The loaded libhhr.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m hash_hierarchical_top_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        pd = ctypes.POINTER(Dims)
        L.hhr_encode_keys.argtypes = [pd, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]
        L.hhr_encode_keys.restype = i32
        L.hhr_kept_max.argtypes = [pd, i32, i32]
        L.hhr_kept_max.restype = i32
        L.hhr_select_workspace_bytes.argtypes = [pd, i32, i32, i32, i32]
        L.hhr_select_workspace_bytes.restype = sz
        po = ctypes.POINTER(SelectOpts)
        L.hhr_select.argtypes = [pd, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                 po, vp, vp, vp, sz, ctypes.POINTER(Trace), vp]
        L.hhr_select.restype = i32
        L.hhr_attn_workspace_bytes.argtypes = [pd, i32]
        L.hhr_attn_workspace_bytes.restype = sz
        L.hhr_sparse_attn.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp, vp,
                                      sz, vp]
        L.hhr_sparse_attn.restype = i32
        L.hhr_read_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.hhr_read_device_status.restype = i32
        L.hhr_profile_next.argtypes = [i32, vp, vp]
        L.hhr_profile_next.restype = i32
        L.hhr_decode_step_workspace_bytes.argtypes = [pd, i32, i32, i32]
        L.hhr_decode_step_workspace_bytes.restype = sz
        L.hhr_decode_step.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32,
                                      i32, po, ctypes.c_float, vp, vp, vp, vp, sz, vp]
        L.hhr_decode_step.restype = i32
        L.hhr_decode_step_kernels.argtypes = [pd, i32, i32, i32]
        L.hhr_decode_step_kernels.restype = i32
        L.hhr_sparse_attn_noalloc.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, i32,
                                              ctypes.c_float, vp, vp]
        L.hhr_sparse_attn_noalloc.restype = i32
        L.hhr_last_cuda_error.argtypes = []
        L.hhr_last_cuda_error.restype = ctypes.c_char_p
        L.hhr_status_string.argtypes = [i32]
        L.hhr_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().hhr_status_string(int(status)).decode()


def make_dims(batch, n_q_heads, n_kv_heads, page_size, max_pages_per_seq, n_phys_pages,
              head_dim=128, code_bits=128, summary_fp16=0, select_per_head=0) -> Dims:
    return Dims(batch, n_q_heads, n_kv_heads, head_dim, page_size, code_bits,
                max_pages_per_seq, n_phys_pages, int(summary_fp16), int(select_per_head))


def sel_rows(d: Dims) -> int:
    """Selection rows per sequence: KV groups, or query heads with select_per_head."""
    return d.n_q_heads if d.select_per_head else d.n_kv_heads


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def _p(t, dtypes, name):
    """Device pointer of a contiguous CUDA tensor of one of ``dtypes`` (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(fn, st):
    if st != HHR_OK:
        raise HHRError(fn, st)


I32 = (torch.int32,)
F32 = (torch.float32,)
SUMMARY = (torch.float32, torch.float16)
U32 = (torch.int32, torch.uint32) if hasattr(torch, "uint32") else (torch.int32,)


def hhr_encode_keys(d, k_cache, page_table, start, n_new, max_new, R, W, page_minmax, codes,
                    block_mean, stream=None):
    _check("hhr_encode_keys", lib().hhr_encode_keys(
        ctypes.byref(d), _p(k_cache, _BF16, "k_cache"), _p(page_table, I32, "page_table"),
        _p(start, I32, "start"), _p(n_new, I32, "n_new"), int(max_new), _p(R, F32, "R"),
        _p(W, F32, "W"), _p(page_minmax, SUMMARY, "page_minmax"), _p(codes, U32, "codes"),
        _p(block_mean, F32, "block_mean"), _s(stream)))


def hhr_kept_max(d, m_pages, keep_div) -> int:
    return int(lib().hhr_kept_max(ctypes.byref(d), int(m_pages), int(keep_div)))


def hhr_select_workspace_bytes(d, mode, m_pages, keep_div, top_k) -> int:
    return int(lib().hhr_select_workspace_bytes(ctypes.byref(d), int(mode), int(m_pages),
                                                int(keep_div), int(top_k)))


def hhr_attn_workspace_bytes(d, top_k) -> int:
    return int(lib().hhr_attn_workspace_bytes(ctypes.byref(d), int(top_k)))


def make_trace(q_rot=None, q_code=None, bounds=None, kept=None, kept_count=None) -> Trace:
    tr = Trace()
    for name, t in (("q_rot", q_rot), ("q_code", q_code), ("bounds", bounds), ("kept", kept),
                    ("kept_count", kept_count)):
        setattr(tr, name, t.data_ptr() if t is not None else None)
    return tr


def hhr_select(d, mode, q, seq_len, q_pos, page_table, R, W, page_minmax, codes, block_mean,
               k_cache, m_pages, keep_div, top_k, out_idx, out_count, workspace, trace=None,
               stream=None, opts=None):
    tr = ctypes.byref(trace) if trace is not None else None
    op = ctypes.byref(opts) if opts is not None else None
    _check("hhr_select", lib().hhr_select(
        ctypes.byref(d), int(mode), _p(q, _BF16, "q"), _p(seq_len, I32, "seq_len"),
        _p(q_pos, I32, "q_pos"), _p(page_table, I32, "page_table"), _p(R, F32, "R"),
        _p(W, F32, "W"), _p(page_minmax, SUMMARY, "page_minmax"), _p(codes, U32, "codes"),
        _p(block_mean, F32, "block_mean"), _p(k_cache, _BF16, "k_cache"), int(m_pages),
        int(keep_div), int(top_k), op, _p(out_idx, I32, "out_idx"),
        _p(out_count, I32, "out_count"),
        _p(workspace, (torch.uint8,), "workspace"), workspace.numel(), tr, _s(stream)))


def hhr_sparse_attn(d, q, k_cache, v_cache, page_table, seq_len, idx, count, top_k, scale, out,
                    workspace, stream=None):
    _check("hhr_sparse_attn", lib().hhr_sparse_attn(
        ctypes.byref(d), _p(q, _BF16, "q"), _p(k_cache, _BF16, "k_cache"),
        _p(v_cache, _BF16, "v_cache"), _p(page_table, I32, "page_table"),
        _p(seq_len, I32, "seq_len"), _p(idx, I32, "idx"), _p(count, I32, "count"), int(top_k),
        float(scale), _p(out, F32, "out"), _p(workspace, (torch.uint8,), "workspace"),
        workspace.numel(), _s(stream)))


def hhr_read_device_status(stream=None):
    """(status, bits): synchronises the stream and clears the device status word."""
    bits = ctypes.c_int(0)
    st = lib().hhr_read_device_status(_s(stream), ctypes.byref(bits))
    if st not in (HHR_OK, HHR_ERR_DEVICE_STATUS):
        raise HHRError("hhr_read_device_status", st)
    return st, bits.value


def hhr_profile_next(kernel, start_event, stop_event):
    """Bracket the next launch of ``kernel`` (name or id) with two torch.cuda.Events."""
    k = KERNEL_ID[kernel] if isinstance(kernel, str) else int(kernel)
    ev = lambda e: ctypes.c_void_p(e.cuda_event) if e is not None else None
    _check("hhr_profile_next", lib().hhr_profile_next(k, ev(start_event), ev(stop_event)))


def hhr_decode_step_kernels(d, m_pages, keep_div, top_k) -> int:
    """Kernels one hhr_decode_step call launches (2 on the small-batch row-cluster path)."""
    n = int(lib().hhr_decode_step_kernels(ctypes.byref(d), int(m_pages), int(keep_div),
                                          int(top_k)))
    if n < 0:
        raise HHRError("hhr_decode_step_kernels", n)
    return n


def hhr_sparse_attn_noalloc(d, q, k_cache, v_cache, page_table, seq_len, idx, count, top_k,
                            scale, out, stream=None):
    """hhr_sparse_attn with the library's fixed 8 MiB device scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/hhr.h)."""
    _check("hhr_sparse_attn_noalloc", lib().hhr_sparse_attn_noalloc(
        ctypes.byref(d), _p(q, _BF16, "q"), _p(k_cache, _BF16, "k_cache"),
        _p(v_cache, _BF16, "v_cache"), _p(page_table, I32, "page_table"),
        _p(seq_len, I32, "seq_len"), _p(idx, I32, "idx"), _p(count, I32, "count"), int(top_k),
        float(scale), _p(out, F32, "out"), _s(stream)))


def hhr_decode_step_workspace_bytes(d, m_pages, keep_div, top_k) -> int:
    return int(lib().hhr_decode_step_workspace_bytes(ctypes.byref(d), int(m_pages),
                                                     int(keep_div), int(top_k)))


def hhr_decode_step(d, q, k_new, v_new, k_cache, v_cache, page_table, seq_len, R, W,
                    page_minmax, codes, m_pages, keep_div, top_k, scale, out_idx, out_count, out,
                    workspace, stream=None, opts=None):
    op = ctypes.byref(opts) if opts is not None else None
    _check("hhr_decode_step", lib().hhr_decode_step(
        ctypes.byref(d), _p(q, _BF16, "q"), _p(k_new, _BF16, "k_new"), _p(v_new, _BF16, "v_new"),
        _p(k_cache, _BF16, "k_cache"), _p(v_cache, _BF16, "v_cache"),
        _p(page_table, I32, "page_table"), _p(seq_len, I32, "seq_len"), _p(R, F32, "R"),
        _p(W, F32, "W"), _p(page_minmax, SUMMARY, "page_minmax"), _p(codes, U32, "codes"),
        int(m_pages), int(keep_div), int(top_k), op, float(scale), _p(out_idx, I32, "out_idx"),
        _p(out_count, I32, "out_count"), _p(out, F32, "out"),
        _p(workspace, (torch.uint8,), "workspace"), workspace.numel(), _s(stream)))
