"""Thin ctypes binding of libekv.so (the C ABI of include/ekv.h).

Argument marshalling only: PyTorch supplies device memory and the current
stream; every step of the decode path runs in the library's CUDA kernels.
There is no fallback — if the library is missing or fails to load, every call
raises ``EkvUnavailable``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "EkvError", "EkvUnavailable", "Cache", "Seqs", "StepParams", "lib", "lib_path",
    "EKV_F32", "EKV_BF16", "EKV_POLICY_TOPK", "EKV_POLICY_GAUSS", "EKV_POLICY_FULL",
    "EKV_OP_SELECT_GAUSS", "EKV_OP_ENTMAX_DECODE", "EKV_OP_DECODE_STEP",
    "EKV_EFLAG_BAD_PAGE", "EKV_EFLAG_BAD_LEN", "EKV_EFLAG_SEL_OVERFLOW", "EKV_EFLAG_BAD_SEL",
    "make_cache", "make_seqs", "workspace", "ekv_build_page_meta", "ekv_append",
    "ekv_score_pages", "ekv_select_topk", "ekv_select_gauss", "ekv_entmax_decode",
    "ekv_decode_step", "ekv_workspace_bytes", "ekv_get_error", "ekv_status_string",
    "ekv_entmax_decode_static_ws", "ekv_step_kernel_count", "ekv_softmax_decode", "EKV_OP_SOFTMAX_DECODE",
    "ekv_exactness_certificate", "EKV_OP_SELECT_TOPK", "ekv_selftest_wait_timeout", "EKV_EFLAG_TIMEOUT",
    "ekv_decode_adaptive", "EKV_OP_DECODE_ADAPTIVE",
]

EKV_F32, EKV_BF16 = 0, 1
EKV_POLICY_TOPK, EKV_POLICY_GAUSS, EKV_POLICY_FULL = 0, 1, 2
EKV_OP_SELECT_GAUSS, EKV_OP_ENTMAX_DECODE, EKV_OP_DECODE_STEP, EKV_OP_SOFTMAX_DECODE = 1, 2, 3, 4
EKV_OP_SELECT_TOPK = 5
EKV_OP_DECODE_ADAPTIVE = 6
EKV_EFLAG_BAD_PAGE, EKV_EFLAG_BAD_LEN, EKV_EFLAG_SEL_OVERFLOW, EKV_EFLAG_BAD_SEL = 1, 2, 4, 8
EKV_EFLAG_TIMEOUT = 16

lib_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libekv.so")


class EkvError(RuntimeError):
    def __init__(self, name, status):
        super().__init__(f"{name}: {ekv_status_string(status)} (status {status})")
        self.status = status


class EkvUnavailable(RuntimeError):
    pass


class Cache(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("num_phys_pages", ctypes.c_int32), ("k_pool", ctypes.c_void_p),
                ("v_pool", ctypes.c_void_p), ("box", ctypes.c_void_p), ("mom", ctypes.c_void_p)]


class Seqs(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_pages", ctypes.c_int32)]


class StepParams(ctypes.Structure):
    _fields_ = [("policy", ctypes.c_int32), ("k", ctypes.c_int32), ("delta", ctypes.c_float),
                ("cap", ctypes.c_int32), ("alpha", ctypes.c_float), ("scale", ctypes.c_float),
                ("dense_v", ctypes.c_int32), ("append", ctypes.c_int32)]


_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_SIGS = {
    "ekv_build_page_meta": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P],
    "ekv_append": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P, _P, _P],
    "ekv_score_pages": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P, _I, _F, _P, _P],
    "ekv_select_topk": [ctypes.POINTER(Seqs), _I, _I, _P, _I, _P, _P, _P, _SZ, _P],
    "ekv_select_gauss": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P, _I, _F, _F, _F, _I,
                         _P, _P, _P, _P, _SZ, _P],
    "ekv_entmax_decode": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P, _I, _F, _F, _P, _P,
                          _I, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "ekv_decode_step": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), ctypes.POINTER(StepParams),
                        _P, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "ekv_workspace_bytes": [_I, ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _I, _I],
    "ekv_softmax_decode": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P, _I, _F, _P, _P, _I, _P, _P,
                           _P, _SZ, _P],
    "ekv_exactness_certificate": [ctypes.POINTER(Seqs), _I, _I, _I, _F, _P, _P, _P, _I, _P, _P, _P],
    "ekv_decode_adaptive": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P, _I, _F, _F, _I, _P, _P, _P, _P, _P,
                            ctypes.POINTER(ctypes.c_int32), _P, _SZ, _P],
    "ekv_selftest_wait_timeout": [ctypes.c_uint32, _P],
    "ekv_step_kernel_count": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), ctypes.POINTER(StepParams), _I],
    "ekv_entmax_decode_static_ws": [ctypes.POINTER(Cache), ctypes.POINTER(Seqs), _P, _I, _F, _F, _P,
                                    _P, _I, _I, _P, _P, _P, _P, _P],
    "ekv_get_error": [ctypes.POINTER(ctypes.c_uint32)],
    "ekv_status_string": [_I],
}


def lib():
    """The loaded libekv.so (raises EkvUnavailable when it is missing)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(lib_path):
            raise EkvUnavailable(f"{lib_path} is missing: build it with sparse_kv_cache_kmax_b200.build_lib.build()")
        try:
            h = ctypes.CDLL(lib_path)
        except OSError as e:
            raise EkvUnavailable(f"cannot load {lib_path}: {e}") from e
        for name, args in _SIGS.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int32
        h.ekv_workspace_bytes.restype = ctypes.c_size_t
        h.ekv_status_string.restype = ctypes.c_char_p
        _LIB = h
    return _LIB


def ekv_status_string(status: int) -> str:
    try:
        return lib().ekv_status_string(int(status)).decode()
    except EkvUnavailable:
        return f"status {status}"


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name, status):
    if status != 0:
        raise EkvError(name, status)


_DTYPES = {torch.float32: EKV_F32, torch.bfloat16: EKV_BF16}


def make_cache(k_pool, v_pool, box=None, mom=None) -> Cache:
    """Describe a paged cache.  k_pool, v_pool: [num_phys, Hkv, S, d];
    box, mom: [Hkv, num_phys, 2, d] (head-major) of the same dtype (allocated
    here if None)."""
    if box is None:
        box = torch.empty(k_pool.shape[1], k_pool.shape[0], 2, k_pool.shape[3], dtype=k_pool.dtype,
                          device=k_pool.device)
    if mom is None:
        mom = torch.empty_like(box)
    for t in (k_pool, v_pool, box, mom):
        if not t.is_contiguous():
            raise ValueError("cache tensors must be contiguous")
    c = Cache(_DTYPES[k_pool.dtype], k_pool.shape[3], k_pool.shape[2], k_pool.shape[1],
              k_pool.shape[0], k_pool.data_ptr(), v_pool.data_ptr(), box.data_ptr(), mom.data_ptr())
    c._keep = (k_pool, v_pool, box, mom)
    c.box_t, c.mom_t = box, mom
    return c


def make_seqs(page_table, seq_lens) -> Seqs:
    """page_table: int32 [B, max_pages]; seq_lens: int32 [B] (device)."""
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    s = Seqs(page_table.data_ptr(), seq_lens.data_ptr(), page_table.shape[0], page_table.shape[1])
    s._keep = (page_table.contiguous(), seq_lens.contiguous())
    return s


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte-aligned device scratch buffer of at least nbytes."""
    t = torch.empty(max(int(nbytes), 1) + 256, dtype=torch.uint8, device=device)
    off = (-t.data_ptr()) % 256
    return t[off: off + max(int(nbytes), 1)]


def ekv_workspace_bytes(op, cache, seqs, num_q_heads, cap) -> int:
    return int(lib().ekv_workspace_bytes(op, ctypes.byref(cache), ctypes.byref(seqs), num_q_heads, cap))


def ekv_build_page_meta(cache, seqs, stream=None):
    _check("ekv_build_page_meta", lib().ekv_build_page_meta(ctypes.byref(cache), ctypes.byref(seqs), _stream(stream)))


def ekv_append(cache, seqs, k_new, v_new, stream=None):
    _check("ekv_append", lib().ekv_append(ctypes.byref(cache), ctypes.byref(seqs), _ptr(k_new),
                                          _ptr(v_new), _stream(stream)))


def ekv_score_pages(cache, seqs, q, scale, ub, stream=None):
    _check("ekv_score_pages", lib().ekv_score_pages(ctypes.byref(cache), ctypes.byref(seqs), _ptr(q),
                                                    q.shape[1], scale, _ptr(ub), _stream(stream)))


def ekv_select_topk(seqs, num_kv_heads, page_size, ub, k, sel, n_sel, stream=None, *, ws=None):
    """ws: ekv_workspace_bytes(EKV_OP_SELECT_TOPK, ..., k) bytes (None when 0,
    or to select long sequences in one stage)."""
    _check("ekv_select_topk", lib().ekv_select_topk(ctypes.byref(seqs), num_kv_heads, page_size, _ptr(ub),
                                                    k, _ptr(sel), _ptr(n_sel), _ptr(ws),
                                                    0 if ws is None else ws.numel(), _stream(stream)))


def ekv_select_gauss(cache, seqs, q, scale, alpha, delta, cap, sel, n_sel, tau_hat, ws, stream=None):
    _check("ekv_select_gauss", lib().ekv_select_gauss(
        ctypes.byref(cache), ctypes.byref(seqs), _ptr(q), q.shape[1], scale, alpha, delta, cap,
        _ptr(sel), _ptr(n_sel), _ptr(tau_hat), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def ekv_entmax_decode(cache, seqs, q, scale, alpha, sel, n_sel, cap, out, ws, *, dense_v=False,
                      tau=None, support_count=None, support_bits=None, stream=None):
    _check("ekv_entmax_decode", lib().ekv_entmax_decode(
        ctypes.byref(cache), ctypes.byref(seqs), _ptr(q), q.shape[1], scale, alpha, _ptr(sel),
        _ptr(n_sel), cap, int(bool(dense_v)), _ptr(out), _ptr(tau), _ptr(support_count),
        _ptr(support_bits), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def ekv_decode_step(cache, seqs, params: StepParams, q, k_new, v_new, sel, n_sel, out, ws, *,
                    tau=None, stream=None):
    _check("ekv_decode_step", lib().ekv_decode_step(
        ctypes.byref(cache), ctypes.byref(seqs), ctypes.byref(params), _ptr(q), q.shape[1],
        _ptr(k_new), _ptr(v_new), _ptr(sel), _ptr(n_sel), _ptr(out), _ptr(tau), _ptr(ws),
        0 if ws is None else ws.numel(), _stream(stream)))


def ekv_softmax_decode(cache, seqs, q, scale, sel, n_sel, cap, out, ws, *, lse=None, stream=None):
    """Softmax decode over the selected pages (sel None: every page)."""
    _check("ekv_softmax_decode", lib().ekv_softmax_decode(
        ctypes.byref(cache), ctypes.byref(seqs), _ptr(q), q.shape[1], scale, _ptr(sel), _ptr(n_sel), cap,
        _ptr(out), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def ekv_exactness_certificate(seqs, num_kv_heads, page_size, alpha, ub, sel, n_sel, tau, certified, *,
                              stream=None):
    """certified[b, hq] = 1 when head hq's sparse output equals its full-cache one."""
    _check("ekv_exactness_certificate", lib().ekv_exactness_certificate(
        ctypes.byref(seqs), num_kv_heads, page_size, tau.shape[1], alpha, _ptr(ub), _ptr(sel), _ptr(n_sel),
        sel.shape[-1], _ptr(tau), _ptr(certified), _stream(stream)))


def ekv_decode_adaptive(cache, seqs, q, scale, alpha, k0, sel, n_sel, out, tau, certified, ws, stream=None) -> int:
    """Top-k decode whose budget doubles from k0 until every head is certified
    exact; returns the final k (sel then holds [batch, Hkv, k])."""
    k_used = ctypes.c_int32(0)
    _check("ekv_decode_adaptive", lib().ekv_decode_adaptive(
        ctypes.byref(cache), ctypes.byref(seqs), _ptr(q), q.shape[1], scale, alpha, int(k0), _ptr(sel), _ptr(n_sel),
        _ptr(out), _ptr(tau), _ptr(certified), ctypes.byref(k_used), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)))
    return int(k_used.value)


def ekv_selftest_wait_timeout(polls=1024, stream=None):
    """One bounded wait that nothing satisfies: raises EKV_EFLAG_TIMEOUT."""
    _check("ekv_selftest_wait_timeout", lib().ekv_selftest_wait_timeout(polls, _stream(stream)))


def ekv_step_kernel_count(cache, seqs, params: StepParams, num_q_heads) -> int:
    """Kernels one ekv_decode_step call with these arguments enqueues."""
    return int(lib().ekv_step_kernel_count(ctypes.byref(cache), ctypes.byref(seqs), ctypes.byref(params),
                                           num_q_heads))


def ekv_entmax_decode_static_ws(cache, seqs, q, scale, alpha, sel, n_sel, cap, out, *, dense_v=False,
                                tau=None, support_count=None, support_bits=None, stream=None):
    """ekv_entmax_decode with the library's static scratch array (no workspace,
    no allocation); see include/ekv.h for its limits."""
    _check("ekv_entmax_decode_static_ws", lib().ekv_entmax_decode_static_ws(
        ctypes.byref(cache), ctypes.byref(seqs), _ptr(q), q.shape[1], scale, alpha, _ptr(sel), _ptr(n_sel),
        cap, int(bool(dense_v)), _ptr(out), _ptr(tau), _ptr(support_count), _ptr(support_bits),
        _stream(stream)))


def ekv_get_error() -> int:
    v = ctypes.c_uint32(0)
    _check("ekv_get_error", lib().ekv_get_error(ctypes.byref(v)))
    return int(v.value)
