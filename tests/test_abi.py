"""The C-ABI library: it loads, exports every symbol include/ekv.h declares,
and its host-side validation rejects bad arguments before any launch (CPU)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from sparse_kv_cache_kmax_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ekv.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"EKV_API\s+[\w\s\*]+?\b(ekv_\w+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 10
    h = B.lib()
    for n in names:
        assert hasattr(h, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", B.lib_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (ekv_\w+)", out))
    assert set(names) <= exported
    assert exported <= set(names), f"undeclared exports: {exported - set(names)}"


def test_status_strings():
    assert B.ekv_status_string(0) == "ok"
    assert "workspace" in B.ekv_status_string(3)


FAKE = 0x1000  # never dereferenced: validation fails before any launch


def _cache(**kw):
    c = dict(dtype=B.EKV_BF16, head_dim=128, page_size=16, num_kv_heads=8, num_phys_pages=10,
             k_pool=FAKE, v_pool=FAKE, box=FAKE, mom=FAKE)
    c.update(kw)
    return B.Cache(**c)


def _seqs(**kw):
    s = dict(page_table=FAKE, seq_lens=FAKE, batch=2, max_pages=5)
    s.update(kw)
    return B.Seqs(**s)


def _decode(cache, seqs, Hq=32, scale=0.1, alpha=1.5, sel=FAKE, n_sel=FAKE, cap=4, out=FAKE,
            ws=0x100000, ws_bytes=1 << 40):
    return B.lib().ekv_entmax_decode(ctypes.byref(cache), ctypes.byref(seqs), FAKE, Hq, scale, alpha,
                                     sel, n_sel, cap, 0, out, None, None, None, ws, ws_bytes, None)


def test_validation_rejects_before_launch():
    L = B.lib()
    c, s = _cache(), _seqs()
    assert L.ekv_build_page_meta(None, ctypes.byref(s), None) == 1
    assert L.ekv_build_page_meta(ctypes.byref(_cache(box=None)), ctypes.byref(s), None) == 1
    assert L.ekv_build_page_meta(ctypes.byref(_cache(head_dim=96)), ctypes.byref(s), None) == 2
    assert L.ekv_build_page_meta(ctypes.byref(_cache(page_size=8)), ctypes.byref(s), None) == 2
    assert L.ekv_build_page_meta(ctypes.byref(_cache(dtype=7)), ctypes.byref(s), None) == 2
    assert L.ekv_build_page_meta(ctypes.byref(c), ctypes.byref(_seqs(batch=0)), None) == 1
    assert L.ekv_append(ctypes.byref(c), ctypes.byref(s), None, FAKE, None) == 1
    assert L.ekv_score_pages(ctypes.byref(c), ctypes.byref(s), FAKE, 12, 0.1, FAKE, None) == 1   # Hq % Hkv
    assert L.ekv_score_pages(ctypes.byref(c), ctypes.byref(s), FAKE, 24, 0.1, FAKE, None) == 2   # G = 3
    assert L.ekv_score_pages(ctypes.byref(c), ctypes.byref(s), FAKE, 32, -1.0, FAKE, None) == 1
    assert L.ekv_select_topk(ctypes.byref(s), 8, 16, FAKE, 0, FAKE, FAKE, None, 0, None) == 1
    assert L.ekv_select_topk(ctypes.byref(s), 8, 12, FAKE, 4, FAKE, FAKE, None, 0, None) == 2
    long = _seqs(max_pages=65536)
    assert B.lib().ekv_workspace_bytes(B.EKV_OP_SELECT_TOPK, ctypes.byref(c), ctypes.byref(s), 32, 4) == 0
    need = B.lib().ekv_workspace_bytes(B.EKV_OP_SELECT_TOPK, ctypes.byref(c), ctypes.byref(long), 32, 512)
    assert need > 0
    assert L.ekv_select_topk(ctypes.byref(long), 8, 16, FAKE, 512, FAKE, FAKE, 0x100000, 16, None) == 3
    assert _decode(c, s, alpha=1.0) == 1
    assert _decode(c, s, alpha=float("nan")) == 1
    assert _decode(c, s, sel=None) == 1                 # sel without n_sel
    assert _decode(c, s, sel=None, n_sel=None, cap=4) == 1   # full cache needs cap ≥ max_pages
    assert _decode(c, s, out=None) == 1
    assert _decode(c, s, ws=0x100010) == 3              # misaligned
    assert _decode(c, s, ws_bytes=16) == 3              # too small
    g = L.ekv_select_gauss(ctypes.byref(c), ctypes.byref(s), FAKE, 32, 0.1, 1.7, 0.5, 8, FAKE, FAKE,
                           None, 0x100000, 1 << 40, None)
    assert g == 2                                       # 1/(α−1) not an integer
    p = B.StepParams(9, 4, 0.5, 4, 1.5, 0.1, 0, 0)
    assert L.ekv_decode_step(ctypes.byref(c), ctypes.byref(s), ctypes.byref(p), FAKE, 32, None, None,
                             FAKE, FAKE, FAKE, None, 0x100000, 1 << 40, None) == 1
    p = B.StepParams(B.EKV_POLICY_TOPK, 8, 0.5, 4, 1.5, 0.1, 0, 0)        # k > cap
    assert L.ekv_decode_step(ctypes.byref(c), ctypes.byref(s), ctypes.byref(p), FAKE, 32, None, None,
                             FAKE, FAKE, FAKE, None, 0x100000, 1 << 40, None) == 1


def test_workspace_sizes_are_host_only_and_monotone():
    c, s = _cache(), _seqs()
    a = B.lib().ekv_workspace_bytes(B.EKV_OP_ENTMAX_DECODE, ctypes.byref(c), ctypes.byref(s), 32, 4)
    b = B.lib().ekv_workspace_bytes(B.EKV_OP_ENTMAX_DECODE, ctypes.byref(c), ctypes.byref(s), 32, 5)
    g = B.lib().ekv_workspace_bytes(B.EKV_OP_SELECT_GAUSS, ctypes.byref(c), ctypes.byref(s), 32, 4)
    st = B.lib().ekv_workspace_bytes(B.EKV_OP_DECODE_STEP, ctypes.byref(c), ctypes.byref(s), 32, 4)
    assert 0 < a < b and g > 0 and st >= a + g
    assert a % 256 == 0
    assert B.lib().ekv_workspace_bytes(99, ctypes.byref(c), ctypes.byref(s), 32, 4) == 0
    assert B.lib().ekv_workspace_bytes(B.EKV_OP_ENTMAX_DECODE, ctypes.byref(c), ctypes.byref(s), 24, 4) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_a_device_reports_cuda_error():
    c, s = _cache(), _seqs()
    assert _decode(c, s) == 4


def test_step_kernel_count_host_side():
    L = B.lib()
    c, s = _cache(), _seqs()
    assert L.ekv_step_kernel_count(ctypes.byref(c), ctypes.byref(s), None, 32) == 0
    assert L.ekv_step_kernel_count(ctypes.byref(c), ctypes.byref(s),
                                   ctypes.byref(B.StepParams(9, 4, 0.5, 4, 1.5, 0.1, 0, 1)), 32) == 0
    assert L.ekv_step_kernel_count(ctypes.byref(c), ctypes.byref(s),
                                   ctypes.byref(B.StepParams(B.EKV_POLICY_TOPK, 4, 0.5, 4, 1.5, 0.1, 0, 1)), 24) == 0
    # fp32 caches never take the fused decode: append + score + top-k + 3 decode kernels
    f32 = _cache(dtype=B.EKV_F32)
    topk = B.StepParams(B.EKV_POLICY_TOPK, 4, 0.5, 4, 1.5, 0.1, 0, 1)
    assert L.ekv_step_kernel_count(ctypes.byref(f32), ctypes.byref(s), ctypes.byref(topk), 32) == 6
    full = B.StepParams(B.EKV_POLICY_FULL, 0, 0.5, 4, 1.5, 0.1, 0, 0)
    assert L.ekv_step_kernel_count(ctypes.byref(f32), ctypes.byref(s), ctypes.byref(full), 32) == 3
    # Gaussian policy: page statistics, τ̂, filter count and filter write
    gauss = B.StepParams(B.EKV_POLICY_GAUSS, 0, 0.5, 4, 1.5, 0.1, 0, 1)
    assert L.ekv_step_kernel_count(ctypes.byref(f32), ctypes.byref(s), ctypes.byref(gauss), 32) == 1 + 4 + 3
