"""ekv_entmax_decode_static_ws: the decode entry point for callers that cannot
allocate device memory (for example a plugin whose host framework owns the
whole device memory pool, or a serving loop that must not call cudaMalloc).

Its scratch is one array compiled into the library, shared by every call.
These tests run it on decode paths that really use that scratch (the scores,
thresholds and split counters of the selected tokens live there), twice in a
row and interleaved with another configuration so that the second call starts
from whatever the previous one left, and compare each call with the
ekv_entmax_decode call that gets a caller workspace and with the float64
oracle.  It must also refuse, before any device work, a configuration whose
scratch does not fit.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.workloads import scaled_down

from gpu_helpers import OUT_TOL, Gpu, check_unit_decode, gen, np64, oracle_unit, row_rel_err

pytestmark = pytest.mark.gpu


def _static_decode(gpu, alpha, sel, n_sel, cap):
    wl = gpu.wl
    out = torch.full((wl.batch, gpu.Hq, wl.head_dim), float("nan"), device="cuda")
    tau = torch.full((wl.batch, gpu.Hq), float("nan"), device="cuda")
    cnt = torch.full((wl.batch, gpu.Hq), -1, dtype=torch.int32, device="cuda")
    words = (cap * wl.page_size + 31) // 32
    bits = torch.zeros(wl.batch, gpu.Hq, words, dtype=torch.int32, device="cuda")
    B.ekv_entmax_decode_static_ws(gpu.cache, gpu.seqs, gpu.inp["q"], gpu.scale, alpha, sel, n_sel, cap, out,
                                  tau=tau, support_count=cnt, support_bits=bits)
    return out, tau, cnt, bits


def _decode_kernels(gpu, cap):
    """Kernels the decode of these sizes launches: a top-k step's count minus
    its page scores and one-stage top-k."""
    p = B.StepParams(B.EKV_POLICY_TOPK, cap, 0.0, cap, 1.5, gpu.scale, 0, 0)
    return B.ekv_step_kernel_count(gpu.cache, gpu.seqs, p, gpu.Hq) - 2


def _case(name, over, seed, k):
    wl = scaled_down(name, **over)
    inp = gen(wl, seed)
    gpu = Gpu(inp)
    gpu.build_meta()
    sel, n_sel = gpu.topk(gpu.score(), k)
    torch.cuda.synchronize()
    return gpu, sel, n_sel


# many bf16 units: the two-launch split decode; fp32 cache: the three-kernel
# decode; both keep their scores, maxima and page ids in the scratch
CASES = {
    "bf16_topk": ("short_scattered", dict(batch=10, context=900, context_min=300), 4242, 24),
    "f32_topk": ("tiny_fp32", dict(batch=2, context=4093), 4243, 32),
}


@pytest.mark.parametrize("case", list(CASES))
def test_static_scratch_decode_matches_workspace_decode_and_oracle_twice(case):
    name, over, seed, k = CASES[case]
    gpu, sel, n_sel = _case(name, over, seed, k)
    other, osel, on = _case("short_scattered", dict(batch=12, context=1500, context_min=700), 4244, 40)
    wl = gpu.wl
    assert B.ekv_workspace_bytes(B.EKV_OP_ENTMAX_DECODE, gpu.cache, gpu.seqs, gpu.Hq, k) > 0
    kernels = _decode_kernels(gpu, k)
    assert kernels == (3 if wl.dtype == "f32" else 2), kernels
    ref = gpu.decode(1.5, sel, n_sel, k)
    torch.cuda.synchronize()
    orcs = {(b, h): oracle_unit(gpu.inp, b, h, sel=sel[b, h, : int(n_sel[b, h])].cpu().numpy())
            for b in range(wl.batch) for h in range(wl.num_kv_heads)}
    for call in range(2):
        out, tau, cnt, bits = _static_decode(gpu, 1.5, sel, n_sel, k)
        torch.cuda.synchronize()
        err = row_rel_err(np64(out).reshape(-1, wl.head_dim), np64(ref[0]).reshape(-1, wl.head_dim))
        assert np.all(err <= OUT_TOL[wl.dtype]), (call, err.max())
        assert torch.allclose(tau, ref[1], rtol=1e-6, atol=1e-6), call
        assert torch.equal(cnt, ref[2]), call
        assert torch.equal(bits, ref[3]), call
        for (b, h), orc in orcs.items():
            check_unit_decode(orc, out, tau, cnt, bits, b, h, wl.group, wl.dtype, what=f"call {call} unit {(b, h)}")
        # another configuration in between leaves its own contents in the array
        o2 = _static_decode(other, 1.5, osel, on, 40)
        r2 = other.decode(1.5, osel, on, 40)
        torch.cuda.synchronize()
        assert torch.equal(o2[2], r2[2]) and torch.allclose(o2[1], r2[1], rtol=1e-6, atol=1e-6)
    assert B.ekv_get_error() == 0


def test_static_scratch_refuses_oversized_configurations():
    fake = 0x1000  # never dereferenced: the size check fails before any device work
    cache = B.Cache(B.EKV_BF16, 128, 16, 8, 1 << 20, fake, fake, fake, fake)
    seqs = B.Seqs(fake, fake, 64, 65536)
    need = B.ekv_workspace_bytes(B.EKV_OP_ENTMAX_DECODE, cache, seqs, 32, 4096)
    assert need > (16 << 20)
    status = B.lib().ekv_entmax_decode_static_ws(
        ctypes.byref(cache), ctypes.byref(seqs), fake, 32, 0.1, 1.5, fake, fake, 4096, 0, fake,
        None, None, None, None)
    assert status == 3
