"""ekv_entmax_decode_static_ws: the decode entry point for callers that cannot
allocate device memory (for example a plugin whose host framework owns the
whole device memory pool, or a serving loop that must not call cudaMalloc).

It must give the same results as ekv_entmax_decode with a caller workspace,
on consecutive calls that reuse the library's static scratch array, and it
must refuse, before any device work, a configuration whose scratch does not
fit in that array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.workloads import scaled_down

from gpu_helpers import OUT_TOL, Gpu, gen, np64, row_rel_err

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


@pytest.mark.parametrize("policy", ["topk", "full"])
def test_static_scratch_decode_matches_workspace_decode_twice(policy):
    wl = scaled_down("clustered_128k", batch=2, context=3005)
    inp = gen(wl, 4242)
    gpu = Gpu(inp)
    gpu.build_meta()
    if policy == "topk":
        cap = 24
        sel, n_sel = gpu.topk(gpu.score(), cap)
    else:
        cap, sel, n_sel = inp["max_pages"], None, None
    ref_out, ref_tau, ref_cnt, ref_bits = gpu.decode(1.5, sel, n_sel, cap)
    torch.cuda.synchronize()
    for call in range(2):
        out, tau, cnt, bits = _static_decode(gpu, 1.5, sel, n_sel, cap)
        torch.cuda.synchronize()
        err = row_rel_err(np64(out).reshape(-1, wl.head_dim), np64(ref_out).reshape(-1, wl.head_dim))
        assert np.all(err <= OUT_TOL[wl.dtype]), (call, err.max())
        assert torch.allclose(tau, ref_tau, rtol=1e-6, atol=1e-6), call
        assert torch.equal(cnt, ref_cnt), call
        assert torch.equal(bits, ref_bits), call


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
