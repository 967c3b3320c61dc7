"""GPU edge cases: single-token and ragged sequences, budgets that cover the
whole sequence, and data errors (bad page ids, lengths, selections, a full
Gaussian selection buffer) that the kernels turn into error flags."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.engine import DecodeEngine
from sparse_kv_cache_kmax_b200.workloads import scaled_down

from gpu_helpers import OUT_TOL, REL_TIE, Gpu, gen, np64, oracle_unit, row_rel_err

pytestmark = pytest.mark.gpu


def _check_outputs(inp, eng, policy, k=None):
    wl = inp["workload"]
    G = wl.group
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            if policy == "full":
                orc = oracle_unit(inp, b, h, policy="all")
            else:
                got = eng.sel[b, h, : int(eng.n_sel[b, h])].cpu().numpy()
                orc = oracle_unit(inp, b, h, sel=got)
            err = row_rel_err(np64(eng.out[b, h * G:(h + 1) * G]), orc["o"])
            assert np.all(err <= OUT_TOL[wl.dtype]), (b, h, err.max())


@pytest.mark.parametrize("lens", [[1, 17, 33], [16, 15, 1]])
def test_tiny_and_ragged_sequences(lens):
    wl = scaled_down("gqa_32k", batch=3, context=64)
    inp = gen(wl, 21)
    inp["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for policy in ("topk", "full", "gauss"):
        eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"],
                           wl.num_q_heads, policy=policy, k=2, delta=0.5, alpha=1.5)
        eng.build_meta()
        eng.step(inp["q"])
        torch.cuda.synchronize()
        assert B.ekv_get_error() == 0
        if policy == "topk":
            P = [-(-L // wl.page_size) for L in lens]
            assert eng.n_sel[:, 0].tolist() == [min(2, p) for p in P]
        _check_outputs(inp, eng, policy)


def test_budget_covering_every_page_selects_all():
    wl = scaled_down("clustered_128k", batch=2, context=200)
    inp = gen(wl, 22)
    gpu = Gpu(inp)
    gpu.build_meta()
    sel, n = gpu.topk(gpu.score(), 64)
    torch.cuda.synchronize()
    P = -(-200 // wl.page_size)
    assert torch.all(n == P)
    assert torch.equal(sel[:, :, :P].cpu(), torch.arange(P, dtype=torch.int32).expand(2, wl.num_kv_heads, P))


def test_bad_page_id_and_length_raise_flags_without_faulting():
    wl = scaled_down("gqa_32k", batch=2, context=300)
    inp = gen(wl, 23)
    assert B.ekv_get_error() == 0
    pt = inp["page_table"].clone()
    pt[0, 3] = inp["num_phys"] + 5            # outside the pool: skipped by every kernel
    lens = inp["seq_lens"].clone()
    lens[1] = wl.max_pages * wl.page_size + 100  # longer than the page table: clamped
    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], pt, lens, wl.num_q_heads, policy="topk", k=8)
    eng.build_meta()
    eng.step(inp["q"])
    torch.cuda.synchronize()
    flags = B.ekv_get_error()
    assert flags & B.EKV_EFLAG_BAD_PAGE and flags & B.EKV_EFLAG_BAD_LEN
    assert torch.isfinite(eng.out).all()
    assert B.ekv_get_error() == 0                # reading clears the word


def test_bad_selection_entries_raise_flag():
    wl = scaled_down("gqa_32k", batch=1, context=300)
    inp = gen(wl, 24)
    gpu = Gpu(inp)
    gpu.build_meta()
    sel = torch.zeros(1, wl.num_kv_heads, 4, dtype=torch.int32, device="cuda")
    sel[0, :, 1] = 10_000                         # past the sequence's pages
    n = torch.full((1, wl.num_kv_heads), 4, dtype=torch.int32, device="cuda")
    out, tau, cnt, bits = gpu.decode(1.5, sel, n, 4)
    torch.cuda.synchronize()
    assert B.ekv_get_error() & B.EKV_EFLAG_BAD_SEL
    assert torch.isfinite(out).all()


def test_gauss_selection_overflow_is_flagged_and_truncated():
    wl = scaled_down("clustered_128k", batch=1, context=800)
    inp = gen(wl, 25)
    gpu = Gpu(inp)
    gpu.build_meta()
    sel, n, tau_hat = gpu.gauss(1.25, 1e6, cap=4)  # Δ huge: every page passes
    torch.cuda.synchronize()
    assert B.ekv_get_error() & B.EKV_EFLAG_SEL_OVERFLOW
    assert torch.all(n == 4)
    assert torch.equal(sel[0, :, :4].cpu(), torch.arange(4, dtype=torch.int32).expand(wl.num_kv_heads, 4))


@pytest.mark.parametrize("alpha", [2.0, 1.5, 1.25])
def test_gauss_point_mass_pages(alpha):
    """Every other page holds one key in all its tokens (zero spread), aligned
    with the group's mean query so that those pages carry the top scores.
    From Jensen's bound the expected mass is then their count (32), the
    solve's far steps pass every page's mean, where no mass is left, and it
    must back off and come back from the right: τ̂ and the kept set still
    match the oracle's bisection.  The other pages drop out of the solve
    (their spread puts them six σ below τ̂)."""
    wl = scaled_down("clustered_128k", batch=2, context=1024)
    inp = gen(wl, 23)
    G, S = wl.group, wl.page_size
    kp = inp["k_pool"]
    for b in range(wl.batch):
        P = -(-int(inp["seq_lens"][b]) // S)
        ids = inp["page_table"][b, :P].long()
        for h in range(wl.num_kv_heads):
            qbar = inp["q"][b, h * G:(h + 1) * G].float().mean(0)
            key = 3.0 * wl.head_dim ** 0.5 * qbar / qbar.norm()
            kp[ids[::2], h] = key.to(kp.dtype)
    gpu = Gpu(inp)
    gpu.build_meta()
    B.ekv_get_error()  # clear what earlier tests left
    delta = 0.5
    sel, n, tau_hat = gpu.gauss(alpha, delta)
    torch.cuda.synchronize()
    assert B.ekv_get_error() == 0
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            gs = oracle_unit(inp, b, h, policy="gauss", delta=delta, alpha=alpha)["gauss"]
            t = np64(tau_hat[b, h * G:(h + 1) * G])
            assert np.allclose(t, gs["tau_hat"], rtol=1e-5, atol=1e-5), (b, h, t, gs["tau_hat"])
            margin = gs["margin"]
            band = REL_TIE * np.maximum(1.0, np.abs(gs["tau_hat"] - delta))[:, None]
            certain_in = np.any(margin > band, axis=0)
            certain_out = np.all(margin < -band, axis=0)
            assert certain_in[::2].all()  # the point-mass pages pass by a wide margin
            got = set(sel[b, h, : int(n[b, h])].cpu().numpy().tolist())
            assert set(np.nonzero(certain_in)[0].tolist()) <= got, (b, h)
            assert not (got & set(np.nonzero(certain_out)[0].tolist())), (b, h)


def test_fp32_cache_full_size_tiny_config():
    """The tiny fp32 configuration at its full size (4096 tokens, 256 pages)."""
    from sparse_kv_cache_kmax_b200.workloads import WORKLOADS

    wl = WORKLOADS["tiny_fp32"]
    inp = gen(wl, 26)
    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], 1,
                       policy="topk", k=wl.topk, alpha=1.5)
    eng.build_meta()
    eng.step(inp["q"])
    torch.cuda.synchronize()
    orc = oracle_unit(inp, 0, 0, policy="topk", k=wl.topk)
    got = eng.sel[0, 0, : int(eng.n_sel[0, 0])].cpu().numpy()
    from gpu_helpers import assert_sel_matches, topk_tie_band
    assert_sel_matches(got, orc["sel"], topk_tie_band(orc["score"], wl.topk), "tiny")
    if not np.array_equal(got, orc["sel"]):
        orc = oracle_unit(inp, 0, 0, sel=got)
    assert row_rel_err(np64(eng.out[0]), orc["o"]).max() <= OUT_TOL["f32"]


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable():
    """Failure detection without a fault: a wait on an mbarrier that nothing
    completes gives up after its poll limit, the sticky error word reports
    EKV_EFLAG_TIMEOUT, and the next library call runs normally."""
    flags = ctypes.c_uint32(0)
    B.lib().ekv_get_error(ctypes.byref(flags))          # start from a clean word
    B.ekv_selftest_wait_timeout(4096)
    assert B.lib().ekv_get_error(ctypes.byref(flags)) == 0
    assert flags.value & B.EKV_EFLAG_TIMEOUT
    assert B.lib().ekv_get_error(ctypes.byref(flags)) == 0 and flags.value == 0   # cleared
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0                      # the context still works
