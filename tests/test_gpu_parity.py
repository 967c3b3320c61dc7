"""GPU parity: every stage of the CUDA path against the float64 oracle on the
same seeded inputs, through the C ABI.  Sizes span several CTA tiles and a
ragged last page; tolerances are those of tests/gpu_helpers.py."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.workloads import scaled_down

from gpu_helpers import (OUT_TOL, REL_TIE, Gpu, assert_sel_matches, check_unit_decode, gen, np64,
                         oracle_unit, q_group, row_rel_err, sel_tensor, topk_tie_band, unit_arrays)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32": dict(context=4093),
    "gqa_32k": dict(batch=2, context=1500),
    "clustered_128k": dict(batch=2, context=3005),
    "short_scattered": dict(batch=5, context=900, context_min=300),
    "long_512k": dict(batch=1, context=4007),
}


def _wl(name):
    return scaled_down(name, **CASES[name])


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    wl = _wl(request.param)
    inp = gen(wl, 1000 + list(CASES).index(request.param), n_new=2)
    gpu = Gpu(inp)
    box, mom = gpu.build_meta()
    torch.cuda.synchronize()
    return wl, inp, gpu, box, mom


def _units(wl, limit=6):
    us = [(b, h) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    if len(us) <= limit:
        return us
    rng = np.random.default_rng(0)
    pick = rng.choice(len(us), limit - 1, replace=False)
    return [us[0]] + [us[i] for i in sorted(pick) if i != 0]


def _bits(t, dtype):
    if dtype == "bf16":
        return t.contiguous().view(torch.int16).cpu().numpy()
    return t.contiguous().view(torch.int32).cpu().numpy()


def test_metadata_bit_exact(case):
    wl, inp, gpu, box, mom = case
    for b in range(wl.batch):
        L = int(inp["seq_lens"][b])
        phys, n_valid = O.unit_pages(inp["page_table"][b].cpu().numpy(), L, wl.page_size)
        for h in range(wl.num_kv_heads):
            meta = O.page_metadata(np64(inp["k_pool"][torch.as_tensor(phys).cuda(), h]), n_valid, wl.dtype)
            tdt = box.dtype
            got_box = _bits(box[h, torch.as_tensor(phys).cuda()], wl.dtype)
            got_mom = _bits(mom[h, torch.as_tensor(phys).cuda()], wl.dtype)
            want_box = _bits(torch.from_numpy(np.stack([meta["kmax"], meta["kmin"]], 1)).to(tdt), wl.dtype)
            want_mom = _bits(torch.from_numpy(np.stack([meta["mean"], meta["var"]], 1)).to(tdt), wl.dtype)
            assert np.array_equal(got_box, want_box), (b, h)
            assert np.array_equal(got_mom, want_mom), (b, h)


def test_bound_matches_oracle_and_dominates_scores(case):
    wl, inp, gpu, box, mom = case
    ub = gpu.score()
    torch.cuda.synchronize()
    for b, h in _units(wl):
        orc = oracle_unit(inp, b, h, policy="all")
        P = orc["score"].size
        got = np64(ub[b, h, :P])
        meta = orc["meta"]
        q = q_group(inp, b, h)
        mag = gpu.scale * (np.abs(q)[:, None, :] * np.maximum(np.abs(meta["kmax"]), np.abs(meta["kmin"]))[None]).sum(-1).max(0)
        assert np.all(np.abs(got - orc["score"]) <= 1e-5 * mag + 1e-30), (b, h)
        # the page score bounds every token score of the group in the page
        zmax = np.full(P, -np.inf)
        np.maximum.at(zmax, orc["token_page"], (orc["u"] / 0.5).max(0))
        assert np.all(got + 1e-5 * mag >= zmax), (b, h)


@pytest.mark.parametrize("k", [1, 7, 64])
def test_topk_exact_on_gpu_scores_and_within_ties_of_oracle(case, k):
    wl, inp, gpu, box, mom = case
    ub = gpu.score()
    sel, n = gpu.topk(ub, k)
    torch.cuda.synchronize()
    for b in range(wl.batch):
        L = int(inp["seq_lens"][b])
        P = -(-L // wl.page_size)
        for h in range(wl.num_kv_heads):
            scores32 = np64(ub[b, h, :P])
            want = O.select_topk(scores32, k)
            got = sel[b, h, : int(n[b, h])].cpu().numpy()
            assert int(n[b, h]) == min(k, P)
            assert np.array_equal(got, want), (b, h)          # integer work on the same scores: exact
    for b, h in _units(wl, 3):
        orc = oracle_unit(inp, b, h, policy="topk", k=k)
        got = sel[b, h, : int(n[b, h])].cpu().numpy()
        assert_sel_matches(got, orc["sel"], topk_tie_band(orc["score"], k), f"unit {(b, h)}")


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25])
def test_decode_on_oracle_selection(case, alpha):
    wl, inp, gpu, box, mom = case
    k = 12
    sels, orcs = {}, {}
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            orcs[(b, h)] = None
    units = _units(wl)
    for b, h in units:
        orcs[(b, h)] = oracle_unit(inp, b, h, policy="topk", k=k, alpha=alpha)
        sels[(b, h)] = orcs[(b, h)]["sel"]
    for key in orcs:
        if orcs[key] is None:
            sels[key] = np.arange(min(k, 1))
    sel, n = sel_tensor(sels, wl.batch, wl.num_kv_heads, k)
    out, tau, cnt, bits = gpu.decode(alpha, sel, n, k)
    torch.cuda.synchronize()
    for b, h in units:
        check_unit_decode(orcs[(b, h)], out, tau, cnt, bits, b, h, wl.group, wl.dtype,
                          what=f"alpha {alpha} unit {(b, h)}")


def test_decode_general_alpha(case):
    wl, inp, gpu, box, mom = case
    alpha = 1.7                                 # β = 1/0.7: the pure Newton path
    out, tau, cnt, bits = gpu.decode(alpha)     # full cache
    torch.cuda.synchronize()
    for b, h in _units(wl, 3):
        orc = oracle_unit(inp, b, h, policy="all", alpha=alpha)
        check_unit_decode(orc, out, tau, cnt, bits, b, h, wl.group, wl.dtype, what=f"unit {(b, h)}")


def test_full_cache_decode_and_dense_variant(case):
    wl, inp, gpu, box, mom = case
    out, tau, cnt, bits = gpu.decode(1.5)
    out_d, tau_d, _, _ = gpu.decode(1.5, dense_v=True)
    torch.cuda.synchronize()
    assert torch.equal(tau, tau_d)
    assert np.all(row_rel_err(np64(out_d).reshape(-1, wl.head_dim), np64(out).reshape(-1, wl.head_dim))
                  <= OUT_TOL[wl.dtype])
    for b, h in _units(wl, 4):
        orc = oracle_unit(inp, b, h, policy="all", alpha=1.5)
        check_unit_decode(orc, out, tau, cnt, bits, b, h, wl.group, wl.dtype, what=f"unit {(b, h)}")


def test_exactness_when_selection_holds_the_support(case):
    """[EntmaxKV] §3: selected pages ⊇ support pages ⇒ sparse output = full output."""
    from gpu_helpers import support_from_bits
    wl, inp, gpu, box, mom = case
    out_f, tau_f, cnt_f, bits_f = gpu.decode(1.5)
    torch.cuda.synchronize()
    cap = inp["max_pages"]
    bits_np = bits_f.cpu().numpy().view(np.uint32)
    sels = {}
    rng = np.random.default_rng(5)
    for b in range(wl.batch):
        L = int(inp["seq_lens"][b])
        P = -(-L // wl.page_size)
        for h in range(wl.num_kv_heads):
            pages = set()
            for g in range(wl.group):
                sup = support_from_bits(bits_np[b, h * wl.group + g], P * wl.page_size)
                pages |= set((np.nonzero(sup)[0] // wl.page_size).tolist())
            pages |= set(rng.choice(P, min(P, 3), replace=False).tolist())
            sels[(b, h)] = np.array(sorted(pages))
    sel, nsel = sel_tensor(sels, wl.batch, wl.num_kv_heads, cap)
    out_s, tau_s, _, _ = gpu.decode(1.5, sel, nsel, cap)
    torch.cuda.synchronize()
    assert np.all(row_rel_err(np64(out_s).reshape(-1, wl.head_dim), np64(out_f).reshape(-1, wl.head_dim))
                  <= 1e-5)
    assert torch.allclose(tau_s, tau_f, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25])
def test_gauss_selection(case, alpha):
    wl, inp, gpu, box, mom = case
    delta = 0.5
    sel, n, tau_hat = gpu.gauss(alpha, delta)
    torch.cuda.synchronize()
    for b, h in _units(wl, 4):
        orc = oracle_unit(inp, b, h, policy="gauss", delta=delta, alpha=alpha)
        gs = orc["gauss"]
        G = wl.group
        t = np64(tau_hat[b, h * G:(h + 1) * G])
        assert np.allclose(t, gs["tau_hat"], rtol=1e-5, atol=1e-5), (t, gs["tau_hat"])
        margin = gs["margin"]
        band = REL_TIE * np.maximum(1.0, np.abs(gs["tau_hat"] - delta))[:, None]
        certain_in = np.any(margin > band, axis=0)
        certain_out = np.all(margin < -band, axis=0)
        got = set(sel[b, h, : int(n[b, h])].cpu().numpy().tolist())
        if certain_in.any():
            assert set(np.nonzero(certain_in)[0].tolist()) <= got, (b, h)
            assert not (got & set(np.nonzero(certain_out)[0].tolist())), (b, h)
        else:
            assert int(n[b, h]) == 1


@pytest.mark.parametrize("policy", ["topk", "gauss", "full"])
def test_decode_step_end_to_end(case, policy):
    wl, inp, gpu, box, mom = case
    from sparse_kv_cache_kmax_b200.engine import DecodeEngine
    k = 16
    eng = DecodeEngine(inp["k_pool"].clone(), inp["v_pool"].clone(), inp["page_table"], inp["seq_lens"],
                       wl.num_q_heads, policy=policy, k=k, delta=0.5, alpha=1.5)
    eng.build_meta()
    out = eng.step(inp["q"], inp["k_new"][0], inp["v_new"][0]).clone()   # re-append the stored token
    torch.cuda.synchronize()
    for b, h in _units(wl, 3):
        if policy == "full":
            orc = oracle_unit(inp, b, h, policy="all")
        else:
            orc = oracle_unit(inp, b, h, policy=policy, k=k, delta=0.5)
            got = eng.sel[b, h, : int(eng.n_sel[b, h])].cpu().numpy()
            if policy == "topk":
                assert_sel_matches(got, orc["sel"], topk_tie_band(orc["score"], k), f"unit {(b, h)}")
            if not np.array_equal(got, orc["sel"]):
                orc = oracle_unit(inp, b, h, sel=got)
        G = wl.group
        err = row_rel_err(np64(out[b, h * G:(h + 1) * G]), orc["o"])
        assert np.all(err <= OUT_TOL[wl.dtype]), (policy, b, h, err.max())
    # the step ran the kernels it says: append + scores + one-stage top-k,
    # then for bf16 the cluster decode (few units) or the two-launch split
    # decode (many units), for fp32 the three-kernel decode
    n_kern = B.ekv_step_kernel_count(eng.cache, eng.seqs, eng.params, wl.num_q_heads)
    if policy == "topk":
        assert n_kern - 3 in ((1, 2) if wl.dtype == "bf16" else (3,)), n_kern


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.7])
def test_streaming_full_cache_decode_ragged_lengths(alpha):
    """Full-cache decode of sequences longer than the scores one thread keeps
    in registers (they are read again from L2 at every pass of the per-head
    CTA), ragged lengths on a scattered pool, 64 units: the two-launch decode
    with its streaming per-head kernel, against the oracle."""
    wl = scaled_down("short_scattered", batch=8, context=40000, context_min=17000)
    inp = gen(wl, 4242)
    gpu = Gpu(inp)
    gpu.build_meta()
    p = B.StepParams(B.EKV_POLICY_FULL, 0, 0.0, inp["max_pages"], alpha, gpu.scale, 0, 0)
    assert B.ekv_step_kernel_count(gpu.cache, gpu.seqs, p, wl.num_q_heads) == 2
    out, tau, cnt, bits = gpu.decode(alpha)
    torch.cuda.synchronize()
    assert B.ekv_get_error() == 0
    for b, h in _units(wl, 4):
        orc = oracle_unit(inp, b, h, policy="all", alpha=alpha)
        check_unit_decode(orc, out, tau, cnt, bits, b, h, wl.group, wl.dtype,
                          what=f"alpha {alpha} unit {(b, h)}")
    # dense V: the same scores and τ, then every valid V row read once per
    # unit by a third launch; zero weights add nothing
    p.dense_v = 1
    assert B.ekv_step_kernel_count(gpu.cache, gpu.seqs, p, wl.num_q_heads) == 3
    out_d, tau_d, cnt_d, _ = gpu.decode(alpha, dense_v=True)
    torch.cuda.synchronize()
    assert torch.equal(tau_d, tau) and torch.equal(cnt_d, cnt)
    assert np.all(row_rel_err(np64(out_d).reshape(-1, wl.head_dim), np64(out).reshape(-1, wl.head_dim)) <= 1e-5)
