"""Parity at the full sizes of the benchmark's workloads, in the launch
configuration the benchmark times: one ``ekv_decode_step`` call (append, page
scores, selection, sparse α-entmax decode) over the whole batch, then sampled
units — unit 0 and a few fixed others — compared with the float64 oracle.

Source: "Résumé Technique : EntmaxKV" §2.C "Attention Entmax Parcimonieuse"
and §3 "Récupération du Support" (the sparse decode over the selected pages,
its threshold and its support).  Per sampled unit the checks are those of
tests/gpu_helpers.py: the selection within the tie band (top-k: pages within
1e-5 relative of the k-th score; Gaussian: margins within 1e-5 of zero), τ
within 1e-5, support bits exact outside |u − τ| < 1e-5, output rows within
2e-3 max relative error (bf16 caches).  Top-k is also exact on the GPU's own
page scores for every unit (integer work on the same keys).

The inputs are the benchmark's own (same generator, same sizes); each
workload is drawn once and shared by its tests."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.engine import DecodeEngine
from sparse_kv_cache_kmax_b200.workloads import WORKLOADS, gauss_cap

from gpu_helpers import (REL_TIE, assert_sel_matches, check_unit_decode, gen, np64, oracle_unit,
                         row_rel_err, topk_tie_band)

pytestmark = pytest.mark.gpu

# (workload, policy, alpha, budget): the benchmark's headline line, its other
# alphas, the Gaussian policy and the full-cache decode, and every other
# workload's own line
CASES = [
    ("clustered_128k", "topk", 1.5, 256),
    ("clustered_128k", "topk", 1.25, 256),
    ("clustered_128k", "topk", 2.0, 256),
    ("clustered_128k", "gauss", 1.5, 0.5),
    ("clustered_128k", "full", 1.5, None),
    ("gqa_32k", "topk", 1.5, 64),
    ("short_scattered", "topk", 1.5, 32),
    ("long_512k", "topk", 1.5, 512),
    ("long_512k", "gauss", 1.5, 0.5),
    ("long_512k", "full", 1.5, None),
    ("ctx_1m", "topk", 1.5, 512),
    ("ctx_1m", "gauss", 1.5, 0.5),
    ("ctx_1m", "full", 1.5, None),
]

_CACHE = {}


def _inputs(name):
    """Full-size inputs of one workload (the benchmark's seed); one at a time."""
    if name not in _CACHE:
        _CACHE.clear()
        torch.cuda.empty_cache()
        _CACHE[name] = gen(WORKLOADS[name], 3000)
    return _CACHE[name]


def _sample_units(wl, n):
    units = [(b, h) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    rng = np.random.default_rng(17)
    rest = rng.choice(np.arange(1, len(units)), size=min(n - 1, len(units) - 1), replace=False)
    return [units[0]] + [units[i] for i in sorted(rest)]


@pytest.mark.parametrize("name,policy,alpha,budget", CASES,
                         ids=[f"{c[0]}-{c[1]}-a{c[2]}" for c in CASES])
def test_fullsize_step_matches_oracle_on_sampled_units(name, policy, alpha, budget):
    inp = _inputs(name)
    wl = inp["workload"]
    k = budget if policy == "topk" else None
    delta = budget if policy == "gauss" else None
    full = policy == "full"
    cap = k if policy == "topk" else (inp["max_pages"] if full else gauss_cap(wl, inp["max_pages"]))
    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], wl.num_q_heads,
                       policy=policy, k=k, delta=delta, alpha=alpha, cap=cap)
    eng.build_meta()
    out = eng.step(inp["q"], inp["k_new"][0], inp["v_new"][0]).clone()   # re-appends the stored token
    sel_all, n_all = eng.sel.clone(), eng.n_sel.clone()
    torch.cuda.synchronize()
    assert B.ekv_get_error() == 0

    # the same decode kernel on the step's selection, with the support outputs
    Hq, S = wl.num_q_heads, wl.page_size
    words = (cap * S + 31) // 32
    out_d = torch.full_like(out, float("nan"))
    tau = torch.full((wl.batch, Hq), float("nan"), device="cuda")
    cnt = torch.full((wl.batch, Hq), -1, dtype=torch.int32, device="cuda")
    bits = torch.zeros(wl.batch, Hq, words, dtype=torch.int32, device="cuda")
    ws = B.workspace(B.ekv_workspace_bytes(B.EKV_OP_ENTMAX_DECODE, eng.cache, eng.seqs, Hq, cap), "cuda")
    B.ekv_entmax_decode(eng.cache, eng.seqs, inp["q"], eng.params.scale, alpha, None if full else sel_all,
                        None if full else n_all, cap, out_d, ws, tau=tau, support_count=cnt, support_bits=bits)
    torch.cuda.synchronize()
    assert torch.equal(out_d, out), "the step's decode and the standalone decode differ"
    if full:
        # the dense-V variant: same τ, every V row read, zero weights add nothing
        out_v = torch.full_like(out, float("nan"))
        tau_v = torch.full_like(tau, float("nan"))
        B.ekv_entmax_decode(eng.cache, eng.seqs, inp["q"], eng.params.scale, alpha, None, None, cap, out_v, ws,
                            dense_v=True, tau=tau_v)
        torch.cuda.synchronize()
        assert torch.equal(tau_v, tau)
        assert np.all(row_rel_err(np64(out_v).reshape(-1, wl.head_dim), np64(out_d).reshape(-1, wl.head_dim)) <= 1e-5)

    scale = float(np.float32(wl.scale))
    if policy == "topk":
        # integer work on the GPU's own page scores: exact, every unit
        ub = torch.empty(wl.batch, wl.num_kv_heads, inp["max_pages"], device="cuda")
        B.ekv_score_pages(eng.cache, eng.seqs, inp["q"], scale, ub)
        ub_h = np64(ub)
        sel_h, n_h = sel_all.cpu().numpy(), n_all.cpu().numpy()
        for b in range(wl.batch):
            P = -(-int(inp["seq_lens"][b]) // S)
            for h in range(wl.num_kv_heads):
                want = O.select_topk(ub_h[b, h, :P], k)
                assert int(n_h[b, h]) == min(k, P)
                assert np.array_equal(sel_h[b, h, : n_h[b, h]], want), (b, h)
    elif policy == "gauss":
        tau_hat = torch.zeros(wl.batch, Hq, device="cuda")
        gsel = torch.zeros_like(sel_all)
        gn = torch.zeros_like(n_all)
        gws = B.workspace(B.ekv_workspace_bytes(B.EKV_OP_SELECT_GAUSS, eng.cache, eng.seqs, Hq, cap), "cuda")
        B.ekv_select_gauss(eng.cache, eng.seqs, inp["q"], scale, alpha, delta, cap, gsel, gn, tau_hat, gws)
        torch.cuda.synchronize()
        assert torch.equal(gn, n_all)
        for b in range(wl.batch):
            for h in range(wl.num_kv_heads):
                n = int(gn[b, h])
                assert torch.equal(gsel[b, h, :n], sel_all[b, h, :n]), (b, h)
        assert B.ekv_get_error() == 0, "a Gaussian selection overflowed the cap"

    G = wl.group
    n_units = 8 if wl.units >= 256 else 4
    for b, h in _sample_units(wl, n_units):
        if full:
            orc = oracle_unit(inp, b, h, policy="all", alpha=alpha)
            check_unit_decode(orc, out_d, tau, cnt, bits, b, h, G, wl.dtype,
                              what=f"{name} full cache alpha {alpha} unit {(b, h)}")
            continue
        got = sel_all[b, h, : int(n_all[b, h])].cpu().numpy()
        orc = oracle_unit(inp, b, h, policy=policy, k=k, delta=delta, alpha=alpha)
        if policy == "topk":
            assert_sel_matches(got, orc["sel"], topk_tie_band(orc["score"], k), f"unit {(b, h)}")
        else:
            gs = orc["gauss"]
            t_hat = np64(tau_hat[b, h * G:(h + 1) * G])
            assert np.allclose(t_hat, gs["tau_hat"], rtol=1e-5, atol=1e-5), (b, h, t_hat, gs["tau_hat"])
            margin = gs["margin"]
            band = REL_TIE * np.maximum(1.0, np.abs(gs["tau_hat"] - delta))[:, None]
            sure_in = np.nonzero(np.any(margin > band, axis=0))[0]
            sure_out = np.nonzero(np.all(margin < -band, axis=0))[0]
            if sure_in.size:
                assert set(sure_in.tolist()) <= set(got.tolist()), (b, h)
                assert not (set(got.tolist()) & set(sure_out.tolist())), (b, h)
        if not np.array_equal(got, orc["sel"]):
            orc = oracle_unit(inp, b, h, alpha=alpha, sel=got)
        check_unit_decode(orc, out_d, tau, cnt, bits, b, h, G, wl.dtype,
                          what=f"{name} {policy} alpha {alpha} unit {(b, h)}")
