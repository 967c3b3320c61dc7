"""GPU exactness certificate ([EntmaxKV] §3 "Récupération du Support"):
against the oracle's certificate on the same selection, certified heads equal
the full-cache decode, and the adaptive budget ends at the full-cache output."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.engine import DecodeEngine
from sparse_kv_cache_kmax_b200.workloads import scaled_down

from gpu_helpers import OUT_TOL, Gpu, gen, np64, oracle_unit, row_rel_err

pytestmark = pytest.mark.gpu

CASES = {
    "clustered_128k": dict(batch=2, context=3005),
    "gqa_32k": dict(batch=2, context=1500),
    "long_512k": dict(batch=1, context=4007),
}


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    wl = scaled_down(request.param, **CASES[request.param])
    inp = gen(wl, 4000 + list(CASES).index(request.param))
    gpu = Gpu(inp)
    gpu.build_meta()
    return wl, inp, gpu


@pytest.mark.parametrize("k", [4, 16])
def test_certificate_matches_oracle_and_certified_heads_are_exact(case, k):
    wl, inp, gpu = case
    alpha = 1.5
    ub = gpu.score()
    sel, n = gpu.topk(ub, k)
    out, tau, _, _ = gpu.decode(alpha, sel, n, k)
    cert = torch.full((wl.batch, gpu.Hq), -1, dtype=torch.int32, device="cuda")
    B.ekv_exactness_certificate(gpu.seqs, wl.num_kv_heads, wl.page_size, alpha, ub, sel, n, tau, cert)
    full, _, _, _ = gpu.decode(alpha)
    torch.cuda.synchronize()
    G = wl.group
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            got_sel = sel[b, h, : int(n[b, h])].cpu().numpy()
            orc = oracle_unit(inp, b, h, sel=got_sel, alpha=alpha)
            want = O.exactness_certificate(orc["score"], got_sel, orc["tau"], alpha)
            rest = np.setdiff1d(np.arange(orc["score"].size), got_sel)
            edge = (alpha - 1) * orc["score"][rest].max() if rest.size else -np.inf
            for g in range(G):
                hq = h * G + g
                c = int(cert[b, hq])
                assert c in (0, 1)
                if abs(edge - orc["tau"][g]) > 1e-5 * max(1.0, abs(orc["tau"][g])):
                    assert c == int(want[g]), (b, hq, edge, orc["tau"][g])
                if c:
                    err = row_rel_err(np64(out[b, hq]), np64(full[b, hq]))
                    assert err <= 2 * OUT_TOL[wl.dtype], (b, hq, err)


def test_selection_of_every_page_is_certified(case):
    wl, inp, gpu = case
    k = inp["max_pages"]
    ub = gpu.score()
    sel, n = gpu.topk(ub, k)
    _, tau, _, _ = gpu.decode(1.5, sel, n, k)
    cert = torch.zeros((wl.batch, gpu.Hq), dtype=torch.int32, device="cuda")
    B.ekv_exactness_certificate(gpu.seqs, wl.num_kv_heads, wl.page_size, 1.5, ub, sel, n, tau, cert)
    assert bool((cert == 1).all())


def test_adaptive_budget_ends_certified_at_full_cache_output(case):
    wl, inp, gpu = case
    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], wl.num_q_heads,
                       policy="topk", k=2, alpha=1.5)
    eng.build_meta()
    out, k = eng.decode_adaptive(inp["q"], k0=2)
    torch.cuda.synchronize()
    assert bool(eng._ad["cert"].all()) or k >= inp["max_pages"]
    G = wl.group
    for b in range(wl.batch):
        for h in range(min(wl.num_kv_heads, 3)):
            orc = oracle_unit(inp, b, h, policy="all", alpha=1.5)
            err = row_rel_err(np64(out[b, h * G:(h + 1) * G]), orc["o"])
            assert np.all(err <= OUT_TOL[wl.dtype]), (b, h, err.max(), k)
