"""Top-k over sequences longer than one CTA holds in registers (16384 pages): the
two-stage selection (chunks keep their k best, then k among those) against the
one-stage kernel and the oracle's rule on the same scores ([EntmaxKV] §2.B)."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmax_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("k,dup", [(512, False), (100, True), (2000, False)])
def test_two_stage_topk_matches_one_stage_and_oracle(k, dup):
    g = torch.Generator(device="cuda").manual_seed(77 + k)
    batch, hkv, S, P = 2, 3, 16, 19000
    lens = torch.tensor([P * S, (P - 777) * S - 5], dtype=torch.int32, device="cuda")
    pt = torch.arange(batch * P, dtype=torch.int32, device="cuda").view(batch, P)
    seqs = B.make_seqs(pt, lens)
    ub = torch.randn(batch, hkv, P, generator=g, device="cuda")
    if dup:  # heavy ties: scores on a coarse grid
        ub = torch.round(ub * 4) / 4
    kv = torch.empty(1, hkv, S, 128, dtype=torch.bfloat16, device="cuda")
    cache = B.make_cache(kv, kv)
    cache.num_phys_pages = batch * P
    need = B.ekv_workspace_bytes(B.EKV_OP_SELECT_TOPK, cache, seqs, 4 * hkv, k)
    assert need > 0
    ws = B.workspace(need, "cuda")
    s2 = torch.full((batch, hkv, k), -1, dtype=torch.int32, device="cuda")
    n2 = torch.zeros(batch, hkv, dtype=torch.int32, device="cuda")
    B.ekv_select_topk(seqs, hkv, S, ub, k, s2, n2, ws=ws)
    s1 = torch.full_like(s2, -1)
    n1 = torch.zeros_like(n2)
    B.ekv_select_topk(seqs, hkv, S, ub, k, s1, n1)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2) and torch.equal(n1, n2)
    ubh = ub.double().cpu().numpy()
    for b in range(batch):
        pages = -(-int(lens[b]) // S)
        for h in range(hkv):
            want = O.select_topk(ubh[b, h, :pages], k)
            assert int(n2[b, h]) == len(want)
            assert np.array_equal(s2[b, h, : len(want)].cpu().numpy(), want), (b, h)


@pytest.mark.parametrize("dup", [False, True])
def test_one_stage_topk_lengths(dup):
    """One CTA per unit at lengths on both sides of 8 and 16 keys per thread,
    rows not 16-byte aligned (odd row pitch), k from 1 to P − 1."""
    g = torch.Generator(device="cuda").manual_seed(5 + dup)
    pages = [5, 300, 8191, 8192, 8193, 12345, 16383]
    batch, hkv, S, maxp = len(pages), 2, 16, 16383
    lens = torch.tensor([p * S - 3 for p in pages], dtype=torch.int32, device="cuda")
    pt = torch.arange(batch * maxp, dtype=torch.int32, device="cuda").view(batch, maxp)
    seqs = B.make_seqs(pt, lens)
    ub = torch.randn(batch, hkv, maxp, generator=g, device="cuda")
    if dup:
        ub = torch.round(ub * 4) / 4
    ubh = ub.double().cpu().numpy()
    for k in (1, 256, 4000):
        sel = torch.full((batch, hkv, k), -1, dtype=torch.int32, device="cuda")
        n = torch.zeros(batch, hkv, dtype=torch.int32, device="cuda")
        B.ekv_select_topk(seqs, hkv, S, ub, k, sel, n)
        torch.cuda.synchronize()
        for b, P in enumerate(pages):
            for h in range(hkv):
                want = O.select_topk(ubh[b, h, :P], k)
                assert int(n[b, h]) == len(want) == min(k, P)
                assert np.array_equal(sel[b, h, : len(want)].cpu().numpy(), want), (k, b, h)
    # k = P − 1 on the longest unit
    k = pages[-1] - 1
    sel = torch.full((batch, hkv, k), -1, dtype=torch.int32, device="cuda")
    n = torch.zeros(batch, hkv, dtype=torch.int32, device="cuda")
    B.ekv_select_topk(seqs, hkv, S, ub, k, sel, n)
    torch.cuda.synchronize()
    for h in range(hkv):
        want = O.select_topk(ubh[-1, h, : pages[-1]], k)
        assert np.array_equal(sel[-1, h, :k].cpu().numpy(), want)
