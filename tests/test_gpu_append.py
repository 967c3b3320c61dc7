"""The cache append of a decode step with a token that is not already stored,
against the float64 oracle: "Résumé Technique : EntmaxKV" §2.A — the cache
grows one token per step and the metadata of the page that receives it
(bounding box, mean, variance) is kept current.

Each case grows every sequence by one token whose position falls on a
different kind of slot (slot 0 of a fresh page, a mid-page slot, the last
slot of a page), on contiguous and on scattered page tables, bf16 and fp32.
The K/V pools after ``ekv_append`` must equal the oracle's ``append_token``
on host copies byte for byte; the touched pages' box/mom rows must equal
``page_metadata`` over the page's valid tokens bit for bit; every other
metadata row must be unchanged.  The whole step with the append
(``ekv_decode_step``, append = 1) is then compared with the oracle's decode
of the grown cache."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.engine import DecodeEngine
from sparse_kv_cache_kmax_b200.workloads import scaled_down

from gpu_helpers import OUT_TOL, assert_sel_matches, gen, np64, oracle_unit, row_rel_err, topk_tie_band

pytestmark = pytest.mark.gpu


def _bits(t):
    t = t.contiguous()
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).cpu().numpy()


def _grown_lengths(lens, S, P_alloc):
    """New lengths (counting the appended token) whose positions L−1 cycle
    through slot 0 of a fresh page, a mid-page slot and the last slot, all
    inside the pages each sequence has."""
    out = []
    for b, L in enumerate(lens):
        cap = P_alloc[b] * S
        kind = b % 3
        base = (min(L, cap) - 1) // S * S          # first token of the last allocated page
        if kind == 0:
            new = base + 1                        # slot 0 (a fresh page)
        elif kind == 1:
            new = base + S // 2 + 1               # slot S/2
        else:
            new = base                            # slot S−1 of the previous page
        out.append(max(2, min(new, cap)))
    return out


CASES = {
    "bf16_contiguous": ("clustered_128k", dict(batch=3, context=3005)),
    "f32_contiguous": ("tiny_fp32", dict(batch=3, context=777)),
    "bf16_scattered": ("short_scattered", dict(batch=6, context=900, context_min=300)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_append_new_token_matches_oracle(case):
    name, over = CASES[case]
    wl = scaled_down(name, **over)
    inp = gen(wl, 5100 + list(CASES).index(case), n_new=2)
    S, Hkv = wl.page_size, wl.num_kv_heads
    lens0 = inp["seq_lens"].tolist()
    P_alloc = [-(-L // S) for L in lens0]
    lens_new = _grown_lengths(lens0, S, P_alloc)
    slots = [(L - 1) % S for L in lens_new]
    assert {0, S // 2, S - 1} <= set(slots), slots

    # metadata of the cache before the append (lengths L − 1)
    inp["seq_lens"].copy_(torch.tensor([L - 1 for L in lens_new], dtype=torch.int32))
    cache = B.make_cache(inp["k_pool"], inp["v_pool"])
    seqs = B.make_seqs(inp["page_table"], inp["seq_lens"])
    B.ekv_build_page_meta(cache, seqs)
    torch.cuda.synchronize()
    box0, mom0 = cache.box_t.clone(), cache.mom_t.clone()
    k_host = np64(inp["k_pool"])
    v_host = np64(inp["v_pool"])

    # the append of a fresh token (variant 1: not the stored one)
    inp["seq_lens"].copy_(torch.tensor(lens_new, dtype=torch.int32))
    k_new, v_new = inp["k_new"][1], inp["v_new"][1]
    B.ekv_append(cache, seqs, k_new, v_new)
    torch.cuda.synchronize()
    assert B.ekv_get_error() == 0
    pt = inp["page_table"].cpu().numpy()
    touched = O.append_token(k_host, v_host, pt, lens_new, np64(k_new), np64(v_new), S)
    assert np.array_equal(np64(inp["k_pool"]), k_host)
    assert np.array_equal(np64(inp["v_pool"]), v_host)

    box, mom = cache.box_t, cache.mom_t
    tdt = box.dtype
    rows = set()
    for b, phys, n_valid in touched:
        assert n_valid == slots[b] + 1
        rows.add(phys)
        for h in range(Hkv):
            meta = O.page_metadata(k_host[phys, h][None], [n_valid], wl.dtype)
            want_box = torch.from_numpy(np.stack([meta["kmax"][0], meta["kmin"][0]])).to(tdt)
            want_mom = torch.from_numpy(np.stack([meta["mean"][0], meta["var"][0]])).to(tdt)
            assert np.array_equal(_bits(box[h, phys]), _bits(want_box)), (b, phys, h, "box")
            assert np.array_equal(_bits(mom[h, phys]), _bits(want_mom)), (b, phys, h, "mom")
    keep = torch.tensor(sorted(set(range(inp["num_phys"])) - rows), dtype=torch.long, device="cuda")
    assert torch.equal(_t(box[:, keep]), _t(box0[:, keep]))
    assert torch.equal(_t(mom[:, keep]), _t(mom0[:, keep]))


def _t(x):
    return x.contiguous().view(torch.int16 if x.dtype == torch.bfloat16 else torch.int32)


@pytest.mark.parametrize("case", ["bf16_contiguous", "bf16_scattered"])
def test_decode_step_with_append_of_a_new_token(case):
    """ekv_decode_step(append = 1) on a grown cache: its output for the new
    token's query equals the oracle's decode of the cache with that token."""
    name, over = CASES[case]
    wl = scaled_down(name, **over)
    inp = gen(wl, 5200 + list(CASES).index(case), n_new=2)
    S = wl.page_size
    lens0 = inp["seq_lens"].tolist()
    lens_new = _grown_lengths(lens0, S, [-(-L // S) for L in lens0])
    inp["seq_lens"].copy_(torch.tensor([L - 1 for L in lens_new], dtype=torch.int32))
    k = 12
    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], wl.num_q_heads,
                       policy="topk", k=k, alpha=1.5)
    eng.build_meta()
    inp["seq_lens"].copy_(torch.tensor(lens_new, dtype=torch.int32))
    out = eng.step(inp["q"], inp["k_new"][1], inp["v_new"][1]).clone()
    torch.cuda.synchronize()
    assert B.ekv_get_error() == 0
    G = wl.group
    for b in range(wl.batch):
        for h in (0, wl.num_kv_heads - 1):
            orc = oracle_unit(inp, b, h, policy="topk", k=k)        # reads the grown pools
            got = eng.sel[b, h, : int(eng.n_sel[b, h])].cpu().numpy()
            assert_sel_matches(got, orc["sel"], topk_tie_band(orc["score"], k), f"unit {(b, h)}")
            if not np.array_equal(got, orc["sel"]):
                orc = oracle_unit(inp, b, h, sel=got)
            err = row_rel_err(np64(out[b, h * G:(h + 1) * G]), orc["o"])
            assert np.all(err <= OUT_TOL[wl.dtype]), (b, h, err.max())
            # the new token takes part: it is in the selected pages' token list
            last_page = (lens_new[b] - 1) // S
            if last_page in set(got.tolist()):
                assert orc["token_page"][-1] == last_page
