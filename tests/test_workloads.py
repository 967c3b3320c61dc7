"""Seeded input generators: determinism, layout and planted structure (CPU)."""
import torch

from sparse_kv_cache_kmax_b200.workloads import WORKLOADS, make_inputs, scaled_down


def _small(name):
    return scaled_down(name, batch=3, context=700, context_min=300 if WORKLOADS[name].context_min else 0)


def test_deterministic_and_layout():
    for name in WORKLOADS:
        wl = _small(name)
        a, b = make_inputs(wl, 5), make_inputs(wl, 5)
        for key in ("k_pool", "v_pool", "page_table", "seq_lens", "q"):
            assert torch.equal(a[key], b[key]), (name, key)
        c = make_inputs(wl, 6)
        assert not torch.equal(a["k_pool"], c["k_pool"])
        S, d = wl.page_size, wl.head_dim
        assert a["k_pool"].shape[1:] == (wl.num_kv_heads, S, d)
        assert a["q"].shape == (wl.batch, wl.num_q_heads, d)
        # every sequence's pages are distinct physical pages inside the pool
        used = []
        for bi, L in enumerate(a["seq_lens"].tolist()):
            P = -(-L // S)
            used += a["page_table"][bi, :P].tolist()
        assert len(set(used)) == len(used) and max(used) < a["num_phys"]
        # the new token equals the stored token at position L - 1
        for bi, L in enumerate(a["seq_lens"].tolist()):
            phys = int(a["page_table"][bi, (L - 1) // S])
            assert torch.equal(a["k_pool"][phys, :, (L - 1) % S], a["k_new"][0][bi])
            assert torch.equal(a["v_pool"][phys, :, (L - 1) % S], a["v_new"][0][bi])


def test_scattered_pool_is_permuted_and_lengths_ranged():
    wl = scaled_down("short_scattered", batch=8, context=900, context_min=400)
    a = make_inputs(wl, 1)
    lens = a["seq_lens"].tolist()
    assert min(lens) >= 400 and max(lens) <= 900 and len(set(lens)) > 1
    first = a["page_table"][:, 0].tolist()
    assert first != sorted(first)


def test_planted_tokens_score_high():
    wl = _small("gqa_32k")
    a = make_inputs(wl, 3)
    q = a["q"].float().view(wl.batch, wl.num_kv_heads, wl.group, -1).mean(2)
    S = wl.page_size
    L = int(a["seq_lens"][0])
    P = -(-L // S)
    K = a["k_pool"][a["page_table"][0, :P].long(), 0].float().reshape(P * S, -1)[:L]
    cos = torch.nn.functional.cosine_similarity(K, q[0, 0][None], dim=1)
    assert int((cos > 0.75).sum()) == max(1, round(0.01 * L))
