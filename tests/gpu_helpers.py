"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the float64 oracle on the same seeded inputs, and compare stage by stage.

Tolerances (written here once, used by every GPU test):
* metadata, selections, support counts: bit-exact / set-exact, except pages
  whose score lies within REL_TIE (1e-5) of the k-th score (top-k), pages whose
  Gaussian margin lies within REL_TIE of zero, and tokens with |u − τ| < 1e-5;
* bounds: |ub − ub₆₄| ≤ 1e-5 · scale · Σ_j |q_j|·max(|kmin_j|, |kmax_j|)
  (fp32 summation of 2·d products);
* outputs: per (sequence, query head) row, max_i |o_i − ô_i| / max(max_i |ô_i|,
  1e-6) ≤ 2e-3 for bf16 caches and ≤ 1e-5 for fp32 caches.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from sparse_kv_cache_kmax_b200 import binding as B
from sparse_kv_cache_kmax_b200.workloads import make_inputs

REL_TIE = 1e-5
TOK_TIE = 1e-5
OUT_TOL = {"bf16": 2e-3, "f32": 1e-5}


def np64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def gen(wl, seed, n_new=1):
    return make_inputs(wl, seed, device="cuda", n_new=n_new)


def unit_arrays(inp, b, h):
    """One unit's pages on the host as float64 (a pool with identity page table)."""
    wl = inp["workload"]
    L = int(inp["seq_lens"][b])
    P = -(-L // wl.page_size)
    ids = inp["page_table"][b, :P].long()
    k = np64(inp["k_pool"][ids, h])[:, None]
    v = np64(inp["v_pool"][ids, h])[:, None]
    return k, v, np.arange(P), L


def q_group(inp, b, h):
    G = inp["workload"].group
    return np64(inp["q"][b, h * G:(h + 1) * G])


def oracle_unit(inp, b, h, *, policy="topk", k=None, delta=None, alpha=1.5, sel=None):
    wl = inp["workload"]
    kp, vp, pt, L = unit_arrays(inp, b, h)
    return O.decode_unit(kp, vp, pt, L, 0, q_group(inp, b, h), page_size=wl.page_size,
                         scale=float(np.float32(wl.scale)), alpha=alpha, dtype=wl.dtype,
                         policy=policy, k=k, delta=delta, sel=sel)


def topk_tie_band(score, k):
    """Pages whose score is within REL_TIE of the k-th largest (ambiguous)."""
    if k >= score.size:
        return np.zeros(score.size, bool)
    kth = np.sort(score)[::-1][k - 1]
    return np.abs(score - kth) <= REL_TIE * max(abs(kth), 1e-30)


def assert_sel_matches(got, want, ambiguous, what=""):
    got, want = set(np.asarray(got).tolist()), set(np.asarray(want).tolist())
    amb = set(np.nonzero(ambiguous)[0].tolist())
    diff = (got ^ want) - amb
    assert not diff, f"{what}: selections differ outside the tie band: {sorted(diff)[:10]}"


def row_rel_err(o, ref):
    return np.max(np.abs(o - ref), axis=-1) / np.maximum(np.max(np.abs(ref), axis=-1), 1e-6)


def support_from_bits(bits_row, n):
    words = np.asarray(bits_row, dtype=np.uint32)
    idx = np.arange(n)
    return ((words[idx // 32] >> (idx % 32).astype(np.uint32)) & 1).astype(bool)


class Gpu:
    """The CUDA path on one workload instance, stage by stage."""

    def __init__(self, inp):
        self.inp = inp
        wl = inp["workload"]
        self.wl = wl
        self.cache = B.make_cache(inp["k_pool"], inp["v_pool"])
        self.seqs = B.make_seqs(inp["page_table"], inp["seq_lens"])
        self.Hq = wl.num_q_heads
        self.scale = float(np.float32(wl.scale))

    def build_meta(self):
        B.ekv_build_page_meta(self.cache, self.seqs)
        return self.cache.box_t, self.cache.mom_t

    def score(self):
        ub = torch.full((self.wl.batch, self.wl.num_kv_heads, self.inp["max_pages"]), float("nan"),
                        device="cuda")
        B.ekv_score_pages(self.cache, self.seqs, self.inp["q"], self.scale, ub)
        return ub

    def topk(self, ub, k):
        sel = torch.full((self.wl.batch, self.wl.num_kv_heads, k), -1, dtype=torch.int32, device="cuda")
        n = torch.zeros(self.wl.batch, self.wl.num_kv_heads, dtype=torch.int32, device="cuda")
        n_tk = B.ekv_workspace_bytes(B.EKV_OP_SELECT_TOPK, self.cache, self.seqs, self.Hq, k)
        ws = B.workspace(n_tk, "cuda") if n_tk else None
        B.ekv_select_topk(self.seqs, self.wl.num_kv_heads, self.wl.page_size, ub, k, sel, n, ws=ws)
        return sel, n

    def gauss(self, alpha, delta, cap=None):
        cap = cap or self.inp["max_pages"]
        sel = torch.full((self.wl.batch, self.wl.num_kv_heads, cap), -1, dtype=torch.int32, device="cuda")
        n = torch.zeros(self.wl.batch, self.wl.num_kv_heads, dtype=torch.int32, device="cuda")
        tau_hat = torch.zeros(self.wl.batch, self.Hq, device="cuda")
        ws = B.workspace(B.ekv_workspace_bytes(B.EKV_OP_SELECT_GAUSS, self.cache, self.seqs, self.Hq, cap), "cuda")
        B.ekv_select_gauss(self.cache, self.seqs, self.inp["q"], self.scale, alpha, delta, cap, sel, n,
                           tau_hat, ws)
        return sel, n, tau_hat

    def decode(self, alpha, sel=None, n_sel=None, cap=None, dense_v=False):
        wl = self.wl
        if sel is None:
            cap = self.inp["max_pages"]
        cap = cap or sel.shape[-1]
        out = torch.full((wl.batch, self.Hq, wl.head_dim), float("nan"), device="cuda")
        tau = torch.full((wl.batch, self.Hq), float("nan"), device="cuda")
        cnt = torch.full((wl.batch, self.Hq), -1, dtype=torch.int32, device="cuda")
        words = (cap * wl.page_size + 31) // 32
        bits = torch.zeros(wl.batch, self.Hq, words, dtype=torch.int32, device="cuda")
        ws = B.workspace(B.ekv_workspace_bytes(B.EKV_OP_ENTMAX_DECODE, self.cache, self.seqs, self.Hq, cap), "cuda")
        B.ekv_entmax_decode(self.cache, self.seqs, self.inp["q"], self.scale, alpha, sel, n_sel, cap, out, ws,
                            dense_v=dense_v, tau=tau, support_count=cnt, support_bits=bits)
        return out, tau, cnt, bits


def sel_tensor(sels, batch, hkv, cap):
    """Pack per-unit host selections into the [B, Hkv, cap] / [B, Hkv] layout."""
    sel = torch.full((batch, hkv, cap), -1, dtype=torch.int32)
    n = torch.zeros(batch, hkv, dtype=torch.int32)
    for (b, h), s in sels.items():
        sel[b, h, : len(s)] = torch.as_tensor(np.asarray(s), dtype=torch.int32)
        n[b, h] = len(s)
    return sel.cuda(), n.cuda()


def check_unit_decode(orc, out, tau, cnt, bits, b, h, G, dtype, *, what=""):
    """Compare one unit's decode outputs with an oracle decode_unit result."""
    rows = slice(h * G, (h + 1) * G)
    o = np64(out[b, rows])
    err = row_rel_err(o, orc["o"])
    assert np.all(err <= OUT_TOL[dtype]), f"{what}: output rel err {err.max():.3e}"
    t = np64(tau[b, rows])
    assert np.allclose(t, orc["tau"], rtol=1e-5, atol=1e-5), f"{what}: tau {t} vs {orc['tau']}"
    n = orc["u"].shape[1]
    bits_np = bits[b, rows].cpu().numpy().view(np.uint32)
    for g in range(G):
        sup = support_from_bits(bits_np[g], n)
        want = orc["p"][g] > 0
        clear = np.abs(orc["u"][g] - orc["tau"][g]) >= TOK_TIE
        assert np.array_equal(sup[clear], want[clear]), f"{what}: support of head {g} differs"
        amb = int((~clear).sum())
        assert abs(int(cnt[b, h * G + g]) - int(want.sum())) <= amb, f"{what}: support count"
