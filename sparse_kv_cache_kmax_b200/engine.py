"""A decode session over one paged cache: owns the metadata pools, the
selection / output buffers and the device workspace, and runs whole decode
steps through ``ekv_decode_step`` (one C-ABI call per step)."""
from __future__ import annotations

import math

import torch

from . import binding as B


class DecodeEngine:
    def __init__(self, k_pool, v_pool, page_table, seq_lens, num_q_heads, *, policy="topk", k=None,
                 delta=None, alpha=1.5, scale=None, cap=None, dense_v=False):
        self.cache = B.make_cache(k_pool, v_pool)
        self.seqs = B.make_seqs(page_table, seq_lens)
        self.device = k_pool.device
        self.Hq = int(num_q_heads)
        self.Hkv = int(k_pool.shape[1])
        self.d = int(k_pool.shape[3])
        self.S = int(k_pool.shape[2])
        self.batch = int(page_table.shape[0])
        self.max_pages = int(page_table.shape[1])
        pol = {"topk": B.EKV_POLICY_TOPK, "gauss": B.EKV_POLICY_GAUSS, "full": B.EKV_POLICY_FULL}[policy]
        if cap is None:
            cap = int(k) if policy == "topk" else self.max_pages
        self.cap = self.max_pages if policy == "full" else int(cap)
        self.params = B.StepParams(pol, int(k or 0), float(delta if delta is not None else 0.0), self.cap,
                                   float(alpha), float(scale if scale is not None else 1.0 / math.sqrt(self.d)),
                                   int(bool(dense_v)), 1)
        dev = self.device
        self.sel = torch.zeros(self.batch, self.Hkv, self.cap, dtype=torch.int32, device=dev)
        self.n_sel = torch.zeros(self.batch, self.Hkv, dtype=torch.int32, device=dev)
        self.out = torch.zeros(self.batch, self.Hq, self.d, dtype=torch.float32, device=dev)
        self.tau = torch.zeros(self.batch, self.Hq, dtype=torch.float32, device=dev)
        nbytes = B.ekv_workspace_bytes(B.EKV_OP_DECODE_STEP, self.cache, self.seqs, self.Hq, self.cap)
        if nbytes == 0:
            raise ValueError("invalid decode configuration")
        self.ws = B.workspace(nbytes, dev)

    @property
    def box(self):
        return self.cache.box_t

    @property
    def mom(self):
        return self.cache.mom_t

    def build_meta(self, stream=None):
        B.ekv_build_page_meta(self.cache, self.seqs, stream)

    def step(self, q, k_new=None, v_new=None, stream=None):
        """One decode step; appends (k_new, v_new) first when given."""
        self.params.append = int(k_new is not None)
        B.ekv_decode_step(self.cache, self.seqs, self.params, q, k_new, v_new, self.sel, self.n_sel,
                          self.out, self.ws, tau=self.tau, stream=stream)
        return self.out

    def decode_adaptive(self, q, k_new=None, v_new=None, k0=None, stream=None):
        """Top-k decode whose budget doubles until every query head is
        certified exact (one ekv_decode_adaptive call: no unselected page can
        hold support, so the output is the full-cache one).  Appends first
        when k_new is given.  Returns (out [B, Hq, d], k used)."""
        Bsz, Hkv, P = self.batch, self.Hkv, self.max_pages
        dev = self.device
        if not hasattr(self, "_ad"):
            ws = B.workspace(B.ekv_workspace_bytes(B.EKV_OP_DECODE_ADAPTIVE, self.cache, self.seqs, self.Hq, P), dev)
            self._ad = dict(sel=torch.empty(Bsz * Hkv * P, dtype=torch.int32, device=dev),
                            n=torch.zeros(Bsz, Hkv, dtype=torch.int32, device=dev),
                            out=torch.zeros(Bsz, self.Hq, self.d, device=dev),
                            tau=torch.zeros(Bsz, self.Hq, device=dev),
                            cert=torch.zeros(Bsz, self.Hq, dtype=torch.int32, device=dev), ws=ws)
        a = self._ad
        if k_new is not None:
            B.ekv_append(self.cache, self.seqs, k_new, v_new, stream)
        k = B.ekv_decode_adaptive(self.cache, self.seqs, q, self.params.scale, self.params.alpha,
                                  max(1, min(int(k0 or self.params.k or 1), P)), a["sel"], a["n"], a["out"],
                                  a["tau"], a["cert"], a["ws"], stream)
        return a["out"], k
