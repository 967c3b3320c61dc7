"""Seeded synthetic decode workloads shaped like the EntmaxKV long-context runs.

This module only draws inputs: paged K/V pools, page tables, sequence lengths
and decode queries.  It holds none of the method's arithmetic, so both the
CUDA path and the float64 oracle can consume its tensors.

The source page ("Résumé Technique : EntmaxKV ...", gist.science/fr/paper/
2605.21649, §4) evaluates on RULER, passkey retrieval and PG19 with 1B-param
models, up to 100k–1M tokens of context.  Neither the data nor the weights are
available, so these synthetic caches stand in for them: planted high-score
tokens play the role of the passkey / needle, clustered pages the role of
locally coherent text, heavy-tailed coordinate scales the role of outlier
key channels.

Layouts (all row-major):
    k_pool, v_pool  [num_phys, Hkv, S, d]   (bf16 or fp32)
    page_table      [B, max_pages] int32    (logical page → physical page)
    seq_lens        [B] int32               (tokens, including the new one)
    q               [B, Hq, d]              (same dtype as the cache)
    k_new, v_new    [B, Hkv, d]             (the token at position L_b − 1)
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "scaled_down"]


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    context: int                 # tokens per sequence (upper end if ranged)
    page_size: int
    dtype: str                   # 'bf16' | 'f32'
    key_model: str               # 'planted' | 'aligned' | 'clustered' | 'heavy_tail'
    context_min: int = 0         # > 0: lengths uniform in [context_min, context]
    scattered: bool = False      # physical pages randomly permuted in a shared pool
    planted_count: int = 0       # 'planted' / 'heavy_tail': tokens per (sequence, KV head)
    planted_fraction: float = 0.0  # 'aligned': fraction of each sequence's tokens
    alphas: tuple = (1.5,)
    topk: int = 0
    delta: float | None = None

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def max_pages(self) -> int:
        return -(-self.context // self.page_size)

    @property
    def units(self) -> int:
        return self.batch * self.num_kv_heads


WORKLOADS = {
    # tiny single head, fp32, 8 planted tokens near 3·q/|q|
    "tiny_fp32": Workload("tiny_fp32", 1, 1, 1, 64, 4096, 16, "f32", "planted",
                          planted_count=8, alphas=(1.5,), topk=32),
    # GQA decode at 32k, 1% of tokens aligned with the group's queries
    "gqa_32k": Workload("gqa_32k", 8, 32, 8, 128, 32768, 16, "bf16", "aligned",
                        planted_fraction=0.01, alphas=(1.5,), topk=64),
    # clustered long context at 128k: page means N(0,1), within-page N(0, 0.3²)
    "clustered_128k": Workload("clustered_128k", 4, 32, 8, 128, 131072, 16, "bf16", "clustered",
                               alphas=(1.5, 1.25, 2.0), topk=256, delta=0.5),
    # many short sequences on a scattered shared pool
    "short_scattered": Workload("short_scattered", 64, 32, 8, 128, 16384, 16, "bf16", "aligned",
                                context_min=4096, scattered=True, planted_fraction=0.005,
                                alphas=(1.5,), topk=32),
    # one 512k sequence, page size 32, heavy-tailed key channels and 16 needles
    "long_512k": Workload("long_512k", 1, 64, 8, 128, 524288, 32, "bf16", "heavy_tail",
                          planted_count=16, alphas=(1.5,), topk=512, delta=0.5),
    # one 1M sequence (the page's measured context length), both policies
    "ctx_1m": Workload("ctx_1m", 1, 32, 8, 128, 1048576, 16, "bf16", "clustered",
                       alphas=(1.5,), topk=512, delta=0.5),
}


def scaled_down(name: str, **overrides) -> Workload:
    """A workload of the same family with some fields replaced (test sizes)."""
    return dataclasses.replace(WORKLOADS[name], **overrides)


def _torch_dtype(dtype: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def _unit(x, dim=-1):
    return x / x.norm(dim=dim, keepdim=True)


def make_inputs(wl: Workload, seed: int, device="cpu", n_new: int = 1) -> dict:
    """Draw one workload instance from a seeded generator on ``device``.

    Values are drawn in fp32 and rounded once to the cache dtype.  ``n_new``
    extra variants of the newest token are drawn for repeated append steps
    (variant 0 is the token stored at position L_b − 1).
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    B, Hq, Hkv, d, S = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.page_size
    G = Hq // Hkv
    f32 = dict(device=device, dtype=torch.float32)

    if wl.context_min > 0:
        lens = torch.randint(wl.context_min, wl.context + 1, (B,), generator=g, device=device)
    else:
        lens = torch.full((B,), wl.context, device=device, dtype=torch.int64)
    lens_list = [int(x) for x in lens.tolist()]
    n_pages = [-(-L // S) for L in lens_list]
    max_pages = max(n_pages)
    Lmax = max_pages * S

    q = torch.randn(B, Hq, d, generator=g, **f32)
    q_mean_dir = _unit(q.view(B, Hkv, G, d).mean(dim=2))        # [B, Hkv, d]

    if wl.key_model == "clustered":
        page_mu = torch.randn(B, Hkv, max_pages, 1, d, generator=g, **f32)
        keys = page_mu + 0.3 * torch.randn(B, Hkv, max_pages, S, d, generator=g, **f32)
        keys = keys.view(B, Hkv, Lmax, d)
        del page_mu
    elif wl.key_model == "heavy_tail":
        chan = torch.exp(torch.randn(B, Hkv, 1, d, generator=g, **f32))
        keys = chan * torch.randn(B, Hkv, Lmax, d, generator=g, **f32)
    else:
        keys = torch.randn(B, Hkv, Lmax, d, generator=g, **f32)
    values = torch.randn(B, Hkv, Lmax, d, generator=g, **f32)

    # planted tokens: positions drawn per (sequence, KV head) among valid tokens
    for b in range(B):
        L = lens_list[b]
        if wl.key_model == "planted":
            count = wl.planted_count
        elif wl.key_model == "aligned":
            count = max(1, int(round(wl.planted_fraction * L)))
        elif wl.key_model == "heavy_tail":
            count = wl.planted_count
        else:
            count = 0
        if count == 0:
            continue
        for h in range(Hkv):
            pos = torch.randperm(L, generator=g, device=device)[:count]
            qbar = q_mean_dir[b, h]
            if wl.key_model == "planted":
                # keys = 3·q/|q| + N(0, 0.1²) per coordinate
                planted = 3.0 * qbar + 0.1 * torch.randn(count, d, generator=g, **f32)
            elif wl.key_model == "aligned":
                # cosine 0.8 with the group's mean query direction, norm √d
                w = torch.randn(count, d, generator=g, **f32)
                w = _unit(w - (w @ qbar)[:, None] * qbar[None])
                planted = math.sqrt(d) * (0.8 * qbar[None] + 0.6 * w)
            else:
                # needle: 6 standard deviations of the ordinary scores along q̄
                spread = torch.sqrt(torch.sum((qbar * chan[b, h, 0]) ** 2))
                planted = (6.0 * spread * qbar)[None].expand(count, d)
            keys[b, h, pos] = planted

    dt = _torch_dtype(wl.dtype)
    # physical pages: contiguous per sequence, or a random permutation of a shared pool
    if wl.scattered:
        num_phys = sum(n_pages)
        perm = torch.randperm(num_phys, generator=g, device=device)
        page_table = torch.zeros(B, max_pages, dtype=torch.int32, device=device)
        offs = 0
        for b in range(B):
            page_table[b, : n_pages[b]] = perm[offs: offs + n_pages[b]].to(torch.int32)
            offs += n_pages[b]
    else:
        num_phys = B * max_pages
        page_table = torch.arange(num_phys, dtype=torch.int32, device=device).view(B, max_pages)

    k_pool = torch.zeros(num_phys, Hkv, S, d, dtype=dt, device=device)
    v_pool = torch.zeros(num_phys, Hkv, S, d, dtype=dt, device=device)
    for b in range(B):
        P = n_pages[b]
        ids = page_table[b, :P].long()
        kb = keys[b, :, : P * S].reshape(Hkv, P, S, d).permute(1, 0, 2, 3)
        vb = values[b, :, : P * S].reshape(Hkv, P, S, d).permute(1, 0, 2, 3)
        tail = lens_list[b] - (P - 1) * S          # valid tokens of the last page
        k_pool[ids] = kb.to(dt)
        v_pool[ids] = vb.to(dt)
        if tail < S:                               # positions past L_b stay zero
            k_pool[ids[-1], :, tail:] = 0
            v_pool[ids[-1], :, tail:] = 0

    last = torch.tensor([L - 1 for L in lens_list], device=device)
    ar = torch.arange(B, device=device)
    k_new = [keys[ar, :, last].to(dt)]
    v_new = [values[ar, :, last].to(dt)]
    for _ in range(1, n_new):
        k_new.append(torch.randn(B, Hkv, d, generator=g, **f32).to(dt))
        v_new.append(torch.randn(B, Hkv, d, generator=g, **f32).to(dt))
    del keys, values

    return {
        "workload": wl,
        "k_pool": k_pool, "v_pool": v_pool,
        "page_table": page_table.contiguous(),
        "seq_lens": torch.tensor(lens_list, dtype=torch.int32, device=device),
        "q": q.to(dt).contiguous(),
        "k_new": k_new, "v_new": v_new,
        "max_pages": max_pages, "num_phys": num_phys,
        "scale": wl.scale,
    }


def gauss_cap(wl: Workload, max_pages: int) -> int:
    """Pages a unit may keep under the Gaussian policy (the ``cap`` of
    ekv_select_gauss / ekv_decode_step, which sizes the selection buffer and
    the decode's scratch): every page of the sequence, at most 65536 tokens'
    worth (4096 pages of 16 tokens, 2048 of 32).  A selection past the cap keeps its
    first cap pages and raises EKV_EFLAG_SEL_OVERFLOW, which the tests check
    is never raised on these workloads."""
    return int(min(max_pages, 65536 // wl.page_size))
