"""Float64 CPU oracle of the EntmaxKV support-aware paged decode step.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or runs anything here, and this file shares no code, table or
helper with it: the two meet only on the seeded input bytes.

Every quantity is computed in float64 from the *stored* values (bf16 / fp32
widened exactly).  Functions cite the passage of the source page they follow:

    "Résumé Technique : EntmaxKV – Décodage Conscient du Support pour
    l'Attention Entmax" (gist.science/fr/paper/2605.21649), cited below as
    [EntmaxKV] with its section.

The page prints no formula.  Where it is silent the plainest reading is taken;
each reading is named in the function that makes it:

* α-entmax: p_i = [(α−1)z_i − τ]_+^{1/(α−1)}, τ such that Σp = 1, with
  z_i = scale·q·k_i (the standard α-entmax of Peters, Niculae & Martins 2019).
* metadata: coordinate-wise max/min over a page's valid tokens; mean and
  *population* variance accumulated in float64 in token order, each rounded
  once (round-to-nearest-even) to the storage dtype.
* bounding-box bound per query head ub = scale·Σ_j max(q_j·kmin_j, q_j·kmax_j);
  a KV head's page score is the max over the query heads of its GQA group.
* top-k: the k highest page scores, ties to the lower logical page index,
  all pages when P ≤ k, returned in ascending page order.
* Gaussian-aware policy: token scores of page p are N(m_p, s_p²) with
  m_p = scale·q·μ_p, s_p² = scale²·Σ_j q_j² σ²_pj (independent coordinates);
  τ̂ solves Σ_p n_p·E[((α−1)z − τ̂)_+^β] = 1 (β = 1/(α−1), an integer);
  page p is kept when (α−1)·(m_p + s_p·√(2 ln n_p)) > τ̂ − Δ for any query
  head of the group; if none passes, the single page with the largest margin.

Parity status of each function is pinned by tests under ``tests/`` (closed
forms, brute force, quadrature, invariants); none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import ndtr

__all__ = [
    "round_bf16", "round_to", "page_metadata", "bbox_upper_bound",
    "page_scores", "select_topk", "gauss_truncated_power_mean",
    "gauss_tau_hat", "select_gauss", "entmax_threshold", "entmax_probs",
    "entmax_attention", "softmax_attention", "softmax_dropped_mass", "unit_pages", "decode_unit",
    "build_page_meta", "append_token", "ENTMAX_SORT_ALPHAS",
    "exactness_certificate", "adaptive_topk",
]

ENTMAX_SORT_ALPHAS = (1.5, 2.0)


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------
def round_bf16(x):
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits and fp32's exponent range: a normal value
    in [2^(e-1), 2^e) is a multiple of 2^(e-8); below 2^-126 the spacing is the
    subnormal quantum 2^-133.  ``np.rint`` rounds half to even.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    qexp = np.maximum(e - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(x, -qexp)), qexp)
    y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, x), y)
    return np.where(x == 0, x, y)


def round_to(x, dtype):
    """Round float64 values once to the storage dtype ('bf16' or 'f32')."""
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


# --------------------------------------------------------------------------
# [EntmaxKV] §2.A — per-page metadata (bounding box + Gaussian statistics)
# --------------------------------------------------------------------------
def page_metadata(k_tokens, n_valid, dtype):
    """Bounding box and first/second moments of each page's keys.

    [EntmaxKV] §2.A "Bornes de Boîte Englobante" (coordinate-wise k_min /
    k_max) and "Statistiques Gaussiennes" (mean and variance of the keys of a
    page).  Only the first ``n_valid[p]`` tokens of page p count.

    k_tokens: [P, S, d] float64 stored key values; n_valid: [P] ints in 1..S.
    Returns dict of [P, d] float64 arrays, each exactly representable in
    ``dtype``: kmax, kmin (exact), mean, var (population variance).
    Sums run in token order, float64, one rounding per operation.
    """
    k_tokens = np.asarray(k_tokens, np.float64)
    P, S, d = k_tokens.shape
    n = np.asarray(n_valid, np.int64)
    if np.any(n < 1) or np.any(n > S):
        raise ValueError("n_valid must lie in 1..S")
    kmax = np.full((P, d), -np.inf)
    kmin = np.full((P, d), np.inf)
    total = np.zeros((P, d))
    for t in range(S):
        live = (t < n)[:, None]
        x = k_tokens[:, t, :]
        kmax = np.where(live, np.maximum(kmax, x), kmax)
        kmin = np.where(live, np.minimum(kmin, x), kmin)
        total = np.where(live, total + x, total)
    mean = total / n[:, None]
    sq = np.zeros((P, d))
    for t in range(S):
        live = (t < n)[:, None]
        dev = k_tokens[:, t, :] - mean
        sq = np.where(live, sq + dev * dev, sq)
    var = sq / n[:, None]
    return {"kmax": kmax, "kmin": kmin,
            "mean": round_to(mean, dtype), "var": round_to(var, dtype)}


# --------------------------------------------------------------------------
# [EntmaxKV] §2.A — bounding-box upper bound
# --------------------------------------------------------------------------
def bbox_upper_bound(q, kmax, kmin, scale):
    """Upper bound of every token score of a page, per query head.

    [EntmaxKV] §2.A: the coordinate-wise box [k_min, k_max] yields a
    deterministic upper bound on the largest attention score any token of the
    page can reach.  For a key inside the box, q_j·k_j ≤ max(q_j·kmin_j,
    q_j·kmax_j) coordinate by coordinate, hence
        ub[h, p] = scale · Σ_j max(q[h, j]·kmin[p, j], q[h, j]·kmax[p, j]).

    q: [G, d]; kmax, kmin: [P, d] → ub [G, P] float64.
    """
    q = np.asarray(q, np.float64)[:, None, :]
    lo = q * np.asarray(kmin, np.float64)[None]
    hi = q * np.asarray(kmax, np.float64)[None]
    return scale * np.maximum(lo, hi).sum(axis=-1)


def page_scores(ub):
    """Score of a page for a KV head: the max of its query heads' bounds.

    Reading (the page is silent on grouped-query attention): selection is
    made once per (sequence, KV head), so a page is worth loading for the
    group as soon as one of the group's query heads may score high in it.
    """
    return np.max(np.asarray(ub, np.float64), axis=0)


# --------------------------------------------------------------------------
# [EntmaxKV] §2.B.1 — top-k page selection
# --------------------------------------------------------------------------
def select_topk(score, k):
    """Indices of the k pages with the highest upper-bound score.

    [EntmaxKV] §2.B "Sélection de Pages Top-k": fixed budget, the k pages with
    the largest bound.  Ties go to the lower page index; when there are at
    most k pages, all are kept.  Returned in ascending page order.
    """
    score = np.asarray(score, np.float64)
    order = np.argsort(-score, kind="stable")
    return np.sort(order[: min(int(k), score.shape[0])])


# --------------------------------------------------------------------------
# [EntmaxKV] §2.B.2 — Gaussian-aware entmax selection
# --------------------------------------------------------------------------
def _normal_partial_moments(c, jmax):
    """M_j(c) = ∫_c^∞ z^j φ(z) dz for j = 0..jmax (standard normal φ).

    M_0 = Q(c) (upper tail), M_1 = φ(c), and integrating z^(j-1)·zφ(z) by
    parts (zφ = −φ') gives M_j = c^(j-1)·φ(c) + (j−1)·M_(j−2).
    """
    c = np.clip(np.asarray(c, np.float64), -60.0, 60.0)
    phi = np.exp(-0.5 * c * c) / math.sqrt(2.0 * math.pi)
    out = [ndtr(-c), phi]
    for j in range(2, jmax + 1):
        out.append(c ** (j - 1) * phi + (j - 1) * out[j - 2])
    return out[: jmax + 1]


def gauss_truncated_power_mean(mu, sigma, tau, beta):
    """E[(u − τ)_+^β] for u ~ N(μ, σ²) and an integer β ≥ 1.

    Binomial expansion around the mean: with u = μ + σZ and c = (τ−μ)/σ,
        (u−τ)^β = Σ_j C(β, j)·(μ−τ)^(β−j)·σ^j·Z^j   on {Z > c},
    so the expectation is Σ_j C(β, j)(μ−τ)^(β−j) σ^j M_j(c).  σ = 0 reduces
    to (μ − τ)_+^β.  Pinned against numerical quadrature in the tests.
    """
    beta = int(beta)
    mu, sigma, tau = np.broadcast_arrays(np.asarray(mu, np.float64),
                                         np.asarray(sigma, np.float64),
                                         np.asarray(tau, np.float64))
    degenerate = sigma <= 0.0
    safe_sigma = np.where(degenerate, 1.0, sigma)
    c = (tau - mu) / safe_sigma
    moments = _normal_partial_moments(c, beta)
    acc = np.zeros(mu.shape)
    for j in range(beta + 1):
        acc = acc + math.comb(beta, j) * (mu - tau) ** (beta - j) * safe_sigma ** j * moments[j]
    point = np.maximum(mu - tau, 0.0) ** beta
    return np.where(degenerate, point, np.maximum(acc, 0.0))


def gauss_tau_hat(mu_u, sig_u, n, beta):
    """Threshold τ̂ of the page-level Gaussian normalisation equation.

    [EntmaxKV] §2.B.2: τ̂ solves an approximate normalisation equation built
    from the page Gaussians.  Reading: the expected entmax mass is one,
        F(τ) = Σ_p n_p · E[(u_p − τ)_+^β] = 1,   u_p ~ N(mu_u[p], sig_u[p]²),
    where u = (α−1)·score.  F decreases strictly while positive, so the root
    is unique.  Bracket: by Jensen, E[(u−τ)_+^β] ≥ (μ−τ)_+^β, so F ≥ 1 at
    τ_lo = max_p (μ_p − n_p^(−1/β)); the upper end doubles a step until
    F < 1.  Plain bisection then runs to float64 resolution.
    """
    mu_u = np.asarray(mu_u, np.float64)
    sig_u = np.asarray(sig_u, np.float64)
    n = np.asarray(n, np.float64)

    def excess(t):
        return float(np.sum(n * gauss_truncated_power_mean(mu_u, sig_u, t, beta))) - 1.0

    lo = float(np.max(mu_u - n ** (-1.0 / beta)))
    step = 1.0
    hi = lo + step
    while excess(hi) >= 0.0:
        step *= 2.0
        hi = lo + step
    while True:
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            break
        if excess(mid) >= 0.0:
            lo = mid
        else:
            hi = mid
    return lo


def select_gauss(q, mean, var, n_valid, scale, alpha, delta):
    """Gaussian-aware entmax page selection for one (sequence, KV head).

    [EntmaxKV] §2.A "Statistiques Gaussiennes" + §2.B.2: each page's token
    scores are modelled as a Gaussian from its stored key mean/variance; τ̂ is
    estimated from those Gaussians; a page is kept when its estimated maximum
    score clears τ̂ minus the safety margin Δ.

    Readings: m = scale·q·μ, s = scale·√(Σ_j q_j² σ²_j); estimated maximum of
    n_p Gaussian scores ŝ = m + s·√(2 ln n_p) (the classical bound on the
    expected maximum of n Gaussians; n_p = 1 gives m); the comparison is made
    in threshold units, (α−1)·ŝ > τ̂ − Δ, per query head, and the group keeps
    the union.  If no page passes, the single page with the largest margin
    (lowest index on ties) is kept.

    q: [G, d]; mean, var: [P, d]; n_valid [P].  Returns a dict: sel
    (ascending), tau_hat [G], m, s, shat [G, P] and margin [G, P] =
    (α−1)ŝ − (τ̂ − Δ).
    """
    beta = 1.0 / (alpha - 1.0)
    if abs(beta - round(beta)) > 1e-12 or round(beta) < 1:
        raise ValueError("the Gaussian policy needs an integer 1/(alpha-1)")
    beta = int(round(beta))
    q = np.asarray(q, np.float64)
    n = np.asarray(n_valid, np.float64)
    m = scale * (q @ np.asarray(mean, np.float64).T)
    s = scale * np.sqrt((q * q) @ np.asarray(var, np.float64).T)
    mu_u = (alpha - 1.0) * m
    sig_u = (alpha - 1.0) * s
    tau_hat = np.array([gauss_tau_hat(mu_u[h], sig_u[h], n, beta) for h in range(q.shape[0])])
    shat = m + s * np.sqrt(2.0 * np.log(n))[None, :]
    margin = (alpha - 1.0) * shat - (tau_hat[:, None] - delta)
    keep = np.any(margin > 0.0, axis=0)
    if not np.any(keep):
        keep[int(np.argmax(np.max(margin, axis=0)))] = True
    return {"sel": np.nonzero(keep)[0], "tau_hat": tau_hat, "m": m, "s": s,
            "shat": shat, "margin": margin}


# --------------------------------------------------------------------------
# [EntmaxKV] §2 / §2.C — α-entmax
# --------------------------------------------------------------------------
def _sparsemax_threshold(u):
    """α = 2: sort descending; τ_k = (Σ_{j≤k} u_(j) − 1)/k; support size
    k* = max{k : u_(k) > τ_k}; τ = τ_{k*}."""
    us = np.sort(u)[::-1]
    k = np.arange(1, us.size + 1, dtype=np.float64)
    tau_k = (np.cumsum(us) - 1.0) / k
    ok = np.nonzero(us > tau_k)[0]
    return float(tau_k[ok[-1]])


def _entmax15_threshold(u):
    """α = 1.5 (β = 2): for the top-k set, Σ_{j≤k}(u_(j) − τ)² = 1 has the
    smaller root τ_k = M_k − √δ_k with M_k, Q_k the mean and mean square of
    the top k and δ_k = (1 − k(Q_k − M_k²))/k; k* = max{k : δ_k ≥ 0 and
    u_(k) > τ_k}."""
    us = np.sort(u)[::-1]
    k = np.arange(1, us.size + 1, dtype=np.float64)
    M = np.cumsum(us) / k
    Q = np.cumsum(us * us) / k
    delta = (1.0 - k * (Q - M * M)) / k
    tau_k = M - np.sqrt(np.maximum(delta, 0.0))
    ok = np.nonzero((delta >= 0.0) & (us > tau_k))[0]
    return float(tau_k[ok[-1]])


def _bisection_threshold(u, alpha):
    """General α: f(τ) = Σ_i [u_i − τ]_+^β − 1 decreases in τ; f ≥ 0 at
    max(u) − 1 and f ≤ 0 at max(u) − n^(1−α); bisect until the midpoint
    equals an endpoint."""
    beta = 1.0 / (alpha - 1.0)
    top = float(np.max(u))
    lo = top - 1.0
    hi = top - float(u.size) ** (1.0 - alpha)

    def f(t):
        return float(np.sum(np.maximum(u - t, 0.0) ** beta)) - 1.0

    while True:
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            break
        if f(mid) >= 0.0:
            lo = mid
        else:
            hi = mid
    return lo


def entmax_threshold(u, alpha, method=None):
    """τ of α-entmax for the shifted scores u = (α−1)·z (1-D array).

    [EntmaxKV] §2: α-entmax (α > 1) gives exact zeros.  Exact sort-based forms
    for α ∈ {1.5, 2}; bisection otherwise (or when method='bisect').
    """
    u = np.asarray(u, np.float64)
    if u.ndim != 1 or u.size == 0:
        raise ValueError("u must be a non-empty 1-D array")
    if alpha <= 1.0:
        raise ValueError("alpha must exceed 1")
    if method is None:
        method = "sort" if alpha in ENTMAX_SORT_ALPHAS else "bisect"
    if method == "sort":
        if alpha == 2.0:
            return _sparsemax_threshold(u)
        if alpha == 1.5:
            return _entmax15_threshold(u)
        raise ValueError("sort form exists only for alpha in {1.5, 2}")
    return _bisection_threshold(u, alpha)


def entmax_probs(z, alpha, method=None):
    """α-entmax probabilities p_i = [(α−1)z_i − τ]_+^{1/(α−1)} (Σp = 1)."""
    u = (alpha - 1.0) * np.asarray(z, np.float64)
    tau = entmax_threshold(u, alpha, method)
    return np.maximum(u - tau, 0.0) ** (1.0 / (alpha - 1.0)), tau


def entmax_attention(q, K, V, scale, alpha):
    """α-entmax attention of query heads over one token set.

    [EntmaxKV] §2.C: attention weights are α-entmax over the loaded tokens
    only.  q: [G, d]; K, V: [T, d] → dict with o [G, d], tau [G], u [G, T]
    (u = (α−1)·scale·q·k), p [G, T].
    """
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    u = (alpha - 1.0) * (scale * (q @ K.T))
    beta = 1.0 / (alpha - 1.0)
    taus = np.array([entmax_threshold(u[h], alpha) for h in range(q.shape[0])])
    p = np.maximum(u - taus[:, None], 0.0) ** beta
    return {"o": p @ V, "tau": taus, "u": u, "p": p}


def softmax_attention(q, K, V, scale):
    """Dense softmax attention (the full-cache softmax decode of [EntmaxKV] §4).

    Also returns lse [G] = log Σ_i e^{z_i}, computed as m + log Σ_i e^{z_i − m}
    with m the row maximum, so that p_i = e^{z_i − lse}."""
    z = scale * (np.asarray(q, np.float64) @ np.asarray(K, np.float64).T)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    s = e.sum(axis=1, keepdims=True)
    w = e / s
    return {"o": w @ np.asarray(V, np.float64), "p": w, "lse": (m + np.log(s))[:, 0]}


def softmax_dropped_mass(q, K, kept, scale):
    """Softmax weight that a kept token set leaves out, per query head.

    [EntmaxKV] §3 "Borne d'Erreur": the error of attending over a subset is
    bounded through the attention mass of the dropped tokens.  Here that mass
    is the full-cache softmax weight summed over the tokens not kept:
    δ_h = Σ_{i ∉ kept} p_{h,i}.  q: [G, d]; K: [T, d] every token; kept: [T]
    booleans.  Returns δ [G]."""
    p = softmax_attention(q, K, np.zeros((np.shape(K)[0], 1)), scale)["p"]
    return p[:, ~np.asarray(kept, bool)].sum(axis=1)


# --------------------------------------------------------------------------
# paged cache plumbing — [EntmaxKV] §2.A "Le cache KV est partitionné en pages"
# --------------------------------------------------------------------------
def unit_pages(page_table_row, seq_len, page_size):
    """Physical page ids and valid token counts of one sequence's pages."""
    n_pages = -(-int(seq_len) // page_size)
    phys = np.asarray(page_table_row[:n_pages], np.int64)
    n_valid = np.minimum(page_size, int(seq_len) - page_size * np.arange(n_pages))
    return phys, n_valid


def build_page_meta(k_pool, page_table, seq_lens, page_size, dtype):
    """Metadata for every (physical page, KV head) a sequence uses.

    k_pool: [num_phys, Hkv, S, d] float64.  Returns {phys: dict(field → [Hkv, d])}.
    """
    out = {}
    for b, L in enumerate(seq_lens):
        phys, n_valid = unit_pages(page_table[b], L, page_size)
        for h in range(k_pool.shape[1]):
            meta = page_metadata(k_pool[phys, h], n_valid, dtype)
            for i, pid in enumerate(phys):
                rec = out.setdefault(int(pid), {f: np.zeros((k_pool.shape[1], k_pool.shape[3])) for f in meta})
                for f in meta:
                    rec[f][h] = meta[f][i]
    return out


def append_token(k_pool, v_pool, page_table, seq_lens, k_new, v_new, page_size):
    """Write each sequence's new token at position seq_len − 1 (in place).

    Returns the list of (b, phys, n_valid) pages whose metadata the append
    must refresh.
    """
    touched = []
    for b, L in enumerate(seq_lens):
        pos = int(L) - 1
        phys = int(page_table[b][pos // page_size])
        k_pool[phys, :, pos % page_size, :] = k_new[b]
        v_pool[phys, :, pos % page_size, :] = v_new[b]
        touched.append((b, phys, pos % page_size + 1))
    return touched


def decode_unit(k_pool, v_pool, page_table_row, seq_len, kv_head, q_group, *,
                page_size, scale, alpha, dtype, policy="topk", k=None,
                delta=None, sel=None):
    """Full decode step of one (sequence, KV head) unit, stage by stage.

    [EntmaxKV] §2 pipeline: metadata (§2.A) → page scores (§2.A) → selection
    (§2.B: 'topk' with budget k, 'gauss' with margin Δ, 'all' = full cache, or
    an explicit ``sel`` of logical pages) → α-entmax attention over the valid
    tokens of the selected pages (§2.C).
    """
    phys, n_valid = unit_pages(page_table_row, seq_len, page_size)
    K_pages = np.asarray(k_pool[phys, kv_head], np.float64)
    V_pages = np.asarray(v_pool[phys, kv_head], np.float64)
    meta = page_metadata(K_pages, n_valid, dtype)
    ub = bbox_upper_bound(q_group, meta["kmax"], meta["kmin"], scale)
    score = page_scores(ub)
    out = {"meta": meta, "ub": ub, "score": score, "n_valid": n_valid}
    if sel is None:
        if policy == "topk":
            sel = select_topk(score, k)
        elif policy == "gauss":
            gs = select_gauss(q_group, meta["mean"], meta["var"], n_valid, scale, alpha, delta)
            sel = gs["sel"]
            out["gauss"] = gs
            out["tau_hat"] = gs["tau_hat"]
            out["margin"] = gs["margin"]
        elif policy == "all":
            sel = np.arange(phys.size)
        else:
            raise ValueError(policy)
    sel = np.asarray(sel, np.int64)
    out["sel"] = sel
    Ks = np.concatenate([K_pages[p, : n_valid[p]] for p in sel])
    Vs = np.concatenate([V_pages[p, : n_valid[p]] for p in sel])
    att = entmax_attention(q_group, Ks, Vs, scale, alpha)
    out.update(att)
    out["token_page"] = np.concatenate([np.full(n_valid[p], p) for p in sel])
    out["token_slot"] = np.concatenate([np.arange(n_valid[p]) for p in sel])
    return out


# --------------------------------------------------------------------------
# exactness certificate — [EntmaxKV] §3 "Récupération du Support"
# --------------------------------------------------------------------------
def exactness_certificate(score, sel, tau, alpha):
    """Per query head: True when no unselected page can hold a support token.

    [EntmaxKV] §3: if the selected tokens contain the α-entmax support, the
    sparse output equals the full-cache one.  Every token score of page p is
    at most the page score (the bound maximised over the group's heads), so
    when (α−1)·max_{p ∉ sel} score_p ≤ τ_h, no unselected token has
    u = (α−1)z > τ_h; τ_h then also solves the full-cache equation (the extra
    tokens add nothing to Σ[u − τ]_+^β), so the outputs agree.  score: [P]
    unit scores; sel: selected page indices; tau: [G].  With nothing left
    unselected the certificate holds trivially.
    """
    score = np.asarray(score, np.float64)
    rest = np.setdiff1d(np.arange(score.shape[0]), np.asarray(sel, np.int64))
    if rest.size == 0:
        return np.ones(np.shape(tau), bool)
    return (alpha - 1.0) * score[rest].max() <= np.asarray(tau, np.float64)


def adaptive_topk(k_pool, v_pool, page_table_row, seq_len, kv_head, q_group, *, page_size,
                  scale, alpha, dtype, k0):
    """Grow the top-k budget (doubling from k0) until every head of the unit is
    certified exact; returns (k, decode_unit result).  The certificate's
    extension of [EntmaxKV] §3 into an adaptive budget."""
    n_pages = -(-int(seq_len) // page_size)
    k = max(1, int(k0))
    while True:
        r = decode_unit(k_pool, v_pool, page_table_row, seq_len, kv_head, q_group, page_size=page_size,
                        scale=scale, alpha=alpha, dtype=dtype, policy="topk", k=k)
        if k >= n_pages or np.all(exactness_certificate(r["score"], r["sel"], r["tau"], alpha)):
            return k, r
        k = min(2 * k, n_pages)
