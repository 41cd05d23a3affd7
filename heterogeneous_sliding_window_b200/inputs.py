"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds none of the method's arithmetic.  It draws random numbers
(Q/K/V values, per-head alpha/beta tables) and searches a single scale factor
for the alpha/beta tables; every span evaluation it needs is done by a
``rules_fn`` the caller passes in (the CUDA library's rule on the product
side, the oracle's rule in tests), so both sides derive their spans
themselves.

Workload shapes follow the pages' evaluation models (Vicuna-7B/13B,
Llama3-8B; "Mixture of Attention" project page, sections "Long-context task
performance" and "Inference speed and memory efficiency").  Values are iid
N(0, 1); bf16 inputs are fp32 draws rounded to bf16 (round-to-nearest-even).
"""

import numpy as np
import torch

# Candidate sets used for the Vicuna-7B-shaped and Llama3-8B-shaped span
# tables (the blog walkthrough's candidate sets are lost on the page, so the
# benchmark workload's own sets are used).
ALPHA_SET_7B = (0.0, 512.0, 1024.0, 2048.0)
BETA_SET_7B = (0.0, 0.125, 0.25, 0.5, 1.0)
# Vicuna-13B-shaped mix: fixed-local heads and elastic heads.
ALPHA_SET_LOCAL_13B = (1024.0, 2048.0)
BETA_SET_ELASTIC_13B = (0.5, 0.9)


def randn(seed, shape, dtype="bf16"):
    """iid N(0,1) as a CPU torch tensor of the requested dtype ('bf16' or 'f32')."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(size=shape, dtype=np.float32)
    t = torch.from_numpy(x)
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def randn_cuda(seed, shape, dtype="bf16", device="cuda"):
    """iid N(0,1) drawn on the GPU by torch's seeded generator (large inputs)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def as_f64(t):
    """Exact float64 copy of a CPU/GPU tensor (bf16 and fp32 upcast exactly)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def draw_alpha_beta(seed, n_heads, alpha_set=ALPHA_SET_7B, beta_set=BETA_SET_7B):
    """Per-head (alpha, beta) drawn uniformly from the candidate sets."""
    rng = np.random.default_rng(seed)
    a = rng.choice(np.asarray(alpha_set, dtype=np.float64), size=n_heads)
    b = rng.choice(np.asarray(beta_set, dtype=np.float64), size=n_heads)
    return a, b


def rescale_to_density(alpha, beta, N, block, density, rules_fn, iters=60):
    """Scale (alpha, beta) by one factor c so the mean span / N is closest to ``density``.

    ``rules_fn(alpha, beta, N, block) -> list of spans`` evaluates the rule.
    The mean of the rounded and clamped spans is non-decreasing in c, so a
    bisection on c brackets the target; the side whose mean lands closer wins.
    Returns (c*alpha, c*beta).
    """
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    target = density * N

    def mean_span(c):
        return float(np.mean(rules_fn(c * alpha, c * beta, N, block)))

    lo, hi = 0.0, 1.0
    while mean_span(hi) < target and hi < 1e12:
        hi *= 2.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if mean_span(mid) < target:
            lo = mid
        else:
            hi = mid
    best = lo if abs(mean_span(lo) - target) <= abs(mean_span(hi) - target) else hi
    return best * alpha, best * beta


def tables_7b(seed, n_heads, N, block, density, rules_fn):
    """Vicuna-7B-shaped per-head table rescaled to a target mean span / N."""
    a, b = draw_alpha_beta(seed, n_heads)
    return rescale_to_density(a, b, N, block, density, rules_fn)


def tables_13b_mix(seed, n_heads, N, block, density, rules_fn):
    """Vicuna-13B-shaped layer: fixed-local heads (beta = 0, alpha in {1024, 2048})
    mixed with elastic heads (alpha = 0, beta in {0.5, 0.9}).

    The count k of elastic heads is the one whose mean span / N lands closest to
    ``density``; which heads are elastic, and their values, are drawn by seed.
    """
    rng = np.random.default_rng(seed)
    loc_a = rng.choice(np.asarray(ALPHA_SET_LOCAL_13B), size=n_heads)
    el_b = rng.choice(np.asarray(BETA_SET_ELASTIC_13B), size=n_heads)
    order = rng.permutation(n_heads)
    best = None
    for k in range(n_heads + 1):
        elastic = np.zeros(n_heads, dtype=bool)
        elastic[order[:k]] = True
        a = np.where(elastic, 0.0, loc_a)
        b = np.where(elastic, el_b, 0.0)
        m = float(np.mean(rules_fn(a, b, N, block))) / N
        if best is None or abs(m - density) < best[0]:
            best = (abs(m - density), a, b)
    return best[1], best[2]


def tiny_tables():
    """Tiny fp32 case: 4 heads with spans {32, 64, 128, 256} (beta = 0, block 32)."""
    return np.array([32.0, 64.0, 128.0, 256.0]), np.zeros(4)


# Global-token counts per head for the band-plus-global-token workloads: a
# seeded draw from a small set (a few StreamingLLM-style sink tokens up to a
# few tiles of them).
SINK_SET = (0, 4, 64, 128, 1024)


def sink_counts(seed, n_heads, choices=SINK_SET):
    """Per-head global token counts drawn uniformly from ``choices``."""
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.choice(np.asarray(choices, dtype=np.int64), size=n_heads)]
