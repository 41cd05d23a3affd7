"""Oracle: the elastic span rule.  TEST INFRASTRUCTURE ONLY.

What the method computes
------------------------
"Mixture of Attention" project page, "Key findings / Finding two": every
attention head h gets a window whose length follows a linear rule in the
input length N,

    S_h = alpha_h + beta_h * N,

with (alpha_h, beta_h) searched per head.  Section "Method design / Elastic
search space" adds that the candidate rules map N to spans that satisfy the
kernel's block-size requirement.  The worked example on the same page
("heads A, B, C" at N = 4k) shows head B with S = 5.6k and beta = 0 drawn as
"100% of the input length" at 4k, so the span is clamped to N.

Readings taken where the pages are silent:

* Rounding to the block: nearest multiple of ``block``, ties rounded up,
  computed as ``block * floor(x / block + 0.5)`` in IEEE binary64 with every
  operation rounded separately (no fused multiply-add).
* Clamp: ``S = min(N, max(block, S))``; when N < block this yields N.
* ``alpha`` and ``beta`` must be finite and non-negative; N >= 1; block >= 1.
"""

import math


def span_rule(alpha, beta, N, block):
    """Span of one head for input length ``N`` (Finding two; Elastic search space).

    x = alpha + beta*N, rounded to the nearest multiple of ``block`` (ties up),
    then clamped to [block, N].  Returns a Python int.
    """
    alpha = float(alpha)
    beta = float(beta)
    N = int(N)
    block = int(block)
    if not (math.isfinite(alpha) and math.isfinite(beta)):
        raise ValueError("alpha and beta must be finite")
    if alpha < 0.0 or beta < 0.0:
        raise ValueError("alpha and beta must be non-negative")
    if N < 1 or block < 1:
        raise ValueError("N and block must be >= 1")
    Nf = float(N)
    bf = float(block)
    prod = beta * Nf          # one rounding
    x = alpha + prod          # a second, separate rounding
    q = math.floor(x / bf + 0.5)
    s = bf * q
    if s < bf:
        s = bf
    if s > Nf:
        s = Nf
    return int(s)


def eval_spans(alphas, betas, N, block):
    """Spans of all heads of one layer: ``[span_rule(a, b, N, block) ...]``."""
    if len(alphas) != len(betas):
        raise ValueError("alpha and beta tables differ in length")
    return [span_rule(a, b, N, block) for a, b in zip(alphas, betas)]
