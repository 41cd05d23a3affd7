"""Oracle: heterogeneous causal sliding-window attention.  TEST INFRASTRUCTURE ONLY.

What the method computes
------------------------
"Mixture of Attention" project page, "Key findings" and the N x N causal
attention figure of "Finding two": each head keeps a diagonal band of the
causal attention matrix whose width is the head's own span S_h; everything
outside the band is masked.  The blog walkthrough ("MoA: Mixture of Sparse
Attention ...", section 2.1) builds the rule on a sliding-window mask, and
its section 5 says the CUDA kernel applies the mask and aggregates attention.

Written out, for batch b, query head h, query row i (0-based):

    window(i)  = { j : i - S_h < j <= i, j >= 0 }        (S_h keys incl. i)
    s_j        = scale * sum_k q[b,h,i,k] * k[b,g,j,k]      for j in window(i)
    p_j        = exp(s_j - max_j s_j)
    o[b,h,i,:] = sum_j p_j v[b,g,j,:] / sum_j p_j

where g = h // (Hq // Hkv) is the key/value head that query head h reads
(grouped-query attention; with Hq == Hkv, g == h).  Subtracting the row
maximum leaves the result unchanged mathematically and keeps exp finite.

Readings taken where the pages are silent: the window holds S_h keys including the
query's own position (S_h = 1 attends to itself only); spans are per query head.
The plain path has no sink or global tokens; ``prefill_sink`` adds them (see
there).

Everything runs in numpy float64 on whatever values the caller passes
(callers upcast the exact bf16 or fp32 values the GPU sees).
"""

import numpy as np


def window(i, S):
    """Inclusive key range [lo, hi] of query row ``i`` under span ``S``."""
    if S < 1:
        raise ValueError("span must be >= 1")
    return max(0, i - S + 1), i


def row_weights(q_i, K, lo, hi, scale):
    """Softmax weights of one query row over keys lo..hi (float64 vector)."""
    s = (np.asarray(K[lo:hi + 1], dtype=np.float64) @ np.asarray(q_i, dtype=np.float64)) * scale
    p = np.exp(s - s.max())
    return p / p.sum()


def attend_row(q_i, K, V, lo, hi, scale):
    """One output row: softmax over keys lo..hi applied to V[lo..hi]."""
    w = row_weights(q_i, K, lo, hi, scale)
    return w @ np.asarray(V[lo:hi + 1], dtype=np.float64)


def prefill(q, k, v, spans, scale, rows=None):
    """Windowed causal attention over a whole prompt.

    q: [B, Hq, N, d]; k, v: [B, Hkv, N, d]; spans: per query head (len Hq).
    Returns float64 [B, Hq, N, d].  With ``rows`` given (an iterable of
    (b, h, i) triples) returns a float64 array [len(rows), d] holding only
    those output rows, for sampled checks at sizes where the full output
    would take too long.
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    if len(spans) != Hq:
        raise ValueError("one span per query head")
    G = Hq // Hkv
    if rows is not None:
        out = np.empty((len(rows), d), dtype=np.float64)
        for n, (b, h, i) in enumerate(rows):
            lo, hi = window(i, int(spans[h]))
            out[n] = attend_row(q[b, h, i], k[b, h // G], v[b, h // G], lo, hi, scale)
        return out
    out = np.empty((B, Hq, N, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            K = np.asarray(k[b, g], dtype=np.float64)
            V = np.asarray(v[b, g], dtype=np.float64)
            S = int(spans[h])
            for i in range(N):
                lo, hi = window(i, S)
                out[b, h, i] = attend_row(q[b, h, i], K, V, lo, hi, scale)
    return out


def chunk(q, k_hist, v_hist, t, spans, scale, rows=None):
    """Windowed causal attention of a chunk of new tokens that continues each sequence.

    The same definition as ``prefill``, at an offset: query i of sequence b
    is the token at position P = t[b] + i and attends to window(P, S_h) of
    that sequence's keys (positions earlier than the chunk included).  This
    is the prefill of a prompt that arrives in pieces while decoding serves
    from the fixed-size cache ("Mixture of Attention" project page, "Demo"
    step 03); with t[b] = 0 it is ``prefill`` of the chunk.

    q: [B, Hq, n, d], queries of positions t[b] .. t[b]+n-1.
    k_hist, v_hist: per sequence b an array [Hkv, t[b]+n, d] with the keys
    and values of every position 0 .. t[b]+n-1 (the chunk's own last).
    t: tokens before the chunk, one per sequence.
    Returns float64 [B, Hq, n, d], or with ``rows`` ((b, h, i) triples) the
    float64 [len(rows), d] of those output rows only.
    """
    q = np.asarray(q)
    B, Hq, n, d = q.shape
    if len(t) != B or len(k_hist) != B or len(v_hist) != B:
        raise ValueError("one history and one position per sequence")
    if len(spans) != Hq:
        raise ValueError("one span per query head")
    Hkv = np.asarray(k_hist[0]).shape[0]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    for b in range(B):
        if np.asarray(k_hist[b]).shape[1] != int(t[b]) + n or np.asarray(v_hist[b]).shape != np.asarray(k_hist[b]).shape:
            raise ValueError("history of sequence %d must hold t[b] + n positions" % b)
    if rows is None:
        rows_list = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(n)]
    else:
        rows_list = list(rows)
    out = np.empty((len(rows_list), d), dtype=np.float64)
    for r, (b, h, i) in enumerate(rows_list):
        P = int(t[b]) + i
        lo, hi = window(P, int(spans[h]))
        out[r] = attend_row(q[b, h, i], k_hist[b][h // G], v_hist[b][h // G], lo, hi, scale)
    if rows is None:
        return out.reshape(B, Hq, n, d)
    return out


def in_window_flops(spans, N, d, B=1):
    """Algorithmic FLOPs of prefill counting only in-window work.

    Row i of head h touches min(i+1, S_h) keys; QK^T and PV each cost 2*d
    flops per (row, key) pair, so the total is 4*d*sum_h sum_i min(i+1, S_h)
    = 4*d*sum_h (S_h*N - S_h*(S_h-1)/2) for S_h <= N.
    """
    total = 0
    for S in spans:
        S = min(int(S), int(N))
        pairs = S * N - S * (S - 1) // 2
        total += 4 * d * pairs
    return B * total


# ---------------------------------------------------------------------------
# Band plus global ("sink") tokens
# ---------------------------------------------------------------------------
# The codewithpapers page for arXiv 2406.14909 ("MoA: Mixture of Sparse
# Attention for Automatic Large Language Model Compression") lists, from the
# official repository, a pattern generator named gen_global_pattern beside
# gen_band_pattern, and density counters named streamingllm_attention_density
# and streamingllm_kv_cache_density; the project page's Table 4 compares with
# StreamingLLM.  The pages give no formula.  Reading taken: a head with k_h
# global tokens attends to its band and, in addition, to the first k_h
# positions of the sequence (those that are causal), every key counted once:
#
#     keys(i) = { j : i - S_h < j <= i }  union  { j : 0 <= j < k_h, j <= i }
#
# k_h = 0 is the plain band; k_h >= N (or S_h >= N) is dense causal attention.


def keys_sink(i, S, k):
    """Sorted key positions of query row ``i`` under span ``S`` and ``k`` global tokens."""
    if S < 1 or k < 0:
        raise ValueError("span must be >= 1 and the global token count >= 0")
    lo, hi = window(i, S)
    band = set(range(lo, hi + 1))
    glob = set(range(0, min(k, i + 1)))
    return sorted(band | glob)


def attend_keys(q_i, K, V, keys, scale):
    """One output row: softmax over the listed key positions applied to their values."""
    idx = np.asarray(keys, dtype=np.int64)
    Ks = np.asarray(K, dtype=np.float64)[idx]
    Vs = np.asarray(V, dtype=np.float64)[idx]
    s = (Ks @ np.asarray(q_i, dtype=np.float64)) * scale
    p = np.exp(s - s.max())
    return (p / p.sum()) @ Vs


def prefill_sink(q, k, v, spans, sinks, scale, rows=None):
    """Windowed causal attention with global tokens over a whole prompt.

    Same shapes and ``rows`` convention as ``prefill``; ``sinks`` holds k_h per
    query head.  Row i of head h attends to ``keys_sink(i, S_h, k_h)``.
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    if len(spans) != Hq or len(sinks) != Hq:
        raise ValueError("one span and one global token count per query head")
    G = Hq // Hkv
    if rows is None:
        rows_list = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N)]
    else:
        rows_list = list(rows)
    out = np.empty((len(rows_list), d), dtype=np.float64)
    for n, (b, h, i) in enumerate(rows_list):
        keys = keys_sink(i, int(spans[h]), int(sinks[h]))
        out[n] = attend_keys(q[b, h, i], k[b, h // G], v[b, h // G], keys, scale)
    if rows is None:
        return out.reshape(B, Hq, N, d)
    return out


def in_window_flops_sink(spans, sinks, N, d, B=1):
    """Algorithmic FLOPs of prefill with global tokens: 4 d per (row, key) pair.

    Row i of head h touches min(i + 1, S_h) band keys and the global keys below
    the band, max(0, min(k_h, i - S_h + 1)) of them.
    """
    total = 0
    for S, kk in zip(spans, sinks):
        S, kk = int(S), int(kk)
        pairs = 0
        for i in range(int(N)):
            pairs += min(i + 1, S) + max(0, min(kk, i - S + 1))
        total += 4 * d * pairs
    return B * total

