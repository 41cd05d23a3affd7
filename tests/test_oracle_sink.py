"""Pins for the oracle's band-plus-global-token attention (CPU only).

The reading: a head with k global tokens attends to its band (i - S, i] and to
the first k positions that are causal, each key once.  Each check fixes the
oracle against something other than itself: brute force over an explicit
N x N mask, the plain band when k = 0, torch's dense causal SDPA when k or S
covers the prompt, a two-key closed form, the count of mask entries, decode
against the last prefill row, and hand-computed byte offsets of the cache.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention, kvcache


def _brute_force_sink(q, k, v, spans, sinks, scale):
    """Pure-Python loops over an explicit N x N mask: band or global, and causal."""
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    out = np.zeros((B, Hq, N, d))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            S, kk = spans[h], sinks[h]
            mask = [[(j <= i) and ((j > i - S) or (j < kk)) for j in range(N)] for i in range(N)]
            for i in range(N):
                scores = []
                for j in range(N):
                    if mask[i][j]:
                        acc = 0.0
                        for c in range(d):
                            acc += float(q[b, h, i, c]) * float(k[b, g, j, c])
                        scores.append((j, acc * scale))
                m = max(s for _, s in scores)
                w = [(j, math.exp(s - m)) for j, s in scores]
                z = sum(p for _, p in w)
                for c in range(d):
                    out[b, h, i, c] = sum(p * float(v[b, g, j, c]) for j, p in w) / z
    return out


SINK_CASES = [
    dict(B=1, Hq=4, Hkv=4, N=19, d=4, spans=[1, 3, 6, 19], sinks=[1, 4, 2, 5]),
    dict(B=2, Hq=4, Hkv=2, N=15, d=3, spans=[2, 5, 4, 7], sinks=[3, 0, 8, 1]),
    dict(B=1, Hq=2, Hkv=1, N=22, d=5, spans=[4, 9], sinks=[6, 22]),
]


@pytest.mark.parametrize("case", SINK_CASES)
def test_sink_matches_brute_force_mask(case):
    rng = np.random.default_rng(11)
    q = rng.standard_normal((case["B"], case["Hq"], case["N"], case["d"]))
    k = rng.standard_normal((case["B"], case["Hkv"], case["N"], case["d"]))
    v = rng.standard_normal((case["B"], case["Hkv"], case["N"], case["d"]))
    scale = 1.0 / math.sqrt(case["d"])
    got = attention.prefill_sink(q, k, v, case["spans"], case["sinks"], scale)
    ref = _brute_force_sink(q, k, v, case["spans"], case["sinks"], scale)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_no_global_tokens_is_the_band():
    rng = np.random.default_rng(12)
    q = rng.standard_normal((2, 3, 40, 6))
    k = rng.standard_normal((2, 3, 40, 6))
    v = rng.standard_normal((2, 3, 40, 6))
    spans = [1, 9, 33]
    got = attention.prefill_sink(q, k, v, spans, [0, 0, 0], 0.4)
    ref = attention.prefill(q, k, v, spans, 0.4)
    assert np.max(np.abs(got - ref)) < 1e-13


def test_global_tokens_or_span_covering_the_prompt_is_dense_causal():
    rng = np.random.default_rng(13)
    B, H, N, d = 1, 4, 50, 8
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, H, N, d))
    v = rng.standard_normal((B, H, N, d))
    spans = [1, 7, N, 2 * N]
    sinks = [N, N + 3, 0, 5]
    got = attention.prefill_sink(q, k, v, spans, sinks, 1.0 / math.sqrt(d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def test_span_one_with_one_global_token_closed_form():
    """S = 1, k = 1: row i >= 1 attends to positions 0 and i only; row 0 to itself."""
    rng = np.random.default_rng(14)
    N, d, scale = 12, 5, 0.7
    q = rng.standard_normal((1, 1, N, d))
    k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, d))
    got = attention.prefill_sink(q, k, v, [1], [1], scale)
    assert np.array_equal(got[0, 0, 0], v[0, 0, 0])
    for i in range(1, N):
        s0 = scale * float(q[0, 0, i] @ k[0, 0, 0])
        si = scale * float(q[0, 0, i] @ k[0, 0, i])
        w0 = 1.0 / (1.0 + math.exp(si - s0))
        expect = w0 * v[0, 0, 0] + (1.0 - w0) * v[0, 0, i]
        assert np.max(np.abs(got[0, 0, i] - expect)) < 1e-13


def test_keys_sink_counts_overlap_once():
    assert attention.keys_sink(2, 3, 2) == [0, 1, 2]
    assert attention.keys_sink(10, 3, 4) == [0, 1, 2, 3, 8, 9, 10]
    assert attention.keys_sink(1, 1, 5) == [0, 1]
    assert attention.keys_sink(0, 4, 0) == [0]


def test_in_window_flops_sink_counts_mask_entries():
    for N, spans, sinks in [(37, [1, 5, 37, 60], [3, 0, 9, 40]), (64, [8, 64], [64, 1])]:
        pairs = 0
        for S, kk in zip(spans, sinks):
            for i in range(N):
                pairs += sum(1 for j in range(N) if j <= i and (j > i - S or j < kk))
        d = 16
        assert attention.in_window_flops_sink(spans, sinks, N, d) == 4 * d * pairs
        if not any(sinks):
            assert attention.in_window_flops(spans, N, d) == 4 * d * pairs


@pytest.mark.parametrize("C,sink_cap,n", [(7, 3, 30), (16, 16, 40), (5, 9, 25)])
def test_sink_decode_equals_last_prefill_row(C, sink_cap, n):
    """The ring (capacity C) plus the global-token rows serve decode exactly: after every
    append, decode equals row t - 1 of prefill_sink over the t tokens so far, also once
    the ring has wrapped past the global tokens."""
    rng = np.random.default_rng(15)
    B, Hkv, G, d = 2, 2, 2, 4
    Hq = Hkv * G
    spans = [min(C, x) for x in (1, C, 3, C - 1)]
    sinks = [min(sink_cap, x) for x in (sink_cap, 2, 0, 1)]
    cache = kvcache.RingCache(B, Hkv, d, [C] * Hkv, [sink_cap] * Hkv)
    K = rng.standard_normal((B, Hkv, n, d))
    V = rng.standard_normal((B, Hkv, n, d))
    Q = rng.standard_normal((B, Hq, n, d))
    for t in range(1, n + 1):
        cache.append(K[:, :, t - 1:t], V[:, :, t - 1:t])
        got = kvcache.decode_sink(cache, Q[:, :, t - 1], spans, sinks, 0.5)
        rows = [(b, h, t - 1) for b in range(B) for h in range(Hq)]
        ref = attention.prefill_sink(Q[:, :, :t], K[:, :, :t], V[:, :, :t], spans, sinks, 0.5, rows=rows)
        assert np.max(np.abs(got.reshape(B * Hq, d) - ref)) < 1e-13, t


def test_sink_image_layout_hand_computed():
    """B=2, Hkv=2, d=2, capacities (3, 2), global tokens (2, 1), f32: the global-token rows
    follow every ring block, per sequence and kv head, row p holding position p."""
    B, Hkv, d = 2, 2, 2
    cache = kvcache.RingCache(B, Hkv, d, [3, 2], [2, 1])
    n = 5
    k = np.zeros((B, Hkv, n, d))
    v = np.zeros((B, Hkv, n, d))
    for b in range(B):
        for g in range(Hkv):
            for r in range(n):
                k[b, g, r] = [1000 * b + 100 * g + r, 0.5]
                v[b, g, r] = [-(1000 * b + 100 * g + r), 0.25]
    cache.append(k, v)
    img = np.frombuffer(kvcache.data_image(cache, "f32"), dtype="<f4")
    assert img.size * 4 == kvcache.buffer_bytes(B, Hkv, d, [3, 2], 4, [2, 1]) - kvcache.header_bytes(B)
    # ring region: (3 + 2) rows x 2 (K and V) x d floats per sequence = 20 per sequence
    ring_floats = B * (3 + 2) * 2 * d
    sink = img[ring_floats:]
    # per sequence: g=0 Ksink[2][2], Vsink[2][2]; g=1 Ksink[1][2], Vsink[1][2] = 12 floats
    assert sink.size == B * 12
    for b in range(B):
        base = b * 12
        assert list(sink[base + 0:base + 4]) == [1000 * b + 0, 0.5, 1000 * b + 1, 0.5]          # K, g=0, p=0,1
        assert list(sink[base + 4:base + 8]) == [-(1000 * b + 0), 0.25, -(1000 * b + 1), 0.25]  # V, g=0
        assert list(sink[base + 8:base + 10]) == [1000 * b + 100, 0.5]                         # K, g=1, p=0
        assert list(sink[base + 10:base + 12]) == [-(1000 * b + 100), 0.25]                    # V, g=1
    # the ring of (b=1, g=0) holds positions 2, 3, 4 at slots 2, 0, 1
    r10 = img[(1 * 5 + 0) * 2 * d:]
    assert list(r10[0:6]) == [1003, 0.5, 1004, 0.5, 1002, 0.5]


def test_sink_decode_rejects_counts_above_the_cache():
    cache = kvcache.RingCache(1, 1, 2, [4], [2])
    cache.append(np.ones((1, 1, 6, 2)), np.ones((1, 1, 6, 2)))
    with pytest.raises(ValueError):
        kvcache.decode_sink(cache, np.ones((1, 1, 2)), [4], [3], 1.0)
    with pytest.raises(ValueError):
        kvcache.decode_sink(cache, np.ones((1, 1, 2)), [5], [1], 1.0)
