"""Pins for the oracle's windowed attention (CPU only).

Each check fixes the oracle against something other than itself: brute force
with an explicit N x N mask, torch's dense causal SDPA when every span covers
the prompt, closed forms (span 1, zero queries), and invariants.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention


def _brute_force(q, k, v, spans, scale):
    """Pure-Python loops over an explicit N x N band mask (tiny inputs only)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = [[[[0.0] * d for _ in range(N)] for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            g = h // G
            S = spans[h]
            mask = [[(j <= i) and (j > i - S) for j in range(N)] for i in range(N)]
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
                    out[b][h][i][c] = sum(p * float(v[b, g, j, c]) for j, p in w) / z
    return np.array(out)


@pytest.mark.parametrize("case", [
    dict(B=1, Hq=3, Hkv=3, N=17, d=5, spans=[1, 4, 17]),
    dict(B=2, Hq=4, Hkv=2, N=13, d=4, spans=[2, 13, 40, 6]),
    dict(B=1, Hq=2, Hkv=1, N=24, d=3, spans=[7, 8]),
])
def test_matches_brute_force_mask(case):
    rng = np.random.default_rng(0)
    q = rng.standard_normal((case["B"], case["Hq"], case["N"], case["d"]))
    k = rng.standard_normal((case["B"], case["Hkv"], case["N"], case["d"]))
    v = rng.standard_normal((case["B"], case["Hkv"], case["N"], case["d"]))
    scale = 1.0 / math.sqrt(case["d"])
    got = attention.prefill(q, k, v, case["spans"], scale)
    ref = _brute_force(q, k, v, case["spans"], scale)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_full_span_equals_dense_causal_sdpa():
    """S_h >= N reduces to dense causal attention (torch SDPA, float64, CPU)."""
    rng = np.random.default_rng(1)
    B, H, N, d = 2, 3, 70, 16
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, H, N, d))
    v = rng.standard_normal((B, H, N, d))
    got = attention.prefill(q, k, v, [N, N + 5, 10 * N], 1.0 / math.sqrt(d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def test_span_one_returns_own_value():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 2, 33, 8))
    k = rng.standard_normal((1, 2, 33, 8))
    v = rng.standard_normal((1, 2, 33, 8))
    got = attention.prefill(q, k, v, [1, 1], 0.3)
    assert np.array_equal(got, v)


def test_zero_query_averages_window():
    """q = 0 gives uniform weights, so o[i] is the mean of v over i-S < j <= i."""
    rng = np.random.default_rng(3)
    N, d = 50, 6
    k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, d))
    q = np.zeros((1, 1, N, d))
    for S in (1, 2, 7, 49, 50, 64):
        got = attention.prefill(q, k, v, [S], 1.0)[0, 0]
        for i in range(N):
            lo = max(0, i - S + 1)
            assert np.allclose(got[i], v[0, 0, lo:i + 1].mean(axis=0), rtol=0, atol=1e-13)


def test_rows_sum_to_one():
    rng = np.random.default_rng(4)
    K = rng.standard_normal((300, 32))
    for S in (1, 5, 128, 300):
        for i in (0, 1, 77, 299):
            lo, hi = attention.window(i, S)
            w = attention.row_weights(rng.standard_normal(32) * 4, K, lo, hi, 0.25)
            assert len(w) == min(S, i + 1)
            assert abs(w.sum() - 1.0) < 1e-12 and np.all(w >= 0)


def test_gqa_equals_repeated_kv():
    """Grouped heads read kv head h // G: same as MHA on repeated K/V."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, N, d = 1, 6, 2, 20, 4
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    spans = [3, 20, 5, 1, 9, 12]
    got = attention.prefill(q, k, v, spans, 0.5)
    ref = attention.prefill(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), spans, 0.5)
    assert np.array_equal(got, ref)


def test_permutation_invariance_within_window():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((40, 8))
    V = rng.standard_normal((40, 8))
    q = rng.standard_normal(8)
    perm = rng.permutation(40)
    a = attention.attend_row(q, K, V, 0, 39, 0.7)
    b = attention.attend_row(q, K[perm], V[perm], 0, 39, 0.7)
    assert np.max(np.abs(a - b)) < 1e-13


def test_peaky_scores_stay_finite():
    """Scores far beyond exp's range: the row-max shift keeps the result finite."""
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, 16, 4)) * 400.0
    k = rng.standard_normal((1, 1, 16, 4))
    v = rng.standard_normal((1, 1, 16, 4))
    got = attention.prefill(q, k, v, [16], 1.0)
    assert np.all(np.isfinite(got))
    ref = _brute_force(q, k, v, [16], 1.0)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_rows_subset_matches_full():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((2, 4, 30, 4))
    k = rng.standard_normal((2, 2, 30, 4))
    v = rng.standard_normal((2, 2, 30, 4))
    spans = [1, 7, 30, 12]
    full = attention.prefill(q, k, v, spans, 0.5)
    rows = [(1, 3, 29), (0, 0, 0), (1, 1, 6), (0, 2, 17)]
    sub = attention.prefill(q, k, v, spans, 0.5, rows=rows)
    for n, (b, h, i) in enumerate(rows):
        assert np.array_equal(sub[n], full[b, h, i])


def test_in_window_flops_counts_mask_entries():
    for N, spans, d in [(10, [1, 3, 10, 20], 8), (257, [64, 128, 1, 300], 128)]:
        count = 0
        for S in spans:
            count += sum(1 for i in range(N) for j in range(N) if j <= i and j > i - S)
        assert attention.in_window_flops(spans, N, d) == 4 * d * count


def test_chunk_equals_prefill_rows_of_the_whole_sequence():
    """A chunk continuing a sequence gives the rows of prefill over the whole
    sequence at the chunk's positions (prefill is pinned to the brute-force
    mask above)."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, d, t, n = 2, 4, 2, 8, 23, 9
    spans = [1, 5, 40, 17]
    k = rng.standard_normal((B, Hkv, t + n, d))
    v = rng.standard_normal((B, Hkv, t + n, d))
    q_full = rng.standard_normal((B, Hq, t + n, d))
    want = attention.prefill(q_full, k, v, spans, 0.3)[:, :, t:, :]
    got = attention.chunk(q_full[:, :, t:, :], [k[b] for b in range(B)], [v[b] for b in range(B)], [t, t], spans, 0.3)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_chunk_at_position_zero_is_prefill_of_the_chunk():
    rng = np.random.default_rng(32)
    q = rng.standard_normal((1, 2, 11, 4))
    k = rng.standard_normal((1, 1, 11, 4))
    v = rng.standard_normal((1, 1, 11, 4))
    got = attention.chunk(q, [k[0]], [v[0]], [0], [3, 11], 0.5)
    np.testing.assert_allclose(got, attention.prefill(q, k, v, [3, 11], 0.5), rtol=0, atol=1e-12)


def test_chunk_of_one_token_equals_ring_decode():
    """n = 1 is one decode step: the ring-buffer emulation (its own pins in
    test_oracle_kvcache) reads the same window through the ring."""
    from oracle import kvcache as okv
    rng = np.random.default_rng(33)
    B, Hq, Hkv, d = 2, 4, 2, 8
    spans = [7, 2, 12, 12]
    caps = okv.group_capacities(spans, Hkv)
    t = [30, 5]
    hist_k = [rng.standard_normal((Hkv, tb + 1, d)) for tb in t]
    hist_v = [rng.standard_normal((Hkv, tb + 1, d)) for tb in t]
    q = rng.standard_normal((B, Hq, 1, d))
    got = attention.chunk(q, hist_k, hist_v, t, spans, 0.25)[:, :, 0, :]
    want = np.empty_like(got)
    for b in range(B):
        ring = okv.RingCache(1, Hkv, d, caps)
        for p in range(t[b] + 1):
            ring.append(hist_k[b][None, :, p:p + 1, :], hist_v[b][None, :, p:p + 1, :])
        want[b] = okv.decode(ring, q[b:b + 1, :, 0, :], spans, 0.25)[0]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_chunk_rows_subset_and_shape_checks():
    rng = np.random.default_rng(34)
    q = rng.standard_normal((2, 2, 5, 4))
    hk = [rng.standard_normal((1, 8, 4)), rng.standard_normal((1, 6, 4))]
    hv = [rng.standard_normal((1, 8, 4)), rng.standard_normal((1, 6, 4))]
    full = attention.chunk(q, hk, hv, [3, 1], [4, 2], 0.5)
    rows = [(1, 0, 4), (0, 1, 0)]
    np.testing.assert_array_equal(attention.chunk(q, hk, hv, [3, 1], [4, 2], 0.5, rows=rows),
                                  np.stack([full[b, h, i] for b, h, i in rows]))
    with pytest.raises(ValueError):
        attention.chunk(q, hk, hv, [3, 2], [4, 2], 0.5)       # history length does not match t + n
