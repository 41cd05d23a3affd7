"""The oracle's pins catch plausible mistakes (CPU only).

Each test plants one mistake in the oracle (a monkeypatched copy of one of its
functions: a window one key too wide, a dropped term, a wrong index, a
transposed operand, a wrong rounding) and checks that at least one of the
existing pins in test_oracle_*.py now fails.  A pin that also passed on the
mutant would not pin that part of the oracle.
"""

import importlib.util
import math
import os

import numpy as np
import pytest

from oracle import attention, kvcache, rules

_HERE = os.path.dirname(os.path.abspath(__file__))


def _pins(name):
    spec = importlib.util.spec_from_file_location("pins_" + name, os.path.join(_HERE, name + ".py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


ATT = _pins("test_oracle_attention")
KV = _pins("test_oracle_kvcache")
RULES = _pins("test_oracle_rules")
BRUTE_CASES = [dict(B=1, Hq=3, Hkv=3, N=17, d=5, spans=[1, 4, 17]),
               dict(B=2, Hq=4, Hkv=2, N=13, d=4, spans=[2, 13, 40, 6])]


def _fails(fn, *args):
    """True when the pin fn(*args) no longer passes."""
    try:
        fn(*args)
    except Exception:      # an assertion or any error raised by the planted mistake
        return True
    return False


def _any_brute_force_fails():
    return any(_fails(ATT.test_matches_brute_force_mask, c) for c in BRUTE_CASES)


def test_pins_pass_on_the_oracle_as_written():
    assert not _any_brute_force_fails()
    assert not _fails(ATT.test_chunk_equals_prefill_rows_of_the_whole_sequence)
    assert not _fails(KV.test_layout_sizes_and_offsets)
    assert not _fails(KV.test_decode_equals_last_prefill_row)
    assert not _fails(KV.test_ring_holds_last_capacity_tokens)
    assert not _fails(ATT.test_in_window_flops_counts_mask_entries)


def test_window_one_key_too_wide_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "window", lambda i, S: (max(0, i - S), i))
    assert _any_brute_force_fails()
    assert _fails(ATT.test_span_one_returns_own_value)


def test_window_without_the_diagonal_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "window", lambda i, S: (max(0, i - S), i - 1))
    assert _any_brute_force_fails()


def test_scale_applied_twice_is_caught(monkeypatch):
    orig = attention.row_weights
    monkeypatch.setattr(attention, "row_weights", lambda q_i, K, lo, hi, scale: orig(q_i, K, lo, hi, scale * scale))
    assert _any_brute_force_fails()
    assert _fails(ATT.test_full_span_equals_dense_causal_sdpa)


def test_keys_used_as_values_is_caught(monkeypatch):
    def attend_row(q_i, K, V, lo, hi, scale):
        w = attention.row_weights(q_i, K, lo, hi, scale)
        return w @ np.asarray(K[lo:hi + 1], dtype=np.float64)      # transposed operand: K for V
    monkeypatch.setattr(attention, "attend_row", attend_row)
    assert _any_brute_force_fails()


def test_unnormalised_weights_are_caught(monkeypatch):
    def row_weights(q_i, K, lo, hi, scale):
        s = (np.asarray(K[lo:hi + 1], dtype=np.float64) @ np.asarray(q_i, dtype=np.float64)) * scale
        return np.exp(s - s.max())                                   # dropped division by the sum
    monkeypatch.setattr(attention, "row_weights", row_weights)
    assert _any_brute_force_fails()
    assert _fails(ATT.test_rows_sum_to_one)


def test_wrong_kv_head_for_a_query_head_is_caught(monkeypatch):
    orig_attend = attention.attend_row

    def prefill(q, k, v, spans, scale, rows=None):
        # query head h reads kv head h % Hkv instead of h // G
        q = np.asarray(q)
        k = np.asarray(k)
        v = np.asarray(v)
        B, Hq, N, d = q.shape
        Hkv = k.shape[1]
        out = np.empty((B, Hq, N, d))
        for b in range(B):
            for h in range(Hq):
                for i in range(N):
                    lo, hi = attention.window(i, int(spans[h]))
                    out[b, h, i] = orig_attend(q[b, h, i], k[b, h % Hkv], v[b, h % Hkv], lo, hi, scale)
        return out
    monkeypatch.setattr(attention, "prefill", prefill)
    assert _fails(ATT.test_gqa_equals_repeated_kv)


def test_chunk_positions_one_early_are_caught(monkeypatch):
    def chunk(q, k_hist, v_hist, t, spans, scale, rows=None):
        q = np.asarray(q)
        B, Hq, n, d = q.shape
        G = Hq // np.asarray(k_hist[0]).shape[0]
        out = np.empty((B, Hq, n, d))
        for b in range(B):
            for h in range(Hq):
                for i in range(n):
                    P = max(int(t[b]) + i - 1, 0)                    # off by one
                    lo, hi = attention.window(P, int(spans[h]))
                    out[b, h, i] = attention.attend_row(q[b, h, i], k_hist[b][h // G], v_hist[b][h // G], lo, hi,
                                                        scale)
        return out
    monkeypatch.setattr(attention, "chunk", chunk)
    assert _fails(ATT.test_chunk_equals_prefill_rows_of_the_whole_sequence)


def test_ring_slot_shifted_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(kvcache.RingCache, "slot", staticmethod(lambda p, C: (p + 1) % C))
    assert _fails(KV.test_layout_sizes_and_offsets)


def test_decode_window_one_key_too_wide_is_caught(monkeypatch):
    def window_positions(self, b, S):
        t = self.t[b]
        return list(range(max(0, t - S - 1), t))
    monkeypatch.setattr(kvcache.RingCache, "window_positions", window_positions)
    assert _fails(KV.test_decode_equals_last_prefill_row)


def _span_variant(rounding, clamp=True):
    def span_rule(alpha, beta, N, block):
        x = float(alpha) + float(beta) * float(N)
        s = float(block) * rounding(x / float(block))
        if clamp:
            s = min(float(N), max(float(block), s))
        return int(s)
    return span_rule


def test_span_rounded_down_is_caught(monkeypatch):
    monkeypatch.setattr(rules, "span_rule", _span_variant(math.floor))
    assert _fails(RULES.test_rule_matches_brute_force_nearest_multiple)


def test_span_ties_rounded_down_is_caught(monkeypatch):
    monkeypatch.setattr(rules, "span_rule", _span_variant(lambda y: math.ceil(y - 0.5)))
    assert _fails(RULES.test_exact_tie_rounds_up)


def test_span_without_the_clamp_is_caught(monkeypatch):
    monkeypatch.setattr(rules, "span_rule", _span_variant(lambda y: math.floor(y + 0.5), clamp=False))
    assert _fails(RULES.test_clamps)
    assert any(_fails(RULES.test_project_page_worked_heads, row) for row in RULES._golden_rows())


def test_ring_keeping_the_first_rows_of_a_long_append_is_caught(monkeypatch):
    def append(self, k, v):
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        B, Hkv, n, d = k.shape
        for b in range(B):
            for g in range(Hkv):
                C = self.C[g]
                for r in range(min(n, C)):                           # the first C rows, not the last
                    s = self.slot(self.t[b] + r, C)
                    self.K[b][g][s] = k[b, g, r]
                    self.V[b][g][s] = v[b, g, r]
                    self.written[b][g][s] = True
            self.t[b] += n
    monkeypatch.setattr(kvcache.RingCache, "append", append)
    assert _fails(KV.test_ring_holds_last_capacity_tokens)


def test_ring_not_advancing_positions_is_caught(monkeypatch):
    orig = kvcache.RingCache.append

    def append(self, k, v):
        t = list(self.t)
        orig(self, k, v)
        self.t = t                                                   # t_b += n dropped
    monkeypatch.setattr(kvcache.RingCache, "append", append)
    assert _fails(KV.test_ring_holds_last_capacity_tokens)


def test_flops_without_the_causal_triangle_is_caught(monkeypatch):
    def in_window_flops(spans, N, d, B=1):
        return B * sum(4 * d * min(int(S), int(N)) * N for S in spans)   # dropped S(S-1)/2 term
    monkeypatch.setattr(attention, "in_window_flops", in_window_flops)
    assert _fails(ATT.test_in_window_flops_counts_mask_entries)


# ---- band plus global tokens -------------------------------------------------
SINK = _pins("test_oracle_sink")


def _any_sink_brute_force_fails():
    return any(_fails(SINK.test_sink_matches_brute_force_mask, c) for c in SINK.SINK_CASES)


def _keys_mutant(glob_fn, join="union"):
    def keys(i, S, k):
        lo, hi = attention.window(i, S)
        band = list(range(lo, hi + 1))
        glob = list(glob_fn(i, k))
        return sorted(set(band) | set(glob)) if join == "union" else sorted(band + glob)
    return keys


def test_sink_pins_pass_on_the_oracle_as_written():
    assert not _any_sink_brute_force_fails()
    for args in [(7, 3, 30), (16, 16, 40), (5, 9, 25)]:
        assert not _fails(SINK.test_sink_decode_equals_last_prefill_row, *args)
    assert not _fails(SINK.test_sink_image_layout_hand_computed)


def test_global_range_one_too_wide_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "keys_sink", _keys_mutant(lambda i, k: range(0, min(k + 1, i + 1))))
    assert _any_sink_brute_force_fails()


def test_global_tokens_ignoring_causality_are_caught(monkeypatch):
    monkeypatch.setattr(attention, "keys_sink", _keys_mutant(lambda i, k: range(0, k)))
    assert _any_sink_brute_force_fails()


def test_keys_in_band_and_global_counted_twice_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "keys_sink", _keys_mutant(lambda i, k: range(0, min(k, i + 1)), join="concat"))
    assert _any_sink_brute_force_fails()


def test_global_rows_read_through_the_ring_is_caught(monkeypatch):
    def gather_ring_only(self, b, g, positions):
        C = self.C[g]
        idx = [p % C for p in positions]
        return self.K[b][g][idx], self.V[b][g][idx]
    monkeypatch.setattr(kvcache.RingCache, "gather_any", gather_ring_only)
    assert any(_fails(SINK.test_sink_decode_equals_last_prefill_row, *a) for a in [(7, 3, 30), (5, 9, 25)])


def test_global_rows_not_kept_at_append_is_caught(monkeypatch):
    orig = kvcache.RingCache.append

    def append_no_globals(self, k, v):
        saved = self.sinks
        self.sinks = [0] * self.Hkv
        try:
            orig(self, k, v)
        finally:
            self.sinks = saved
    monkeypatch.setattr(kvcache.RingCache, "append", append_no_globals)
    assert _fails(SINK.test_sink_image_layout_hand_computed)
    assert any(_fails(SINK.test_sink_decode_equals_last_prefill_row, *a) for a in [(7, 3, 30), (5, 9, 25)])
