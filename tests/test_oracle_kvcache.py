"""Pins for the oracle's ring-buffer cache and decode (CPU only)."""

import collections
import math
import struct

import numpy as np
import pytest

from oracle import attention, kvcache


def test_ring_holds_last_capacity_tokens():
    """After any number of appends, the ring holds exactly the last C tokens (deque)."""
    rng = np.random.default_rng(0)
    B, Hkv, d = 2, 3, 2
    caps = [1, 4, 7]
    cache = kvcache.RingCache(B, Hkv, d, caps)
    ref = [[collections.deque(maxlen=c) for c in caps] for _ in range(B)]
    pos = 0
    for n in [3, 1, 1, 9, 2, 1, 15, 1]:
        k = rng.standard_normal((B, Hkv, n, d))
        v = rng.standard_normal((B, Hkv, n, d))
        cache.append(k, v)
        for b in range(B):
            for g in range(Hkv):
                for r in range(n):
                    ref[b][g].append((pos + r, k[b, g, r].copy(), v[b, g, r].copy()))
        pos += n
        for b in range(B):
            assert cache.t[b] == pos
            for g in range(Hkv):
                held = list(ref[b][g])
                K, V = cache.gather(b, g, [p for p, _, _ in held])
                assert np.array_equal(K, np.array([x for _, x, _ in held]))
                assert np.array_equal(V, np.array([x for _, _, x in held]))


def test_gather_rejects_evicted_positions():
    cache = kvcache.RingCache(1, 1, 1, [4])
    cache.append(np.zeros((1, 1, 10, 1)), np.zeros((1, 1, 10, 1)))
    with pytest.raises(ValueError):
        cache.gather(0, 0, [5])
    cache.gather(0, 0, [6, 7, 8, 9])


def test_decode_equals_last_prefill_row():
    """Decode at position t equals row t of prefill over t+1 tokens, bit for bit."""
    rng = np.random.default_rng(1)
    B, Hq, Hkv, d, N = 2, 4, 2, 8, 40
    spans = [3, 16, 9, 40]
    caps = kvcache.group_capacities(spans, Hkv)
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    cache = kvcache.RingCache(B, Hkv, d, caps)
    cache.append(k[:, :, :25], v[:, :, :25])
    full = attention.prefill(q, k, v, spans, 0.3)
    for t in range(25, N):
        cache.append(k[:, :, t:t + 1], v[:, :, t:t + 1])
        out = kvcache.decode(cache, q[:, :, t], spans, 0.3)
        assert np.array_equal(out, full[:, :, t])


def test_decode_rejects_span_above_capacity():
    cache = kvcache.RingCache(1, 1, 2, [4])
    cache.append(np.zeros((1, 1, 5, 2)), np.zeros((1, 1, 5, 2)))
    with pytest.raises(ValueError):
        kvcache.decode(cache, np.zeros((1, 1, 2)), [5], 1.0)


def test_group_capacities():
    assert kvcache.group_capacities([3, 9, 2, 2, 8, 1], 3) == [9, 2, 8]
    assert kvcache.group_capacities([5, 6], 2) == [5, 6]


def test_layout_sizes_and_offsets():
    """Hand-computed byte offsets of a small bf16 buffer."""
    B, Hkv, d = 2, 2, 4
    caps = [2, 3]
    assert kvcache.header_bytes(1) == 256
    assert kvcache.header_bytes(30) == 256
    assert kvcache.header_bytes(31) == 512
    assert kvcache.buffer_bytes(B, Hkv, d, caps, 2) == 256 + 2 * 5 * 2 * 4 * 2
    cache = kvcache.RingCache(B, Hkv, d, caps)
    # token values chosen exactly representable in bf16: value = 1 + pos/8 + b*4 + g*2
    for t in range(4):
        k = np.zeros((B, Hkv, 1, d))
        v = np.zeros((B, Hkv, 1, d))
        for b in range(B):
            for g in range(Hkv):
                k[b, g, 0, :] = 1 + t / 8 + b * 4 + g * 2
                v[b, g, 0, :] = -(1 + t / 8 + b * 4 + g * 2)
        cache.append(k, v)
    img = kvcache.data_image(cache, "bf16")
    assert len(img) == 2 * 5 * 2 * 4 * 2

    def bf16_at(elem_offset):
        (u,) = struct.unpack_from("<H", img, 2 * elem_offset)
        return struct.unpack("<f", struct.pack("<I", u << 16))[0]

    # b=1, g=1: element offset (b*sumC + P_g) * 2 * d = (1*5 + 2) * 8 = 56.
    # capacity 3, tokens 0..3 -> slots: token 3 in slot 0, tokens 1, 2 in slots 1, 2.
    base = 56
    assert bf16_at(base + 0 * d) == 1 + 3 / 8 + 4 + 2
    assert bf16_at(base + 1 * d) == 1 + 1 / 8 + 4 + 2
    assert bf16_at(base + 2 * d) == 1 + 2 / 8 + 4 + 2
    # V block follows the K block: + C_g * d
    assert bf16_at(base + 3 * d + 0 * d) == -(1 + 3 / 8 + 4 + 2)
    # b=0, g=0: capacity 2 -> token 2 in slot 0, token 3 in slot 1
    assert bf16_at(0) == 1 + 2 / 8
    assert bf16_at(d) == 1 + 3 / 8


def test_image_rejects_unrepresentable_values():
    cache = kvcache.RingCache(1, 1, 1, [1])
    cache.append(np.full((1, 1, 1, 1), 1.0 + 2.0 ** -12), np.zeros((1, 1, 1, 1)))
    with pytest.raises(ValueError):
        kvcache.data_image(cache, "bf16")
    kvcache.data_image(cache, "f32")
