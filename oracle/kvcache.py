"""Oracle: fixed-size per-head ring-buffer KV cache and decode.  TEST INFRASTRUCTURE ONLY.

What the method computes
------------------------
"Mixture of Attention" project page, section "Demo", step 03: inference is
deployed with a fixed-size, sparse KV cache whose size differs per head; the
section "Inference speed and memory efficiency" says MoA bounds the KV cache
size.  The blog walkthrough (section 5) implements a static KV cache in its
CUDA kernel.  A head with span S only ever reads its last S keys, so a
cache of capacity C >= S that keeps the last C rows serves it exactly.

Readings taken where the pages are silent:

* Spans are evaluated once, at the configured context length N, and stay
  fixed through decoding (the cache is static).
* Grouped-query attention: the cache of key/value head g has capacity
  C_g = max of the spans of the query heads reading it.
* Ring addressing: token position p of a sequence lives in slot p mod C_g.
* Append-then-attend: a decode step first appends the new token's k, v at
  position t (the count of tokens already cached), then the query at
  position t attends to positions j with t - S_h < j <= t.

Byte image of the device buffer
-------------------------------
The device cache is one caller-owned buffer laid out as

* header of ``align_up(16 + 8*B, 256)`` bytes: uint32 error word at byte 0,
  bytes 4..15 reserved, then int64 ``t[B]`` (tokens cached per sequence);
* data: for b in 0..B-1, for g in 0..Hkv-1, the K block [C_g, d] followed by
  the V block [C_g, d], row-major, elements of the cache dtype;
* for a cache that keeps global tokens (k_g of them for kv head g), after
  that: for b, for g, Ksink [k_g, d] then Vsink [k_g, d], position p < k_g at
  row p.

:func:`data_image` rebuilds the data region byte for byte from this
description so tests can compare the GPU buffer bit-exactly.
"""

import numpy as np

from .attention import attend_row


class RingCache:
    """Python emulation of the per-(sequence, kv-head) ring buffers."""

    def __init__(self, B, Hkv, d, capacities, sinks=None):
        if len(capacities) != Hkv:
            raise ValueError("one capacity per kv head")
        if any(int(c) < 1 for c in capacities):
            raise ValueError("capacities must be >= 1")
        sinks = [0] * Hkv if sinks is None else [int(x) for x in sinks]
        if len(sinks) != Hkv or any(x < 0 for x in sinks):
            raise ValueError("one global token count >= 0 per kv head")
        self.B, self.Hkv, self.d = int(B), int(Hkv), int(d)
        self.C = [int(c) for c in capacities]
        self.K = [[np.zeros((c, d), dtype=np.float64) for c in self.C] for _ in range(B)]
        self.V = [[np.zeros((c, d), dtype=np.float64) for c in self.C] for _ in range(B)]
        self.written = [[np.zeros(c, dtype=bool) for c in self.C] for _ in range(B)]
        # global tokens: positions p < sinks[g] are also kept, for good, at sink slot p
        self.sinks = sinks
        self.Ks = [[np.zeros((x, d), dtype=np.float64) for x in sinks] for _ in range(B)]
        self.Vs = [[np.zeros((x, d), dtype=np.float64) for x in sinks] for _ in range(B)]
        self.t = [0] * B

    @staticmethod
    def slot(p, C):
        """Ring slot of token position ``p`` in a buffer of capacity ``C``."""
        return p % C

    def append(self, k, v):
        """Append ``n`` tokens per sequence: k, v are [B, Hkv, n, d].

        Every row is written in order to slot (t_b + r) mod C_g, so when n > C_g
        later rows overwrite earlier ones and the ring ends up holding the last
        C_g of them.  Then t_b += n.
        """
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        B, Hkv, n, d = k.shape
        if (B, Hkv, d) != (self.B, self.Hkv, self.d) or v.shape != k.shape:
            raise ValueError("append shape mismatch")
        for b in range(B):
            for g in range(Hkv):
                C = self.C[g]
                for r in range(n):
                    s = self.slot(self.t[b] + r, C)
                    self.K[b][g][s] = k[b, g, r]
                    self.V[b][g][s] = v[b, g, r]
                    self.written[b][g][s] = True
                    if self.t[b] + r < self.sinks[g]:
                        self.Ks[b][g][self.t[b] + r] = k[b, g, r]
                        self.Vs[b][g][self.t[b] + r] = v[b, g, r]
            self.t[b] += n

    def window_positions(self, b, S):
        """Token positions the newest query of sequence b attends to under span S."""
        t = self.t[b]
        if t < 1:
            raise ValueError("no tokens cached")
        return list(range(max(0, t - S), t))

    def gather(self, b, g, positions):
        """K and V rows of the given token positions, read through the ring."""
        C = self.C[g]
        t = self.t[b]
        for p in positions:
            if p < t - C or p >= t:
                raise ValueError("position %d is not held by the ring" % p)
        idx = [self.slot(p, C) for p in positions]
        return self.K[b][g][idx], self.V[b][g][idx]


    def gather_any(self, b, g, positions):
        """K and V rows of the given positions, each read from the ring when the ring still
        holds it, else from the global-token rows (positions below sinks[g])."""
        C = self.C[g]
        t = self.t[b]
        Ks, Vs = [], []
        for p in positions:
            if t - C <= p < t:
                Ks.append(self.K[b][g][self.slot(p, C)])
                Vs.append(self.V[b][g][self.slot(p, C)])
            elif 0 <= p < min(self.sinks[g], t):
                Ks.append(self.Ks[b][g][p])
                Vs.append(self.Vs[b][g][p])
            else:
                raise ValueError("position %d is held neither by the ring nor as a global token" % p)
        return np.array(Ks), np.array(Vs)


def decode_sink(cache, q, spans, sinks, scale):
    """One decode step with global tokens: the query of position t = t_b - 1 of (b, h) attends
    to keys_sink(t, S_h, k_h) of kv head g = h // (Hq // Hkv) (its band through the ring, the
    first k_h positions through the global-token rows).  Needs S_h <= C_g and k_h <= sinks[g].
    Returns float64 [B, Hq, d]."""
    from .attention import keys_sink
    q = np.asarray(q)
    B, Hq, d = q.shape
    if Hq % cache.Hkv != 0 or len(spans) != Hq or len(sinks) != Hq:
        raise ValueError("shape mismatch")
    G = Hq // cache.Hkv
    out = np.empty((B, Hq, d), dtype=np.float64)
    for b in range(B):
        if cache.t[b] < 1:
            raise ValueError("no tokens cached")
        for h in range(Hq):
            g = h // G
            S, kk = int(spans[h]), int(sinks[h])
            if S > cache.C[g] or kk > cache.sinks[g]:
                raise ValueError("span or global token count exceeds the kv head's cache")
            keys = keys_sink(cache.t[b] - 1, S, kk)
            K, V = cache.gather_any(b, g, keys)
            out[b, h] = attend_row(q[b, h], K, V, 0, len(keys) - 1, scale)
    return out


def decode(cache, q, spans, scale):
    """One decode step: q [B, Hq, d] is the query of the token at position t_b - 1.

    For each (b, h) attends to positions j in (t_b - 1 - S_h, t_b - 1], read
    from the ring of kv head g = h // (Hq // Hkv).  Returns float64 [B, Hq, d].
    """
    q = np.asarray(q)
    B, Hq, d = q.shape
    if Hq % cache.Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // cache.Hkv
    out = np.empty((B, Hq, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            S = int(spans[h])
            if S > cache.C[g]:
                raise ValueError("span exceeds the kv head's capacity")
            pos = cache.window_positions(b, S)
            K, V = cache.gather(b, g, pos)
            out[b, h] = attend_row(q[b, h], K, V, 0, len(pos) - 1, scale)
    return out


def group_capacities(spans, Hkv):
    """C_g = max span over the query heads that read kv head g."""
    Hq = len(spans)
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    return [max(int(s) for s in spans[g * G:(g + 1) * G]) for g in range(Hkv)]


def header_bytes(B):
    """Size of the buffer header: 16 bytes + int64 t[B], rounded up to 256."""
    return ((16 + 8 * int(B)) + 255) // 256 * 256


def buffer_bytes(B, Hkv, d, capacities, elem_bytes, sinks=None):
    """Total size of the device buffer for the documented layout (global-token rows after the ring)."""
    rows = sum(int(c) for c in capacities) + (sum(int(x) for x in sinks) if sinks else 0)
    return header_bytes(B) + int(B) * rows * 2 * int(d) * int(elem_bytes)


def _to_bits(x, dtype):
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        f = x.astype(np.float32)
        if not np.array_equal(f.astype(np.float64), x):
            raise ValueError("value not representable in fp32")
        return f.view(np.uint32).astype("<u4").tobytes()
    if dtype == "bf16":
        f = x.astype(np.float32)
        u = f.view(np.uint32)
        if not np.array_equal(f.astype(np.float64), x) or np.any(u & 0xFFFF):
            raise ValueError("value not representable in bf16")
        return (u >> 16).astype("<u2").tobytes()
    raise ValueError("dtype must be 'f32' or 'bf16'")


def data_image(cache, dtype):
    """Bytes of the data region: per b, per g, K[C_g, d] then V[C_g, d]; then, when the cache
    keeps global tokens, per b, per g, Ksink[k_g, d] then Vsink[k_g, d] (slot p = position p)."""
    parts = []
    for b in range(cache.B):
        for g in range(cache.Hkv):
            parts.append(_to_bits(cache.K[b][g], dtype))
            parts.append(_to_bits(cache.V[b][g], dtype))
    for b in range(cache.B):
        for g in range(cache.Hkv):
            if cache.sinks[g]:
                parts.append(_to_bits(cache.Ks[b][g], dtype))
                parts.append(_to_bits(cache.Vs[b][g], dtype))
    return b"".join(parts)


def block_from_image(data, b, g, B, Hkv, d, capacities, dtype):
    """K and V rows [C_g, d] of (sequence b, kv head g) read from a data-region image.

    ``data`` is a bytes-like image of the data region laid out as documented
    above; returns float64 arrays in slot order.
    """
    eb = 4 if dtype == "f32" else 2
    sumC = sum(int(c) for c in capacities)
    C = int(capacities[g])
    start = (b * sumC + sum(int(c) for c in capacities[:g])) * 2 * d
    raw = np.frombuffer(bytes(data[start * eb:(start + 2 * C * d) * eb]),
                        dtype="<u4" if eb == 4 else "<u2")
    if eb == 4:
        vals = raw.view("<f4").astype(np.float64)
    else:
        vals = (raw.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    vals = vals.reshape(2, C, d)
    return vals[0].copy(), vals[1].copy()


def decode_row_from_ring(K, V, t, S, q, scale):
    """Decode output of one (b, h) whose ring (slot order) is K, V after t tokens.

    Attends to positions max(0, t - S) .. t - 1, each read from slot p mod C.
    """
    C = K.shape[0]
    if S > C:
        raise ValueError("span exceeds capacity")
    pos = list(range(max(0, t - S), t))
    idx = [p % C for p in pos]
    return attend_row(q, K[idx], V[idx], 0, len(idx) - 1, scale)
