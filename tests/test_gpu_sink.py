"""GPU parity of the band-plus-global-token path against the fp64 oracle.

Reading (codewithpapers page for arXiv 2406.14909: the official repository's
gen_global_pattern and StreamingLLM density counters): head h attends to its
band (i - S_h, i] and to the first k_h positions (those <= i), each key once.
Tolerances as for the plain path: fp32 max-abs 1e-5, bf16 max-abs 2e-2 against
the oracle on the same bf16 values; cache bytes (ring and global-token rows)
bit-exact against the oracle's byte image.  Outputs are pre-filled with NaN.
"""

import math

import numpy as np
import pytest
import torch

from heterogeneous_sliding_window_b200 import inputs, moa
from oracle import attention as oatt, kvcache as okv

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
F32_TOL = 1e-5
DEV = "cuda"


def _nan(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, device=DEV)


def _prefill_sink(q, k, v, spans, sinks, scale, dt, fill=None):
    B, Hq, N, d = q.shape
    o = _nan((B, Hq, N, d), q.dtype)
    ws = moa.Workspace(moa.MOA_OP_PREFILL, B, Hq, N, d, spans) if dt == "bf16" else None
    moa.moa_prefill_sink(q, k, v, o, B, Hq, k.shape[1], N, d, dt, spans, sinks, scale,
                         ws.ptr if ws else None, ws.nbytes if ws else 0, fill.handle if fill is not None else None)
    if ws is not None:
        moa.moa_workspace_check(ws.ptr)
    torch.cuda.synchronize()
    return o


def _group_max(x, Hkv):
    G = len(x) // Hkv
    return [max(x[g * G:(g + 1) * G]) for g in range(Hkv)]


def test_tiny_fp32_prefill_fill_and_decode_with_global_tokens():
    """Tiny fp32 layer (B=1, 4 heads, d=64, N=256, spans {32, 64, 128, 256}) with 4, 16, 0 and
    100 global tokens: prefill with the cache fill, then 16 fused decode steps, at 1e-5, with the
    ring and global-token bytes bit-exact after the prompt and after the steps."""
    B, H, d, N = 1, 4, 64, 256
    spans, sinks = [32, 64, 128, 256], [4, 16, 0, 100]
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn(600, (B, H, N, d), "f32")
    k = inputs.randn(601, (B, H, N, d), "f32")
    v = inputs.randn(602, (B, H, N, d), "f32")
    cache = moa.KVCache(B, H, d, "f32", spans, sink_capacity=sinks)
    o = _prefill_sink(q.to(DEV), k.to(DEV), v.to(DEV), spans, sinks, scale, "f32", fill=cache)
    ref = oatt.prefill_sink(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, sinks, scale)
    assert np.max(np.abs(inputs.as_f64(o) - ref)) <= F32_TOL
    ring = okv.RingCache(B, H, d, spans, sinks)
    ring.append(inputs.as_f64(k), inputs.as_f64(v))
    assert cache.positions() == ring.t == [N]
    assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "f32")
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, H, 0, d, spans)
    nb = moa.moa_workspace_bytes_sink(moa.MOA_OP_DECODE, B, H, 0, d, spans, sinks)
    wsb = torch.zeros(nb + 256, dtype=torch.uint8, device=DEV)
    wptr = (wsb.data_ptr() + 255) // 256 * 256
    del ws
    for step in range(16):
        qt = inputs.randn(610 + step, (B, H, d), "f32")
        kt = inputs.randn(630 + step, (B, H, 1, d), "f32")
        vt = inputs.randn(650 + step, (B, H, 1, d), "f32")
        ot = _nan((B, H, d), torch.float32)
        moa.moa_decode_append_sink(cache.handle, qt.to(DEV), kt.to(DEV), vt.to(DEV), ot, H, spans, sinks, scale,
                                   wptr, nb)
        torch.cuda.synchronize()
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        ref_t = okv.decode_sink(ring, inputs.as_f64(qt), spans, sinks, scale)
        assert np.max(np.abs(inputs.as_f64(ot) - ref_t)) <= F32_TOL, step
    assert cache.positions() == ring.t == [N + 16]
    assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "f32")


PREFILL_CASES = [
    # (B, Hq, Hkv, N, spans, sinks)
    (1, 4, 4, 1000, [1, 64, 200, 1000], [4, 300, 129, 0]),        # global tiles below and inside the band
    (2, 8, 2, 700, [1, 127, 128, 129, 256, 300, 700, 64], [1, 128, 127, 700, 5000, 256, 3, 385]),
    (1, 2, 1, 513, [384, 100], [64, 513]),                        # odd number of query tiles
    (1, 3, 3, 128, [128, 1, 37], [5, 128, 1]),                    # exactly one tile
    (1, 2, 2, 1, [1, 5], [1, 7]),                                 # a single token
    (1, 4, 2, 2300, [64, 256, 500, 129], [256, 1, 1024, 640]),    # several global tiles, long bands
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "B%d_H%d_%d_N%d" % c[:4])
def test_bf16_prefill_with_global_tokens_matches_oracle(case):
    B, Hq, Hkv, N, spans, sinks = case
    d = 128
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn(701, (B, Hq, N, d))
    k = inputs.randn(702, (B, Hkv, N, d))
    v = inputs.randn(703, (B, Hkv, N, d))
    o = _prefill_sink(q.to(DEV), k.to(DEV), v.to(DEV), spans, sinks, scale, "bf16")
    ref = oatt.prefill_sink(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, sinks, scale)
    err = np.max(np.abs(inputs.as_f64(o) - ref))
    assert err <= BF16_TOL, err


def test_bf16_prefill_without_global_tokens_equals_plain_prefill():
    """sinks all 0 through moa_prefill_sink gives moa_prefill's output bit for bit."""
    B, Hq, Hkv, N, d = 2, 8, 2, 700, 128
    spans = [1, 127, 128, 129, 256, 300, 700, 5000]
    q = inputs.randn(711, (B, Hq, N, d)).to(DEV)
    k = inputs.randn(712, (B, Hkv, N, d)).to(DEV)
    v = inputs.randn(713, (B, Hkv, N, d)).to(DEV)
    o1 = _prefill_sink(q, k, v, spans, [0] * Hq, 0.088, "bf16")
    o2 = _nan((B, Hq, N, d), torch.bfloat16)
    ws = moa.Workspace(moa.MOA_OP_PREFILL, B, Hq, N, d, spans)
    moa.moa_prefill(q, k, v, o2, B, Hq, Hkv, N, d, "bf16", spans, 0.088, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_bf16_prefill_fill_keeps_global_rows_bit_exact():
    """The prefill kernel's cache writer fills the ring and the global-token rows of a GQA
    cache, after a prompt that already sits in the cache (positions continue)."""
    B, Hq, Hkv, N, d = 2, 4, 2, 600, 128
    spans, sinks = [64, 256, 600, 100], [100, 3, 0, 300]
    caps, scaps = _group_max(spans, Hkv), [128, 300]
    cache = moa.KVCache(B, Hkv, d, "bf16", caps, sink_capacity=scaps)
    ring = okv.RingCache(B, Hkv, d, caps, scaps)
    for rep, n in enumerate([N, 77]):
        q = inputs.randn(720 + rep, (B, Hq, n, d))
        k = inputs.randn(730 + rep, (B, Hkv, n, d))
        v = inputs.randn(740 + rep, (B, Hkv, n, d))
        o = _prefill_sink(q.to(DEV), k.to(DEV), v.to(DEV), spans, sinks, 0.1, "bf16", fill=cache)
        ring.append(inputs.as_f64(k), inputs.as_f64(v))
        assert cache.positions() == ring.t
        assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16"), rep
        ref = oatt.prefill_sink(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, sinks, 0.1)
        assert np.max(np.abs(inputs.as_f64(o) - ref)) <= BF16_TOL, rep


def test_append_keeps_global_rows_bit_exact():
    B, Hkv, d = 3, 3, 128
    caps, scaps = [1, 70, 300], [5, 0, 600]
    cache = moa.KVCache(B, Hkv, d, "bf16", caps, sink_capacity=scaps)
    ring = okv.RingCache(B, Hkv, d, caps, scaps)
    for step, n in enumerate([3, 1, 299, 1, 64, 700, 1]):
        k = inputs.randn(750 + step, (B, Hkv, n, d))
        v = inputs.randn(760 + step, (B, Hkv, n, d))
        cache.append(k.to(DEV), v.to(DEV))
        ring.append(inputs.as_f64(k), inputs.as_f64(v))
        torch.cuda.synchronize()
        assert cache.positions() == ring.t
        assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16"), step


DECODE_CASES = [
    # (B, Hq, Hkv, dtype, d, prefix, spans, sinks, steps)
    (2, 4, 4, "bf16", 128, 900, [1, 256, 257, 900], [4, 600, 0, 1], 3),         # a head with two global splits
    (3, 8, 2, "bf16", 128, 50, [40, 7, 64, 64, 300, 1, 299, 17], [8, 64, 0, 3, 100, 1, 60, 64], 4),  # GQA, short
    (1, 4, 1, "bf16", 128, 2000, [1000, 513, 2000, 1], [1000, 16, 0, 1024], 2),  # ring wraps past the globals
    (2, 16, 2, "bf16", 128, 700, [700, 3, 300, 301, 64, 1, 699, 500,
                                  2, 500, 512, 513, 257, 5, 600, 40], [4] * 16, 2),   # 8 heads per KV head
    (2, 4, 2, "f32", 64, 0, [1, 5, 32, 17], [2, 0, 40, 40], 48),                 # from an empty cache
    # 4 heads per KV head, global-token counts differing within each group, two global splits
    (2, 8, 2, "bf16", 128, 2600, [2000, 300, 2500, 64, 1200, 1, 800, 2100], [1500, 0, 3, 1100, 0, 0, 2000, 64], 2),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "B%d_H%d_%d_%s_T%d" % (c[0], c[1], c[2], c[3], c[5]))
def test_decode_with_global_tokens_matches_oracle(case):
    """moa_decode_append_sink against the oracle's decode with global tokens, and moa_kv_append
    followed by moa_decode_sink giving the same bits, cache bytes and positions."""
    B, Hq, Hkv, dt, d, prefix, spans, sinks, steps = case
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    bits = torch.int16 if dt == "bf16" else torch.int32
    tol = BF16_TOL if dt == "bf16" else F32_TOL
    scale = 1.0 / math.sqrt(d)
    caps, scaps = _group_max(spans, Hkv), _group_max(sinks, Hkv)
    one = moa.KVCache(B, Hkv, d, dt, caps, sink_capacity=scaps)
    two = moa.KVCache(B, Hkv, d, dt, caps, sink_capacity=scaps)
    ring = okv.RingCache(B, Hkv, d, caps, scaps)
    if prefix:
        k0 = inputs.randn(770, (B, Hkv, prefix, d), dt)
        v0 = inputs.randn(771, (B, Hkv, prefix, d), dt)
        for c in (one, two):
            c.append(k0.to(DEV), v0.to(DEV))
        ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
    nb = moa.moa_workspace_bytes_sink(moa.MOA_OP_DECODE, B, Hq, 0, d, spans, sinks)
    wbuf = [torch.zeros(nb + 256, dtype=torch.uint8, device=DEV) for _ in range(2)]
    wp = [(w.data_ptr() + 255) // 256 * 256 for w in wbuf]
    for step in range(steps):
        qt = (inputs.randn(780 + step, (B, Hq, d), "f32") * (1 + step % 3)).to(tdt)
        kt = inputs.randn(800 + step, (B, Hkv, 1, d), dt)
        vt = inputs.randn(820 + step, (B, Hkv, 1, d), dt)
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        o1 = _nan((B, Hq, d), tdt)
        o2 = _nan((B, Hq, d), tdt)
        moa.moa_decode_append_sink(one.handle, qt.to(DEV), kt.to(DEV), vt.to(DEV), o1, Hq, spans, sinks, scale,
                                   wp[0], nb)
        two.append(kt.to(DEV), vt.to(DEV))
        moa.moa_decode_sink(two.handle, qt.to(DEV), o2, Hq, spans, sinks, scale, wp[1], nb)
        torch.cuda.synchronize()
        ref = okv.decode_sink(ring, inputs.as_f64(qt), spans, sinks, scale)
        err = np.max(np.abs(inputs.as_f64(o1) - ref))
        assert err <= tol, (step, err)
        assert torch.equal(o1.view(bits), o2.view(bits)), step
        assert torch.equal(one.data_bytes(), two.data_bytes()), step
    assert one.positions() == two.positions() == ring.t
    assert bytes(one.data_bytes().cpu().numpy()) == okv.data_image(ring, dt)


def test_plain_decode_on_a_cache_with_global_rows():
    """moa_decode (no global tokens) on a cache that keeps global-token rows attends to the band
    only and still keeps the rows of the positions it appends."""
    B, Hq, Hkv, d, prefix = 2, 8, 2, 128, 3
    spans, scaps = [40, 38, 64, 64, 300, 299, 299, 280], [8, 8]
    caps = _group_max(spans, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps, sink_capacity=scaps)
    ring = okv.RingCache(B, Hkv, d, caps, scaps)
    k0 = inputs.randn(840, (B, Hkv, prefix, d))
    v0 = inputs.randn(841, (B, Hkv, prefix, d))
    cache.append(k0.to(DEV), v0.to(DEV))
    ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    for step in range(10):
        qt = inputs.randn(850 + step, (B, Hq, d))
        kt = inputs.randn(870 + step, (B, Hkv, 1, d))
        vt = inputs.randn(890 + step, (B, Hkv, 1, d))
        ot = _nan((B, Hq, d), torch.bfloat16)
        moa.moa_decode_append(cache.handle, qt.to(DEV), kt.to(DEV), vt.to(DEV), ot, Hq, spans, 0.088, ws.ptr,
                              ws.nbytes)
        torch.cuda.synchronize()
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        ref = okv.decode(ring, inputs.as_f64(qt), spans, 0.088)
        assert np.max(np.abs(inputs.as_f64(ot) - ref)) <= BF16_TOL, step
    assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16")


def test_chunked_prefill_keeps_global_rows():
    """Chunks appended by moa_prefill_chunk land in the global-token rows too (the chunk itself
    attends to its bands only), so a later decode with global tokens sees them."""
    B, Hq, Hkv, d = 1, 4, 2, 128
    spans, sinks = [64, 256, 300, 100], [130, 3, 0, 200]
    caps, scaps = _group_max(spans, Hkv), _group_max(sinks, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps, sink_capacity=scaps)
    ring = okv.RingCache(B, Hkv, d, caps, scaps)
    for c, n in enumerate([100, 150, 300]):
        q = inputs.randn(900 + c, (B, Hq, n, d)).to(DEV)
        k = inputs.randn(910 + c, (B, Hkv, n, d))
        v = inputs.randn(920 + c, (B, Hkv, n, d))
        nb = moa.moa_chunk_workspace_bytes(cache.handle, Hq, n, spans)
        wbuf = torch.empty(nb + 256, dtype=torch.uint8, device=DEV)
        wptr = (wbuf.data_ptr() + 255) // 256 * 256
        o = _nan((B, Hq, n, d), torch.bfloat16)
        moa.moa_prefill_chunk(cache.handle, q, k.to(DEV), v.to(DEV), o, Hq, n, spans, 0.088, wptr, nb)
        torch.cuda.synchronize()
        ring.append(inputs.as_f64(k), inputs.as_f64(v))
        assert cache.positions() == ring.t
        assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16"), c
    nb = moa.moa_workspace_bytes_sink(moa.MOA_OP_DECODE, B, Hq, 0, d, spans, sinks)
    wbuf = torch.zeros(nb + 256, dtype=torch.uint8, device=DEV)
    wptr = (wbuf.data_ptr() + 255) // 256 * 256
    qt = inputs.randn(930, (B, Hq, d))
    kt = inputs.randn(931, (B, Hkv, 1, d))
    vt = inputs.randn(932, (B, Hkv, 1, d))
    ot = _nan((B, Hq, d), torch.bfloat16)
    moa.moa_decode_append_sink(cache.handle, qt.to(DEV), kt.to(DEV), vt.to(DEV), ot, Hq, spans, sinks, 0.088,
                               wptr, nb)
    torch.cuda.synchronize()
    ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
    ref = okv.decode_sink(ring, inputs.as_f64(qt), spans, sinks, 0.088)
    assert np.max(np.abs(inputs.as_f64(ot) - ref)) <= BF16_TOL


def test_bf16_prefill_with_global_tokens_vicuna7b_sampled():
    """The bench's global-token prompt: B=1, 32 heads, d=128, N=8192, spans at 25 % density,
    global tokens per head from {0, 4, 64, 128, 1024}; sampled rows."""
    from oracle import rules as orules
    B, H, N, d = 1, 32, 8192, 128
    a, b = inputs.tables_7b(1, H, N, 64, 0.25, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    sinks = inputs.sink_counts(7, H)
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(11, (B, H, N, d))
    k = inputs.randn_cuda(12, (B, H, N, d))
    v = inputs.randn_cuda(13, (B, H, N, d))
    cache = moa.KVCache(B, H, d, "bf16", spans, sink_capacity=sinks)
    o = _prefill_sink(q, k, v, spans, sinks, scale, "bf16", fill=cache)
    assert not torch.isnan(o).any()
    rng = np.random.default_rng(9)
    rows = [(0, h, i) for h in range(0, H, 3) for i in (0, 3, 127, 128, 1100, N - 1)]
    rows += [(0, int(rng.integers(H)), int(rng.integers(N))) for _ in range(40)]
    ref = oatt.prefill_sink(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, sinks, scale, rows=rows)
    got = np.stack([inputs.as_f64(o[b_, h_, i_]) for b_, h_, i_ in rows])
    assert np.max(np.abs(got - ref)) <= BF16_TOL
    assert cache.positions() == [N]


def test_decode_with_global_tokens_llama3_gqa_layer_sampled():
    """A Llama3-8B-shaped GQA decode layer with global tokens (B=4, 32 query heads on 8 KV heads,
    d=128, context 8192, 50 % spans, global-token counts from {0, 4, 64, 128, 1024}): the
    tensor-core group kernel's global splits at full size, sampled (b, h) against the oracle's
    row decode over the ring and the global rows."""
    from oracle import rules as orules
    B, Hq, Hkv, d, N = 4, 32, 8, 128, 8192
    G = Hq // Hkv
    a, b = inputs.tables_7b(1001, Hq, N, 64, 0.5, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    sinks = inputs.sink_counts(11, Hq)
    caps, scaps = _group_max(spans, Hkv), _group_max(sinks, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps, sink_capacity=scaps)
    data = cache.data_bytes().view(torch.bfloat16)
    data.copy_(inputs.randn_cuda(31, (data.numel(),)))       # ring rows and global-token rows
    cache.set_positions([N] * B)
    host = cache.data_bytes().cpu().numpy().tobytes()
    scale = 1.0 / math.sqrt(d)
    qt = inputs.randn_cuda(32, (B, Hq, d))
    kt = inputs.randn_cuda(33, (B, Hkv, 1, d))
    vt = inputs.randn_cuda(34, (B, Hkv, 1, d))
    nb = moa.moa_workspace_bytes_sink(moa.MOA_OP_DECODE, B, Hq, 0, d, spans, sinks)
    wbuf = torch.zeros(nb + 256, dtype=torch.uint8, device=DEV)
    ot = _nan((B, Hq, d), torch.bfloat16)
    moa.moa_decode_append_sink(cache.handle, qt, kt, vt, ot, Hq, spans, sinks, scale,
                               (wbuf.data_ptr() + 255) // 256 * 256, nb)
    torch.cuda.synchronize()
    assert cache.positions() == [N + 1] * B
    kt64, vt64, qt64, ot64 = (inputs.as_f64(x) for x in (kt, vt, qt, ot))
    ring_bytes = B * sum(caps) * 2 * d * 2
    sumK = sum(scaps)
    rng = np.random.default_rng(12)
    picks = [(int(rng.integers(B)), int(rng.integers(Hq))) for _ in range(24)] + [(0, 0), (B - 1, Hq - 1)]
    for bb, hh in picks:
        g = hh // G
        K, V = (x.copy() for x in okv.block_from_image(host, bb, g, B, Hkv, d, caps, "bf16"))
        C = caps[g]
        K[N % C] = kt64[bb, g, 0]                      # the appended token's slot
        V[N % C] = vt64[bb, g, 0]
        Kg = scaps[g]
        start = (bb * sumK + sum(scaps[:g])) * 2 * d * 2
        raw = np.frombuffer(host[ring_bytes + start: ring_bytes + start + 2 * Kg * d * 2], dtype="<u2")
        glob = (raw.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(2, Kg, d)
        # the band comes through the ring, the global tokens below it from the global-token
        # rows (the fill is random, so the two copies of a position differ: the call's documented
        # source decides)
        t = N + 1
        keys = oatt.keys_sink(t - 1, spans[hh], sinks[hh])
        Ks = np.stack([K[p % C] if p >= t - spans[hh] else glob[0][p] for p in keys])
        Vs = np.stack([V[p % C] if p >= t - spans[hh] else glob[1][p] for p in keys])
        ref = oatt.attend_row(qt64[bb, hh], Ks, Vs, 0, len(keys) - 1, scale)
        assert np.max(np.abs(ot64[bb, hh] - ref)) <= BF16_TOL, (bb, hh)


@pytest.mark.parametrize("shape", ["vicuna13b", "llama3_gqa"])
def test_bf16_prefill_with_global_tokens_full_size_sampled(shape):
    """Global tokens on the full-size prompts: a Vicuna-13B-shaped layer (40 heads, N=16384, 50 %
    fixed-local and elastic heads) and the Llama3-8B-shaped GQA prompt (32/8 heads, N=32768, 25 %),
    global-token counts from {0, 4, 64, 128, 1024}; sampled rows against the oracle."""
    from oracle import rules as orules
    d = 128
    if shape == "vicuna13b":
        B, Hq, Hkv, N = 1, 40, 40, 16384
        a, b = inputs.tables_13b_mix(5, Hq, N, 64, 0.5, orules.eval_spans)
    else:
        B, Hq, Hkv, N = 1, 32, 8, 32768
        a, b = inputs.tables_7b(4000, Hq, N, 64, 0.25, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    sinks = inputs.sink_counts(13, Hq)
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(41, (B, Hq, N, d))
    k = inputs.randn_cuda(42, (B, Hkv, N, d))
    v = inputs.randn_cuda(43, (B, Hkv, N, d))
    o = _prefill_sink(q, k, v, spans, sinks, scale, "bf16")
    assert not torch.isnan(o).any()
    rng = np.random.default_rng(14)
    rows = [(0, h, i) for h in (0, Hq // 3, Hq - 1) for i in (0, 5, 127, 1100, N // 2, N - 1)]
    rows += [(0, int(rng.integers(Hq)), int(rng.integers(N))) for _ in range(24)]
    ref = oatt.prefill_sink(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, sinks, scale, rows=rows)
    got = np.stack([inputs.as_f64(o[b_, h_, i_]) for b_, h_, i_ in rows])
    assert np.max(np.abs(got - ref)) <= BF16_TOL
