"""GPU parity: libmoa's kernels (through the C ABI) against the fp64 CPU oracle.

Tolerances: bf16 inputs with fp32 accumulation, max-abs 2e-2 against the
oracle run on the same bf16 values in fp64; fp32 path max-abs 1e-5; span
evaluation and ring-buffer bytes bit-exact.  Output buffers are pre-filled
with NaN so an unwritten element fails the comparison.
"""

import math

import numpy as np
import pytest
import torch

from heterogeneous_sliding_window_b200 import inputs, moa
from oracle import attention as oatt, kvcache as okv, rules as orules

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
F32_TOL = 1e-5
DEV = "cuda"


def _nan_like(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, device=DEV)


def _bf16_prefill(q, k, v, spans, scale, fill=None):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    o = _nan_like((B, Hq, N, d), torch.bfloat16)
    ws = moa.Workspace(moa.MOA_OP_PREFILL, B, Hq, N, d, spans)
    moa.moa_prefill(q, k, v, o, B, Hq, Hkv, N, d, "bf16", spans, scale, ws.ptr, ws.nbytes,
                    fill.handle if fill is not None else None)
    moa.moa_workspace_check(ws.ptr)
    torch.cuda.synchronize()
    return o


# ---------------------------------------------------------------------------
# Tiny fp32 configuration: B=1, 4 heads, d=64, N=256, spans {32,64,128,256}
# (beta = 0, block 32); full prefill, then 16 decode steps through the ring.
# ---------------------------------------------------------------------------
def test_tiny_fp32_prefill_fill_and_16_decode_steps():
    B, H, d, N = 1, 4, 64, 256
    a, b = inputs.tiny_tables()
    spans = moa.moa_rules_eval(a, b, N, 32)
    assert spans == orules.eval_spans(a, b, N, 32) == [32, 64, 128, 256]
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn(100, (B, H, N, d), "f32")
    k = inputs.randn(101, (B, H, N, d), "f32")
    v = inputs.randn(102, (B, H, N, d), "f32")
    cache = moa.KVCache(B, H, d, "f32", spans)
    o = _nan_like((B, H, N, d), torch.float32)
    moa.moa_prefill(q.to(DEV), k.to(DEV), v.to(DEV), o, B, H, H, N, d, "f32", spans, scale,
                    None, 0, cache.handle)
    torch.cuda.synchronize()
    ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, scale)
    assert np.max(np.abs(inputs.as_f64(o) - ref)) <= F32_TOL

    ring = okv.RingCache(B, H, d, spans)
    ring.append(inputs.as_f64(k), inputs.as_f64(v))
    assert cache.positions() == ring.t == [N]
    assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "f32")

    ws = moa.Workspace(moa.MOA_OP_DECODE, B, H, 0, d, spans)
    for step in range(16):
        qt = inputs.randn(200 + step, (B, H, d), "f32")
        kt = inputs.randn(300 + step, (B, H, 1, d), "f32")
        vt = inputs.randn(400 + step, (B, H, 1, d), "f32")
        cache.append(kt.to(DEV), vt.to(DEV))
        ot = _nan_like((B, H, d), torch.float32)
        moa.moa_decode(cache.handle, qt.to(DEV), ot, H, spans, scale, ws.ptr, ws.nbytes)
        torch.cuda.synchronize()
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        ref_t = okv.decode(ring, inputs.as_f64(qt), spans, scale)
        assert np.max(np.abs(inputs.as_f64(ot) - ref_t)) <= F32_TOL, step
    assert cache.positions() == ring.t == [N + 16]
    assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "f32")


# ---------------------------------------------------------------------------
# bf16 tensor-core prefill
# ---------------------------------------------------------------------------
PREFILL_CASES = [
    # (B, Hq, Hkv, N, spans, q_gain)   -- ragged N, spans around tile edges, GQA
    (1, 4, 4, 1000, [1, 64, 200, 1000], 1.0),
    (2, 8, 2, 700, [1, 127, 128, 129, 256, 300, 700, 5000], 1.0),
    (1, 2, 1, 513, [384, 100], 4.0),              # peaky scores: stresses the lazy rescale
    (1, 3, 3, 128, [128, 1, 37], 1.0),            # exactly one tile
    (1, 2, 2, 1, [1, 5], 1.0),                    # a single token
    (3, 4, 4, 300, [300, 300, 300, 300], 2.0),    # dense causal (S = N)
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "B%d_H%d_%d_N%d" % c[:4])
def test_bf16_prefill_matches_oracle(case):
    B, Hq, Hkv, N, spans, gain = case
    d = 128
    scale = 1.0 / math.sqrt(d)
    q = (inputs.randn(1, (B, Hq, N, d), "f32") * gain).to(torch.bfloat16)
    k = inputs.randn(2, (B, Hkv, N, d))
    v = inputs.randn(3, (B, Hkv, N, d))
    o = _bf16_prefill(q.to(DEV), k.to(DEV), v.to(DEV), spans, scale)
    ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, scale)
    err = np.max(np.abs(inputs.as_f64(o) - ref))
    assert err <= BF16_TOL, err


def test_bf16_prefill_output_only_16_byte_aligned():
    """Output rows go out in 32-byte stores when o is 32-byte aligned, else in
    16-byte stores: an o 16 bytes past a 32-byte boundary takes the second path,
    and nothing outside o is written."""
    B, Hq, Hkv, N, d = 1, 4, 2, 700, 128
    spans = [1, 129, 300, 700]
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn(21, (B, Hq, N, d))
    k = inputs.randn(22, (B, Hkv, N, d))
    v = inputs.randn(23, (B, Hkv, N, d))
    n = B * Hq * N * d
    flat = _nan_like((n + 32,), torch.bfloat16)
    off = ((16 - flat.data_ptr() % 32) % 32) // 2
    o = flat[off:off + n].view(B, Hq, N, d)
    assert o.data_ptr() % 32 == 16
    ws = moa.Workspace(moa.MOA_OP_PREFILL, B, Hq, N, d, spans)
    moa.moa_prefill(q.to(DEV), k.to(DEV), v.to(DEV), o, B, Hq, Hkv, N, d, "bf16", spans, scale, ws.ptr, ws.nbytes)
    moa.moa_workspace_check(ws.ptr)
    torch.cuda.synchronize()
    ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, scale)
    err = np.max(np.abs(inputs.as_f64(o) - ref))
    assert err <= BF16_TOL, err
    assert torch.isnan(flat[:off]).all() and torch.isnan(flat[off + n:]).all()


def test_bf16_prefill_scores_growing_along_the_sequence():
    """Key norms grow with position, so later tiles' maxima jump far above the
    running maximum (the kernel's rescale path) and early tiles underflow."""
    B, Hq, N, d = 1, 4, 900, 128
    spans = [900, 300, 129, 640]
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn(31, (B, Hq, N, d), "f32")
    k = inputs.randn(32, (B, Hq, N, d), "f32")
    growth = torch.linspace(0.2, 12.0, N).view(1, 1, N, 1)
    k = (k * growth).to(torch.bfloat16)
    q = (q * 2.0).to(torch.bfloat16)
    v = inputs.randn(33, (B, Hq, N, d))
    o = _bf16_prefill(q.to(DEV), k.to(DEV), v.to(DEV), spans, scale)
    ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, scale)
    err = np.max(np.abs(inputs.as_f64(o) - ref))
    assert err <= BF16_TOL, err


def test_bf16_prefill_scores_beyond_the_exponent_range():
    """q x 16 and key norms growing to 12x along the sequence: scores reach several hundred
    in log2 units, so 2^(s - m) overflows fp32 (ex2 gives inf above 128) unless the softmax
    moves its reference first.  Element by element against the oracle, no NaN or inf."""
    B, Hq, N, d = 1, 4, 900, 128
    spans = [900, 300, 129, 640]
    scale = 1.0 / math.sqrt(d)
    q = (inputs.randn(41, (B, Hq, N, d), "f32") * 16.0).to(torch.bfloat16)
    growth = torch.linspace(0.2, 12.0, N).view(1, 1, N, 1)
    k = (inputs.randn(42, (B, Hq, N, d), "f32") * growth).to(torch.bfloat16)
    v = inputs.randn(43, (B, Hq, N, d))
    q64, k64, v64 = inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v)
    s_max = max(float(np.max(q64[0, h] @ k64[0, h].T)) for h in range(Hq)) * scale * math.log2(math.e)
    assert s_max > 128.0, s_max          # the case reaches past the exponent range
    o = _bf16_prefill(q.to(DEV), k.to(DEV), v.to(DEV), spans, scale)
    assert torch.isfinite(o.float()).all()
    ref = oatt.prefill(q64, k64, v64, spans, scale)
    err = np.max(np.abs(inputs.as_f64(o) - ref))
    assert err <= BF16_TOL, err


@pytest.mark.parametrize("Hkv", [4, 1], ids=["per_head", "group_mma"])
def test_bf16_decode_scores_beyond_the_exponent_range(Hkv):
    """Decode with q x 16 and cached keys up to 8x: scores far above 128 in log2 units, on the
    per-head kernel and on the tensor-core group kernel."""
    B, Hq, d, prefix = 2, 4, 128, 900
    spans = [900, 513, 64, 700] if Hkv == 4 else [900, 880, 700, 600]
    scale = 1.0 / math.sqrt(d)
    caps = okv.group_capacities(spans, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    growth = torch.linspace(1.0, 8.0, prefix).view(1, 1, prefix, 1)
    k0 = (inputs.randn(44, (B, Hkv, prefix, d), "f32") * growth).to(torch.bfloat16)
    v0 = inputs.randn(45, (B, Hkv, prefix, d))
    cache.append(k0.to(DEV), v0.to(DEV))
    ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    for step in range(2):
        qt = (inputs.randn(46 + step, (B, Hq, d), "f32") * 16.0).to(torch.bfloat16)
        kt = (inputs.randn(48 + step, (B, Hkv, 1, d), "f32") * 8.0).to(torch.bfloat16)
        vt = inputs.randn(50 + step, (B, Hkv, 1, d))
        cache.append(kt.to(DEV), vt.to(DEV))
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        ot = _nan_like((B, Hq, d), torch.bfloat16)
        moa.moa_decode(cache.handle, qt.to(DEV), ot, Hq, spans, scale, ws.ptr, ws.nbytes)
        torch.cuda.synchronize()
        assert torch.isfinite(ot.float()).all()
        ref = okv.decode(ring, inputs.as_f64(qt), spans, scale)
        err = np.max(np.abs(inputs.as_f64(ot) - ref))
        assert err <= BF16_TOL, (step, err)
    assert cache.positions() == ring.t


def test_bf16_prefill_fill_cache_bytes():
    B, Hq, Hkv, N, d = 2, 4, 2, 600, 128
    spans = [64, 256, 600, 100]
    caps = okv.group_capacities(spans, Hkv)
    q = inputs.randn(7, (B, Hq, N, d))
    k = inputs.randn(8, (B, Hkv, N, d))
    v = inputs.randn(9, (B, Hkv, N, d))
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    _bf16_prefill(q.to(DEV), k.to(DEV), v.to(DEV), spans, 0.1, fill=cache)
    ring = okv.RingCache(B, Hkv, d, caps)
    ring.append(inputs.as_f64(k), inputs.as_f64(v))
    assert cache.positions() == [N, N]
    assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16")


def test_bf16_prefill_fill_after_cached_tokens():
    """The prefill kernel's cache writer appends after tokens already held:
    per-sequence positions differ, the ring wraps inside a prompt, MHA and
    GQA, a prompt longer than some capacities.  Bytes and positions equal the
    ring emulation's, and the attention output is unchanged by the fill."""
    for (B, Hq, Hkv, N, spans, t0) in [(2, 3, 3, 700, [64, 300, 700], [0, 0]),
                                       (2, 4, 2, 333, [129, 64, 256, 200], [5, 300]),
                                       (3, 2, 1, 128, [1, 128], [7, 0, 1000]),
                                       (1, 2, 2, 5, [1, 5], [3]),
                                       (2, 1, 1, 1, [1], [0, 9])]:
        d = 128
        caps = okv.group_capacities(spans, Hkv)
        seed = 40 + N
        k0 = inputs.randn(seed, (B, Hkv, max(t0) or 1, d))
        v0 = inputs.randn(seed + 1, (B, Hkv, max(t0) or 1, d))
        q = inputs.randn(seed + 2, (B, Hq, N, d))
        k = inputs.randn(seed + 3, (B, Hkv, N, d))
        v = inputs.randn(seed + 4, (B, Hkv, N, d))
        cache = moa.KVCache(B, Hkv, d, "bf16", caps)
        ring = okv.RingCache(B, Hkv, d, caps)
        # a history: max(t0) tokens appended to every sequence, then each
        # sequence's position set to t0[b] (the ring bytes stay, only the
        # positions move), in the emulation as well
        if max(t0) > 0:
            moa.moa_kv_append(cache.handle, k0.to(DEV), v0.to(DEV), max(t0))
            ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
            cache.set_positions(t0)
            ring.t = list(t0)
        o = _bf16_prefill(q.to(DEV), k.to(DEV), v.to(DEV), spans, 0.1, fill=cache)
        ring.append(inputs.as_f64(k), inputs.as_f64(v))
        assert cache.positions() == [t + N for t in t0]
        assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16")
        ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, 0.1)
        assert np.max(np.abs(inputs.as_f64(o) - ref)) <= BF16_TOL


def _sample_rows(B, H, N, rng, n=96):
    rows = set()
    for b in range(B):
        for h in range(H):
            for i in (0, 1, 127, 128, N - 1, N - 2):
                if 0 <= i < N:
                    rows.add((b, h, i))
    rows = sorted(rows)
    extra = [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))) for _ in range(n)]
    return rows + extra


def test_bf16_prefill_vicuna7b_full_size_sampled():
    """B=1, 32 heads, d=128, N=8192, 25% density spans: the bench launch, sampled rows."""
    B, H, N, d = 1, 32, 8192, 128
    a, b = inputs.tables_7b(1, H, N, 64, 0.25, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    assert spans == orules.eval_spans(a, b, N, 64)
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(11, (B, H, N, d))
    k = inputs.randn_cuda(12, (B, H, N, d))
    v = inputs.randn_cuda(13, (B, H, N, d))
    o = _bf16_prefill(q, k, v, spans, scale)
    assert not torch.isnan(o).any()
    rows = _sample_rows(B, H, N, np.random.default_rng(0), n=64)
    rows = [r for r in rows if r[1] % 4 == 0 or r[2] in (N - 1,)][:160]
    ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, scale, rows=rows)
    got = np.stack([inputs.as_f64(o[b_, h_, i_]) for b_, h_, i_ in rows])
    assert np.max(np.abs(got - ref)) <= BF16_TOL


def test_bf16_prefill_vicuna13b_mixed_spans_sampled():
    """A Vicuna-13B-shaped layer: B=1, 40 heads, d=128, N=16384, fixed-local heads mixed with
    elastic heads at 50% density (config 4), sampled rows."""
    B, H, N, d = 1, 40, 16384, 128
    a, b = inputs.tables_13b_mix(5, H, N, 64, 0.5, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    assert spans == orules.eval_spans(a, b, N, 64)
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(21, (B, H, N, d))
    k = inputs.randn_cuda(22, (B, H, N, d))
    v = inputs.randn_cuda(23, (B, H, N, d))
    o = _bf16_prefill(q, k, v, spans, scale)
    assert not torch.isnan(o).any()
    rows = _sample_rows(B, H, N, np.random.default_rng(1), n=64)
    rows = [r for r in rows if r[1] % 5 == 0 or r[2] in (N - 1,)][:120]
    ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, scale, rows=rows)
    got = np.stack([inputs.as_f64(o[b_, h_, i_]) for b_, h_, i_ in rows])
    assert np.max(np.abs(got - ref)) <= BF16_TOL


def test_decode_append_replayed_from_cuda_graph():
    """Two layers of moa_decode_append captured once in a CUDA graph and replayed for four
    steps (new q, k, v copied into the captured buffers each time) match the oracle."""
    B, Hq, Hkv, d, prefix = 2, 8, 2, 128, 300
    layers = [[300, 7, 64, 64, 250, 1, 299, 17], [40, 38, 64, 64, 300, 299, 299, 280]]
    scale = 1.0 / math.sqrt(d)
    state = []
    for li, spans in enumerate(layers):
        caps = okv.group_capacities(spans, Hkv)
        cache = moa.KVCache(B, Hkv, d, "bf16", caps)
        ring = okv.RingCache(B, Hkv, d, caps)
        k0 = inputs.randn(110 + li, (B, Hkv, prefix, d))
        v0 = inputs.randn(120 + li, (B, Hkv, prefix, d))
        cache.append(k0.to(DEV), v0.to(DEV))
        ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
        ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
        bufs = [torch.zeros((B, Hq, d), dtype=torch.bfloat16, device=DEV),
                torch.zeros((B, Hkv, 1, d), dtype=torch.bfloat16, device=DEV),
                torch.zeros((B, Hkv, 1, d), dtype=torch.bfloat16, device=DEV),
                torch.zeros((B, Hq, d), dtype=torch.bfloat16, device=DEV)]
        state.append((spans, cache, ring, ws, bufs))
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for spans, cache, ring, ws, (q, k, v, o) in state:
            moa.moa_decode_append(cache.handle, q, k, v, o, Hq, spans, scale, ws.ptr, ws.nbytes, stream)
    torch.cuda.synchronize()
    for step in range(4):
        host = []
        for li, (spans, cache, ring, ws, (q, k, v, o)) in enumerate(state):
            qt = inputs.randn(130 + 10 * step + li, (B, Hq, d))
            kt = inputs.randn(170 + 10 * step + li, (B, Hkv, 1, d))
            vt = inputs.randn(210 + 10 * step + li, (B, Hkv, 1, d))
            q.copy_(qt)
            k.copy_(kt)
            v.copy_(vt)
            ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
            host.append(qt)
        graph.replay()
        torch.cuda.synchronize()
        for (spans, cache, ring, ws, (q, k, v, o)), qt in zip(state, host):
            ref = okv.decode(ring, inputs.as_f64(qt), spans, scale)
            assert np.max(np.abs(inputs.as_f64(o) - ref)) <= BF16_TOL, step
    for spans, cache, ring, ws, bufs in state:
        assert cache.positions() == ring.t == [prefix + 4] * B


def test_bf16_prefill_llama3_gqa_dense_sampled():
    """Hq=32 / Hkv=8, N=32768, every span = N (the dense causal check), sampled rows."""
    B, Hq, Hkv, N, d = 1, 32, 8, 32768, 128
    spans = [N] * Hq
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(21, (B, Hq, N, d))
    k = inputs.randn_cuda(22, (B, Hkv, N, d))
    v = inputs.randn_cuda(23, (B, Hkv, N, d))
    o = _bf16_prefill(q, k, v, spans, scale)
    rows = [(0, h, i) for h in (0, 5, 31) for i in (0, 129, 4095, 20000, N - 1)]
    ref = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, scale, rows=rows)
    got = np.stack([inputs.as_f64(o[b_, h_, i_]) for b_, h_, i_ in rows])
    assert np.max(np.abs(got - ref)) <= BF16_TOL


def test_bf16_prefill_llama3_gqa_density_sweep_sampled():
    """Hq=32 / Hkv=8, d=128, N=32768 at the sweep's 12.5, 25 and 50 % mean densities (per query
    head spans, heterogeneous within each group), each KV group's cache sized to the group's
    largest span and filled by the call, as the bench launches it; sampled rows, and the ring
    bytes of sampled slots."""
    B, Hq, Hkv, N, d = 1, 32, 8, 32768, 128
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(4100, (B, Hq, N, d))
    k = inputs.randn_cuda(4101, (B, Hkv, N, d))
    v = inputs.randn_cuda(4102, (B, Hkv, N, d))
    q64, k64, v64 = inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v)
    rng = np.random.default_rng(5)
    for dens in (0.125, 0.25, 0.5):
        a, b = inputs.tables_7b(4000, Hq, N, 64, dens, orules.eval_spans)
        spans = moa.moa_rules_eval(a, b, N, 64)
        assert spans == orules.eval_spans(a, b, N, 64)
        caps = okv.group_capacities(spans, Hkv)
        cache = moa.KVCache(B, Hkv, d, "bf16", caps)
        o = _bf16_prefill(q, k, v, spans, scale, fill=cache)
        assert not torch.isnan(o).any()
        rows = [(0, h, i) for h in (0, 9, 22, 31) for i in (0, 127, 128, 16383, N - 129, N - 1)]
        rows += [(0, int(rng.integers(Hq)), int(rng.integers(N))) for _ in range(24)]
        ref = oatt.prefill(q64, k64, v64, spans, scale, rows=rows)
        got = np.stack([inputs.as_f64(o[b_, h_, i_]) for b_, h_, i_ in rows])
        assert np.max(np.abs(got - ref)) <= BF16_TOL, dens
        # the ring holds the last C_g positions of every group at slot p mod C_g
        assert cache.positions() == [N]
        data, goff = cache.layout()
        blk = cache.data_bytes().view(torch.bfloat16)
        for g in (0, Hkv - 1):
            C = caps[g]
            for p in (N - 1, N - C, N - 1 - int(rng.integers(C))):
                base = goff[g] * 2 * d + (p % C) * d
                assert torch.equal(blk[base:base + d].view(torch.int16), k[0, g, p].view(torch.int16))
                assert torch.equal(blk[base + C * d:base + C * d + d].view(torch.int16), v[0, g, p].view(torch.int16))
        del cache


# ---------------------------------------------------------------------------
# Ring-buffer append and bf16 decode
# ---------------------------------------------------------------------------
def test_append_bytes_bit_exact():
    B, Hkv, d = 3, 3, 128
    caps = [1, 70, 300]
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    for step, n in enumerate([5, 1, 299, 1, 1, 64, 700, 1, 3]):
        k = inputs.randn(50 + step, (B, Hkv, n, d))
        v = inputs.randn(60 + step, (B, Hkv, n, d))
        cache.append(k.to(DEV), v.to(DEV))
        ring.append(inputs.as_f64(k), inputs.as_f64(v))
        torch.cuda.synchronize()
        assert cache.positions() == ring.t
        assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16")


DECODE_CASES = [
    # (B, Hq, Hkv, prefix, spans, steps)
    (2, 4, 4, 900, [1, 256, 257, 900], 3),         # multi-split heads, single-split heads
    (3, 8, 2, 50, [40, 7, 64, 64, 300, 1, 299, 17], 4),  # prefix shorter than spans, GQA
    (1, 4, 1, 2000, [1000, 513, 2000, 1], 2),       # window smaller than ring: wraps
    (2, 8, 4, 700, [700, 1, 300, 513, 64, 65, 2, 699], 3),     # 2 query heads per KV head
    # windows of a group overlapping enough (sum > 2.2x the group window) for the group-shared kernel
    (3, 8, 2, 50, [40, 38, 64, 64, 300, 299, 299, 280], 3),
    (1, 16, 2, 1500, [1500, 3, 700, 701, 64, 1, 1499, 900,     # 8 query heads per KV head
                      2, 1000, 1024, 513, 257, 5, 1200, 40], 2),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "B%d_H%d_%d_T%d" % c[:4])
def test_bf16_decode_matches_oracle(case):
    B, Hq, Hkv, prefix, spans, steps = case
    d = 128
    scale = 1.0 / math.sqrt(d)
    caps = okv.group_capacities(spans, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    k0 = inputs.randn(70, (B, Hkv, prefix, d))
    v0 = inputs.randn(71, (B, Hkv, prefix, d))
    cache.append(k0.to(DEV), v0.to(DEV))
    ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    for step in range(steps):
        qt = (inputs.randn(80 + step, (B, Hq, d), "f32") * (1 + step)).to(torch.bfloat16)
        kt = inputs.randn(90 + step, (B, Hkv, 1, d))
        vt = inputs.randn(95 + step, (B, Hkv, 1, d))
        cache.append(kt.to(DEV), vt.to(DEV))
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        ot = _nan_like((B, Hq, d), torch.bfloat16)
        moa.moa_decode(cache.handle, qt.to(DEV), ot, Hq, spans, scale, ws.ptr, ws.nbytes)
        torch.cuda.synchronize()
        ref = okv.decode(ring, inputs.as_f64(qt), spans, scale)
        err = np.max(np.abs(inputs.as_f64(ot) - ref))
        assert err <= BF16_TOL, (step, err)
    assert cache.positions() == ring.t


FUSED_CASES = [
    # (B, Hq, Hkv, dtype, d, prefix, spans, steps)
    (2, 4, 4, "bf16", 128, 900, [1, 256, 257, 900], 3),                    # per-head kernel
    (3, 8, 2, "bf16", 128, 50, [40, 7, 64, 64, 300, 1, 299, 17], 4),       # GQA, per-head kernel
    (3, 8, 2, "bf16", 128, 50, [40, 38, 64, 64, 300, 299, 299, 280], 3),   # GQA, group kernel
    (1, 16, 2, "bf16", 128, 1500, [1500, 3, 700, 701, 64, 1, 1499, 900,
                                   2, 1000, 1024, 513, 257, 5, 1200, 40], 2),  # 8 heads per group
    (1, 4, 1, "bf16", 128, 2000, [1000, 513, 2000, 1], 2),                 # ring wraps
    (2, 4, 2, "f32", 64, 0, [1, 5, 32, 17], 40),                           # from an empty cache
    # the SIMT group kernel (fp32 or d = 64 with 4 or 8 heads per KV head and
    # windows overlapping more than 2.2x); bf16 d = 128 groups take the tensor-core kernel
    (2, 8, 2, "f32", 64, 50, [40, 38, 40, 36, 64, 60, 64, 63], 3),
    (2, 8, 2, "bf16", 64, 700, [600, 580, 512, 599, 64, 60, 64, 63], 3),
    (1, 16, 2, "f32", 64, 30, [30, 29, 28, 27, 26, 25, 24, 23, 20, 20, 20, 20, 20, 20, 20, 19], 3),
]


@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: "B%d_H%d_%d_%s_T%d" % (c[0], c[1], c[2], c[3], c[5]))
def test_decode_append_equals_append_then_decode(case):
    """moa_decode_append gives, bit for bit, the outputs, cache bytes and positions of
    moa_kv_append followed by moa_decode, and matches the oracle."""
    B, Hq, Hkv, dt, d, prefix, spans, steps = case
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    tol = BF16_TOL if dt == "bf16" else F32_TOL
    scale = 1.0 / math.sqrt(d)
    caps = okv.group_capacities(spans, Hkv)
    two = moa.KVCache(B, Hkv, d, dt, caps)
    one = moa.KVCache(B, Hkv, d, dt, caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    if prefix:
        k0 = inputs.randn(72, (B, Hkv, prefix, d), dt)
        v0 = inputs.randn(73, (B, Hkv, prefix, d), dt)
        for c in (two, one):
            c.append(k0.to(DEV), v0.to(DEV))
        ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
    ws2 = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    ws1 = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    for step in range(steps):
        qt = inputs.randn(82 + step, (B, Hq, d), dt)
        kt = inputs.randn(92 + step, (B, Hkv, 1, d), dt)
        vt = inputs.randn(97 + step, (B, Hkv, 1, d), dt)
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        o2 = _nan_like((B, Hq, d), tdt)
        o1 = _nan_like((B, Hq, d), tdt)
        two.append(kt.to(DEV), vt.to(DEV))
        moa.moa_decode(two.handle, qt.to(DEV), o2, Hq, spans, scale, ws2.ptr, ws2.nbytes)
        moa.moa_decode_append(one.handle, qt.to(DEV), kt.to(DEV), vt.to(DEV), o1, Hq, spans, scale,
                              ws1.ptr, ws1.nbytes)
        torch.cuda.synchronize()
        assert torch.equal(o1.view(torch.int16 if dt == "bf16" else torch.int32),
                           o2.view(torch.int16 if dt == "bf16" else torch.int32)), step
        assert torch.equal(one.data_bytes(), two.data_bytes()), step
        ref = okv.decode(ring, inputs.as_f64(qt), spans, scale)
        assert np.max(np.abs(inputs.as_f64(o1) - ref)) <= tol, step
    assert one.positions() == two.positions() == ring.t


def test_bf16_decode_vicuna7b_layer_full_size_sampled():
    """One layer of the decode workload: B=32, 32 heads, context 4096, 50% density."""
    B, H, d, N = 32, 32, 128, 4096
    a, b = inputs.tables_7b(1000, H, N, 64, 0.5, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    cache = moa.KVCache(B, H, d, "bf16", spans)
    data = cache.data_bytes().view(torch.bfloat16)
    data.copy_(inputs.randn_cuda(5, (data.numel(),)))
    cache.set_positions([N] * B)
    rng = np.random.default_rng(3)
    picks = [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(24)] + [(0, 0), (B - 1, H - 1)]
    blocks = {}
    host = None
    for bb, hh in picks:
        if (bb, hh) not in blocks:
            if host is None:
                host = cache.data_bytes().cpu().numpy().tobytes()
            blocks[(bb, hh)] = okv.block_from_image(host, bb, hh, B, H, d, spans, "bf16")
    scale = 1.0 / math.sqrt(d)
    qt = inputs.randn_cuda(6, (B, H, d))
    kt = inputs.randn_cuda(7, (B, H, 1, d))
    vt = inputs.randn_cuda(8, (B, H, 1, d))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, H, 0, d, spans)
    cache.append(kt, vt)
    ot = _nan_like((B, H, d), torch.bfloat16)
    moa.moa_decode(cache.handle, qt, ot, H, spans, scale, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert cache.positions() == [N + 1] * B
    kt64, vt64, qt64, ot64 = (inputs.as_f64(x) for x in (kt, vt, qt, ot))
    for bb, hh in picks:
        K, V = blocks[(bb, hh)]
        C = spans[hh]
        K[N % C] = kt64[bb, hh, 0]          # the appended token's slot
        V[N % C] = vt64[bb, hh, 0]
        ref = okv.decode_row_from_ring(K, V, N + 1, spans[hh], qt64[bb, hh], scale)
        assert np.max(np.abs(ot64[bb, hh] - ref)) <= BF16_TOL, (bb, hh)


@pytest.mark.parametrize("B", [1, 4])
def test_bf16_decode_vicuna7b_layer_small_batch(B):
    """The same layer at batch 1 and 4, where the launch has under 1 024 splits of 512 entries
    and the kernel takes half-size splits (up to 16 per head here): every head, fused append,
    against the oracle's ring decode; the appended rows bit-exact."""
    H, d, N = 32, 128, 4096
    a, b = inputs.tables_7b(1000, H, N, 64, 0.5, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    cache = moa.KVCache(B, H, d, "bf16", spans)
    data = cache.data_bytes().view(torch.bfloat16)
    data.copy_(inputs.randn_cuda(15 + B, (data.numel(),)))
    cache.set_positions([N] * B)
    host = cache.data_bytes().cpu().numpy().tobytes()
    scale = 1.0 / math.sqrt(d)
    qt = inputs.randn_cuda(16 + B, (B, H, d))
    kt = inputs.randn_cuda(17 + B, (B, H, 1, d))
    vt = inputs.randn_cuda(18 + B, (B, H, 1, d))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, H, 0, d, spans)
    ot = _nan_like((B, H, d), torch.bfloat16)
    moa.moa_decode_append(cache.handle, qt, kt, vt, ot, H, spans, scale, ws.ptr, ws.nbytes)
    moa.moa_workspace_check(ws.ptr)
    torch.cuda.synchronize()
    assert cache.positions() == [N + 1] * B
    after = cache.data_bytes().cpu().numpy().tobytes()
    kt64, vt64, qt64, ot64 = (inputs.as_f64(x) for x in (kt, vt, qt, ot))
    for bb in range(B):
        for hh in range(H):
            K, V = okv.block_from_image(host, bb, hh, B, H, d, spans, "bf16")
            C = spans[hh]
            K[N % C] = kt64[bb, hh, 0]      # the appended token's slot
            V[N % C] = vt64[bb, hh, 0]
            K2, V2 = okv.block_from_image(after, bb, hh, B, H, d, spans, "bf16")
            assert np.array_equal(K2[N % C], K[N % C]) and np.array_equal(V2[N % C], V[N % C]), (bb, hh)
            ref = okv.decode_row_from_ring(K, V, N + 1, spans[hh], qt64[bb, hh], scale)
            assert np.max(np.abs(ot64[bb, hh] - ref)) <= BF16_TOL, (bb, hh)


def test_bf16_decode_llama3_gqa_layer_full_size_sampled():
    """A Llama3-8B-shaped GQA decode layer: B=4, 32 query heads on 8 KV heads, context 8192,
    per-head spans at 50% density (heterogeneous within each group), one appended token."""
    B, Hq, Hkv, d, N = 4, 32, 8, 128, 8192
    a, b = inputs.tables_7b(1001, Hq, N, 64, 0.5, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    caps = okv.group_capacities(spans, Hkv)
    G = Hq // Hkv
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    data = cache.data_bytes().view(torch.bfloat16)
    data.copy_(inputs.randn_cuda(15, (data.numel(),)))
    cache.set_positions([N] * B)
    rng = np.random.default_rng(4)
    picks = [(int(rng.integers(B)), int(rng.integers(Hq))) for _ in range(24)] + [(0, 0), (B - 1, Hq - 1)]
    host = cache.data_bytes().cpu().numpy().tobytes()
    blocks = {}
    for bb, hh in picks:
        if (bb, hh // G) not in blocks:
            blocks[(bb, hh // G)] = okv.block_from_image(host, bb, hh // G, B, Hkv, d, caps, "bf16")
    scale = 1.0 / math.sqrt(d)
    qt = inputs.randn_cuda(16, (B, Hq, d))
    kt = inputs.randn_cuda(17, (B, Hkv, 1, d))
    vt = inputs.randn_cuda(18, (B, Hkv, 1, d))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    cache.append(kt, vt)
    ot = _nan_like((B, Hq, d), torch.bfloat16)
    moa.moa_decode(cache.handle, qt, ot, Hq, spans, scale, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert cache.positions() == [N + 1] * B
    kt64, vt64, qt64, ot64 = (inputs.as_f64(x) for x in (kt, vt, qt, ot))
    for bb, hh in picks:
        g = hh // G
        K, V = (x.copy() for x in blocks[(bb, g)])
        C = caps[g]
        K[N % C] = kt64[bb, g, 0]           # the appended token's slot
        V[N % C] = vt64[bb, g, 0]
        ref = okv.decode_row_from_ring(K, V, N + 1, spans[hh], qt64[bb, hh], scale)
        assert np.max(np.abs(ot64[bb, hh] - ref)) <= BF16_TOL, (bb, hh)


@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 1)], ids=["mha", "gqa"])
def test_decode_empty_sequence_sets_error_bit(H, Hkv):
    B, d = 2, 128
    spans = [8] * H
    cache = moa.KVCache(B, Hkv, d, "bf16", [8] * Hkv)
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, H, 0, d, spans)
    q = inputs.randn_cuda(1, (B, H, d))
    o = _nan_like((B, H, d), torch.bfloat16)
    moa.moa_decode(cache.handle, q, o, H, spans, 0.1, ws.ptr, ws.nbytes)
    with pytest.raises(moa.MoaError) as e:
        cache.positions()
    assert e.value.status == moa.MOA_ERR_INVALID_ARG
    assert torch.all(o.float() == 0)


def test_decode_rejects_span_above_capacity():
    cache = moa.KVCache(1, 1, 128, "bf16", [64])
    ws = moa.Workspace(moa.MOA_OP_DECODE, 1, 1, 0, 128, [64])
    q = inputs.randn_cuda(1, (1, 1, 128))
    with pytest.raises(moa.MoaError) as e:
        moa.moa_decode(cache.handle, q, q.clone(), 1, [65], 0.1, ws.ptr, ws.nbytes)
    assert e.value.status == moa.MOA_ERR_CAPACITY


@pytest.mark.parametrize("nbytes", [0, 16, 48, (64 << 20) + 4096 + 48])
def test_stream_read_checksum(nbytes):
    """The read-only bandwidth probe reads every byte once: its checksum is the
    XOR of the even-indexed 32-bit words (high half) and of the odd-indexed
    words (low half), recomputed here on the host."""
    rng = np.random.default_rng(7)
    host = rng.integers(0, 2 ** 32, size=max(nbytes // 4, 1), dtype=np.uint32)[: nbytes // 4]
    buf = torch.from_numpy(host.view(np.int32).copy()).to(DEV) if nbytes else torch.empty(4, dtype=torch.int32,
                                                                                          device=DEV)
    out = torch.full((1,), -1, dtype=torch.int64, device=DEV)
    moa.moa_stream_read(buf, nbytes, out)
    torch.cuda.synchronize()
    got = int(out.cpu().numpy().view(np.uint64)[0])
    hi = int(np.bitwise_xor.reduce(host[0::2])) if nbytes else 0
    lo = int(np.bitwise_xor.reduce(host[1::2])) if nbytes else 0
    assert got == (hi << 32) | lo


# ---------------------------------------------------------------------------
# Chunked prefill: pieces of a prompt attend to the ring's window and to
# themselves, then are appended
# ---------------------------------------------------------------------------
def _chunk_call(cache, q, k, v, Hq, spans, scale):
    B, _, n, d = q.shape
    nb = moa.moa_chunk_workspace_bytes(cache.handle, Hq, n, spans)
    buf = torch.empty(nb + 256, dtype=torch.uint8, device=DEV)
    ptr = (buf.data_ptr() + 255) // 256 * 256
    o = _nan_like((B, Hq, n, d), torch.bfloat16)
    moa.moa_prefill_chunk(cache.handle, q, k, v, o, Hq, n, spans, scale, ptr, nb)
    torch.cuda.synchronize()
    return o


CHUNK_CASES = [
    # (B, Hq, Hkv, spans, chunk sizes in order)
    (2, 4, 2, [300, 64, 129, 1], [500, 200, 77]),                # first chunk into an empty cache
    (1, 2, 1, [40, 700], [128, 1, 300, 256, 129]),               # tile-aligned, one token, ragged
    (3, 8, 2, [40, 38, 64, 64, 300, 299, 299, 280], [257, 130]),  # GQA, 4 query heads per kv head
    (1, 4, 4, [1, 2, 3, 1000], [700, 700]),                      # ring wraps inside a chunk
]


@pytest.mark.parametrize("case", CHUNK_CASES, ids=lambda c: "B%d_H%d_%d_%s" % (c[0], c[1], c[2],
                                                                            "-".join(map(str, c[4]))))
def test_bf16_prefill_chunks_match_oracle(case):
    B, Hq, Hkv, spans, pieces = case
    d = 128
    scale = 1.0 / math.sqrt(d)
    T = sum(pieces)
    q = inputs.randn(80, (B, Hq, T, d))
    k = inputs.randn(81, (B, Hkv, T, d))
    v = inputs.randn(82, (B, Hkv, T, d))
    caps = okv.group_capacities(spans, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    qf, kf, vf = inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v)
    t = 0
    for n in pieces:
        sl = slice(t, t + n)
        o = _chunk_call(cache, q[:, :, sl].contiguous().to(DEV), k[:, :, sl].contiguous().to(DEV),
                        v[:, :, sl].contiguous().to(DEV), Hq, spans, scale)
        want = oatt.chunk(qf[:, :, sl], [kf[b, :, :t + n] for b in range(B)], [vf[b, :, :t + n] for b in range(B)],
                          [t] * B, spans, scale)
        err = np.max(np.abs(inputs.as_f64(o) - want))
        assert err <= BF16_TOL, (t, n, err)
        ring.append(kf[:, :, sl], vf[:, :, sl])
        t += n
        assert cache.positions() == [t] * B
        assert bytes(cache.data_bytes().cpu().numpy()) == okv.data_image(ring, "bf16")


def test_bf16_prefill_chunk_with_a_different_history_per_sequence():
    """Sequences at different positions (one shorter than every window, one
    empty): rows of negative positions are masked per sequence."""
    B, Hq, Hkv, d = 3, 4, 2, 128
    spans = [333, 64, 700, 5]
    scale = 1.0 / math.sqrt(d)
    t = [1000, 37, 0]
    n = 190
    caps = okv.group_capacities(spans, Hkv)
    hist_k = [inputs.randn(90 + b, (1, Hkv, t[b] + n, d)) for b in range(B)]
    hist_v = [inputs.randn(95 + b, (1, Hkv, t[b] + n, d)) for b in range(B)]
    image = b""
    for b in range(B):
        ring = okv.RingCache(1, Hkv, d, caps)
        if t[b]:
            ring.append(inputs.as_f64(hist_k[b][:, :, :t[b]]), inputs.as_f64(hist_v[b][:, :, :t[b]]))
        image += okv.data_image(ring, "bf16")
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    cache.data_bytes().copy_(torch.frombuffer(bytearray(image), dtype=torch.uint8).to(DEV))
    cache.set_positions(t)
    q = inputs.randn(99, (B, Hq, n, d))
    kc = torch.cat([hist_k[b][:, :, t[b]:] for b in range(B)], dim=0)
    vc = torch.cat([hist_v[b][:, :, t[b]:] for b in range(B)], dim=0)
    o = _chunk_call(cache, q.to(DEV), kc.contiguous().to(DEV), vc.contiguous().to(DEV), Hq, spans, scale)
    want = oatt.chunk(inputs.as_f64(q), [inputs.as_f64(hist_k[b])[0] for b in range(B)],
                      [inputs.as_f64(hist_v[b])[0] for b in range(B)], t, spans, scale)
    assert np.max(np.abs(inputs.as_f64(o) - want)) <= BF16_TOL
    assert cache.positions() == [tb + n for tb in t]


def test_bf16_prefill_chunk_then_decode():
    """Decode after a chunked prompt reads the cache the chunks left."""
    B, Hq, Hkv, d = 2, 4, 2, 128
    spans = [257, 64, 500, 3]
    scale = 1.0 / math.sqrt(d)
    caps = okv.group_capacities(spans, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    t = 0
    for i, n in enumerate([300, 211]):
        q = inputs.randn(110 + i, (B, Hq, n, d))
        k = inputs.randn(120 + i, (B, Hkv, n, d))
        v = inputs.randn(130 + i, (B, Hkv, n, d))
        _chunk_call(cache, q.to(DEV), k.to(DEV), v.to(DEV), Hq, spans, scale)
        ring.append(inputs.as_f64(k), inputs.as_f64(v))
        t += n
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    qd = inputs.randn(140, (B, Hq, d))
    kd = inputs.randn(141, (B, Hkv, 1, d))
    vd = inputs.randn(142, (B, Hkv, 1, d))
    o = _nan_like((B, Hq, d), torch.bfloat16)
    moa.moa_decode_append(cache.handle, qd.to(DEV), kd.to(DEV), vd.to(DEV), o, Hq, spans, scale, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    ring.append(inputs.as_f64(kd), inputs.as_f64(vd))
    want = okv.decode(ring, inputs.as_f64(qd), spans, scale)
    assert np.max(np.abs(inputs.as_f64(o) - want)) <= BF16_TOL


def test_bf16_prefill_chunk_vicuna7b_shaped_sampled():
    """A 1024-token chunk after a 4096-token prompt, 32 heads at 25 % density:
    sampled rows against the oracle, the rest checked finite."""
    B, H, d, t, n = 1, 32, 128, 4096, 1024
    pa, pb = inputs.tables_7b(5, H, t + n, 64, 0.25, orules.eval_spans)
    spans = [int(s) for s in orules.eval_spans(pa, pb, t + n, 64)]
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(150, (B, H, t + n, d))
    k = inputs.randn_cuda(151, (B, H, t + n, d))
    v = inputs.randn_cuda(152, (B, H, t + n, d))
    caps = okv.group_capacities(spans, H)
    cache = moa.KVCache(B, H, d, "bf16", caps)
    _chunk_call(cache, q[:, :, :t].contiguous(), k[:, :, :t].contiguous(), v[:, :, :t].contiguous(), H, spans, scale)
    o = _chunk_call(cache, q[:, :, t:].contiguous(), k[:, :, t:].contiguous(), v[:, :, t:].contiguous(), H, spans,
                    scale)
    assert torch.isfinite(o.float()).all()
    rng = np.random.default_rng(3)
    rows = [(0, int(h), int(i)) for h, i in zip(rng.integers(0, H, 48), rng.integers(0, n, 48))]
    rows += [(0, 0, 0), (0, H - 1, n - 1)]
    kf = inputs.as_f64(k)
    vf = inputs.as_f64(v)
    want = oatt.chunk(inputs.as_f64(q[:, :, t:]), [kf[0]], [vf[0]], [t], spans, scale, rows=rows)
    got = inputs.as_f64(o)
    err = max(np.max(np.abs(got[b, h, i] - want[r])) for r, (b, h, i) in enumerate(rows))
    assert err <= BF16_TOL
    assert cache.positions() == [t + n]


def test_prefill_chunk_errors():
    cache = moa.KVCache(1, 2, 128, "bf16", [64, 64])
    with pytest.raises(moa.MoaError) as e:
        moa.moa_chunk_workspace_bytes(cache.handle, 4, 10, [65, 1, 1, 1])
    assert e.value.status == moa.MOA_ERR_CAPACITY
    f32 = moa.KVCache(1, 1, 64, "f32", [8])
    with pytest.raises(moa.MoaError) as e:
        moa.moa_chunk_workspace_bytes(f32.handle, 1, 10, [8])
    assert e.value.status == moa.MOA_ERR_UNSUPPORTED
    spans = [64, 1, 1, 1]
    nb = moa.moa_chunk_workspace_bytes(cache.handle, 4, 10, spans)
    buf = torch.empty(nb + 256, dtype=torch.uint8, device=DEV)
    ptr = (buf.data_ptr() + 255) // 256 * 256
    q = torch.zeros((1, 4, 10, 128), dtype=torch.bfloat16, device=DEV)
    kv = torch.zeros((1, 2, 10, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moa.MoaError) as e:
        moa.moa_prefill_chunk(cache.handle, q, kv, kv, q.clone(), 4, 10, spans, 0.088, ptr, nb - 1)
    assert e.value.status == moa.MOA_ERR_WORKSPACE
    with pytest.raises(moa.MoaError) as e:
        moa.moa_prefill_chunk(cache.handle, q, kv, kv, q.clone(), 4, 0, spans, 0.088, ptr, nb)
    assert e.value.status == moa.MOA_ERR_INVALID_ARG
    assert cache.positions() == [0]


# ---------------------------------------------------------------------------
# Largest head count the ABI takes (MOA_MAX_HEADS = 128) and a large batch
# ---------------------------------------------------------------------------
def test_bf16_prefill_at_the_head_limit():
    """128 query heads on 8 KV heads (16 per group), ragged N, spans from 1 to
    beyond N: every output row against the oracle."""
    B, Hq, Hkv, N, d = 1, 128, 8, 300, 128
    rng = np.random.default_rng(11)
    spans = [int(s) for s in rng.integers(1, 400, Hq)]
    spans[0], spans[1], spans[-1] = 1, 300, 399
    q = inputs.randn(160, (B, Hq, N, d))
    k = inputs.randn(161, (B, Hkv, N, d))
    v = inputs.randn(162, (B, Hkv, N, d))
    o = _bf16_prefill(q.to(DEV), k.to(DEV), v.to(DEV), spans, 1 / math.sqrt(d))
    want = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, 1 / math.sqrt(d))
    assert np.max(np.abs(inputs.as_f64(o) - want)) <= BF16_TOL


def test_bf16_decode_at_the_head_limit():
    """128 query heads on 16 KV heads (8 per group), three fused steps.  The
    windows overlap enough (the sum of the spans is well above 2.2 times the
    sum of the group capacities) for the group-shared decode kernel; half of
    the groups hold near-equal windows, the other half spans from 1 to 700."""
    B, Hq, Hkv, d, prefix = 2, 128, 16, 128, 700
    rng = np.random.default_rng(12)
    spans = [int(s) for s in rng.integers(1, 701, Hq)]
    for h in range(0, 64):            # first half of the groups: near-equal windows (group kernel)
        spans[h] = 600 + (h % 8) * 12
    scale = 1.0 / math.sqrt(d)
    caps = okv.group_capacities(spans, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    k0 = inputs.randn(170, (B, Hkv, prefix, d))
    v0 = inputs.randn(171, (B, Hkv, prefix, d))
    cache.append(k0.to(DEV), v0.to(DEV))
    ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    for step in range(3):
        qt = inputs.randn(180 + step, (B, Hq, d))
        kt = inputs.randn(185 + step, (B, Hkv, 1, d))
        vt = inputs.randn(190 + step, (B, Hkv, 1, d))
        ot = _nan_like((B, Hq, d), torch.bfloat16)
        moa.moa_decode_append(cache.handle, qt.to(DEV), kt.to(DEV), vt.to(DEV), ot, Hq, spans, scale, ws.ptr,
                              ws.nbytes)
        torch.cuda.synchronize()
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        ref = okv.decode(ring, inputs.as_f64(qt), spans, scale)
        assert np.max(np.abs(inputs.as_f64(ot) - ref)) <= BF16_TOL, step
    assert cache.positions() == ring.t


def test_bf16_decode_large_batch_sampled():
    """1024 sequences at different positions (set through moa_kv_set_positions
    over caches filled in one append): per-sequence counters and positions,
    sampled sequences against the oracle."""
    B, Hq, Hkv, d, prefix = 1024, 4, 2, 128, 96
    spans = [1, 37, 96, 64]
    scale = 1.0 / math.sqrt(d)
    caps = okv.group_capacities(spans, Hkv)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    k0 = inputs.randn_cuda(200, (B, Hkv, prefix, d))
    v0 = inputs.randn_cuda(201, (B, Hkv, prefix, d))
    cache.append(k0, v0)
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    q = inputs.randn_cuda(202, (B, Hq, d))
    kn = inputs.randn_cuda(203, (B, Hkv, 1, d))
    vn = inputs.randn_cuda(204, (B, Hkv, 1, d))
    o = _nan_like((B, Hq, d), torch.bfloat16)
    moa.moa_decode_append(cache.handle, q, kn, vn, o, Hq, spans, scale, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert cache.positions() == [prefix + 1] * B
    assert torch.isfinite(o.float()).all()
    kf, vf, qf = inputs.as_f64(k0), inputs.as_f64(v0), inputs.as_f64(q)
    knf, vnf = inputs.as_f64(kn), inputs.as_f64(vn)
    got = inputs.as_f64(o)
    for b in [0, 1, 511, 777, B - 1]:
        hist_k = np.concatenate([kf[b], knf[b]], axis=1)
        hist_v = np.concatenate([vf[b], vnf[b]], axis=1)
        want = oatt.chunk(qf[b:b + 1, :, None, :], [hist_k], [hist_v], [prefix], spans, scale)[0, :, 0]
        assert np.max(np.abs(got[b] - want)) <= BF16_TOL, b


def test_prefill_bounded_waits_report_a_timeout():
    """Failure path without a fault: the prefill kernel launched with its work
    units withheld gives up on its first waits after 2 s, the workspace error
    word reads MOA_ERR_TIMEOUT, and a normal prefill on the same context still
    matches the oracle."""
    import time
    d = 128
    x = torch.zeros((1, 1, 128, d), dtype=torch.bfloat16, device=DEV)
    o = torch.zeros_like(x)
    ws = moa.Workspace(moa.MOA_OP_PREFILL, 1, 1, 128, d, [128])
    torch.cuda.synchronize()
    t0 = time.time()
    moa.moa_prefill_stall_test(x, x, x, o, ws.ptr, ws.nbytes)
    with pytest.raises(moa.MoaError) as e:
        moa.moa_workspace_check(ws.ptr)
    assert e.value.status == moa.MOA_ERR_TIMEOUT
    assert 1.5 < time.time() - t0 < 60
    spans = [200, 7]
    q = inputs.randn(170, (1, 2, 300, d))
    k = inputs.randn(171, (1, 1, 300, d))
    v = inputs.randn(172, (1, 1, 300, d))
    out = _bf16_prefill(q.to(DEV), k.to(DEV), v.to(DEV), spans, 1 / math.sqrt(d))
    want = oatt.prefill(inputs.as_f64(q), inputs.as_f64(k), inputs.as_f64(v), spans, 1 / math.sqrt(d))
    assert np.max(np.abs(inputs.as_f64(out) - want)) <= BF16_TOL


def test_bf16_decode_vicuna13b_mixed_layer_sampled():
    """One layer of the 13B decode workload: B=8, 40 heads, context 16384, fixed-local
    and elastic heads mixed to 50 % density, fused append; sampled heads against the
    oracle's ring decode."""
    B, H, d, N = 8, 40, 128, 16384
    a, b = inputs.tables_13b_mix(9, H, N, 64, 0.5, orules.eval_spans)
    spans = moa.moa_rules_eval(a, b, N, 64)
    cache = moa.KVCache(B, H, d, "bf16", spans)
    data = cache.data_bytes().view(torch.bfloat16)
    data.copy_(inputs.randn_cuda(15, (data.numel(),)))
    cache.set_positions([N] * B)
    rng = np.random.default_rng(13)
    picks = [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(16)] + [(0, 0), (B - 1, H - 1)]
    host = cache.data_bytes().cpu().numpy().tobytes()
    blocks = {(bb, hh): okv.block_from_image(host, bb, hh, B, H, d, spans, "bf16") for bb, hh in picks}
    scale = 1.0 / math.sqrt(d)
    qt = inputs.randn_cuda(16, (B, H, d))
    kt = inputs.randn_cuda(17, (B, H, 1, d))
    vt = inputs.randn_cuda(18, (B, H, 1, d))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, H, 0, d, spans)
    ot = _nan_like((B, H, d), torch.bfloat16)
    moa.moa_decode_append(cache.handle, qt, kt, vt, ot, H, spans, scale, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert cache.positions() == [N + 1] * B
    kt64, vt64, qt64, ot64 = (inputs.as_f64(x) for x in (kt, vt, qt, ot))
    for bb, hh in picks:
        K, V = blocks[(bb, hh)]
        C = spans[hh]
        K[N % C] = kt64[bb, hh, 0]
        V[N % C] = vt64[bb, hh, 0]
        ref = okv.decode_row_from_ring(K, V, N + 1, spans[hh], qt64[bb, hh], scale)
        assert np.max(np.abs(ot64[bb, hh] - ref)) <= BF16_TOL, (bb, hh)
