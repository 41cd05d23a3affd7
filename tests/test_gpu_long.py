"""GPU parity at a very long prompt: 2^22 + 77 tokens, through the C ABI.

A GQA pair (2 query heads on 1 KV head) with spans 4 096 and 100 000 runs the
tensor-core prefill with its cache fill, then a 333-token chunk and one fused
decode step after it.  Row offsets, tile indices and ring slots are far beyond
the other tests' sizes here.  The full fp64 output would not fit, so sampled
rows are checked with the oracle's own row routine on each row's key window
(``oracle.attention.window`` / ``attend_row``), cache slots against the oracle's
ring layout bit for bit, and the decode row with ``decode_row_from_ring``.
"""

import math

import numpy as np
import pytest
import torch

from heterogeneous_sliding_window_b200 import inputs, moa
from oracle import attention as oatt, kvcache as okv

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def test_bf16_prefill_chunk_and_decode_after_four_million_tokens_sampled():
    B, Hq, Hkv, N, d = 1, 2, 1, (1 << 22) + 77, 128
    spans = [4096, 100_000]
    scale = 1.0 / math.sqrt(d)
    q = inputs.randn_cuda(71, (B, Hq, N, d))
    k = inputs.randn_cuda(72, (B, Hkv, N, d))
    v = inputs.randn_cuda(73, (B, Hkv, N, d))
    o = torch.full((B, Hq, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    caps = okv.group_capacities(spans, Hkv)
    assert caps == [100_000]
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    ws = moa.Workspace(moa.MOA_OP_PREFILL, B, Hq, N, d, spans)
    moa.moa_prefill(q, k, v, o, B, Hq, Hkv, N, d, "bf16", spans, scale, ws.ptr, ws.nbytes, cache.handle)
    moa.moa_workspace_check(ws.ptr)
    torch.cuda.synchronize()
    assert cache.positions() == [N]

    rng = np.random.default_rng(7)
    fixed = [0, 1, 127, 128, 4095, 4096, 99_999, 100_000, (1 << 21) - 1, 1 << 21, N - 129, N - 128, N - 78,
             N - 77, N - 1]
    for h in range(Hq):
        rows = sorted(set(fixed) | set(int(x) for x in rng.integers(0, N, size=12)))
        for i in rows:
            lo, hi = oatt.window(i, spans[h])
            Kw = inputs.as_f64(k[0, 0, lo:hi + 1])
            Vw = inputs.as_f64(v[0, 0, lo:hi + 1])
            ref = oatt.attend_row(inputs.as_f64(q[0, h, i]), Kw, Vw, 0, hi - lo, scale)
            got = inputs.as_f64(o[0, h, i])
            err = float(np.max(np.abs(got - ref)))
            assert err <= BF16_TOL, (h, i, err)

    # The ring holds positions N - C .. N - 1, position p at slot p mod C.
    C = caps[0]
    Kr, Vr = okv.block_from_image(cache.data_bytes().cpu().numpy(), 0, 0, B, Hkv, d, caps, "bf16")
    for p in sorted(set([N - C, N - C + 1, N - 1, N - 2]) | set(int(x) for x in rng.integers(N - C, N, size=64))):
        s = okv.RingCache.slot(p, C)
        assert np.array_equal(Kr[s], inputs.as_f64(k[0, 0, p])), p
        assert np.array_equal(Vr[s], inputs.as_f64(v[0, 0, p])), p

    # A 333-token chunk continues the sequence: positions N .. N + 332 attend to the ring's window
    # (positions below N, which the ring holds, as checked above) and to the chunk itself.
    n = 333
    qc = inputs.randn_cuda(77, (B, Hq, n, d))
    kc = inputs.randn_cuda(78, (B, Hkv, n, d))
    vc = inputs.randn_cuda(79, (B, Hkv, n, d))
    oc = torch.full((B, Hq, n, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    nb = moa.moa_chunk_workspace_bytes(cache.handle, Hq, n, spans)
    cbuf = torch.empty(nb + 256, dtype=torch.uint8, device="cuda")
    cptr = (cbuf.data_ptr() + 255) // 256 * 256
    moa.moa_prefill_chunk(cache.handle, qc, kc, vc, oc, Hq, n, spans, scale, cptr, nb)
    torch.cuda.synchronize()
    assert cache.positions() == [N + n]
    for h in range(Hq):
        for i in (0, 1, 127, 128, 200, 255, 256, n - 1):
            lo, hi = oatt.window(N + i, spans[h])
            Kw = np.concatenate([inputs.as_f64(k[0, 0, lo:N]), inputs.as_f64(kc[0, 0, :i + 1])])
            Vw = np.concatenate([inputs.as_f64(v[0, 0, lo:N]), inputs.as_f64(vc[0, 0, :i + 1])])
            assert Kw.shape[0] == hi - lo + 1
            ref = oatt.attend_row(inputs.as_f64(qc[0, h, i]), Kw, Vw, 0, hi - lo, scale)
            err = float(np.max(np.abs(inputs.as_f64(oc[0, h, i]) - ref)))
            assert err <= BF16_TOL, ("chunk", h, i, err)
    Kr, Vr = okv.block_from_image(cache.data_bytes().cpu().numpy(), 0, 0, B, Hkv, d, caps, "bf16")
    for i in (0, 1, 200, n - 1):
        s = okv.RingCache.slot(N + i, C)
        assert np.array_equal(Kr[s], inputs.as_f64(kc[0, 0, i])) and np.array_equal(Vr[s], inputs.as_f64(vc[0, 0, i]))
    t = N + n

    # One decode step at position t: the step's k, v are appended in the same launch.
    qt = inputs.randn_cuda(74, (B, Hq, d))
    kt = inputs.randn_cuda(75, (B, Hkv, 1, d))
    vt = inputs.randn_cuda(76, (B, Hkv, 1, d))
    ot = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    moa.moa_decode_append(cache.handle, qt, kt, vt, ot, Hq, spans, scale, dws.ptr, dws.nbytes)
    moa.moa_workspace_check(dws.ptr)
    torch.cuda.synchronize()
    assert cache.positions() == [t + 1]
    Kr, Vr = okv.block_from_image(cache.data_bytes().cpu().numpy(), 0, 0, B, Hkv, d, caps, "bf16")
    s = okv.RingCache.slot(t, C)
    assert np.array_equal(Kr[s], inputs.as_f64(kt[0, 0, 0])) and np.array_equal(Vr[s], inputs.as_f64(vt[0, 0, 0]))
    for h in range(Hq):
        ref = okv.decode_row_from_ring(Kr, Vr, t + 1, spans[h], inputs.as_f64(qt[0, h]), scale)
        err = float(np.max(np.abs(inputs.as_f64(ot[0, h]) - ref)))
        assert err <= BF16_TOL, (h, err)
