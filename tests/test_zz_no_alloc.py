"""moa_decode_static_ws: decode for callers that cannot allocate device memory.

Some callers -- an operator plugin handed only input and output pointers, a
runtime whose device memory belongs entirely to another allocator, code that
must not call cudaMalloc because it synchronises the device -- cannot supply
moa_decode's workspace.  moa_decode_static_ws runs the same decode with its
scratch in a fixed 8 MiB array inside libmoa's device image.  These checks
call it through the C ABI and compare it with moa_decode (which uses a caller
workspace) on two calls in a row: both run the same kernel on the same inputs,
so the outputs must be identical bit for bit, and the second call shows that
the shared array's leftover contents from the first do no harm.  One case is
also compared with the oracle's ring decode, and one checks that the calls
take no device memory.

This file is named to be collected last; it passes alone in a fresh process
and after the rest of the suite.
"""

import math

import numpy as np
import pytest
import torch

from heterogeneous_sliding_window_b200 import inputs, moa
from oracle import kvcache as okv

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
F32_TOL = 1e-5

CASES = [
    # (B, Hq, Hkv, dtype, d, prefix, spans)
    # overlapping windows of 4 heads per KV head: the tensor-core group kernel
    (3, 8, 2, "bf16", 128, 700, [40, 38, 300, 290, 600, 550, 599, 513]),
    # one query head per KV head, multi-split heads: the per-head kernel
    (2, 4, 4, "bf16", 128, 900, [1, 256, 257, 900]),
    # fp32, d = 64, one query head per KV head: the per-head fp32 kernel
    (2, 4, 4, "f32", 64, 600, [32, 64, 513, 600]),
]


def _bits(x):
    return x.view(torch.int16 if x.dtype == torch.bfloat16 else torch.int32)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_H%d_%d_%s_d%d" % c[:5])
def test_static_scratch_decode_equals_workspace_decode_twice(case):
    B, Hq, Hkv, dt, d, prefix, spans = case
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    tol = BF16_TOL if dt == "bf16" else F32_TOL
    G = Hq // Hkv
    caps = [max(spans[g * G:(g + 1) * G]) for g in range(Hkv)]
    scale = 1.0 / math.sqrt(d)
    cache = moa.KVCache(B, Hkv, d, dt, caps)
    ring = okv.RingCache(B, Hkv, d, caps)
    k0 = inputs.randn(1, (B, Hkv, prefix, d), dt)
    v0 = inputs.randn(2, (B, Hkv, prefix, d), dt)
    cache.append(k0.cuda(), v0.cuda())
    ring.append(inputs.as_f64(k0), inputs.as_f64(v0))
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    for call in range(2):
        kt = inputs.randn(10 + call, (B, Hkv, 1, d), dt)
        vt = inputs.randn(20 + call, (B, Hkv, 1, d), dt)
        cache.append(kt.cuda(), vt.cuda())
        ring.append(inputs.as_f64(kt), inputs.as_f64(vt))
        q = inputs.randn(30 + call, (B, Hq, d), dt)
        ref = torch.full((B, Hq, d), float("nan"), dtype=tdt, device="cuda")
        got = torch.full((B, Hq, d), float("nan"), dtype=tdt, device="cuda")
        moa.moa_decode(cache.handle, q.cuda(), ref, Hq, spans, scale, ws.ptr, ws.nbytes)
        moa.moa_decode_static_ws(cache.handle, q.cuda(), got, Hq, spans, scale)
        torch.cuda.synchronize()
        assert torch.equal(_bits(got), _bits(ref)), call
        expect = okv.decode(ring, inputs.as_f64(q), spans, scale)
        err = float(np.max(np.abs(inputs.as_f64(got) - expect)))
        assert err <= tol, (call, err)
    assert cache.positions() == ring.t == [prefix + 2] * B


def test_static_scratch_decode_takes_no_device_memory():
    B, Hq, Hkv, d, prefix = 2, 8, 2, 128, 500
    spans = [40, 38, 300, 290, 500, 450, 499, 413]
    caps = [max(spans[g * 4:(g + 1) * 4]) for g in range(Hkv)]
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    cache.append(inputs.randn(3, (B, Hkv, prefix, d)).cuda(), inputs.randn(4, (B, Hkv, prefix, d)).cuda())
    q = inputs.randn(5, (B, Hq, d)).cuda()
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    moa.moa_decode_static_ws(cache.handle, q, o, Hq, spans, 0.1)    # first call: per-device set-up
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        moa.moa_decode_static_ws(cache.handle, q, o, Hq, spans, 0.1)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == torch_before
    # a cudaMalloc of any size takes at least one 2 MiB page from the free pool
    assert torch.cuda.mem_get_info()[0] >= free_before


def test_static_scratch_rejects_requests_above_its_size():
    # 64 sequences x 32 query heads x 8 splits of 520 B each need ~8.5 MB > 8 MiB.
    # The workspace does not depend on the KV heads, so one KV head keeps the
    # cache small (134 MB); the call is refused on the host before any launch.
    B, Hq, Hkv, d = 64, 32, 1, 128
    spans = [4096] * Hq
    cache = moa.KVCache(B, Hkv, d, "bf16", [4096])
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    with pytest.raises(moa.MoaError) as e:
        moa.moa_decode_static_ws(cache.handle, q, o, Hq, spans, 0.1)
    assert e.value.status == moa.MOA_ERR_WORKSPACE
