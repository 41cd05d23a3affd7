"""moa_decode_static_ws: decode for callers that cannot allocate device memory.

Some callers -- an operator plugin handed only input and output pointers, a
runtime whose device memory belongs entirely to another allocator, code that
must not call cudaMalloc because it synchronises the device -- cannot supply
moa_decode's workspace.  moa_decode_static_ws runs the same decode with its
scratch in a fixed 8 MiB array inside libmoa's device image.  These checks
call it through the C ABI and compare it with moa_decode (which uses a caller
workspace) on two calls in a row, so the second call also proves that the
shared array's leftover contents from the first call do no harm.

This file is named to be collected last; it passes alone in a fresh process
and after the rest of the suite.
"""

import math

import numpy as np
import pytest
import torch

from heterogeneous_sliding_window_b200 import inputs, moa

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def test_static_scratch_decode_matches_workspace_decode_twice():
    B, Hq, Hkv, d, prefix = 3, 8, 2, 128, 700
    spans = [40, 38, 300, 290, 600, 550, 599, 513]      # overlapping windows: the group-shared kernel
    caps = [max(spans[g * 4:(g + 1) * 4]) for g in range(Hkv)]
    scale = 1.0 / math.sqrt(d)
    cache = moa.KVCache(B, Hkv, d, "bf16", caps)
    cache.append(inputs.randn(1, (B, Hkv, prefix, d)).cuda(), inputs.randn(2, (B, Hkv, prefix, d)).cuda())
    ws = moa.Workspace(moa.MOA_OP_DECODE, B, Hq, 0, d, spans)
    for call in range(2):
        cache.append(inputs.randn(10 + call, (B, Hkv, 1, d)).cuda(), inputs.randn(20 + call, (B, Hkv, 1, d)).cuda())
        q = inputs.randn(30 + call, (B, Hq, d)).cuda()
        ref = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        got = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        moa.moa_decode(cache.handle, q, ref, Hq, spans, scale, ws.ptr, ws.nbytes)
        moa.moa_decode_static_ws(cache.handle, q, got, Hq, spans, scale)
        torch.cuda.synchronize()
        err = float(np.max(np.abs(inputs.as_f64(got) - inputs.as_f64(ref))))
        assert err <= BF16_TOL, (call, err)
    assert cache.positions() == [prefix + 2] * B


def test_static_scratch_rejects_requests_above_its_size():
    # 64 sequences x 32 heads x 8 splits of 520 B each need ~8.5 MB > 8 MiB.
    B, H, d = 64, 32, 128
    spans = [4096] * H
    cache = moa.KVCache(B, H, d, "bf16", spans)
    q = torch.zeros((B, H, d), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    with pytest.raises(moa.MoaError) as e:
        moa.moa_decode_static_ws(cache.handle, q, o, H, spans, 0.1)
    assert e.value.status == moa.MOA_ERR_WORKSPACE
