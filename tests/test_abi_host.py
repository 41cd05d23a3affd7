"""Host-side checks of libmoa's C ABI: symbols, span rule, schedule, sizes, argument errors.

No test here launches a kernel; each runs without a GPU.
"""

import ctypes
import os
import random
import re

import numpy as np
import pytest

from heterogeneous_sliding_window_b200 import moa
from heterogeneous_sliding_window_b200 import inputs
from oracle import rules as orules, kvcache as okv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not os.path.exists(moa.LIB_PATH):
        from heterogeneous_sliding_window_b200 import build
        build.build()
    moa.load()


def _declared_symbols():
    names = set()
    with open(os.path.join(ROOT, "include", "moa.h")) as f:
        text = f.read()
    for m in re.finditer(r"^\s*(?:const\s+)?[\w\s\*]+?\b(moa_\w+)\s*\(", text, re.M):
        names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported():
    declared = _declared_symbols()
    assert len(declared) >= 15, declared
    lib = ctypes.CDLL(moa.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(moa.EXPORTS)


def test_rules_bit_exact_against_oracle():
    """10^6 random (alpha, beta, N, block) tuples, exact ties included."""
    rnd = np.random.default_rng(11)
    n_done = 0
    while n_done < 1_000_000:
        N = int(rnd.integers(1, 1 << 20))
        block = int(rnd.choice([1, 16, 32, 64, 128, 256]))
        n = 1000
        kind = rnd.integers(0, 3)
        if kind == 0:      # arbitrary doubles
            a = rnd.uniform(0, 3 * N, n)
            b = rnd.uniform(0, 1.5, n)
        elif kind == 1:    # exact ties: alpha = (k + 1/2) * block, beta = 0
            a = (rnd.integers(0, 2 * N // block + 2, n) + 0.5) * block
            b = np.zeros(n)
        else:              # candidate-set-like values
            a = rnd.choice([0.0, 512.0, 1024.0, 2048.0, 1600.0, 5600.0], n) * rnd.choice([1.0, 0.37, 1.91], n)
            b = rnd.choice([0.0, 0.125, 0.25, 0.5, 0.9, 1.0], n) * rnd.choice([1.0, 0.37, 1.91], n)
        got = moa.moa_rules_eval(a, b, N, block)
        ref = [orules.span_rule(x, y, N, block) for x, y in zip(a.tolist(), b.tolist())]
        assert got == ref, (N, block)
        n_done += n


def test_rules_project_page_heads():
    assert moa.moa_rules_eval([1600, 5600, 0], [0, 0, 0.9], 4096, 64) == [1600, 4096, 3712]
    assert moa.moa_rules_eval([1600, 5600, 0], [0, 0, 0.9], 16384, 64) == [1600, 5632, 14720]


@pytest.mark.parametrize("a,b,N,blk", [
    (float("nan"), 0.0, 10, 1), (0.0, float("inf"), 10, 1), (-1.0, 0.0, 10, 1),
    (1.0, 0.0, 0, 1), (1.0, 0.0, 10, 0), (1.0, 0.0, 1 << 31, 1)])
def test_rules_invalid(a, b, N, blk):
    with pytest.raises(moa.MoaError) as e:
        moa.moa_rules_eval([a], [b], N, blk)
    assert e.value.status == moa.MOA_ERR_INVALID_ARG


def _tiles_needed_brute(m, S, N):
    """Key tiles that hold at least one in-window key of some row of q-tile m."""
    need = set()
    for i in range(128 * m, min(128 * m + 128, N)):
        for j in range(max(0, i - S + 1), i + 1):
            need.add(j // 128)
    return need


@pytest.mark.parametrize("N,spans,n_ctas", [(1000, [1, 64, 127, 128, 129, 300, 1000, 5000], 7),
                                            (128, [1, 128], 148), (129, [2, 129], 3), (5, [3], 1),
                                            (640, [256, 700], 2), (8192, [64, 4736, 576, 5568], 148)])
def test_prefill_schedule_covers_band(N, spans, n_ctas):
    B = 2
    Hq = len(spans)
    rows = moa.moa_prefill_schedule(B, Hq, N, spans, n_ctas)
    M = (N + 127) // 128
    assert rows.shape == (B * Hq * M, 7)
    seen = set()
    unit_tiles = {}
    unit_cta = {}
    order = []
    for cta, unit, b, h, m, lo, hi in rows.tolist():
        assert (b, h, m) not in seen
        seen.add((b, h, m))
        assert hi == m
        need = _tiles_needed_brute(m, spans[h], N) if N <= 1000 else set(
            range(max(0, 128 * m - spans[h] + 1) // 128, m + 1))
        assert set(range(lo, hi + 1)) == need   # exactly the band's tiles, none skipped, none extra
        unit_tiles.setdefault(unit, []).append((m, lo, hi))
        assert unit_cta.setdefault(unit, cta) == cta
        if not order or order[-1] != unit:
            order.append(unit)
    assert len(seen) == B * Hq * M
    assert order == sorted(order)               # rows of a unit adjacent, units numbered in run order
    n_used = len(set(unit_cta.values()))
    assert n_used == min(n_ctas, len(order))
    # a unit is two consecutive query tiles of one head (one tile only at a head's end)
    for unit, ts in unit_tiles.items():
        ms = [t[0] for t in ts]
        assert ms[0] % 2 == 0 and ms == list(range(ms[0], ms[0] + len(ms))) and len(ms) <= 2
    # each CTA runs its units longest first; the lists are balanced within one unit (greedy LPT bound)
    cost = {u: sum(hi - lo + 1 for _, lo, hi in ts) + 4 for u, ts in unit_tiles.items()}
    load = {}
    for u in order:
        c = unit_cta[u]
        load.setdefault(c, []).append(cost[u])
    for c, cs in load.items():
        assert cs == sorted(cs, reverse=True)
    totals = [sum(cs) for cs in load.values()]
    assert max(totals) - min(totals) <= max(cost.values())


def _greedy_lpt(B, Hq, N, spans, n_ctas):
    """The schedule rule in plain Python: units of query tiles (m, m+1) of one
    (b, h), cost = their key-tile count + 4, sorted by cost (longest first,
    ties in (b, h, m) order), each dealt to the list with the least work
    (ties: the lowest list).  Returns the rows moa_prefill_schedule reports."""
    M = (N + 127) // 128
    first = lambda t, S: max(0, 128 * t - S + 1) // 128     # noqa: E731
    units = []
    for b in range(B):
        for h in range(Hq):
            for m in range(0, M, 2):
                cost = m - first(m, spans[h]) + 1 + 4
                if m + 1 < M:
                    cost += m + 1 - first(m + 1, spans[h]) + 1
                units.append((cost, b, h, m))
    order = sorted(range(len(units)), key=lambda i: -units[i][0])   # Python's sort is stable
    n = max(1, min(n_ctas, len(units)))
    work = [0] * n
    lists = [[] for _ in range(n)]
    for i in order:
        c = min(range(n), key=lambda j: (work[j], j))
        lists[c].append(i)
        work[c] += units[i][0]
    rows, k = [], 0
    for c in range(n):
        for i in lists[c]:
            _, b, h, m = units[i]
            for t in range(m, min(m + 2, M)):
                rows.append((c, k, b, h, t, first(t, spans[h]), t))
            k += 1
    return rows


@pytest.mark.parametrize("B,N,spans,n_ctas", [(1, 8192, None, 148), (2, 1000, [1, 64, 300, 1000, 129], 7),
                                              (3, 640, [256, 700], 5), (1, 129, [2, 129], 148)])
def test_prefill_schedule_is_the_greedy_lpt_rule(B, N, spans, n_ctas):
    if spans is None:                        # the bench prompt's spans
        a, b = inputs.tables_7b(1, 32, N, 64, 0.25, orules.eval_spans)
        spans = orules.eval_spans(a, b, N, 64)
    got = [tuple(r) for r in moa.moa_prefill_schedule(B, len(spans), N, spans, n_ctas).tolist()]
    assert got == _greedy_lpt(B, len(spans), N, spans, n_ctas)


def test_prefill_schedule_arguments():
    with pytest.raises(moa.MoaError):
        moa.moa_prefill_schedule(1, 1, 128, [64], 0)
    with pytest.raises(moa.MoaError):
        moa.moa_prefill_schedule(1, 1, 128, [64], 1025)


def test_host_memory_failure_is_a_status():
    """A plan whose host vectors cannot be allocated (about 2^61 work units) comes back as
    MOA_ERR_HOST: no C++ exception crosses the C boundary, and the process goes on."""
    with pytest.raises(moa.MoaError) as e:
        moa.moa_prefill_schedule(2**31 - 1, 128, 2**31 - 1, [1] * 128, 148)
    assert e.value.status == moa.MOA_ERR_HOST
    lib = moa.load()
    assert lib.moa_status_string(moa.MOA_ERR_HOST) == b"MOA_ERR_HOST"
    assert len(moa.moa_prefill_schedule(1, 1, 128, [64], 1)) == 1


def test_kv_sizes_match_layout():
    for B, Hkv, d, caps, dt, eb in [(2, 2, 4 * 16, [2, 3], "bf16", 2), (31, 3, 128, [5, 1, 9], "f32", 4),
                                   (32, 32, 128, [2048] * 32, "bf16", 2)]:
        assert moa.moa_kv_header_bytes(B) == okv.header_bytes(B)
        assert moa.moa_kv_bytes(B, Hkv, d, dt, caps) == okv.buffer_bytes(B, Hkv, d, caps, eb)


def test_kv_invalid():
    with pytest.raises(moa.MoaError):
        moa.moa_kv_bytes(1, 1, 96, "bf16", [4])       # head dim not supported
    with pytest.raises(moa.MoaError):
        moa.moa_kv_bytes(1, 2, 128, "bf16", [4, 0])   # zero capacity
    with pytest.raises(moa.MoaError) as e:
        moa.moa_kv_alloc(256, 10, 1, 1, 128, "bf16", [4])  # buffer too small
    assert e.value.status == moa.MOA_ERR_CAPACITY
    with pytest.raises(moa.MoaError) as e:
        moa.moa_kv_alloc(8, 1 << 20, 1, 1, 128, "bf16", [4])  # misaligned
    assert e.value.status == moa.MOA_ERR_INVALID_ARG


def test_prefill_argument_errors_need_no_gpu():
    ok = dict(q=4096, k=4096, v=4096, o=4096, B=1, Hq=4, Hkv=2, N=256, d=128, dtype="bf16",
              spans=[64] * 4, scale=0.088, ws=None, ws_bytes=0, stream=0)
    bad = [dict(q=None), dict(q=4097), dict(Hq=3), dict(N=0), dict(d=96), dict(spans=[0, 1, 1, 1]),
           dict(scale=float("nan"))]
    for change in bad:
        args = dict(ok)
        args.update(change)
        with pytest.raises(moa.MoaError) as e:
            moa.moa_prefill(**args)
        assert e.value.status == moa.MOA_ERR_INVALID_ARG, change
    args = dict(ok)
    with pytest.raises(moa.MoaError) as e:      # bf16 needs a workspace
        moa.moa_prefill(**args)
    assert e.value.status == moa.MOA_ERR_WORKSPACE
    args.update(d=64, ws=4096, ws_bytes=1 << 20)
    with pytest.raises(moa.MoaError) as e:      # bf16 d=64 not implemented
        moa.moa_prefill(**args)
    assert e.value.status == moa.MOA_ERR_UNSUPPORTED


def test_stream_read_argument_errors_need_no_gpu():
    for buf, nbytes, out in [(None, 16, 4096), (4096, 16, None), (4104, 16, 4096), (4096, 24, 4096),
                             (4096, 16, 4100)]:
        with pytest.raises(moa.MoaError) as e:
            moa.moa_stream_read(buf, nbytes, out, 0)
        assert e.value.status == moa.MOA_ERR_INVALID_ARG, (buf, nbytes, out)


def test_prefill_chunk_argument_errors_need_no_gpu():
    with pytest.raises(moa.MoaError) as e:
        moa.moa_chunk_workspace_bytes(None, 4, 128, [64] * 4)
    assert e.value.status == moa.MOA_ERR_INVALID_ARG
    with pytest.raises(moa.MoaError) as e:
        moa.moa_prefill_chunk(None, 4096, 4096, 4096, 4096, 4, 128, [64] * 4, 0.088, 4096, 1 << 20, 0)
    assert e.value.status == moa.MOA_ERR_INVALID_ARG
    with pytest.raises(moa.MoaError) as e:      # misaligned q is rejected before the cache is looked at
        moa.moa_prefill_chunk(None, 4100, 4096, 4096, 4096, 4, 128, [64] * 4, 0.088, 4096, 1 << 20, 0)
    assert e.value.status == moa.MOA_ERR_INVALID_ARG


def test_prefill_stall_test_argument_errors_need_no_gpu():
    with pytest.raises(moa.MoaError) as e:
        moa.moa_prefill_stall_test(None, 4096, 4096, 4096, 4096, 1 << 20, 0)
    assert e.value.status == moa.MOA_ERR_INVALID_ARG
    with pytest.raises(moa.MoaError) as e:          # workspace not 256-byte aligned
        moa.moa_prefill_stall_test(4096, 4096, 4096, 4096, 4096 + 16, 1 << 20, 0)
    assert e.value.status == moa.MOA_ERR_WORKSPACE


def test_workspace_sizes():
    spans = [64, 300, 4096, 1]
    d = moa.moa_workspace_bytes(moa.MOA_OP_DECODE, 2, 4, 0, 128, spans)
    p = moa.moa_workspace_bytes(moa.MOA_OP_PREFILL, 2, 4, 1000, 128, spans)
    assert d % 256 == 0 and d >= 256 + 2 * 4 * 4
    assert p >= 256 + 2 * 4 * 8 * 16   # one unit per 128-row query tile
    with pytest.raises(moa.MoaError):
        moa.moa_workspace_bytes(moa.MOA_OP_DECODE, 2, 4, 0, 128, [64, 0, 1, 1])


def test_decode_workspace_holds_the_small_batch_splits():
    """A decode launch with under 1 024 splits of 512 entries takes 256-entry splits, so its
    workspace must hold twice as many partials (m, l and d floats each) as 512-entry splits."""
    d, Hq = 128, 32
    spans = [4096] * Hq                           # 8 splits of 512 per head
    def partial_bytes(B, chunk):
        return B * Hq * (-(-4096 // chunk)) * (d + 2) * 4
    small = moa.moa_workspace_bytes(moa.MOA_OP_DECODE, 1, Hq, 0, d, spans)       # 256 at 512: half-size splits
    large = moa.moa_workspace_bytes(moa.MOA_OP_DECODE, 32, Hq, 0, d, spans)      # 8192 at 512
    assert small >= partial_bytes(1, 256)
    assert large >= partial_bytes(32, 512)
    assert large < partial_bytes(32, 256)          # large launches keep 512-entry splits


def test_input_tables_reach_target_density():
    """The seeded table generator lands near the requested mean span / N."""
    for density, N in [(0.25, 8192), (0.5, 4096), (0.125, 32768)]:
        a, b = inputs.tables_7b(3, 32, N, 64, density, orules.eval_spans)
        spans = orules.eval_spans(a, b, N, 64)
        assert abs(np.mean(spans) / N - density) < 0.02
        assert all(s % 64 == 0 for s in spans)
        # the product-side rule gives the same tables and spans
        a2, b2 = inputs.tables_7b(3, 32, N, 64, density, moa.moa_rules_eval)
        assert np.array_equal(a, a2) and np.array_equal(b, b2)
        assert moa.moa_rules_eval(a2, b2, N, 64) == spans
    a, b = inputs.tables_13b_mix(5, 40, 16384, 64, 0.5, orules.eval_spans)
    spans = orules.eval_spans(a, b, 16384, 64)
    assert abs(np.mean(spans) / 16384 - 0.5) < 0.05
    assert set(np.unique(b)) <= {0.0, 0.5, 0.9}


def test_sink_cache_sizes_and_errors():
    for B, Hkv, d, caps, sinks, dt, eb in [(2, 2, 64, [3, 2], [2, 1], "f32", 4),
                                          (3, 4, 128, [5, 1, 9, 4], [0, 0, 7, 0], "bf16", 2),
                                          (1, 1, 128, [8], [0], "bf16", 2)]:
        assert moa.moa_kv_bytes_sink(B, Hkv, d, dt, caps, sinks) == okv.buffer_bytes(B, Hkv, d, caps, eb, sinks)
    assert moa.moa_kv_bytes_sink(2, 2, 128, "bf16", [3, 5], [0, 0]) == moa.moa_kv_bytes(2, 2, 128, "bf16", [3, 5])
    with pytest.raises(moa.MoaError) as e:
        moa.moa_kv_bytes_sink(1, 2, 128, "bf16", [4, 4], [1, -1])     # negative global-token rows
    assert e.value.status == moa.MOA_ERR_INVALID_ARG
    with pytest.raises(moa.MoaError) as e:
        moa.moa_kv_bytes_sink(1, 2, 128, "bf16", [4, 4], [1 << 30, 1 << 30])   # sum above 2^31 - 1
    assert e.value.status == moa.MOA_ERR_INVALID_ARG


def test_sink_prefill_and_workspace_argument_errors_need_no_gpu():
    ok = dict(q=4096, k=4096, v=4096, o=4096, B=1, Hq=4, Hkv=2, N=256, d=128, dtype="bf16",
              spans=[64] * 4, sinks=[4] * 4, scale=0.088, ws=None, ws_bytes=0, stream=0)
    for change, status in [(dict(sinks=[4, -1, 0, 0]), moa.MOA_ERR_INVALID_ARG),
                           (dict(spans=[0, 1, 1, 1]), moa.MOA_ERR_INVALID_ARG),
                           (dict(), moa.MOA_ERR_WORKSPACE)]:
        args = dict(ok)
        args.update(change)
        with pytest.raises(moa.MoaError) as e:
            moa.moa_prefill_sink(**args)
        assert e.value.status == status, change
    spans, sinks = [64, 300, 4096, 1], [0, 600, 4, 1]
    plain = moa.moa_workspace_bytes(moa.MOA_OP_DECODE, 2, 4, 0, 128, spans)
    more = moa.moa_workspace_bytes_sink(moa.MOA_OP_DECODE, 2, 4, 0, 128, spans, sinks)
    assert more > plain and more % 256 == 0
    assert moa.moa_workspace_bytes_sink(moa.MOA_OP_DECODE, 2, 4, 0, 128, spans, [0] * 4) == plain
    assert moa.moa_workspace_bytes_sink(moa.MOA_OP_PREFILL, 2, 4, 1000, 128, spans, sinks) == \
        moa.moa_workspace_bytes(moa.MOA_OP_PREFILL, 2, 4, 1000, 128, spans)
    with pytest.raises(moa.MoaError):
        moa.moa_workspace_bytes_sink(moa.MOA_OP_DECODE, 2, 4, 0, 128, spans, [0, -2, 0, 0])

