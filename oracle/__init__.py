"""CPU oracle for heterogeneous sliding-window attention (MoA).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
link this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

The oracle is a plain, slow, obviously-correct restatement of what the
method computes, written in numpy float64 with Python integer arithmetic
for every index.  It shares no code with the CUDA library under
``heterogeneous_sliding_window_b200/``: no kernels, no headers, no layout or
table generators.  The only module both sides use is the seeded input
generator ``heterogeneous_sliding_window_b200/inputs.py``, which holds none
of the method's arithmetic.

Sources (web pages on the method; cited by title and section):

* "Mixture of Attention" project page (MoA, COLM 2025), section "Key
  findings / Finding two: windows change with input length" -- the per-head
  linear span rule S = alpha + beta * N and the worked heads A, B, C with
  their figure caption; section "Method design / Elastic search space" --
  candidate rules must respect the kernel's block size; section "Demo",
  step 03 -- deployment with a fixed-size, sparse, per-head KV cache.
* "MoA: Mixture of Sparse Attention for Automatic Large Language Model
  Compression" (blog walkthrough), section 2.1 "Elastic sparse rules" --
  sliding-window mask per head with a linear span; section 5 "Usage guide
  and implementation details" -- a CUDA kernel with a static KV cache and
  masked attention aggregation.

Modules:

* :mod:`oracle.rules`     -- span rule (rounding to the block, clamping).
* :mod:`oracle.attention` -- windowed causal softmax attention (prefill).
* :mod:`oracle.kvcache`   -- per-head ring-buffer cache emulation, its byte
  image, and decode attention served from the ring.

Parity status: every public function here is pinned by ``-m "not gpu"``
tests against values or properties fixed outside the oracle itself (the
project page's worked examples, torch's dense causal SDPA, brute force with
an explicit N x N mask, closed forms).  No function is "parity unpinned".
"""

from . import rules, attention, kvcache  # noqa: F401

__all__ = ["rules", "attention", "kvcache"]
