"""CPU oracle for CoSA's prefill path (KAP proxy, page remap, OSK attention).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
the benchmark's CPU-baseline / reference legs may import this package.  The
library's product path never calls into it, and it shares no code with the
CUDA kernels: no helpers, tables, constants or pre/post-processing.

It is deliberately plain and slow: numpy, one step after another in the order
the pages describe ("CoSA: Accelerating Long-Context Inference via
Proxy-Kernel Co-Designed Sparse Attention", §4 CoSA and Appendix C), with the
open points fixed as stated in each function.

  kap      -- Kernel-Aware Proxy: pooled block scores, HRM flags, flag-grouped
              ordering, budget cut (§4.2; Appendix C.1, Figure A).  fp32
              arithmetic, because its integer outputs must be reproduced bit
              for bit; every fp32 step is a single IEEE operation.
  remap    -- ordered block list -> physical KV page list (§4.3, "Any-order
              page visiting").
  osk      -- Ordered-Skipping Kernel semantics: visit the selected blocks in
              order, online softmax, in-kernel skip of the value side
              (§3.3, §4.3, Appendix C.2 / Algorithm A, Appendix D.1).  fp64.
  dense    -- brute-force dense causal softmax attention, fp64 (§3.1), used as
              the closed form the OSK oracle must reduce to at budget 100% and
              tau = 0.
  parallel -- OraclePool: osk tiles evaluated in spawned worker processes
              (tiles are independent; the pool only distributes them).
  _layout  -- which q-blocks exist and where their rows sit in the packed Q,
              for full prefill and for prefill after a cached prefix
              (q_len < kv_len; a reading, the pages treat full prefill only).

Parity status: the proxy's score and HRM definitions are this oracle's own
reading of the empty "Block ranking" paragraph (§4.2); they are pinned by
bounds, brute force and constructed cases, but not by any value the pages
print (none survive), so the score semantics beyond that are parity
unpinned.  The skip rule (Eq. (5) is missing from the pages) is pinned by the
constructions of §3.3's two limitations and by its error bound.
"""
