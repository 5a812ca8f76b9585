"""fp64 CPU oracle for ring-blockwise causal attention (MM-SP hot path).

TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library and
its Python binding) imports, calls or links anything here; only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` do. The
oracle shares no code with the CUDA path: it receives the same seeded input
arrays (built by ``mmsp_inputs``) and nothing else.

Sources ("page" = the web page the method is described on):

* "LongVILA Guide: 2M Context Multi-Modal AI Model" (aifetchly blog),
  section "Multi-Modal Sequence Parallelism (MM-SP) Mechanics", Ring-SP
  paragraph: each rank holds N/P tokens and the KV blocks travel around a
  ring in P-1 shifts;
* same page, section "Implementation: PyTorch Distributed Pipeline and Token
  Routing", class ``LongVILAMultiModalAttention`` (ring loop, scale 1/sqrt(d),
  (B,S,H,D) layout) and class ``LongVILAParallelContext`` (ring neighbours:
  receive from the previous ring rank, send to the next).

Readings where the pages are silent or wrong:
the partial results of the ring steps are combined with the log-sum-exp merge
(the page's sketch sums separately normalised blocks, which is not attention);
the causal mask is j <= i over global positions; zigzag sharding gives rank r
chunks r and 2P-1-r; GQA maps query head h to kv head floor(h*Hkv/Hq); LSE is
a natural log; a row with no visible key has LSE = -inf and O = 0.

Modules:
  sharder   -- naive zigzag sharder (Python loops)
  attention -- causal softmax attention by its definition, forward and
               backward, whole-sequence and sampled rows/keys
  merge     -- the log-sum-exp merge and a ring simulation over P virtual
               ranks that uses it
Every function here is pinned by tests/test_oracle_*.py (closed forms, hand
worked examples under tests/golden/, brute force and library cross-checks).
"""
from . import sharder, attention, merge  # noqa: F401
