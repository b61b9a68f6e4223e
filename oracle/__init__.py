"""CPU oracle for the LSA hot path -- TEST INFRASTRUCTURE, not part of the product.

Only the test suite, the smoke check in ``__graft_entry__`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and shares no
code with it; the two meet only in the seeded inputs of ``lsa_synth``.

Everything is computed in float64 from the exactly decoded stored inputs (BF16 bits,
FP8 e4m3 codes times their per-token scale), by the plain definitions:

* ``formats``  -- BF16 and OCP FP8 e4m3 decoding, written from the format definitions.
* ``lsa``      -- indexer score, block keys / block scores, full-sort top-k with the
                  (score desc, index asc) order, the sink / window union, softmax
                  attention over the selected rows, and the log-sum-exp merge of partials.
* ``run``      -- the whole path for one query token of a synthetic workload.

Sources (web pages on LongCat-2.0 and its sparse attention, LSA):

* [explainer]  "如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？", section
               "① LSA：从“每个 Query 全量扫”改成“先索引、再稀疏读”" (with its
               sub-headings "DSA 的瓶颈" and "LSA 的改法") and section "③ KVP 解码切分示意".
* [release]    "美团大模型LongCat-2.0 正式发布，总参数量达 1.6 万亿，使用国产算力集群",
               section "LongCat 稀疏注意力" (the SI, CLI and HI bullets and the MTP
               paragraph) and section "确定性与可靠性".
* [notes]      "LongCat-2.0 深度技术解读", section "2. 架构改进一：LSA".

The pages describe LSA in words only; they print no formula, shape or worked example.
The readings taken where they are silent are listed in each function's docstring.
"""
from . import formats, lsa  # noqa: F401
