"""CPU fp64 oracle for the tensor-parallel (column/row) linear block.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may use it. It shares no code with the CUDA
library (no kernels, headers, helpers or tables); the only thing both sides share
is the seeded input generator in ``workloads.py``, which holds none of the
block's arithmetic.

Everything here is plain numpy in float64 on the exact values of the bf16
inputs, written from the definitions on the source pages:

* "Tensor Parallel：当一张 GPU 放不下一个大模型" (mini vLLM tutorial), sections
  "Column Parallel Linear：按输出维度切", "Row Parallel Linear：按输入维度切",
  "Attention 里的 tensor parallel", "MLP 里的 tensor parallel",
  "如何验证 tensor parallel 正确", "lm_head 怎么处理" (vocab-parallel greedy argmax).
* "张量并行（Tensor Parallelism）推理部署实战：从 Megatron-LM 切分原理到 vLLM 多卡配置与性能调优",
  sections 1.1 (column-parallel), 1.2 (row-parallel), 二 (Megatron MLP), 2.1
  (attention), 6.3 (TP size must divide the head count).
* "Tensor Parallel 深入解析：多加 GPU，推理为什么可能更慢", sections
  "两张卡如何共同算出一层" (the hand-computed worked example) and
  "权重变小，不代表所有显存都按比例变小" (GQA KV-head replication).

Pins (see ``tests/test_oracle_pins.py``): the worked example, brute-force loops
on tiny integer inputs for every divisor tp, the column-concat / row-sum
invariants, textbook values of GELU and SiLU and their odd-part identities,
torch's own bf16 cast on float32-exact values, hand-picked bf16 ties, and an
exhaustive property check of the GQA head map; for attention on local heads, the
closed forms of uniform weights (Q = 0: means and prefix means of V), one key,
dominant-score selection, torch's own scaled_dot_product_attention (with its
grouped-query option) and sharded-equals-unsharded for every valid tp. Float
workloads at full size are
parity-pinned only through these (no page prints results at those shapes).
"""

from .tp_oracle import *  # noqa: F401,F403
