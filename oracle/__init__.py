"""CPU oracle for the fused attention forward and its quantized block-sparse variant.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or execute
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, helpers or tables); the two meet only in the
seeded inputs of ``workloads``.

Sources (web pages, cited by title and section):

* npu_fusion_attention guide -- "昇腾 NPU 融合注意力算子详解与迁移指南":
  §2 算子数学原理 (the attention formula), §4.2 (atten_mask: 1 = masked, 0 = kept;
  BNSS / B1SS / SS), §4.3 (sparse_mode 0 / 2 / 3; cumulative actual_seq_qlen /
  actual_seq_kvlen), §5 输出说明 (attention_out, softmax_max, softmax_sum),
  §6.1 (the discrete matmul -> +mask -> softmax -> matmul composition), §7 (GQA).
* EagleQBSA article -- "昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍":
  section "EagleQBSA量化叠加稀疏方案设计" with Fig 2.1 (Q/K per-block INT8, V
  per-channel FP8, P to FP8), section "昇腾亲和的量化叠加稀疏Attention算子优化"
  (P rounded to FP8) and section "MindIE SD调用方式" (block_sparse_mask,
  block_shape=[128,128], scale_value, per-tensor scales).

Modules:

* ``formats``  -- bf16 decoding and the OCP E4M3 (FP8) codec, from the format definitions.
* ``dense``    -- the plain definition Softmax(Mask(Q Kᵀ·scale + pse))·V in fp64, plus a
  pure-Python loop version for tiny inputs and the K-tile sets a tiled kernel must visit.
* ``quant``    -- the Q/K per-block INT8 and V per-channel E4M3 quantisers and the
  quantized block-sparse forward, step by step in the article's order.
* ``estimate`` -- block-mask estimation (block mean pooling, block scores, top-k), a plain
  reading of the block selection the EagleQBSA article names but does not describe.

Parity status of every function is stated in its docstring; none is "parity unpinned"
except where a docstring says so.
"""

from . import formats, dense, quant, estimate  # noqa: F401
