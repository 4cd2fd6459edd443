"""CPU oracle for exact blockwise (Ring / Striped) causal attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library and imports nothing from it.

Everything here is plain NumPy in float64 and follows the definitions on the
source pages:

* ``attention``    -- the plain definition Softmax(QK^T * scale + C) V
  ("Striped Attention: Faster Ring Attention for Causal Transformers",
  section 三 技术架构 / 核心公式, causal mask C) with the score scale of
  "ICLR 2024論文解説: Ring Attention", ステップ3.
* ``partition``    -- contiguous (Ring) and modulo-striped (Striped) token
  placement (Ring Attention explainer ステップ1; Striped review 分区策略对比).
* ``masks``        -- the two GetMask procedures (Striped review, GetMask 函数)
  and the same masks derived from global token positions.
* ``ring``         -- the method itself, restated step by step: Q block fixed,
  KV blocks visiting in ring order, online-softmax fold per round (Ring
  Attention explainer ステップ2/ステップ3 and its 実装例); one device's
  per-round partial (``block_attention``) and the ring restated as a merge
  of those partials (``ring_by_merge``, 1cademy page).
* ``work``         -- the per-device/per-round work formulas (Striped review,
  Ring Attention 工作负载 / Striped Attention 工作负载) and brute-force counts.
* ``backward``     -- gradients dQ, dK, dV of the definition (the pages give
  no backward; the textbook softmax derivative of 核心公式).
* ``rope``         -- rotary position embedding at the original token
  positions, then the stripe (Striped review, 位置编码处理 names RoPE; the
  rotation itself is RoFormer's, not defined on the pages).
* ``merge``        -- merging two partial (O, lse) results by splitting the
  softmax denominator into per-node partial sums (1cademy page "Computing
  Attention Weights in Sequence Parallelism").

Pins: every function is checked in ``tests/test_oracle_*.py`` against
something other than itself (brute force on tiny inputs, closed forms, the
worked striping example printed on the Striped review page, invariants).
Functions with no such pin say "parity unpinned" in their docstring; there are
none at present.
"""

from . import attention, backward, merge, masks, partition, ring, rope, work  # noqa: F401
