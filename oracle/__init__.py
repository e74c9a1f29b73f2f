"""fp64 CPU oracle for the differential attention forward.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product path (the CUDA library and its Python binding) never
imports, links or calls anything here, and this package imports nothing from
the product path.

Sources (page title, section):
  * "差分注意力" tutorial (aiknowledge.cn), sections 差分思路, V1 到 V2 的 diff,
    二、从零实现 Step 1-4 -- the main algorithmic authority.
  * "【架构革新】Differential Transformer：用“差分降噪”重塑LLM注意力机制"
    (mcipr.com), section 3 工程实践 -- the lambda_init layer schedule.
  * "Understanding Differential Transformer Unchains Pretrained
    Self-Attentions" (paper note), section 关键设计 -- A_diff = A1 - lambda*A2.

Modules:
  diffattn -- definition-level NumPy fp64 implementation (library matmul as a
              step, no blocking beyond a row chunk that does not change the math).
  brute    -- pure-Python per-element loops for tiny shapes; an independent twin
              used to cross-check ``diffattn``.
  backward -- the chain rule of the forward (dQ, dK, dV, dlambda and lambda's
              parameter gradients) in fp64, pinned by finite differences and an
              independent autograd derivation (tests/test_oracle_backward.py).
  lowrank  -- the fixed low-rank substitute for A2 (paper note, sections
              基于分析的改进建议 and 亮点与洞察), under the reading in its
              header, pinned in tests/test_oracle_lowrank.py.

Parity status: every function is pinned by tests in ``tests/test_oracle.py``
except the page's claimed noise-floor percentages and the SNR claim of the
tutorial's Step 3, which are "parity unpinned" (see ``diffattn.noise_probe``).
"""

from . import backward, brute, diffattn, lowrank  # noqa: F401
