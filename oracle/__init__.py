"""fp64 CPU oracle for the Ring Attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package may import, call
or execute anything under this directory; only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` use it.  It shares no code, table or constant with the
CUDA path and imports nothing from the product package.

Sources (web pages, cited by title and section / equation / table):

* "AI 推理系列（十一）：Ring Attention 如何让多张 GPU 共同计算一条超长序列"
  (wiblog.cn) -- ring schedule, online-softmax accumulation, causal skip.
* "LLM长文本推理Ring Attention环形注意力机制实现与优化" (yunthe.com) --
  the blockwise update with running max / exp-sum / beta / gamma.
* "长上下文的第一性挑战" (t6page) -- Eq. (lc-ch-attention), Eq.
  (lc-ch-kv-memory), tables kv-size and decode-bw.
* "上下文并行 (CP) 收益评估实验设计" (t6page) -- Eq. (cpeval-comp), the pass-KV
  byte count, pass-Q decode, self-consistency checks.

Modules:

* ``attention``   -- the plain definition softmax(scale*QK^T + mask)V in fp64.
* ``blockwise``   -- the pages' blockwise ring algorithm, step by step, used
                     only to pin the definition against the method's invariants.
* ``merge``       -- N-way (O, LSE) merge of normalised partials.
* ``block_class`` -- SKIP / PARTIAL / FULL per tile from the explicit mask.
* ``backward``    -- the gradients dQ, dK, dV of the definition (chain rule),
                     whole-row and block by block in ring order.
* ``costs``       -- FLOP / byte formulas of the pages.

Every function here is pinned by ``tests/test_oracle_*.py`` against brute
force, closed forms and the pages' worked numbers.
"""
