"""CPU oracle for the On-Demand Attention (ODA) decode step.  TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 numpy restatement of what the decode hot path computes, used to check
the CUDA path.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it; the product path never does, and this package imports nothing
from the product package (the two share only the seeded input generators in
``workload/``).

Citations name the method-notes page titled
"On-Demand Attention：让语言模型按需读取完整历史" (notes checked against the full
28-page paper) as [notes §n ...], with the section and equation; and the summary page titled
"On-Demand Attention：模型知道自己什么时候需要回头看" as [summary ...].

Modules
  sets       index sets S^F and S^L                        [notes §2.1, eq. S^F / S^L]
  attention  softmax attention over an index set           [notes §2.1, eq. o_t]
  head       recall head R(h_{t-1}, E(x_t), h_t^L) -> q_t   [notes §2.2, eq. q_t]
  gate       full iff q_t > theta or q_t non-finite         [notes §2.3]
  delta      gated-delta recurrent layer (hybrid stand-in) [notes §2.3, hybrid state]
  step       one decode step: local pass, head, retry from the pre-step state,
             transactional commit, snapshot / restore       [notes §2.3, eq. h_t, C_t]
  labels     gain, penalised label, Huber loss, Delta F     [notes §2.1-§2.3]

Parity pins: every function is pinned in tests/test_oracle_*.py against page-given facts,
closed forms, invariants or library routines.  The recall head's layer details are a
reading of the page (which fixes topology and the exact parameter count only); against the
paper's trained head its values are "parity unpinned" (no weights exist).
"""
