"""CPU float64 oracle for the gated local/full decode-attention path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path
(``gated_local_full_b200``) never imports, links or executes it, and shares no
code with it.

Sources (the web pages this oracle restates):
  [SUM]  "On-Demand Attention (ODA)" summary, picx.dev
  [CARD] "On-Demand Attention: Language Models Know When to Recall", dair.ai paper card
  [EXPL] "Let models trigger full attention only when recall helps -- On-Demand
         Attention recall-head gating", learnaivisually explainer
  [DA-1] zhichai.net post on Declarative Attention (the "<focus>" mode)
  [DA-2] "Declarative Attention: Letting LLMs Control Their Own Attention",
         kongchang.com article ("<focus> Mode: Precise Region Targeting")

Parity status per function is listed in ``oracle/oda_oracle.py``'s header.
"""

from .oda_oracle import *  # noqa: F401,F403
