"""Test infrastructure: the CPU oracle for the deterministic attention backward.

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
arm of ``bench.py`` may import anything from this package.  The product path
(``persistent_sm_attn_b200``) never imports it and shares no code with it.

Sources.  The method is described in three explainer pages of the paper
"DASH: Deterministic Attention Scheduling for High-throughput Reproducible LLM
Training".  Citations below use:

* "DASH summary §n" -- the Spanish technical summary, "Resumen Técnico: DASH –
  Programación de Atención Determinista para el Entrenamiento de LLM de Alto
  Rendimiento", section n (§1 problem, §2.1 DAG formulation, §2.2.A descending
  Q-tile iteration, §2.2.B shift / symmetric shift and the lemma, §4 results).
* "DASH zh summary §n" -- the same technical summary in the Chinese page
  ("DASH: Deterministic Attention Scheduling for High-throughput Reproducible
  LLM Training", 技术摘要 section n).

The pages print no attention formulas; ``attention`` follows the textbook
softmax-attention definition that the method's backward differentiates.

Modules:
  attention  -- fp64 forward and backward from the definitions
  schedules  -- the visiting order and dQ accumulation order of each schedule
  dag        -- brute-force critical paths of the schedule DAG (tiny sizes)
"""
