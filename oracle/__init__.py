"""CPU oracle for the tiered-KV decode path (TEST INFRASTRUCTURE ONLY).

Plain, slow, float64 NumPy restatement of what the pages define. Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import it; the product path (the CUDA library and its
Python binding) never does, and this package imports nothing from it.

Functions and where they come from (page title, section):

* ``attend`` -- softmax attention of one query head over a set of keys;
  "Resumo Técnico: QEvict", Mecanismos Principais / Implementação (GQA decode).
* ``int2_quantize`` / ``int2_dequantize`` -- the recoverable INT2 tier;
  "Resumo Técnico: QEvict", Metodologia (Nível Quantizado Recuperável) and the
  write-once ledger (Hierarquia Recuperável).
* ``vwo_l1norm`` -- ||V_i W_O^h||_1; "Resumo Técnico: CriticalKV",
  Framework Teórico (projected values V W_O) and Algoritmo, Etapa 2.
* ``two_stage`` -- budget b split into alpha*b on attention mass and the rest on
  the perturbation score; "Resumo Técnico: CriticalKV", Algoritmo, Etapas 1-2.
* ``QEvictUnit`` -- one (batch, kv-head) unit of the window-routed three-tier
  cache; "Resumo Técnico: QEvict", Metodologia and Mecanismos Principais.
* ``route_global`` -- one routing event under budgets shared by every layer and kv
  head of a sequence; "Make Each Token Count", Metodologia 3 (Orçamento Global)
  applied to the window tiers of "Resumo Técnico: QEvict", Metodologia.
* ``observation_mass`` / ``criticalkv_select`` -- CriticalKV selection with a
  SnapKV-style observation window; "Resumo Técnico: CriticalKV", Algoritmo.
* ``trim_global_topm`` -- DBTrimKV global budget over r = beta^(t-i);
  "Make Each Token Count", Metodologia 2 (Retenção Geométrica) and 3
  (Orçamento Global), 4 (Implementação, paged variable-length heads).
* ``output_perturbation`` -- L = ||o - o_hat||_1; "Resumo Técnico: CriticalKV",
  Framework Teórico (Definição de Perturbação). Diagnostic only.
* ``sekv_segment`` / ``sekv_summaries`` / ``sekv_gates`` / ``sekv_attend`` -- SEKV's
  entropy-guided spans, surprisal-weighted span summaries and mixed-resolution attention
  with the size correction; "Resumo Técnico: SEKV", Metodologia 1-3.
* ``tier_diagnostics`` / ``future_missed_mass`` -- selection churn, global
  latent importance reactivation and future missed mass; "Resumo Técnico:
  QEvict", Principais Contribuições 1.

Parity status of each function is listed in ``oracle/qevict_oracle.py``.
"""
from .qevict_oracle import *  # noqa: F401,F403
