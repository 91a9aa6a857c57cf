"""The oracle: a plain, slow, fp64 CPU restatement of one FlashLoop loop step.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
product package (``cross_loop_sparse_step_b200``) never imports it, and it never
imports the product package: the two share no code. Inputs come from the seeded
generators in ``cross_loop_sparse_step_b200.synth``, which hold no arithmetic of
the method.

Source of every definition: the pages about *FlashLoop: Fast and Memory-Efficient
Looped Transformers via Lazy Updates* (arXiv 2609.29812), chiefly the paper text
(§1 Introduction, §3 Cross-Loop Redundancy, §4 FlashLoop, Appendix E "Quantization
Setting"). Where the pages are silent the module that needs a reading states it in
its docstring; all readings are collected in the repository's design notes.

Modules
  codec      exact fp32/fp16 group quantiser of the KV store (§4.3, App. E)
  kvstore    base + per-loop residual KV store and its reconstruction (§3.3, §4.3)
  block      RMSNorm, RoPE, projections, SwiGLU FFN of the shared block (§1)
  attention  dense causal attention + column statistics; loop-aware sparse
             attention with cached mass and unselected contribution (§4.2)
  select     normalized hidden-state change and top-k token selection (§4.1)
  loop       the R-loop driver that strings the above together (§4)

Parity status: every function here is pinned by a ``-m "not gpu"`` test against
closed forms, brute force, exact rational arithmetic or invariants; none is
pinned to a worked number from the pages because the pages print none
("parity with the paper unpinned" in that narrow sense; see the design notes).
"""
