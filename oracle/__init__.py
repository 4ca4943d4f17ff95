"""fp64 CPU oracle for tree-packed chunkwise KDA -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct implementations of what the hot path
computes, written from the HARTS pages ("HARTS: A Prefix-Sharing Training
System for Agentic RL with Hybrid-Attention Models", abstract and
Figures 1, 2, C.1) and from the gated delta-rule recurrence the workload
fixes:  S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,
o_t = S_t^T q_t.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It
shares no code with the CUDA path (``tree_packed_chunkwise_b200``) and
never imports it; both read their inputs from ``synth``.

Modules
  planner    round planner (dynamic program + brute force), compact layout
  kda        token-by-token recurrence, forward and hand adjoint
  chunkwise  chunkwise form and fp64 tree executor (rounds, slots, replay)
  attention  tree-masked softmax attention (per trajectory, causal)
  logprob    per-position log-probabilities from one logit row per unique row
  layers     the 3 KDA + 1 latent-attention group (torch fp64 autograd)
"""
