"""CPU oracle for the Kimi Delta Attention (KDA) hot path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. It is plain, slow and
written to be checked by eye against the definition; it shares no code with
the CUDA library (``hybrid_linear_attention_04_b200``) and neither imports the
other. The product path never falls back to it.

Contents
  native.py     : ctypes loader for kda_oracle.c, the fp64 token recurrence in C
                  (the oracle the GPU is compared with at size).
  recurrence.py : the same token recurrence in numpy fp64 (small cases), the
                  snapshot rule, and the chunked (WY/UT) form derived from it.
  exact.py      : the definition as an explicit product of rational matrices,
                  in exact arithmetic (fractions.Fraction), for T <= 8.
  frontend.py   : the q/k front-end (short causal depthwise convolution with a
                  carried conv state, Swish, L2 normalisation), for the next row
                  of the path; pinned in tests/test_frontend_oracle.py.
  segments.py   : affine state maps of token segments and their composition (the
                  algebra of splitting one sequence across workers); pinned in
                  tests/test_segment_maps.py.

Source of the definition: Kimi K3 technical FAQ (runpod.io), "What is KDA, and
why does a serving engineer care?" (delta-rule recurrence, per-channel forget
gate, d_k x d_v state, chunked parallel-within / recurrent-across form), and the
vLLM day-0 blog, "Kimi Delta Attention" (state snapshots at block boundaries).
The equation is the standard gated-delta form
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t / sqrt(d_k).

Pins (tests/test_oracle_pins.py): every function here is checked against the
exact rational product form, closed forms (beta = 0; orthogonal keys), the
overwrite property (beta = 1, unit keys), linearity, boundedness and the
chunked = token identity. No function is left unpinned.
"""
from .recurrence import (kda_recurrence, kda_chunked, snapshot_positions, snapshot_count,
                         normwise_rel_err)
from .native import oracle_sequence, oracle_packed, load as load_native, build as build_native

__all__ = ["kda_recurrence", "kda_chunked", "snapshot_positions", "snapshot_count",
           "normwise_rel_err", "oracle_sequence", "oracle_packed", "load_native",
           "build_native"]
