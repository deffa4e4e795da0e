"""Reference oracle for the GPTQ-family per-layer solve: TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 CPU code that states what the solve computes, step by step, in
the notation of the source pages. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the library path never does, and the
two share no code.

Pins (tests/test_oracle_pins.py) tie every function here to something other than
itself: the worked examples printed on the pages, closed forms, special cases,
brute force and independent least-squares solves. Two readings are only partly
pinned and say so where they are defined: which weight value multiplies the
GPTAQ residual row (``gptaq`` arguments below), and likewise which weight values
enter the compensation-aware row (``cae`` arguments). The first-order term
(``first_order_*``) has no formula on the pages at all: its parity is unpinned
against them and rests on internal pins only.
"""

from .gptq_oracle import (  # noqa: F401
    gram,
    cross_gram,
    dead_and_damp,
    damped_diagonal,
    is_positive_definite,
    symmetric_scale,
    quantize_codes,
    dequantize,
    obq_sweep,
    upper_factor,
    gptaq_p1,
    cae_p2,
    row_form_sweep,
    replay_row_form,
    layer_error,
    solve_layer,
    brute_force_best,
    act_order,
    static_group_scales,
    obq_sweep_grouped,
    replay_row_form_grouped,
    pack_codes,
    unpack_codes,
    first_order_obq_sweep,
    first_order_shift,
    trust_region_beta,
)
