"""CPU fp64 oracle for the log-linear attention forward (test infrastructure only).

Only tests, the smoke check and the bench's CPU-baseline / reference arm use
this package; the product path (hierarchical_fenwick_state_b200) never imports it.
"""
from .llattn_oracle import (  # noqa: F401
    fenwick_level, fenwick_level_matrix,
    llattn_bruteforce_seq, llattn_quadratic_seq, llattn_recurrent_seq, mamba2_recurrent_seq,
    llattn_single, llattn_bruteforce, llattn_quadratic, llattn_recurrent, mamba2_recurrent,
    llattn_sampled, rel_max_err,
    llattn_level_states, llattn_decode_step, llattn_decode_sequence, llattn_decode_batch,
    llattn_backward_seq, llattn_backward, llattn_backward_sampled,
)
from .gdn_oracle import (  # noqa: F401
    gdn_bruteforce_seq, gdn_recurrent_seq, gated_deltanet_seq, gdn_single,
    gdn_recurrent, gdn_bruteforce, gated_deltanet, gdn_sampled,
)
