"""CPU oracle of the DSpark draft/verify round (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never imports it.
"""
from .dspark_oracle import *  # noqa: F401,F403
from .dspark_oracle import (NEAR_TIE, THETA_NEAR_TIE, SCHED_ARGMAX, SCHED_EARLY_STOP, scaled_logits, softmax,
                            greedy_choice, inverse_cdf, markov_bias, draft_step, markov_draft, rnn_state, rnn_draft, verify_request,
                            verify, tv_labels, ragged_offsets, ragged_tags, pack_ragged, verify_ragged,
                            tv_labels_ragged, ECE_BINS, ece, sts_scale, sts_fit, prefix_survival, schedule_order, prefix_schedule,
                            schedule_at_capacity, prefix_schedule_t2,
                            exhaustive_schedule)
