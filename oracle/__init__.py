"""fp64 CPU oracle for the CompKV decode step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. The CUDA path never imports, links or executes anything here, and nothing here
imports the CUDA path. See ``oracle/compkv.py`` for the sources and the readings taken.

Parity status: every function is pinned (tests/test_oracle_pins.py); none is "parity unpinned".
"""
from .compkv import *  # noqa: F401,F403
from .compkv import (MODES, Summaries, StepResult, block_summaries, block_mean_logits,  # noqa: F401
                     logit_variance_estimate, second_order_log_mass, head_scores, group_scores,
                     n_select, select_blocks, token_logits, compensated_attention,
                     dense_attention, compensated_distribution, kl_divergence, log_partitions,
                     block_residuals, brute_force_best_subset, decode_step, dense_step,
                     default_scale, n_blocks, block_bounds, logsumexp, empty_summaries,
                     append_token, average_ranks, rank_correlation, residual_capture,
                     group_residual_criterion, store)
