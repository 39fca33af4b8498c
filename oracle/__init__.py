"""CPU fp64 oracle for the VanillaMarkov transition-bias head.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path
(the CUDA library and its Python binding) never imports it, and this package
imports nothing from the product.

Parity status of each function against something other than itself is
recorded in the module docstrings and in the tests under ``tests/`` whose
names start with ``test_oracle``.
"""
from .markov import (  # noqa: F401
    GREEDY_TEMPERATURE,
    apply_block_logits,
    apply_block_logits_backward,
    apply_step_logits,
    compute_step_bias,
    fused_lm_head_exact,
    fused_lm_head_logits,
    get_prev_embeddings,
    project_bias,
    sample_block_tokens,
    sample_tokens,
    select_greedy,
    temperature_scores,
    transition_logits,
)
from .philox import gumbel_noise, noise_words, philox4x32, uniform_from_word  # noqa: F401
from .rounding import round_to, round_to_bfloat16, round_to_float32, ulp_bfloat16  # noqa: F401
from .checks import (accumulation_bound, check_logits, check_sampled_block, check_tokens,  # noqa: F401
                     fused_accumulation_bound)
