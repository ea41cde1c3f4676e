"""Reference oracle for the speculative-decoding scoring / resampling path.

TEST INFRASTRUCTURE ONLY.  Plain, slow, obviously-correct NumPy code in fp64
that states what the GPU library computes.  It shares no code, header, table or
constant generator with the CUDA library in ``resample_online_log_b200`` and
neither imports the other.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product path never does.

Sources (summaries on gist.science; each function cites its passage):
  * "Faster LLM Inference via Sequential Monte Carlo" (SMC-SD) -- particles,
    importance weights, evict/duplicate resampling, bonus token, KV page
    metadata copy (section 2, Methodology).
  * METASD (multi-drafter speculative decoding) -- Block Divergence reward built
    on the total-variation distance between drafter and target distributions,
    drafter selection by an upper-confidence-bound bandit (section 2,
    Methodology); standard SD verification (section 1).
  * STAND (stochastic adaptive n-gram drafting) -- the logit n-gram store
    (top-10 (index, probability) rows, weighted-average merge, truncation) and
    Gumbel-Top-K sampling without replacement from its rows (Methodology,
    items 1 and 2); stochastic drafting from a distribution rather than its
    argmax (Methodology, item 1).

Every function's parity status is stated in its docstring.  Functions whose
randomness is defined by counter-based Philox draws are "pinned by
definition + statistics": the pages print no worked example with values.
"""

from .philox import (philox4x32_10, uniform_from_bits, gumbel_from_uniform,  # noqa: F401
                     stream_words, STREAM_BONUS, STREAM_ACCEPT, STREAM_RESIDUAL,
                     STREAM_RESAMPLE, STREAM_TOPK_DENSE, STREAM_TOPK_SPARSE, STREAM_DRAFT)
from .score import (row_log_softmax, total_variation, smcsd_score,  # noqa: F401
                    DEV_TOKEN_OOB, DEV_NONFINITE, DEV_ZERO_RESIDUAL, DEV_PAGE_OOB,
                    DEV_ANCESTOR_OOB)
from .resample import smcsd_resample, smcsd_resample_adaptive, systematic_ancestors  # noqa: F401
from .pagetable import kv_pagetable_remap  # noqa: F401
from .verify import sd_verify_reject, accept_probability, residual_distribution  # noqa: F401
from .topk import gumbel_topk, gumbel_topk_sparse  # noqa: F401
from .draft import sd_draft_sample  # noqa: F401
from .bandit import metasd_ucb_step, block_reward, ucb_choice, DEV_ARM_OOB, REWARD_BD, REWARD_BE  # noqa: F401,E501
from .ngram import NgramStore, observe_topk, merge as ngram_merge  # noqa: F401
