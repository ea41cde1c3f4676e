"""Seeded synthetic inputs shared by the tests, the bench and the oracle's callers.

This module holds the input recipes only, none of the scoring / resampling
arithmetic.  It is implemented twice from one counter-based definition:
``synth.gen`` in NumPy (host) and ``synth/csrc/synth.cu`` (device, built into
``synth/libsynth.so``) for inputs too large to build on the host.  Both use only
integer operations and individually rounded fp32 additions, multiplications
and divisions, so they agree bit for bit (tests/test_synth.py checks the NumPy
side against itself and, on a GPU, against the device side).
"""

from .gen import (CONFIGS, SynthConfig, bf16_bits_to_f32, f32_to_bf16_bits,  # noqa: F401
                  gen_rows, draft_tokens_for_rows, page_table, sparse_rows, normal_table,
                  head_boosts, row_ids_for, gen_config_rows)
