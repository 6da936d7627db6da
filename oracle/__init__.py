"""CPU oracle for certified quantized decode attention.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the decode path computes, used to prove the CUDA path
right.  Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it; the library itself never does, and it
shares no code, table or constant with the CUDA sources.
"""

from .cqa_oracle import (  # noqa: F401
    BLOCK,
    VGROUP,
    fp16_round_up,
    quantize_keys_block,
    quantize_values_block,
    pack_int4,
    unpack_int4,
    build_unit,
    dense_attention,
    e_key_bound,
    coverage_kstar,
    rank_consistent,
    rank_discordance,
    decode,
    Thresholds,
)
