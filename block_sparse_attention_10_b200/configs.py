"""The five synthetic MSA workloads (shapes, needles, seeds).

Shapes use B (batch), Tq (query tokens per sequence), Hq/Hkv (attention
heads), D (head dim), HI/DI (indexer heads/dim); the context length L of a
sequence includes its own Tq query tokens.  Block size 128 and top-16 come from
"vLLM Adds Day-0 Support for MiniMax-M3.1-Flash" (ainewsbites.com), section
"A model built for efficient inference"; 1 committed + 7 draft query tokens
from its section "Getting started and RL support".
"""
from .synth import Workload

TINY = Workload("tiny_decode_b1_4k", B=1, Tq=1, Hq=8, Hkv=1, D=128, HI=4, DI=64,
                seq_len=4096, needles=3, seed=1235)
DECODE_B32_64K = Workload("decode_b32_64k", B=32, Tq=1, Hq=32, Hkv=4, D=128, HI=8, DI=128,
                          seq_len=65536, needles=8, seed=1236)
LONG_RAGGED_256K = Workload("long_decode_b8_192k_256k_ragged", B=8, Tq=1, Hq=8, Hkv=1, D=128, HI=4, DI=64,
                            seq_len_range=(196608, 262144), needles=16, seed=1237)
SPEC_VERIFY_512K = Workload("spec_verify_b4_512k_tq8", B=4, Tq=8, Hq=8, Hkv=1, D=128, HI=4, DI=64,
                            seq_len=524288, needles=16, seed=1238)
PREFILL_4K_ON_128K = Workload("prefill_b2_4k_on_128k", B=2, Tq=4096, Hq=32, Hkv=4, D=128, HI=8, DI=128,
                              seq_len=131072 + 4096, needles=0, seed=1239)

ALL = [TINY, DECODE_B32_64K, LONG_RAGGED_256K, SPEC_VERIFY_512K, PREFILL_4K_ON_128K]
BY_NAME = {w.name: w for w in ALL}
