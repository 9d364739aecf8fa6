"""The oracle's pins are strong enough: each plausible mistake planted in a copy of the
oracle (a dropped term, a wrong sign, index or operand) makes at least one pin fail.

Every mutation is applied to a temporary copy of oracle/msa_oracle.c, compiled on the
CPU and swapped in for the real library while the pin tests run; nothing here touches
the CUDA path.
"""
import ctypes
import inspect
import os
import shutil
import subprocess

import pytest

import oracle
from tests import test_oracle_codec, test_oracle_msa

SRC = os.path.join(os.path.dirname(oracle.__file__), "msa_oracle.c")
HDR = os.path.join(os.path.dirname(oracle.__file__), "msa_oracle.h")

MUTATIONS = {
    "indexer_drops_relu": ("s += wh * (dot > 0.0 ? dot : 0.0);", "s += wh * dot;"),
    "indexer_ignores_weights": ("double wh = w_idx ? (double)w_idx[((int64_t)b * Tq + t) * HI + h] : 1.0;",
                                "double wh = 1.0;"),
    "pool_divides_by_block_size": ("bs[j / ORC_BLOCK] = pool_mode == 1 ? acc : acc / (double)cnt;",
                                   "bs[j / ORC_BLOCK] = pool_mode == 1 ? acc : acc / 128.0;"),
    "select_tie_prefers_high_index": ("return ia < ib;", "return ia > ib;"),
    "select_forces_wrong_block": ("const int64_t r = pos / ORC_BLOCK;           /* forced",
                                  "const int64_t r = pos / ORC_BLOCK - (pos >= ORC_BLOCK); /* forced"),
    "attention_drops_scale": ("sc[i] = dot * scale;", "sc[i] = dot;"),
    "attention_wrong_gqa_head": ("const int hk = h / g;", "const int hk = h % Hkv;"),
    "attention_sees_future_key": ("if (j <= pos)\n                            keys[nk++] = j;",
                                  "if (j <= pos + 1)\n                            keys[nk++] = j;"),
    "decode_swaps_nibbles": ("uint8_t code = (d & 1) ? (byte >> 4) : (byte & 0xF);",
                             "uint8_t code = (d & 1) ? (byte & 0xF) : (byte >> 4);"),
    "decode_drops_tensor_scale": ("volatile float r = p * s_tensor;", "volatile float r = p;"),
    "e2m1_ties_away_from_zero": ("return nearbyint(a / q) * q;", "return round(a / q) * q;"),
    "encoder_ignores_tensor_scale": ("volatile float denom = (float)orc_e4m3_value(sc) * s_tensor;",
                                     "volatile float denom = (float)orc_e4m3_value(sc);"),
    "e4m3_wrong_bias": ("mag = ldexp(1.0 + m / 8.0, e - 7);", "mag = ldexp(1.0 + m / 8.0, e - 8);"),
}


def _pins():
    for mod in (test_oracle_codec, test_oracle_msa):
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if name.startswith("test_") and fn.__module__ == mod.__name__:
                yield f"{mod.__name__}.{name}", fn


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(mutation, tmp_path, monkeypatch):
    old, new = MUTATIONS[mutation]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not found once: {mutation}"
    (tmp_path / "msa_oracle.c").write_text(src.replace(old, new))
    shutil.copy(HDR, tmp_path / "msa_oracle.h")
    so = str(tmp_path / "liboracle_mutant.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
                           str(tmp_path / "msa_oracle.c"), "-o", so, "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(so)))
    caught = []
    for name, fn in _pins():
        try:
            fn()
        except AssertionError:
            caught.append(name)
    assert caught, f"no pin caught {mutation}"
