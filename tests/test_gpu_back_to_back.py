"""Back-to-back steps on one workspace: two problems (identical inputs, separate status
words and outputs) run alternately, many times, with no host synchronisation between
steps, so every kernel of the launch chain (programmatic dependent launches included)
overlaps its neighbours as it does in a serving loop.  Every step must finish with a
clean status and produce, bit for bit, the output of a single isolated step (the
path is deterministic: list filling order does not reach the arithmetic).
"""
import dataclasses

import pytest
import torch

from block_sparse_attention_10_b200 import configs, msa
from block_sparse_attention_10_b200.profile_case import build

pytestmark = pytest.mark.gpu

STEPS = 60


def _checksum(x: torch.Tensor) -> torch.Tensor:
    """Order-independent checksum of the bit patterns (int64 sum of the 32-bit words)."""
    return x.contiguous().view(torch.int32).to(torch.int64).sum()


@pytest.mark.parametrize("name", ["prefill_b2_4k_on_128k", "decode_b32_64k", "long_decode_b8_192k_256k_ragged"])
def test_back_to_back_steps_bitwise(name):
    torch.cuda.set_device(0)
    w = configs.BY_NAME[name]
    pa = build(w, with_kv=True)
    pb = dataclasses.replace(pa, status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    ws = msa.alloc_workspace(pa)
    out_ref, lse_ref, _ = msa.outputs(pa)
    msa.msa_decode(pa, ws, out_ref, lse_ref, None)
    torch.cuda.synchronize()
    assert int(pa.status.item()) == 0
    ref = (_checksum(out_ref), _checksum(lse_ref))
    outs = [msa.outputs(pa)[:2] for _ in range(2)]
    sums = []
    for i in range(STEPS):
        o, l = outs[i % 2]
        msa.msa_decode(pa if i % 2 == 0 else pb, ws, o, l, None)
        sums.append((_checksum(o), _checksum(l)))
    torch.cuda.synchronize()
    assert int(pa.status.item()) == 0 and int(pb.status.item()) == 0
    bad = [i for i, (so, sl) in enumerate(sums) if int(so) != int(ref[0]) or int(sl) != int(ref[1])]
    assert not bad, f"steps with outputs different from an isolated step: {bad[:10]}"
    assert torch.equal(outs[(STEPS - 1) % 2][0], out_ref) and torch.equal(outs[(STEPS - 1) % 2][1], lse_ref)
