"""GPU NVFP4 codec (msa_nvfp4_encode / decode / amax) bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import msa, synth
from tests._common import golden_dict

pytestmark = pytest.mark.gpu


def _gpu_encode(x: np.ndarray, st: float):
    c = msa.encode_cache(torch.from_numpy(x).cuda(), st)
    torch.cuda.synchronize()
    return c.data.cpu().numpy(), c.scale.cpu().numpy()


def test_encode_random_bit_exact():
    x = synth.normal_tensor(5, synth.TID_K, 64, 4096).numpy().reshape(-1, 128) * np.float32(3.0)
    for st in (oracle.tensor_scale(x), np.float32(7.0 / 2688), np.float32(1e-3), np.float32(0.5)):
        d, s = _gpu_encode(x, float(st))
        ref = oracle.nvfp4_encode(x, float(st))
        assert np.array_equal(s.reshape(-1), ref.scale.reshape(-1)), "scales differ"
        assert np.array_equal(d.reshape(-1), ref.data.reshape(-1)), "codes differ"


def test_encode_ties_and_edges_bit_exact():
    """Values placed exactly on E2M1 midpoints of their group's denominator, zeros, negatives."""
    rng = np.random.default_rng(7)
    st = np.float32(0.01)
    groups = []
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.0, 0.5, 3.0, 4.0], dtype=np.float64)
    for i in range(4096):
        sc = oracle.e4m3_value(int(rng.integers(0x08, 0x7E)))
        denom = np.float32(np.float32(sc) * st)
        m = rng.choice(mids, 16) * rng.choice([-1.0, 1.0], 16)
        m[0] = 6.0  # pins amax so that the group scale is exactly sc
        groups.append((m * np.float64(denom)).astype(np.float32))
    x = np.stack(groups).reshape(-1, 64)
    x[::97] = 0.0
    d, s = _gpu_encode(x, float(st))
    ref = oracle.nvfp4_encode(x, float(st))
    assert np.array_equal(s.reshape(-1), ref.scale.reshape(-1))
    assert np.array_equal(d.reshape(-1), ref.data.reshape(-1))


def test_encode_handworked_group():
    g = golden_dict("nvfp4_group.txt")
    x = np.array([float(v) for v in g["x"]], dtype=np.float32).reshape(1, 16)
    d, s = _gpu_encode(x, float(g["tensor_scale"][0]))
    assert list(d.reshape(-1)) == [int(b, 16) for b in g["bytes"]]
    assert list(s.reshape(-1)) == [int(g["scale"][0], 16)]


def test_decode_bit_exact_all_codes():
    """Every (byte, scale byte) pair of the format decodes exactly like the oracle."""
    idx = np.arange(256 * 256)
    data = np.repeat((idx // 256).astype(np.uint8)[:, None], 8, axis=1)  # vector i: all bytes = i // 256
    scale = (idx % 256).astype(np.uint8)[:, None]                           # scale byte = i % 256
    scale[(scale == 0x7F) | (scale == 0xFF)] = 0x7E  # E4M3 NaN codes are never written by the encoder
    n = data.shape[0]
    for st in (np.float32(1.0), np.float32(7.0 / 2688)):
        ref = oracle.nvfp4_decode(oracle.Nvfp4(data, scale, float(st)))
        out = torch.empty(n, 16, dtype=torch.float32, device="cuda")
        msa.msa_nvfp4_decode(torch.from_numpy(data).cuda(), torch.from_numpy(scale).cuda(), float(st), out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_amax():
    x = synth.normal_tensor(9, synth.TID_V, 3, 100001).cuda()
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    msa.msa_nvfp4_amax(x, out)
    assert out.item() == x.abs().max().item()
    st = np.float32(out.item()) / np.float32(2688.0)
    assert st == oracle.tensor_scale(x.cpu().numpy())
