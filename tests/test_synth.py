"""The seeded input generators: published SplitMix64 vectors, host/torch
agreement, slices equal to the full stream, value ranges."""
import numpy as np
import torch

from block_quantized_expert_mxfp4_b200 import synth
from conftest import golden


def test_splitmix64_published_vectors():
    want = [int(l, 16) for l in open(golden("splitmix64_vectors.txt")) if l[0] != "#" and l.strip()]
    state = 0
    for v in want:
        assert synth.splitmix64_int(state) == v
        state = (state + 0x9E3779B97F4A7C15) % 2 ** 64
    xs = np.array([0, 0x9E3779B97F4A7C15, 2 * 0x9E3779B97F4A7C15 % 2 ** 64], np.uint64)
    assert [int(v) for v in synth.splitmix64_np(xs)] == want
    got = synth.splitmix64_torch(torch.tensor([synth._to_i64(int(x)) for x in xs]))
    assert [int(v) % 2 ** 64 for v in got] == want


def test_numpy_and_torch_streams_agree():
    key = synth.tensor_key(3, 17)
    idx = np.arange(1000, 5000, dtype=np.uint64) + np.uint64(key)
    a = synth.splitmix64_np(idx).view(np.int64)
    b = synth.splitmix64_torch(torch.arange(1000, 5000, dtype=torch.int64) + synth._to_i64(key))
    assert np.array_equal(a, b.numpy())


def test_expert_slices_equal_full_tensor():
    q, s = synth.mx_expert_bytes(0, 0, synth.TID.GATE, 16, 256, 118, 127, None, 8)
    q2, s2 = synth.mx_expert_bytes(0, 0, synth.TID.GATE, 16, 256, 118, 127, [5, 2], 8)
    assert torch.equal(q2[0], q[5]) and torch.equal(q2[1], q[2])
    assert torch.equal(s2[0], s[5]) and torch.equal(s2[1], s[2])
    assert int(s.min()) == 118 and int(s.max()) == 127
    assert q.dtype == torch.uint8 and q.shape == (8, 16, 128)


def test_fp8_codes_skip_nan():
    c = synth.fp8_codes(0, 1, 200000)
    assert not torch.any((c == 0x7F) | (c == 0xFF))
    assert len(torch.unique(c)) == 254


def test_zipf_logits_are_skewed_and_select_k():
    z = synth.zipf_logits(0, 2048, 256, 6)
    fin = torch.isfinite(z)
    assert torch.all(fin.sum(1) == 6)
    counts = fin.sum(0).sort(descending=True).values
    assert counts[0] > 10 * counts[128] and int(counts[-1]) >= 1


def test_determinism():
    assert torch.equal(synth.activations(1, 2, 64), synth.activations(1, 2, 64))
    assert not torch.equal(synth.activations(1, 2, 64), synth.activations(2, 2, 64))
    assert torch.equal(synth.random_bytes(1, 2, 64), synth.random_bytes(1, 2, 64))
