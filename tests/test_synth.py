"""The seeded input generator: its words are SplitMix64 outputs (checked against a numpy uint64
restatement), its fp16 normals have the normal law's moments, and any subset of rows can be
regenerated without the rest."""
import math

import numpy as np
import torch

from kv_cache_vector_norm_b200 import synth


def _np_words(seed, stream, idx):
    g = np.uint64(0x9E3779B97F4A7C15)
    state = np.uint64(synth.stream_state(seed, stream))
    z = state + (idx.astype(np.uint64) + np.uint64(1)) * g
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def test_words_are_splitmix64():
    idx = np.arange(0, 5000, 7, dtype=np.int64)
    w = synth.random_words(3, 2, torch.from_numpy(idx)).numpy().view(np.uint64)
    assert np.array_equal(w, _np_words(3, 2, idx))


def test_normal_fp16_moments_and_subsets():
    x = synth.normal_fp16(0, synth.STREAM_K, (1 << 20,)).double()
    se = 1 / math.sqrt(x.numel())
    assert abs(x.mean().item()) < 5 * se
    assert abs(x.var().item() - 1) < 5 * math.sqrt(2) * se
    shape = (2, 3, 40, 64)
    sc = synth.channel_scales(1, 3, 64)
    full = synth.kv_tensor(1, synth.STREAM_V, *shape, scales=sc)
    rows = torch.tensor([0, 5, 39, 40, 200, 239])
    assert torch.equal(synth.kv_rows(1, synth.STREAM_V, shape, rows, scales=sc), full.reshape(-1, 64)[rows])


def test_channel_scales_and_block_table():
    sc = synth.channel_scales(0, 8, 128)
    assert sc.shape == (8, 128) and torch.all(sc > 0)
    # exactly one outlier channel (round(0.01 * 128) = 1) per head sits far above the lognormal bulk
    assert torch.all((sc > 20 * torch.exp(torch.tensor(-3.0))).sum(1) >= 1)
    bt = synth.block_table(0, 4, 8, 40)
    assert bt.shape == (4, 8) and len(set(bt.flatten().tolist())) == 32 and int(bt.max()) < 40


def test_score_fidelity_metrics_on_known_cases():
    from kv_cache_vector_norm_b200 import fidelity
    e = torch.tensor([[[1.0, 5.0, 2.0, 0.5, 0.1, 3.0]]])
    m = fidelity.score_fidelity(e.clone(), e)
    assert abs(m["cosine"] - 1.0) < 1e-12 and m["top1"] == 1.0 and m["top5"] == 1.0
    a = torch.tensor([[[1.0, 2.9, 2.0, 0.5, 0.1, 3.0]]])          # argmax moves to the last token
    m = fidelity.score_fidelity(a, e)
    ev, av = e.double().numpy().ravel(), a.double().numpy().ravel()
    assert abs(m["cosine"] - ev @ av / (np.linalg.norm(ev) * np.linalg.norm(av))) < 1e-12
    assert m["top1"] == 0.0 and m["top5"] == 1.0
    assert fidelity.score_fidelity(a, e, k=1)["top1"] == 0.0
    assert fidelity.score_fidelity(a, e, seq_lens=[0])["pairs"] == 0
