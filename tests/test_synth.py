"""The seeded input generator: published SplitMix64 words, exactness of the normals,
bf16 rounding against torch's conversion, and the workload recipes."""
import os

import numpy as np
import pytest

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden_ints(name):
    with open(os.path.join(GOLD, name)) as f:
        return [int(x) for x in f if x.strip() and not x.startswith("#")]


def test_splitmix64_reference_words():
    want = _golden_ints("splitmix64_seed1234567.txt")
    L = synth.lib()
    assert [L.syn_word(1234567, i) for i in range(5)] == want


def test_normal_exact_and_moments():
    x = synth.normal(7, synth.tag(synth.K), (1 << 20,))
    # every value is an integer multiple of 2^-17 and lies in [-6, 6]
    assert np.all(np.abs(x) <= 6.0)
    assert np.array_equal(x * 131072.0, np.round(x * 131072.0))
    assert abs(float(x.mean())) < 5e-3
    assert abs(float(x.var()) - 1.0) < 5e-3
    # deterministic, and distinct tags give distinct streams
    assert np.array_equal(x, synth.normal(7, synth.tag(synth.K), (1 << 20,)))
    y = synth.normal(7, synth.tag(synth.V), (1 << 20,))
    assert abs(float(np.corrcoef(x, y)[0, 1])) < 5e-3


def test_normal_offset_is_a_window():
    a = synth.normal(3, 99, (1000,))
    b = synth.normal(3, 99, (400,), first=600)
    assert np.array_equal(a[600:], b)


def test_bf16_matches_torch_rne():
    import torch
    x = synth.normal(1, 5, (50000,)) * np.float32(3.7)
    x = np.concatenate([x, np.array([0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8,
                                     -1.0 - 2.0 ** -8], np.float32)])
    mine = synth.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    # the bf16 draw equals the rounded fp32 draw
    assert np.array_equal(synth.normal(1, 5, (1000,), "bf16"),
                          synth.f32_to_bf16(synth.normal(1, 5, (1000,))))


def test_uniform_and_distinct():
    u = synth.uniform(0, 1, 100000, 10)
    assert u.min() == 0 and u.max() == 9
    assert np.all(np.abs(np.bincount(u) / 1e5 - 0.1) < 0.01)
    d = synth.distinct(0, 2, 50, 60)
    assert len(set(d.tolist())) == 50 and d.min() >= 0 and d.max() < 60


def test_planted_rows_point_at_query():
    w = synth.C3.scaled(n_docs=64, B=2)
    inp = synth.make_bank_workload(w)
    qr = synth.as_f32(inp["Q_r"], w.dtype).astype(np.float64)
    kr = synth.as_f32(inp["Kbar_r"], w.dtype).astype(np.float64)
    coff = inp["doc_chunk_off"]
    for b in range(w.B):
        p = int(inp["planted"][b, 0])
        rows = kr[coff[p]:coff[p + 1]]
        q = qr[b, 0]
        cos = (rows * q[None]).sum(-1) / (np.linalg.norm(rows, axis=-1) *
                                           np.linalg.norm(q, axis=-1)[None])
        assert cos.mean() > 0.7  # 0.6 / sqrt(0.36 + 0.16) ~ 0.83


def test_workload_shapes():
    w = synth.C1
    inp = synth.make_token_workload(w)
    assert inp["K"].shape == (64 * 512, 2, 64) and inp["K"].dtype == np.float32
    assert inp["Q"].shape == (1, 16, 4, 64)
    assert inp["Q_r"].shape == (1, 16, 2, 64)
    assert inp["K_loc"].shape == (1, 16, 2, 64)
    assert len(inp["planted"]) == 4
    off = synth.doc_tok_offsets(w.scaled(ragged=True, n_docs=50))
    assert off[0] == 0 and np.all(np.diff(off) >= 1)
