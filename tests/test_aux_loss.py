"""The auxiliary routing loss on the GPU (msa_aux_routing_loss) against the oracle's
``aux_routing_loss`` on the same stored inputs.

Parity unpinned: the pages name a supervised contrastive loss between relevant and irrelevant
chunks but print no formula, so both sides implement the same reading (softmax over the chunk
scores at temperature tau, mean log-probability of the positives); the oracle's own arithmetic
is pinned by autograd and a closed form in test_oracle_pins.py. Both sides compute from the
same stored values (fp32, or bf16 decoded exactly), the kernels in fp32: loss within 1e-5
relative, gradients within 1e-4 of their tensor's largest entry.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


def _bits(pos):
    B, n = pos.shape
    words = (n + 31) // 32
    bits = np.zeros((B, words), np.uint32)
    for b in range(B):
        for c in np.nonzero(pos[b])[0]:
            bits[b, c // 32] |= np.uint32(1 << (c % 32))
    return bits


@pytest.mark.parametrize("dt,B,T,h_qr,h_kv,d,n,tau", [
    ("fp32", 3, 5, 4, 2, 64, 300, 0.1),     # two router heads per key head, one query without
                                            # positives
    ("bf16", 2, 16, 8, 8, 128, 512, 0.05),  # the configurations' head layout
    ("bf16", 4, 1, 8, 8, 128, 1000, 0.2),   # decode-shaped queries
])
def test_aux_loss_matches_oracle(msa, gpu, dt, B, T, h_qr, h_kv, d, n, tau):
    rng = np.random.default_rng(n + T)
    Q = synth.normal(n, 301, (B, T, h_qr, d), dt)
    K = synth.normal(n, 302, (n, h_kv, d), dt)
    K[7] = 0  # a zero chunk row: cosine 0, no gradient
    pos = np.zeros((B, n), bool)
    for b in range(B):
        if dt == "fp32" and b == 1:
            continue  # no positives: the query is left out of the mean
        pos[b, rng.choice(n, 8, replace=False)] = True
    loss, dQ, dK = oracle.aux_routing_loss(synth.as_f32(Q, dt), synth.as_f32(K, dt), pos, tau)
    bits = torch.from_numpy(_bits(pos).view(np.int32)).to(gpu)
    g_loss, g_dQ, g_dK = msa.aux_routing_loss(to_dev(Q, gpu), to_dev(K, gpu), bits, tau)
    torch.cuda.synchronize()
    assert abs(float(g_loss.item()) - loss) <= 1e-5 * abs(loss)
    for got, ref in ((g_dQ, dQ), (g_dK, dK)):
        got = got.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) <= 1e-4 * np.max(np.abs(ref))
    assert np.all(g_dK.cpu().numpy()[7] == 0)
