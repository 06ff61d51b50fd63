"""The backward of the sparse attention (msa_sparse_attend_backward) and the scatter of the
gathered rows' gradients into the bank (msa_scatter_bank_grad) against the oracle's reverse
mode of the same attention (``oracle.attend_backward``, double precision).

Tolerance: 2e-2 relative per gradient tensor (max-abs error / max-abs oracle value), the
attention's bf16 tolerance: the kernel forms the probabilities and dS in bf16 before the
tensor-core products (rounding 2^-9 relative) and accumulates in fp32. Per row (error over the
row / the row's max-abs oracle value, floored at 1e-2 of the tensor's largest row) the bound is
1e-1: where dP - D nearly cancels in a row of dS (a query token that sees few keys), the row's
own scale is small against the terms it is made of, and the bf16 rounding of those terms shows
at the few-percent level of that small scale; a wrong row (a mask, an index, a rotation) is off
by O(1) and fails either check.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import to_dev

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2      # per tensor
ROW_TOL = 1e-1       # per row, floored at 1e-2 of the tensor's largest row


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


def _rel_tensor(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(got - ref).max() / max(float(np.abs(ref).max()), 1e-30))


def _rel_rows(got, ref):
    got = np.asarray(got, np.float64).reshape(-1, ref.shape[-1])
    ref = np.asarray(ref, np.float64).reshape(-1, ref.shape[-1])
    scale = np.abs(ref).max(axis=-1)
    floor = 1e-2 * max(float(scale.max()), 1e-30)
    return np.abs(got - ref).max(axis=-1) / np.maximum(scale, floor)


def _case(msa, gpu, B, T, h_q, h_kv, L, ctx, pos0, base, seed=0, nan_tail=True):
    dt, d = "bf16", 128
    rng = np.random.default_rng(seed)
    n_ctx = np.array(ctx, np.int32)
    n_bank = max(int(n_ctx.max()) * 2, 4)
    Q = synth.normal(seed, 201, (B, T, h_q, d), dt)
    Kl = synth.normal(seed, 202, (B, L, h_kv, d), dt)
    Vl = synth.normal(seed, 203, (B, L, h_kv, d), dt)
    Kb = synth.normal(seed, 204, (n_bank, h_kv, d), dt)
    Vb = synth.normal(seed, 205, (n_bank, h_kv, d), dt)
    dO = synth.normal(seed, 206, (B, T, h_q, d), dt)
    max_ctx = max(int(n_ctx.max()), 1)
    gi = np.full((B, max_ctx), -1, np.int32)
    for b in range(B):  # distinct rows per query; two queries may share a bank row
        gi[b, :n_ctx[b]] = rng.choice(n_bank, n_ctx[b], replace=False)
    ref = oracle.attend_backward(Q, Kl, Vl, Kb, Vb, gi, n_ctx, pos0, base, synth.bf16_to_f32(dO))
    cK = np.zeros((B, max_ctx, h_kv, d), np.uint16)
    cV = np.zeros((B, max_ctx, h_kv, d), np.uint16)
    for b in range(B):
        cK[b, :n_ctx[b]] = Kb[gi[b, :n_ctx[b]]]
        cV[b, :n_ctx[b]] = Vb[gi[b, :n_ctx[b]]]
        if nan_tail:  # rows past ctx_len hold whatever the buffer held: NaN here
            cK[b, n_ctx[b]:] = 0x7FC0
            cV[b, n_ctx[b]:] = 0x7FC0
    t = lambda x: to_dev(x, gpu)  # noqa: E731
    cl = torch.from_numpy(n_ctx).to(gpu)
    g = msa.sparse_attend_backward(t(Q), t(Kl), t(Vl), t(cK), t(cV), cl, pos0, base, t(dO))
    torch.cuda.synchronize()
    gi_t = torch.from_numpy(gi).to(gpu)
    dKb, dVb = msa.scatter_bank_grad(gi_t, cl, g["dK_ctx"], g["dV_ctx"], n_bank)
    torch.cuda.synchronize()
    got = {k: g[k].cpu().numpy() for k in ("dQ", "dK_loc", "dV_loc", "dK_ctx", "dV_ctx")}
    got["dKbar"], got["dVbar"] = dKb.cpu().numpy(), dVb.cpu().numpy()
    worst = {}
    for name, x in got.items():  # the bank rows: gathered gradients summed per bank row
        assert np.all(np.isfinite(x)), f"{name}: non-finite values"
        worst[name] = (_rel_tensor(x, ref[name]), float(_rel_rows(x, ref[name]).max()))
    print(worst)
    for name, (t, r) in worst.items():
        assert t < GRAD_TOL, f"{name}: rel err {t:.3e} ({worst})"
        assert r < ROW_TOL, f"{name}: row rel err {r:.3e} ({worst})"
    return worst


@pytest.mark.parametrize("B,T,h_q,h_kv,L,ctx,pos0,base", [
    (1, 256, 32, 8, 1300, [64], 8, 1e6),        # interleave-round shape (4 heads per KV head)
    (4, 1, 32, 8, 2048, [128, 77, 0, 128], 16, 1e6),  # decode shape of the 10M/100M banks
    (2, 40, 8, 2, 300, [200, 5], 3, 1e4),       # partial memory tile, partial query tile
    (2, 70, 4, 4, 70, [0, 130], 0, 0.0),        # one head per KV head, RoPE off, L = T
    (1, 16, 64, 8, 500, [100], 5, 1e6),         # 8 heads per KV head
])
def test_attend_backward_matches_oracle(msa, gpu, B, T, h_q, h_kv, L, ctx, pos0, base):
    _case(msa, gpu, B, T, h_q, h_kv, L, ctx, pos0, base, seed=T + L)


def test_attend_backward_rejects_unsupported(msa, gpu):
    Q = torch.zeros((1, 4, 6, 128), dtype=torch.bfloat16, device=gpu)  # 3 heads per KV head
    K = torch.zeros((1, 8, 2, 128), dtype=torch.bfloat16, device=gpu)
    c = torch.zeros((1, 1, 2, 128), dtype=torch.bfloat16, device=gpu)
    cl = torch.zeros(1, dtype=torch.int32, device=gpu)
    with pytest.raises(msa.MSAError) as e:
        msa.sparse_attend_backward(Q, K, K, c, c, cl, 0, 0.0, Q)
    assert e.value.status == 2
