"""GPU parity of sparse generation: a growing local K/V cache (msa_kv_append) and the decode
step (msa_decode_step: append the step's tokens, attend over [gathered memory ; cache])
against the oracle's token-by-token loop, on the same seeded inputs; a captured step replayed
as a CUDA graph; the overflow of a full cache.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import check_attention, stored_f64, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


def _case(seed, B, T, h_q, h_kv, d, L0, S, n_ctx, dt="bf16"):
    """Seeded inputs: memory bank rows + gather indices, prompt K/V, per-step Q/K/V."""
    rng = np.random.default_rng(seed)
    n_bank = max(int(max(n_ctx)) * 2, 1)
    max_ctx = max(int(max(n_ctx)), 1)
    Kb = synth.normal(seed, 104, (n_bank, h_kv, d), dt)
    Vb = synth.normal(seed, 105, (n_bank, h_kv, d), dt)
    gi = np.full((B, max_ctx), -1, np.int32)
    for b in range(B):
        gi[b, :n_ctx[b]] = rng.choice(n_bank, n_ctx[b], replace=False)
    Kp = synth.normal(seed, 102, (B, L0, h_kv, d), dt)
    Vp = synth.normal(seed, 103, (B, L0, h_kv, d), dt)
    Qs = [synth.normal(seed, 200 + 3 * s, (B, T, h_q, d), dt) for s in range(S)]
    Ks = [synth.normal(seed, 201 + 3 * s, (B, T, h_kv, d), dt) for s in range(S)]
    Vs = [synth.normal(seed, 202 + 3 * s, (B, T, h_kv, d), dt) for s in range(S)]
    ctxK = np.zeros((B, max_ctx, h_kv, d), Kb.dtype)
    ctxV = np.zeros((B, max_ctx, h_kv, d), Vb.dtype)
    for b in range(B):
        ctxK[b, :n_ctx[b]] = Kb[gi[b, :n_ctx[b]]]
        ctxV[b, :n_ctx[b]] = Vb[gi[b, :n_ctx[b]]]
    return dict(Kb=Kb, Vb=Vb, gi=gi, n_ctx=np.asarray(n_ctx, np.int32), Kp=Kp, Vp=Vp, Qs=Qs,
                Ks=Ks, Vs=Vs, ctxK=ctxK, ctxV=ctxV)


@pytest.mark.parametrize("B,T,h_q,h_kv,L0,S,n_ctx,pos0,base,cap", [
    (3, 1, 32, 8, 70, 20, [0, 40, 17], 16, 1e6, 128),   # ragged prompt, one query without memory
    (2, 2, 16, 4, 5, 6, [64, 9], 4, 1e4, 40),           # two tokens per step: 8 rows per KV head
    (1, 1, 8, 1, 0, 9, [30], 3, 0.0, 16),               # empty prompt, one KV head, RoPE off
    (4, 1, 32, 8, 2040, 16, [128, 128, 77, 128], 16, 1e6, 2304),  # 100M-bank decode shape
])
def test_decode_step_matches_oracle(msa, gpu, B, T, h_q, h_kv, L0, S, n_ctx, pos0, base, cap):
    d = 128
    c = _case(7, B, T, h_q, h_kv, d, L0, S, n_ctx)
    ref = oracle.generate(c["Qs"], c["Ks"], c["Vs"], c["Kp"], c["Vp"], c["Kb"], c["Vb"], c["gi"],
                          c["n_ctx"], pos0, base)
    cache = msa.LocalCache(B, cap, h_kv, d, pos0=pos0, rope_base=base, device=gpu)
    if L0:
        cache.append(to_dev(c["Kp"], gpu), to_dev(c["Vp"], gpu))
    ctxK, ctxV = to_dev(c["ctxK"], gpu), to_dev(c["ctxV"], gpu)
    cl = torch.from_numpy(c["n_ctx"]).to(gpu)
    worst = 0.0
    for s in range(S):
        O = msa.decode_step(cache, to_dev(c["Qs"][s], gpu), to_dev(c["Ks"][s], gpu),
                            to_dev(c["Vs"][s], gpu), ctxK, ctxV, cl)
        torch.cuda.synchronize()
        worst = max(worst, check_attention(O, ref[s], "bf16"))
    n = L0 + S * T
    assert int(cache.length.item()) == n
    # the cache holds [prompt ; every step's tokens]: V bit for bit, K rotated at pos0 + row
    # (the oracle's RoPE, within one bf16 rounding)
    K_all = np.concatenate([c["Kp"]] + c["Ks"], axis=1)
    V_all = np.concatenate([c["Vp"]] + c["Vs"], axis=1)
    got_v = cache.V[:, :n].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got_v, V_all)
    got_k = to_np(cache.K[:, :n])
    K64 = stored_f64(K_all, "bf16")
    for b in range(B):
        for j in range(0, n, max(1, n // 37)):
            for hh in range(h_kv):
                ref_k = oracle.rope(K64[b, j, hh], pos0 + j, base) if base > 0 else K64[b, j, hh]
                assert np.all(np.abs(got_k[b, j, hh] - ref_k) <= 2.0 ** -8 * np.abs(ref_k) + 1e-6)


def test_decode_step_without_routed_memory(msa, gpu):
    """max_ctx = 0 (nothing gathered): the cache alone is the context."""
    B, T, h_q, h_kv, d, L0, S, pos0, base = 2, 1, 32, 8, 128, 33, 5, 16, 1e6
    c = _case(13, B, T, h_q, h_kv, d, L0, S, [1, 1])
    gi = np.zeros((B, 0), np.int32)
    cl = np.zeros(B, np.int32)
    ref = oracle.generate(c["Qs"], c["Ks"], c["Vs"], c["Kp"], c["Vp"], c["Kb"], c["Vb"], gi, cl,
                          pos0, base)
    cache = msa.LocalCache(B, L0 + S, h_kv, d, pos0=pos0, rope_base=base, device=gpu)
    cache.append(to_dev(c["Kp"], gpu), to_dev(c["Vp"], gpu))
    empty = torch.empty((B, 0, h_kv, d), dtype=torch.bfloat16, device=gpu)
    cl_dev = torch.from_numpy(cl).to(gpu)
    for s in range(S):
        O = msa.decode_step(cache, to_dev(c["Qs"][s], gpu), to_dev(c["Ks"][s], gpu),
                            to_dev(c["Vs"][s], gpu), empty, empty, cl_dev)
        torch.cuda.synchronize()
        check_attention(O, ref[s], "bf16")
    assert int(cache.length.item()) == L0 + S


def test_kv_append_fills_in_pieces_and_advances_the_length(msa, gpu):
    B, h_kv, d, cap = 3, 8, 128, 100
    K = synth.normal(3, 110, (B, 87, h_kv, d), "bf16")
    V = synth.normal(3, 111, (B, 87, h_kv, d), "bf16")
    cache = msa.LocalCache(B, cap, h_kv, d, device=gpu)  # no RoPE: stored as given
    cache.append(to_dev(K[:, :37], gpu), to_dev(V[:, :37], gpu))
    cache.append(to_dev(K[:, 37:], gpu), to_dev(V[:, 37:], gpu))
    torch.cuda.synchronize()
    assert int(cache.length.item()) == 87
    assert msa.msa_workspace_status(cache.ws) == 0
    for got, want in ((cache.K, K), (cache.V, V)):
        g = got[:, :87].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(g, want)


def test_full_cache_is_flagged_and_left_unchanged(msa, gpu):
    B, T, h_q, h_kv, d, L0 = 2, 1, 32, 8, 128, 30
    c = _case(5, B, T, h_q, h_kv, d, L0, 2, [10, 20])
    cache = msa.LocalCache(B, L0 + 1, h_kv, d, pos0=16, rope_base=1e6, device=gpu)
    cache.append(to_dev(c["Kp"], gpu), to_dev(c["Vp"], gpu))
    ctxK, ctxV = to_dev(c["ctxK"], gpu), to_dev(c["ctxV"], gpu)
    cl = torch.from_numpy(c["n_ctx"]).to(gpu)
    ws = torch.empty(msa.msa_decode_step_workspace(B, T, h_q, h_kv, d, ctxK.shape[1], L0 + 1),
                     dtype=torch.uint8, device=gpu)
    O = torch.empty((B, T, h_q, d), dtype=torch.bfloat16, device=gpu)
    msa.decode_step(cache, to_dev(c["Qs"][0], gpu), to_dev(c["Ks"][0], gpu),
                    to_dev(c["Vs"][0], gpu), ctxK, ctxV, cl, O=O, ws=ws)
    assert msa.msa_workspace_status(ws) == 0
    before = cache.K.clone()
    O.fill_(7.0)
    msa.decode_step(cache, to_dev(c["Qs"][1], gpu), to_dev(c["Ks"][1], gpu),
                    to_dev(c["Vs"][1], gpu), ctxK, ctxV, cl, O=O, ws=ws)
    assert msa.msa_workspace_status(ws) == 2      # the context overflow code
    assert int(cache.length.item()) == L0 + 1
    assert torch.equal(cache.K.view(torch.int16), before.view(torch.int16))
    assert bool((O == 7.0).all())                 # no output written


def test_captured_step_replays_as_the_cache_grows(msa, gpu):
    """Two routed layers' decode steps captured once in a CUDA graph and replayed S times
    (new inputs copied into the captured buffers between replays) give the outputs of the
    same steps launched one by one, bit for bit, and advance both caches."""
    B, T, h_q, h_kv, d, L0, S, pos0, base = 4, 1, 32, 8, 128, 300, 12, 16, 1e6
    cases = [_case(11 + l, B, T, h_q, h_kv, d, L0, S, [128, 100, 0, 64]) for l in range(2)]
    cap = L0 + S
    st = torch.cuda.Stream()

    def setup():
        out = []
        for c in cases:
            cache = msa.LocalCache(B, cap, h_kv, d, pos0=pos0, rope_base=base, device=gpu)
            with torch.cuda.stream(st):
                cache.append(to_dev(c["Kp"], gpu), to_dev(c["Vp"], gpu), stream=st)
            out.append(dict(cache=cache, ctxK=to_dev(c["ctxK"], gpu), ctxV=to_dev(c["ctxV"], gpu),
                            cl=torch.from_numpy(c["n_ctx"]).to(gpu),
                            ws=torch.empty(msa.msa_decode_step_workspace(
                                B, T, h_q, h_kv, d, c["ctxK"].shape[1], cap),
                                dtype=torch.uint8, device=gpu),
                            Q=torch.empty((B, T, h_q, d), dtype=torch.bfloat16, device=gpu),
                            K=torch.empty((B, T, h_kv, d), dtype=torch.bfloat16, device=gpu),
                            V=torch.empty((B, T, h_kv, d), dtype=torch.bfloat16, device=gpu),
                            O=torch.empty((B, T, h_q, d), dtype=torch.bfloat16, device=gpu)))
        st.synchronize()
        return out

    def load(layers, s):
        for c, x in zip(cases, layers):
            x["Q"].copy_(to_dev(c["Qs"][s], gpu))
            x["K"].copy_(to_dev(c["Ks"][s], gpu))
            x["V"].copy_(to_dev(c["Vs"][s], gpu))
        torch.cuda.synchronize()

    def step(layers):
        for x in layers:
            msa.decode_step(x["cache"], x["Q"], x["K"], x["V"], x["ctxK"], x["ctxV"], x["cl"],
                            O=x["O"], ws=x["ws"], stream=st)

    eager = setup()
    want = []
    for s in range(S):
        load(eager, s)
        with torch.cuda.stream(st):
            step(eager)
        st.synchronize()
        want.append([x["O"].clone() for x in eager])
    graphed = setup()
    load(graphed, 0)
    g = torch.cuda.CUDAGraph()
    # capture advances nothing: kernels are recorded, not run
    with torch.cuda.graph(g, stream=st):
        step(graphed)
    assert [int(x["cache"].length.item()) for x in graphed] == [L0, L0]
    for s in range(S):
        load(graphed, s)
        with torch.cuda.stream(st):
            g.replay()
        st.synchronize()
        for l in range(2):
            assert torch.equal(graphed[l]["O"].view(torch.int16), want[s][l].view(torch.int16))
    assert [int(x["cache"].length.item()) for x in graphed] == [cap, cap]
    del g
