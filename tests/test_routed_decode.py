"""The routed-layer decode step of the package (``engine.RoutedDecode``) against the oracle.

The step is the benchmarked one: every routed layer routes over its whole bank, fetches the
selected documents' K̄/V̄ from a bank in pinned host memory (zero-copy gather on a side
stream, or cudaMemcpyAsync runs) or from device memory, and attends; layer l+1's fetch
overlaps layer l's attention, and the gathered rows rotate through two buffer sets. Each
layer's ids, gather indices, context lengths and output are compared with the oracle's
routing, gather and attention on that layer's inputs, eagerly and replayed from a CUDA graph,
so an ordering slip between the streams or a buffer reused too early shows up here.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import SCORE_TOL, check_attention, check_topk, to_dev

pytestmark = pytest.mark.gpu

# the 100M-token-bank decode configuration (B = 4, T = 1, 32 query heads, 8 KV heads, k = 16,
# 2,048 local rows) over 4 routed layers of a reduced, ragged bank
W = synth.C4.scaled(n_docs=2500, layers=4, ragged=True, seed=77)


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


@pytest.fixture(scope="module")
def host_layers():
    return [synth.make_bank_workload(W, layer=l) for l in range(W.layers)]


def _build(msa, gpu, host_layers, fetch, scan, cached=False):
    """With ``cached``, every layer's local context is a rotated cache holding the first
    L_loc - 1 rows, and the step appends the last row (the query token's own K/V) before
    attending: the same attention as the uncached step over K_loc/V_loc."""
    from long_context_doc_b200.engine import DecodeLayer, RoutedDecode
    layers = []
    lens = torch.zeros(len(host_layers), dtype=torch.int32, device=gpu)
    for l, inp in enumerate(host_layers):
        if fetch == "device":
            Kb, Vb = to_dev(inp["Kbar"], gpu), to_dev(inp["Vbar"], gpu)
        else:
            Kb, Vb = (to_dev(inp[n], "cpu").pin_memory() for n in ("Kbar", "Vbar"))
        Krb = to_dev(inp["Kbar_r"], gpu)
        kw = (dict(Kbar_r_hat=msa.kr_normalize(Krb)) if scan == "tc" else
              dict(Kbar_r=Krb, kr_inv_norm=msa.kr_inv_norm(Krb)))
        Kl, Vl = to_dev(inp["K_loc"], gpu), to_dev(inp["V_loc"], gpu)
        if cached:
            c = msa.LocalCache(W.B, W.L_loc, W.h_kv, W.d, pos0=W.k, rope_base=W.rope_base,
                               device=gpu, length=lens[l:l + 1])
            c.append(Kl[:, :-1].contiguous(), Vl[:, :-1].contiguous())
            kw.update(cache=c, K_new=Kl[:, -1:].contiguous(), V_new=Vl[:, -1:].contiguous())
            Kl = Vl = None
        layers.append(DecodeLayer(to_dev(inp["Q_r"], gpu), to_dev(inp["Q"], gpu), Kl, Vl, Kb, Vb,
                                  **kw))
    rd = RoutedDecode(layers, host_layers[0]["doc_chunk_off"], W.k, W.rope_base, fetch=fetch)
    rd.test_lens = lens  # the caches' lengths, reset to L_loc - 1 before every step
    return rd


def _check_against_oracle(rd, host_layers):
    tol = SCORE_TOL["bf16"]
    ids_all = rd.ids.cpu().numpy()
    sc_all = rd.scores.cpu().numpy().astype(np.float64)
    gi_all = rd.gather_idx.cpu().numpy()
    cl_all = rd.ctx_len.cpu().numpy()
    for l, inp in enumerate(host_layers):
        coff = inp["doc_chunk_off"]
        r_ids, r_sc, r_ds = oracle.route(inp["Q_r"], inp["Kbar_r"], coff, W.k)
        check_topk(ids_all[l], sc_all[l], r_ids, r_sc, r_ds, tol)
        assert np.array_equal(ids_all[l][:, 0], inp["planted"][:, 0])
        r_gi, r_cl = oracle.gather(ids_all[l], coff, rd.max_ctx)
        assert np.array_equal(gi_all[l], r_gi), f"layer {l}: gather indices"
        assert np.array_equal(cl_all[l], r_cl), f"layer {l}: context lengths"
        O_ref = oracle.attend(inp["Q"], inp["K_loc"], inp["V_loc"], inp["Kbar"], inp["Vbar"],
                              r_gi, r_cl, W.k, W.rope_base)
        check_attention(rd.O[l], O_ref, "bf16")


def _poison(rd):
    rd.ids.fill_(-5)
    rd.scores.fill_(float("nan"))
    rd.gather_idx.fill_(-5)
    rd.ctx_len.fill_(-5)
    rd.O.fill_(float("nan"))
    for bf in rd.buf:
        bf["cK"].fill_(float("nan"))
        bf["cV"].fill_(float("nan"))


@pytest.mark.parametrize("fetch,scan,graph,cached", [
    ("zerocopy", "tc", False, False),  # the host-bank schedule, launched eagerly
    ("zerocopy", "tc", True, False),   # ... and replayed from a CUDA graph
    ("memcpy", "tc", False, False),    # host-issued cudaMemcpyAsync runs
    ("device", "cc", True, False),     # device bank, CUDA-core scan, graph
    ("zerocopy", "tc", True, True),    # rotated local caches, the benchmarked form
    ("memcpy", "tc", False, True),
], ids=["zerocopy_eager", "zerocopy_graph", "memcpy_eager", "device_cc_graph",
        "zerocopy_graph_cached", "memcpy_eager_cached"])
def test_routed_decode_step_matches_oracle(msa, gpu, host_layers, fetch, scan, graph, cached):
    rd = _build(msa, gpu, host_layers, fetch, scan, cached)
    assert rd.nbuf == 2 and rd.L == 4
    reset = lambda: rd.test_lens.fill_(W.L_loc - 1)  # noqa: E731
    reset()
    torch.cuda.synchronize()
    rd.step()
    torch.cuda.synchronize()
    if graph:
        rd.capture()
        _poison(rd)
        torch.cuda.synchronize()
        for _ in range(2):  # a second step on the same buffers (cross-step ordering)
            with torch.cuda.stream(rd.stream):
                reset()
            rd.replay()
    else:
        _poison(rd)
        torch.cuda.synchronize()
        with torch.cuda.stream(rd.stream):
            for _ in range(2):
                reset()
                rd.step()
    torch.cuda.synchronize()
    if cached:
        assert rd.test_lens.cpu().tolist() == [W.L_loc] * rd.L
    for bf in rd.buf:
        assert msa.msa_workspace_status(bf["ws_r"]) == 0
        assert msa.msa_workspace_status(bf["ws_g"]) == 0
        assert msa.msa_workspace_status(bf["ws_a"]) == 0
    _check_against_oracle(rd, host_layers)


def test_routed_decode_waits_for_local_inputs(msa, gpu, host_layers):
    """``step(local_ready=ev)``: the local K/V rows of the query token, written on another
    stream behind a ~25 ms spin (long after the first layers have routed), reach the first
    attention because the step's stream waits on the event: the outputs equal, bit for bit,
    those of the same step with the rows already in place."""
    rd = _build(msa, gpu, host_layers, "zerocopy", "tc")
    torch.cuda.synchronize()
    rd.step()
    torch.cuda.synchronize()
    O_ref = rd.O.clone()
    ids_ref = rd.ids.clone()
    rows = [(la.K_loc[:, -1:].clone(), la.V_loc[:, -1:].clone()) for la in rd.layers]
    for la in rd.layers:
        la.K_loc[:, -1:].zero_()
        la.V_loc[:, -1:].zero_()
    torch.cuda.synchronize()
    side = torch.cuda.Stream(gpu)
    ready = torch.cuda.Event()
    with torch.cuda.stream(side):
        torch.cuda._sleep(50_000_000)
        for la, (k, v) in zip(rd.layers, rows):
            la.K_loc[:, -1:].copy_(k)
            la.V_loc[:, -1:].copy_(v)
        ready.record(side)
    rd.step(local_ready=ready)
    torch.cuda.synchronize()
    assert torch.equal(rd.ids, ids_ref)
    assert torch.equal(rd.O, O_ref)
    _check_against_oracle(rd, host_layers)


def test_routed_decode_rejects_bad_configurations(msa, gpu, host_layers):
    """A fetch mode that does not match where the bank lives is refused, and so is capturing the
    cudaMemcpyAsync fetch (it waits on the host for every layer's ids)."""
    from long_context_doc_b200.engine import RoutedDecode
    rd = _build(msa, gpu, host_layers[:1], "device", "tc")
    with pytest.raises(ValueError):
        RoutedDecode(rd.layers, host_layers[0]["doc_chunk_off"], W.k, W.rope_base,
                     fetch="zerocopy")
    rd = _build(msa, gpu, host_layers[:2], "memcpy", "tc")
    assert not rd.capturable
    with pytest.raises(RuntimeError):
        rd.capture()
