"""GPU parity: every libmsa entry point against the CPU oracle on the same seeded inputs.

Small cases span several tiles, ragged tails, empty documents and the degenerate shapes of
the method; the full-size banks (1M-token encode, 10M-token bank, 100M-token bank layer)
are checked in the launch configuration the benchmark times, on outputs the oracle can
compute one by one (sampled documents / chunks) and on properties that hold at any size.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import (ATT_TOL, SCORE_TOL, check_attention, check_pooled, check_topk, stored_f64,
                   to_dev, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


# ----------------------------------------------------------------------------- generator
def test_device_generator_is_bit_identical(gpu):
    for dt, td in (("fp32", torch.float32), ("bf16", torch.bfloat16)):
        t = torch.empty(100_003, dtype=td, device=gpu)
        synth.dev_normal(t, 5, synth.tag(synth.K, 3), first=12345, scale=1.0)
        h = synth.normal(5, synth.tag(synth.K, 3), (100_003,), dt, first=12345)
        got = t.view(torch.int16).cpu().numpy().view(np.uint16) if dt == "bf16" else t.cpu().numpy()
        assert np.array_equal(got, h)


# ----------------------------------------------------------------------------- encode
def _encode_case(msa, gpu, w):
    inp = synth.make_token_workload(w)
    ref = {}
    Kb, Vb, Rb, coff = oracle.encode_pool(inp["K"], inp["V"], inp["K_r"], inp["doc_tok_off"],
                                          w.chunk, w.rope_base)
    out = msa.encode_pool(to_dev(inp["K"], gpu), to_dev(inp["V"], gpu), to_dev(inp["K_r"], gpu),
                          inp["doc_tok_off"], w.chunk, w.rope_base)
    torch.cuda.synchronize()
    assert msa.msa_encode_pool_status() == 0  # no device wait ran out
    assert np.array_equal(out["doc_chunk_off"].cpu().numpy(), coff)
    check_pooled(out["Kbar"], Kb, w.dtype, "Kbar")
    check_pooled(out["Vbar"], Vb, w.dtype, "Vbar")
    check_pooled(out["Kbar_r"], Rb, w.dtype, "Kbar_r")
    stored = to_np(out["Kbar_r"])
    nrm = np.sqrt((stored ** 2).sum(-1))
    inv = np.where(nrm > 0, 1.0 / np.where(nrm > 0, nrm, 1), 0.0)
    np.testing.assert_allclose(out["kr_inv_norm"].cpu().numpy(), inv, rtol=2e-6, atol=0)
    return inp, out, (Kb, Vb, Rb, coff)


@pytest.mark.parametrize("w", [
    synth.C1,                                                            # tiny fp32, full size
    synth.C1.scaled(n_docs=37, doc_len=150, ragged=True, seed=3),        # ragged, partial chunks
    synth.C2.scaled(n_docs=12, doc_len=300, ragged=True, n_planted=2),   # Qwen3-4B heads, bf16
    synth.C2.scaled(n_docs=6, doc_len=1024, n_planted=1, chunk=128),     # chunk > table block
    synth.C1.scaled(n_docs=9, doc_len=5, chunk=1, n_planted=0),          # chunk = 1
    synth.C2.scaled(n_docs=40, doc_len=90, ragged=True, h_q=16, h_kv=4, h_qr=4, n_planted=1,
                    seed=5),                                             # bf16, 4 KV heads
    synth.C2.scaled(n_docs=17, doc_len=200, ragged=True, n_planted=1, rope_base=0.0,
                    chunk=48, seed=6),                                   # bf16, no RoPE, chunk 48
], ids=["c1_full", "ragged_fp32", "qwen3_bf16_ragged", "chunk128", "chunk1", "bf16_hkv4",
        "bf16_norope_chunk48"])
def test_encode_pool_matches_oracle(msa, gpu, w):
    _encode_case(msa, gpu, w)


@pytest.mark.parametrize("dt,h_kv,d", [(torch.float32, 2, 64), (torch.bfloat16, 8, 128)],
                         ids=["fp32", "bf16_bulk_copies"])
def test_encode_pool_constant_chunk_and_empty_docs(msa, gpu, dt, h_kv, d):
    lens = np.array([7, 0, 64, 65, 0])
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(off[-1])
    c = torch.full((n, h_kv, d), 0.75, dtype=dt, device=gpu)
    out = msa.encode_pool(c, c, c, off, 64, 0.0)  # RoPE disabled
    torch.cuda.synchronize()
    assert msa.msa_encode_pool_status() == 0
    for key in ("Kbar", "Vbar", "Kbar_r"):
        assert torch.all(out[key] == 0.75)
    assert out["doc_chunk_off"].cpu().tolist() == [0, 1, 1, 2, 4, 4]
    inv = out["kr_inv_norm"].cpu().numpy()
    np.testing.assert_allclose(inv, 1.0 / np.sqrt(d * 0.75 ** 2), rtol=1e-6)


def test_encode_pool_full_1m_token_bank_sampled(msa, gpu):
    """1M-token bank (1024 docs x 1024 tokens, 8 KV heads, d=128, bf16): full GPU encode;
    the oracle recomputes a sample of documents from the same generator."""
    w = synth.C2
    inp = synth.dev_token_workload(w, gpu)
    out = msa.encode_pool(inp["K"], inp["V"], inp["K_r"], inp["doc_tok_off"], w.chunk,
                          w.rope_base)
    torch.cuda.synchronize()
    off = inp["doc_tok_off"]
    coff = synth.chunk_offsets_from_lengths(np.diff(off), w.chunk)
    assert np.array_equal(out["doc_chunk_off"].cpu().numpy(), coff)
    docs = sorted(set([0, w.n_docs - 1] + list(inp["planted"][:2]) +
                      list(synth.uniform(9, 1, 3, w.n_docs))))
    for dd in docs:
        a, b = int(off[dd]), int(off[dd + 1])
        rows = {n: synth.host_token_rows(w, n, a, b) for n in ("K", "V", "K_r")}
        Kb, Vb, Rb, _ = oracle.encode_pool(rows["K"], rows["V"], rows["K_r"],
                                           np.array([0, b - a]), w.chunk, w.rope_base)
        c0, c1 = int(coff[dd]), int(coff[dd + 1])
        check_pooled(out["Kbar"][c0:c1], Kb, "bf16", f"Kbar doc {dd}")
        check_pooled(out["Vbar"][c0:c1], Vb, "bf16", f"Vbar doc {dd}")
        check_pooled(out["Kbar_r"][c0:c1], Rb, "bf16", f"Kbar_r doc {dd}")


# ----------------------------------------------------------------------------- routing
def _bank_inputs(w, gpu, layer=0):
    inp = synth.make_bank_workload(w, layer)
    d = {k: to_dev(inp[k], gpu) for k in ("Kbar_r", "Kbar", "Vbar", "Q", "Q_r", "K_loc", "V_loc")}
    d["doc_chunk_off"] = torch.from_numpy(inp["doc_chunk_off"]).to(gpu)
    return inp, d


def _route_check(msa, gpu, Q_r_np, Krb_np, coff_np, k, dtype, exclude=None):
    Q_r, Krb = to_dev(Q_r_np, gpu), to_dev(Krb_np, gpu)
    coff = torch.from_numpy(np.ascontiguousarray(coff_np, np.int64)).to(gpu)
    inv = msa.kr_inv_norm(Krb)
    ex = None if exclude is None else torch.from_numpy(exclude.view(np.int32)).to(gpu)
    ids, sc, ds = msa.route_topk(Q_r, Krb, inv, coff, k, exclude_bits=ex, doc_scores=True)
    torch.cuda.synchronize()
    r_ids, r_sc, r_ds = oracle.route(Q_r_np, Krb_np, coff_np, k, exclude)
    tol = SCORE_TOL[dtype]
    gds = ds.cpu().numpy().astype(np.float64)
    fin = np.isfinite(r_ds)
    assert np.array_equal(np.isfinite(gds), fin)
    assert np.max(np.abs(gds[fin] - r_ds[fin]), initial=0.0) <= tol
    ids_np, sc_np = ids.cpu().numpy(), sc.cpu().numpy().astype(np.float64)
    if exclude is None:
        n_exact = check_topk(ids_np, sc_np, r_ids, r_sc, r_ds, tol)
    else:
        masked = r_ds.copy()
        for b in range(masked.shape[0]):
            for i in range(masked.shape[1]):
                if (exclude[b, i // 32] >> (i % 32)) & 1:
                    masked[b, i] = -np.inf
        n_exact = check_topk(ids_np, sc_np, r_ids, r_sc, masked, tol)
    return ids_np, sc_np, gds, n_exact


def test_route_tiny_fp32_config(msa, gpu):
    w = synth.C1
    inp = synth.make_token_workload(w)
    ref = oracle.pipeline(w, inp)
    ids, sc, ds, n_exact = _route_check(msa, gpu, inp["Q_r"], ref["Kbar_r"], ref["doc_chunk_off"],
                                        w.k, "fp32")
    assert n_exact == 1


@pytest.mark.parametrize("B,T,dt,n_docs,ragged", [
    (8, 1, "bf16", 3000, False),   # decode batch, several tiles per CTA
    (4, 1, "bf16", 2501, True),    # ragged docs, partial chunks, empty-free
    (3, 5, "bf16", 700, True),     # 15 rows per pass
    (1, 16, "fp32", 300, True),
    (40, 1, "bf16", 500, False),   # three passes of <= 16 queries
    (2, 2, "fp32", 1, False),      # a single document
])
def test_route_matches_oracle(msa, gpu, B, T, dt, n_docs, ragged):
    w = synth.C3.scaled(n_docs=n_docs, B=B, T=T, dtype=dt, ragged=ragged, seed=B * 7 + T,
                        k=min(16, n_docs), n_planted=1 if n_docs >= B else 0)
    inp = synth.make_bank_workload(w)
    ids, sc, ds, n_exact = _route_check(msa, gpu, inp["Q_r"], inp["Kbar_r"], inp["doc_chunk_off"],
                                        w.k, dt)
    if w.n_planted:  # planted docs rank first
        assert np.array_equal(ids[:, 0], inp["planted"][:, 0])


def test_route_router_head_groups_and_empty_docs(msa, gpu):
    rng = np.random.default_rng(1)
    lens = rng.integers(0, 400, 257)
    lens[[0, 5, 256]] = 0
    coff = synth.chunk_offsets_from_lengths(lens, 64)
    n_ch = int(coff[-1])
    Krb = synth.normal(2, 7, (n_ch, 4, 64), "bf16")
    Qr = synth.normal(2, 8, (3, 2, 8, 64), "bf16")  # h_qr = 2 * h_kv
    ids, sc, ds, _ = _route_check(msa, gpu, Qr, Krb, coff, 12, "bf16")
    assert np.all(np.isneginf(ds[:, [0, 5, 256]]))


def test_route_k_equals_n_docs_and_duplicate_ties(msa, gpu):
    n_docs, cpd = 24, 3
    coff = np.arange(0, cpd * n_docs + 1, cpd, dtype=np.int64)
    Krb = synth.normal(4, 1, (cpd * n_docs, 2, 64), "fp32")
    Krb[cpd * 5:cpd * 6] = Krb[cpd * 17:cpd * 18]
    Krb[cpd * 9:cpd * 10] = Krb[cpd * 17:cpd * 18]
    Qr = synth.normal(4, 2, (2, 1, 2, 64), "fp32")
    Qr[1, 0] = Krb[cpd * 17 + 1]
    ids, sc, ds, _ = _route_check(msa, gpu, Qr, Krb, coff, n_docs, "fp32")
    assert sorted(ids[0].tolist()) == list(range(n_docs))
    assert ds[1, 5] == ds[1, 9] == ds[1, 17]          # bit-identical on the GPU too
    assert list(ids[1, :3]) == [5, 9, 17]               # ties to the lower id
    assert abs(sc[1, 0] - 1.0) < 1e-5


def test_route_exclusion_bits(msa, gpu):
    w = synth.C3.scaled(n_docs=999, B=4, seed=11)
    inp = synth.make_bank_workload(w)
    words = (w.n_docs + 31) // 32
    ex = np.zeros((w.B, words), np.uint32)
    rng = np.random.default_rng(2)
    for b in range(w.B):
        for i in rng.choice(w.n_docs, 300, replace=False).tolist() + [int(inp["planted"][b, 0])]:
            ex[b, i // 32] |= np.uint32(1 << (i % 32))
    ids, sc, ds, _ = _route_check(msa, gpu, inp["Q_r"], inp["Kbar_r"], inp["doc_chunk_off"], w.k,
                                  "bf16", exclude=ex)
    for b in range(w.B):
        for i in ids[b]:
            assert not (ex[b, i // 32] >> (i % 32)) & 1


def test_route_fewer_eligible_than_k(msa, gpu):
    n_docs = 40
    coff = np.arange(0, 2 * n_docs + 1, 2, dtype=np.int64)
    Krb = synth.normal(6, 1, (2 * n_docs, 2, 64), "fp32")
    Qr = synth.normal(6, 2, (1, 1, 2, 64), "fp32")
    ex = np.array([[0xFFFFFFFF, 0xFFFFFFFF & ~0b101]], np.uint32)  # only docs 32 and 34 eligible
    Q_r, K_r = to_dev(Qr, gpu), to_dev(Krb, gpu)
    ids, sc, _ = msa.route_topk(Q_r, K_r, msa.kr_inv_norm(K_r), torch.from_numpy(coff).to(gpu), 5,
                                exclude_bits=torch.from_numpy(ex.view(np.int32)).to(gpu))
    r_ids, r_sc, _ = oracle.route(Qr, Krb, coff, 5, ex)
    assert ids.cpu().numpy().tolist() == r_ids.tolist()
    assert np.all(np.isneginf(sc.cpu().numpy()[0, 2:]))


def test_route_full_10m_token_bank(msa, gpu):
    """10M-token bank (20,000 docs x 8 chunks, bf16), 8 decode queries: every doc score
    against the oracle, exact top-16."""
    w = synth.C3
    dv = synth.dev_bank_workload(w, gpu, with_kv=False)
    coff = dv["doc_chunk_off"]
    inv = msa.kr_inv_norm(dv["Kbar_r"])
    ids, sc, ds = msa.route_topk(dv["Q_r"], dv["Kbar_r"], inv, torch.from_numpy(coff).to(gpu), w.k,
                                 doc_scores=True)
    torch.cuda.synchronize()
    Krb = synth.host_bank_rows(w, "Kbar_r", 0, dv["n_chunks"], coff=coff, Q_r=dv["Q_r_host"])
    r_ids, r_sc, r_ds = oracle.route(dv["Q_r_host"], Krb, coff, w.k)
    gds = ds.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(gds - r_ds)) <= SCORE_TOL["bf16"]
    check_topk(ids.cpu().numpy(), sc.cpu().numpy().astype(np.float64), r_ids, r_sc, r_ds,
               SCORE_TOL["bf16"])
    assert np.array_equal(ids.cpu().numpy()[:, 0], dv["planted"][:, 0])


@pytest.fixture(scope="module")
def bank100m_layer(gpu):
    """One routed layer of the 100M-token bank (200,000 docs x 8 chunks = 1.6M chunks, bf16,
    3.3 GB) on the device, its host twin, and the oracle's routing of the 4 decode queries
    over every chunk."""
    w = synth.C4
    dv = synth.dev_bank_workload(w, gpu, layer=0, with_kv=False)
    coff = dv["doc_chunk_off"]
    Krb = synth.host_bank_rows(w, "Kbar_r", 0, dv["n_chunks"], coff=coff, Q_r=dv["Q_r_host"])
    ref = oracle.route(dv["Q_r_host"], Krb, coff, w.k)
    del Krb
    yield w, dv, ref
    del dv
    torch.cuda.empty_cache()


@pytest.mark.slow
@pytest.mark.parametrize("scan", ["tc", "cc"], ids=["tensor_core_scan", "cuda_core_scan"])
def test_route_full_100m_token_bank_layer(msa, gpu, bank100m_layer, scan):
    """A full 100M-token bank layer (1.6M chunks, 3.3 GB) routed for the 4 decode queries of
    the benchmarked configuration, in the launch configuration the benchmark times for
    ``tc`` (the tensor-core scan over the normalised bank, without K̄_r or its norms): every
    one of the 200,000 document scores against the oracle's full routing within the bf16
    tolerance, and the top-16 against the oracle's ids under the gap rule."""
    w, dv, (r_ids, r_sc, r_ds) = bank100m_layer
    coff = torch.from_numpy(dv["doc_chunk_off"]).to(gpu)
    if scan == "tc":
        hat = msa.kr_normalize(dv["Kbar_r"])
        ids, sc, ds = msa.route_topk(dv["Q_r"], None, None, coff, w.k, doc_scores=True,
                                     Kbar_r_hat=hat)
    else:
        inv = msa.kr_inv_norm(dv["Kbar_r"])
        ids, sc, ds = msa.route_topk(dv["Q_r"], dv["Kbar_r"], inv, coff, w.k, doc_scores=True)
    torch.cuda.synchronize()
    gds = ds.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(gds))
    err = np.max(np.abs(gds - r_ds))
    assert err <= SCORE_TOL["bf16"], err
    check_topk(ids.cpu().numpy(), sc.cpu().numpy().astype(np.float64), r_ids, r_sc, r_ds,
               SCORE_TOL["bf16"])
    assert np.array_equal(ids.cpu().numpy()[:, 0], dv["planted"][:, 0])


def test_route_reports_small_workspace(msa, gpu):
    w = synth.C3.scaled(n_docs=100, B=2)
    inp, d = _bank_inputs(w, gpu)
    inv = msa.kr_inv_norm(d["Kbar_r"])
    ws = torch.empty(300, dtype=torch.uint8, device=gpu)
    with pytest.raises(msa.MSAError) as e:
        msa.route_topk(d["Q_r"], d["Kbar_r"], inv, d["doc_chunk_off"], w.k, ws=ws)
    assert e.value.status == 3


# ----------------------------------------------------------------------------- gather
@pytest.mark.parametrize("k", [16, 32])  # 32: every lane of the ranking warp holds an id
def test_gather_indices_exact_and_rows_copied(msa, gpu, k):
    w = synth.C3.scaled(n_docs=300, B=5, ragged=True, seed=5, k=k)
    inp, d = _bank_inputs(w, gpu)
    coff = inp["doc_chunk_off"]
    rng = np.random.default_rng(3)
    ids = np.stack([rng.choice(w.n_docs, w.k, replace=False) for _ in range(w.B)]).astype(np.int32)
    ids[2, 3] = -1
    ids[4, k - 1] = -1  # an empty last slot
    max_ctx = int(w.k * np.max(np.diff(coff)))
    gi, cl, cK, cV = msa.gather(torch.from_numpy(ids).to(gpu), d["doc_chunk_off"], d["Kbar"],
                                d["Vbar"], max_ctx)
    torch.cuda.synchronize()
    r_gi, r_cl = oracle.gather(ids, coff, max_ctx)
    assert np.array_equal(gi.cpu().numpy(), r_gi) and np.array_equal(cl.cpu().numpy(), r_cl)
    kb = d["Kbar"].view(torch.int16).cpu().numpy()
    vb = d["Vbar"].view(torch.int16).cpu().numpy()
    ck = cK.view(torch.int16).cpu().numpy()
    cv = cV.view(torch.int16).cpu().numpy()
    for b in range(w.B):
        n = r_cl[b]
        assert np.array_equal(ck[b, :n], kb[r_gi[b, :n]])
        assert np.array_equal(cv[b, :n], vb[r_gi[b, :n]])


def test_gather_overflow_is_flagged_and_bounded(msa, gpu):
    w = synth.C3.scaled(n_docs=50, B=1)
    inp, d = _bank_inputs(w, gpu)
    ids = torch.arange(16, dtype=torch.int32, device=gpu)[None]
    ws = torch.zeros(256, dtype=torch.uint8, device=gpu)
    gi, cl, cK, cV = msa.gather(ids, d["doc_chunk_off"], d["Kbar"], d["Vbar"], 20, ws=ws)
    assert msa.msa_workspace_status(ws) == 2
    assert cl.item() == 20
    assert gi.cpu().numpy()[0].tolist() == list(range(20))


def test_fetch_from_pinned_host_bank_equals_device_gather(msa, gpu):
    w = synth.C3.scaled(n_docs=400, B=4, seed=8)
    inp, d = _bank_inputs(w, gpu)
    coff = inp["doc_chunk_off"]
    Kh = d["Kbar"].cpu().pin_memory()
    Vh = d["Vbar"].cpu().pin_memory()
    rng = np.random.default_rng(4)
    ids_np = np.stack([rng.choice(w.n_docs, w.k, replace=False) for _ in range(w.B)]).astype(np.int32)
    ids_np[0, :3] = [10, 11, 12]  # adjacent docs: merged copies
    ids = torch.from_numpy(ids_np).to(gpu)
    max_ctx = w.k * w.cpd
    gi, cl, cK, cV = msa.gather(ids, d["doc_chunk_off"], d["Kbar"], d["Vbar"], max_ctx)
    f = msa.Fetcher(w.B, w.k)
    gi2 = torch.empty_like(gi)
    cl2 = torch.empty_like(cl)
    cK2 = torch.zeros_like(cK)
    cV2 = torch.zeros_like(cV)
    ws = torch.zeros(256, dtype=torch.uint8, device=gpu)
    copy_stream = torch.cuda.Stream()
    f.begin(ids, d["doc_chunk_off"], max_ctx, gi2, cl2, ws)
    f.finish(coff, Kh, Vh, max_ctx, cK2, cV2, copy_stream=copy_stream)
    torch.cuda.synchronize()
    assert torch.equal(gi, gi2) and torch.equal(cl, cl2)
    assert torch.equal(cK.view(torch.int16), cK2.view(torch.int16))
    assert torch.equal(cV.view(torch.int16), cV2.view(torch.int16))
    # the same gather kernel reading the pinned host bank directly (zero-copy)
    gi3, cl3, cK3, cV3 = msa.gather(ids, d["doc_chunk_off"], Kh, Vh, max_ctx)
    torch.cuda.synchronize()
    assert torch.equal(cK.view(torch.int16), cK3.view(torch.int16))
    f.close()


def test_fetch_wait_is_bounded(msa, gpu):
    """A host wait that runs out returns MSA_ERR_TIMEOUT and the context stays usable."""
    w = synth.C3.scaled(n_docs=64, B=1)
    inp, d = _bank_inputs(w, gpu)
    coff = inp["doc_chunk_off"]
    Kh = d["Kbar"].cpu().pin_memory()
    Vh = d["Vbar"].cpu().pin_memory()
    ids = torch.arange(w.k, dtype=torch.int32, device=gpu)[None]
    max_ctx = w.k * w.cpd
    gi = torch.empty((1, max_ctx), dtype=torch.int32, device=gpu)
    cl = torch.empty(1, dtype=torch.int32, device=gpu)
    cK = torch.zeros((1, max_ctx, 8, 128), dtype=torch.bfloat16, device=gpu)
    cV = torch.zeros_like(cK)
    ws = torch.zeros(256, dtype=torch.uint8, device=gpu)
    f = msa.Fetcher(1, w.k)
    torch.cuda._sleep(200_000_000)  # keep the stream busy (~0.1 s) so the ids are not ready
    f.begin(ids, d["doc_chunk_off"], max_ctx, gi, cl, ws)
    with pytest.raises(msa.MSAError) as e:
        f.finish(coff, Kh, Vh, max_ctx, cK, cV, timeout_ms=0)
    assert e.value.status == 5
    f.finish(coff, Kh, Vh, max_ctx, cK, cV, timeout_ms=10_000)
    torch.cuda.synchronize()
    assert torch.equal(cK[0, :max_ctx].view(torch.int16), d["Kbar"][:max_ctx].view(torch.int16))
    f.close()


# ----------------------------------------------------------------------------- attention
def _attend_case(msa, gpu, dt, B, T, h_q, h_kv, d, L, n_ctx, pos0, base, seed=0):
    rng = np.random.default_rng(seed)
    n_bank = max(int(n_ctx.max()) * 2, 1)
    Q = synth.normal(seed, 101, (B, T, h_q, d), dt)
    Kl = synth.normal(seed, 102, (B, L, h_kv, d), dt)
    Vl = synth.normal(seed, 103, (B, L, h_kv, d), dt)
    Kb = synth.normal(seed, 104, (n_bank, h_kv, d), dt)
    Vb = synth.normal(seed, 105, (n_bank, h_kv, d), dt)
    max_ctx = max(int(n_ctx.max()), 1)
    gi = np.full((B, max_ctx), -1, np.int32)
    for b in range(B):
        gi[b, :n_ctx[b]] = rng.choice(n_bank, n_ctx[b], replace=False)
    ref = oracle.attend(Q, Kl, Vl, Kb, Vb, gi, n_ctx.astype(np.int32), pos0, base)
    ctxK = np.zeros((B, max_ctx, h_kv, d), Kb.dtype)
    ctxV = np.zeros((B, max_ctx, h_kv, d), Vb.dtype)
    for b in range(B):
        ctxK[b, :n_ctx[b]] = Kb[gi[b, :n_ctx[b]]]
        ctxV[b, :n_ctx[b]] = Vb[gi[b, :n_ctx[b]]]
    O = msa.sparse_attend(to_dev(Q, gpu), to_dev(Kl, gpu), to_dev(Vl, gpu), to_dev(ctxK, gpu),
                          to_dev(ctxV, gpu), torch.from_numpy(n_ctx.astype(np.int32)).to(gpu),
                          pos0, base)
    torch.cuda.synchronize()
    return check_attention(O, ref, dt)


@pytest.mark.parametrize("dt,B,T,h_q,h_kv,d,L,ctx,pos0,base", [
    ("fp32", 1, 16, 4, 2, 64, 16, [32], 4, 1e6),        # tiny config shape
    ("bf16", 2, 1, 32, 8, 128, 2048, [128, 77], 16, 1e6),  # decode, 10M/100M-bank shape
    ("bf16", 1, 128, 32, 8, 128, 128, [256], 16, 1e6),  # 1M-bank prefill shape
    ("fp32", 3, 5, 8, 2, 128, 40, [0, 9, 33], 7, 1e4),  # T < L, one query without memory
    ("bf16", 2, 3, 4, 4, 64, 3, [5, 300], 2, 0.0),      # RoPE off, MHA, long memory
    # decode-shaped (bf16, d = 128, <= 8 query rows per KV head): the streaming decode kernel
    ("bf16", 3, 2, 16, 4, 128, 100, [0, 64, 130], 16, 1e6),  # 8 rows, causal over 2 tokens
    ("bf16", 2, 1, 8, 2, 128, 40, [20, 3], 4, 1e6),     # one tile per pair (no split merge)
    ("bf16", 2, 1, 4, 4, 128, 300, [50, 0], 3, 1e4),    # one row per KV head, no memory
    ("bf16", 1, 1, 8, 2, 128, 200, [70], 2, 0.0),       # RoPE off
    ("bf16", 2, 1, 32, 8, 128, 1024, [96, 128], 5000, 1e6),  # positions up to 6k
    ("fp32", 1, 1, 2, 1, 64, 1, [1], 0, 1e6),           # one memory row + the query itself
    ("bf16", 2, 1, 32, 8, 128, 2048, [256, 200], 32, 1e6),  # k = 32 docs of 8 chunks (max k)
    # long queries (bf16, d = 128, >= 64 query rows per KV head): the tensor-core kernel
    ("bf16", 2, 64, 16, 4, 128, 300, [0, 200], 9, 1e6),  # 2 query tiles, padded L, no memory
    ("bf16", 1, 40, 64, 8, 128, 40, [70], 3, 1e4),      # 8 heads per KV head, partial tile, L = T
    ("bf16", 2, 128, 8, 8, 128, 256, [64, 5], 0, 0.0),  # one head per KV head, RoPE off
    ("bf16", 1, 256, 32, 8, 128, 1300, [64], 8, 1e6),   # interleave-round shape, 11 local tiles
    ("bf16", 1, 128, 32, 8, 128, 128, [512], 32, 1e6),  # prefill shape at k = 32 (512 memory rows)
])
def test_attend_matches_oracle(msa, gpu, dt, B, T, h_q, h_kv, d, L, ctx, pos0, base):
    _attend_case(msa, gpu, dt, B, T, h_q, h_kv, d, L, np.array(ctx), pos0, base)


def test_attend_full_10m_bank_decode_batch(msa, gpu):
    """Decode attention at the 10M-bank config size: B=8, 32 query heads, 128 memory rows +
    2048 local rows, bf16."""
    rel = _attend_case(msa, gpu, "bf16", 8, 1, 32, 8, 128, 2048, np.full(8, 128), 16, 1e6, seed=2)
    assert rel < ATT_TOL["bf16"]


# ----------------------------------------------------------------------------- pipeline
@pytest.mark.parametrize("w", [synth.C1, synth.C1.scaled(ragged=True, n_docs=23, seed=4)],
                         ids=["c1", "c1_ragged"])
def test_pipeline_tiny_config(msa, gpu, w):
    inp = synth.make_token_workload(w)
    ref = oracle.pipeline(w, inp)
    t = lambda x: to_dev(x, gpu)  # noqa: E731
    enc = msa.encode_pool(t(inp["K"]), t(inp["V"]), t(inp["K_r"]), inp["doc_tok_off"], w.chunk,
                          w.rope_base)
    ids, sc, ds = msa.route_topk(t(inp["Q_r"]), enc["Kbar_r"], enc["kr_inv_norm"],
                                 enc["doc_chunk_off"], w.k, doc_scores=True)
    max_ctx = ref["gather_idx"].shape[1]
    gi, cl, cK, cV = msa.gather(ids, enc["doc_chunk_off"], enc["Kbar"], enc["Vbar"], max_ctx)
    O = msa.sparse_attend(t(inp["Q"]), t(inp["K_loc"]), t(inp["V_loc"]), cK, cV, cl, w.k,
                          w.rope_base)
    torch.cuda.synchronize()
    check_topk(ids.cpu().numpy(), sc.cpu().numpy().astype(np.float64), ref["top_ids"],
               ref["top_scores"], ref["doc_scores"], SCORE_TOL[w.dtype])
    _check_downstream_of_selection(w, inp, ref, ids, gi, cl, O, max_ctx)


def _check_downstream_of_selection(w, inp, ref, ids, gi, cl, O, max_ctx):
    """Gather and attention checked on the GPU's own selection (a valid top-k under the gap
    rule, already checked): the oracle gathers and attends with the GPU's ids, and the GPU's
    gather indices must equal the oracle's bit for bit and its output the oracle's within the
    attention tolerance. Runs whatever the selection, so it never skips."""
    g_ids = ids.cpu().numpy()
    r_gi, r_cl = oracle.gather(g_ids, ref["doc_chunk_off"], max_ctx)
    assert np.array_equal(gi.cpu().numpy(), r_gi)
    assert np.array_equal(cl.cpu().numpy(), r_cl)
    O_ref = oracle.attend(inp["Q"], inp["K_loc"], inp["V_loc"], ref["Kbar"], ref["Vbar"], r_gi,
                          r_cl, w.k, w.rope_base)
    check_attention(O, O_ref, w.dtype)
    if np.array_equal(g_ids, ref["top_ids"]):  # same selection: the oracle's pipeline output
        assert np.array_equal(r_gi, ref["gather_idx"])
        check_attention(O, ref["O64"], w.dtype)


# ----------------------------------------------------------------------------- tensor-core scan
def _route_tc_check(msa, gpu, Qr, Krb, coff, k, exclude=None):
    """Long queries: bf16 tensor-core scan from the normalised bank; scores within the bf16
    tolerance, exact top-k under the gap rule."""
    Q_r, K_r = to_dev(Qr, gpu), to_dev(Krb, gpu)
    cof = torch.from_numpy(np.ascontiguousarray(coff, np.int64)).to(gpu)
    inv = msa.kr_inv_norm(K_r)
    hat = msa.kr_normalize(K_r)
    ex = None if exclude is None else torch.from_numpy(exclude.view(np.int32)).to(gpu)
    ws = torch.zeros(msa.msa_route_topk_workspace(Qr.shape[0], Qr.shape[1], Qr.shape[2],
                                                  Krb.shape[1], Krb.shape[2], 1, len(coff) - 1,
                                                  Krb.shape[0], k), dtype=torch.uint8, device=gpu)
    ids, sc, ds = msa.route_topk(Q_r, K_r, inv, cof, k, exclude_bits=ex, doc_scores=True, ws=ws,
                                 Kbar_r_hat=hat)
    torch.cuda.synchronize()
    assert msa.msa_workspace_status(ws) == 0
    r_ids, r_sc, r_ds = oracle.route(Qr, Krb, coff, k, exclude)
    gds = ds.cpu().numpy().astype(np.float64)
    fin = np.isfinite(r_ds)
    assert np.array_equal(np.isfinite(gds), fin)
    err = np.max(np.abs(gds[fin] - r_ds[fin]), initial=0.0)
    assert err <= SCORE_TOL["bf16"], err
    masked = r_ds.copy()
    if exclude is not None:
        for b in range(masked.shape[0]):
            for i in range(masked.shape[1]):
                if (exclude[b, i // 32] >> (i % 32)) & 1:
                    masked[b, i] = -np.inf
    check_topk(ids.cpu().numpy(), sc.cpu().numpy().astype(np.float64), r_ids, r_sc, masked,
               SCORE_TOL["bf16"])
    return ids.cpu().numpy(), err


@pytest.mark.parametrize("B,T,n_docs,ragged", [
    (1, 128, 300, True),     # 1M-bank prefill shape, partial last chunk tile
    (3, 40, 150, False),     # several queries per row tile, padded N
    (2, 256, 200, True),     # interleave-round query length, one query per tile
    (1, 17, 5, False),       # shortest query on the tensor path, fewer chunks than a tile
])
def test_route_tensor_core_matches_oracle(msa, gpu, B, T, n_docs, ragged):
    w = synth.C5.scaled(n_docs=n_docs, B=B, T=T, ragged=ragged, seed=T + B, k=min(8, n_docs),
                        n_planted=1)
    inp = synth.make_bank_workload(w)
    ids, err = _route_tc_check(msa, gpu, inp["Q_r"], inp["Kbar_r"], inp["doc_chunk_off"], w.k)
    if T <= 16:  # a long query's mean direction is nearly orthogonal to each of its tokens
        assert np.array_equal(ids[:, 0], inp["planted"][:, 0])


@pytest.mark.parametrize("B,T,n_docs,ragged", [
    (8, 1, 3000, False),     # 10M-bank decode batch shape
    (7, 1, 1900, True),      # 7 queries: the 8-warp form, a warp with no query in the merge
    (4, 1, 2501, True),      # 100M-bank decode batch shape, ragged docs
    (40, 1, 700, False),     # wide decode batch: one 48-column tile
    (3, 5, 400, True),       # short multi-token queries
])
def test_route_tensor_core_decode_matches_oracle(msa, gpu, B, T, n_docs, ragged):
    w = synth.C3.scaled(n_docs=n_docs, B=B, T=T, ragged=ragged, seed=100 + B + T)
    inp = synth.make_bank_workload(w)
    ids, err = _route_tc_check(msa, gpu, inp["Q_r"], inp["Kbar_r"], inp["doc_chunk_off"], w.k)
    assert np.array_equal(ids[:, 0], inp["planted"][:, 0])


@pytest.mark.parametrize("scan,B,n_docs,k", [
    ("tc", 8, 900, 32),    # the largest k: a full 32-lane list per query
    ("cc", 8, 900, 32),
    ("tc", 64, 600, 32),   # the largest tensor-core batch (one 64-column query tile)
    ("tc", 4, 20, 20),     # every document selected, fewer chunk tiles than SMs
], ids=["tc_k32", "cc_k32", "tc_b64_k32", "tc_all_docs"])
def test_route_largest_k_and_batch(msa, gpu, scan, B, n_docs, k):
    """Maximum sizes of the routing call: k = 32 (the fused top-k's one-warp list), 64 decode
    queries in one tensor-core tile, and k = n_docs (every document ranked)."""
    w = synth.C3.scaled(n_docs=n_docs, B=B, T=1, ragged=True, seed=500 + B + k, k=k)
    inp = synth.make_bank_workload(w)
    if scan == "tc":
        ids, _ = _route_tc_check(msa, gpu, inp["Q_r"], inp["Kbar_r"], inp["doc_chunk_off"], k)
    else:
        ids = _route_check(msa, gpu, inp["Q_r"], inp["Kbar_r"], inp["doc_chunk_off"], k,
                           "bf16")[0]
    assert np.array_equal(ids[:, 0], inp["planted"][:, 0])
    if k == n_docs:
        assert all(sorted(r) == list(range(n_docs)) for r in ids.tolist())


def test_route_tensor_core_full_10m_token_bank_decode(msa, gpu):
    w = synth.C3
    dv = synth.dev_bank_workload(w, gpu, with_kv=False)
    coff = dv["doc_chunk_off"]
    Krb = synth.host_bank_rows(w, "Kbar_r", 0, dv["n_chunks"], coff=coff, Q_r=dv["Q_r_host"])
    ids, err = _route_tc_check(msa, gpu, dv["Q_r_host"], Krb, coff, w.k)
    assert np.array_equal(ids[:, 0], dv["planted"][:, 0])


def test_route_tensor_core_head_groups_and_exclusion(msa, gpu):
    rng = np.random.default_rng(12)
    lens = rng.integers(0, 700, 90)
    lens[[3, 89]] = 0
    coff = synth.chunk_offsets_from_lengths(lens, 64)
    Krb = synth.normal(3, 5, (int(coff[-1]), 4, 128), "bf16")
    Qr = synth.normal(3, 6, (2, 64, 8, 128), "bf16")  # h_qr = 2 * h_kv
    ex = np.zeros((2, 3), np.uint32)
    ex[0, 0] = 0xF0F0F0F0
    ex[1, 2] = 0x3FFFFFF
    _route_tc_check(msa, gpu, Qr, Krb, coff, 12, exclude=ex)


def test_route_tensor_core_full_1m_token_bank(msa, gpu):
    """Routing at the 1M-token-bank size (16,384 chunks, 8 KV heads, d=128) for a 128-token
    query, on a synthetic pooled bank; every document score against the oracle."""
    w = synth.C5.scaled(n_docs=1024, doc_len=1024, B=1, T=128, k=16, n_planted=1, seed=21)
    dv = synth.dev_bank_workload(w, gpu, with_kv=False)
    coff = dv["doc_chunk_off"]
    Krb = synth.host_bank_rows(w, "Kbar_r", 0, dv["n_chunks"], coff=coff, Q_r=dv["Q_r_host"])
    ids, err = _route_tc_check(msa, gpu, dv["Q_r_host"], Krb, coff, w.k)
    assert ids[0, 0] == dv["planted"][0, 0]


def test_pipeline_1m_bank_shape_reduced(msa, gpu):
    """The 1M-token-bank configuration's full path at 24 documents: doc-wise RoPE + pooling,
    tensor-core routing of the 128-token query, gather, global-RoPE attention (bf16)."""
    w = synth.C2.scaled(n_docs=24, n_planted=2)
    inp = synth.make_token_workload(w)
    ref = oracle.pipeline(w, inp)
    t = lambda x: to_dev(x, gpu)  # noqa: E731
    enc = msa.encode_pool(t(inp["K"]), t(inp["V"]), t(inp["K_r"]), inp["doc_tok_off"], w.chunk,
                          w.rope_base)
    check_pooled(enc["Kbar_r"], ref["Krbar64"], "bf16", "Kbar_r")
    hat = msa.kr_normalize(enc["Kbar_r"])
    ids, sc, ds = msa.route_topk(t(inp["Q_r"]), enc["Kbar_r"], enc["kr_inv_norm"],
                                 enc["doc_chunk_off"], w.k, doc_scores=True, Kbar_r_hat=hat)
    max_ctx = ref["gather_idx"].shape[1]
    gi, cl, cK, cV = msa.gather(ids, enc["doc_chunk_off"], enc["Kbar"], enc["Vbar"], max_ctx)
    O = msa.sparse_attend(t(inp["Q"]), t(inp["K_loc"]), t(inp["V_loc"]), cK, cV, cl, w.k,
                          w.rope_base)
    torch.cuda.synchronize()
    assert np.max(np.abs(ds.cpu().numpy() - ref["doc_scores"])) <= SCORE_TOL["bf16"]
    check_topk(ids.cpu().numpy(), sc.cpu().numpy().astype(np.float64), ref["top_ids"],
               ref["top_scores"], ref["doc_scores"], SCORE_TOL["bf16"])
    _check_downstream_of_selection(w, inp, ref, ids, gi, cl, O, max_ctx)
