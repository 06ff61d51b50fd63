"""Memory Interleaving rounds: properties of the oracle's loop (CPU) and parity of the
engine over libmsa against it (GPU)."""
import numpy as np
import pytest

import oracle
import synth
from _util import SCORE_TOL, check_attention, check_topk, to_dev


def _case(B=2, T=32, n_docs=150, doc_len=100, layers=2, k=4, seed=5):
    w = synth.C5.scaled(n_docs=n_docs, doc_len=doc_len, B=B, T=T, L_loc=T, k=k, h_q=8, h_kv=2,
                        h_qr=2, layers=layers, rounds=3, n_planted=1, seed=seed)
    lays = []
    for l in range(layers):
        inp = synth.make_bank_workload(w, l)
        lays.append(dict(Kbar_r=inp["Kbar_r"], Kbar=inp["Kbar"], Vbar=inp["Vbar"],
                         doc_chunk_off=inp["doc_chunk_off"], Q_r=inp["Q_r"], Q=inp["Q"],
                         K_q=inp["K_loc"], V_q=inp["V_loc"]))
    return w, lays


def test_oracle_interleave_round_structure():
    w, lays = _case()
    res = oracle.interleave(lays, w.k, 3, w.rope_base, lambda l, d: synth.appended_doc_kv(w, l, d))
    # round 0 is the plain routed layer with the query tokens as the local context
    for l, lay in enumerate(lays):
        ids, _, _ = oracle.route(lay["Q_r"], lay["Kbar_r"], lay["doc_chunk_off"], w.k)
        assert np.array_equal(res["ids"][0][l], ids)
    for b in range(w.B):
        app = res["appended"][b]
        assert len(app) == 3 * w.k and len(set(app)) == len(app)  # k new docs per round
        assert app[:w.k] == sorted(res["ids"][0][-1][b].tolist())
        assert app[w.k:2 * w.k] == sorted(res["ids"][1][-1][b].tolist())
        for r in (1, 2):  # appended docs are never routed again
            for l in range(len(lays)):
                assert not set(res["ids"][r][l][b].tolist()) & set(app[:r * w.k])


def test_oracle_interleave_follows_selected_docs_and_stops():
    """Generative retrieval stood in for by a schedule: the docs a round selects are appended in
    the order given (duplicates skipped), excluded from later routing, and a None ends the loop.
    (Every query appends the same number of new documents per round: one local length per
    batch.)"""
    w, lays = _case()
    dk = lambda l, d: synth.appended_doc_kv(w, l, d)  # noqa: E731
    sched = {0: [[5, 3], [9, 4]], 1: [[3, 7], [2, 9]]}  # one new doc each in round 1
    seen = []

    def sel(r, ids_r):
        assert len(ids_r) == len(lays) and ids_r[0].shape == (w.B, w.k)
        seen.append(r)
        return sched.get(r)

    res = oracle.interleave(lays, w.k, 4, w.rope_base, dk, select=sel)
    assert res["rounds"] == 3 and seen == [0, 1, 2]
    assert res["appended"] == [[5, 3, 7], [9, 4, 2]]
    for l in range(len(lays)):
        assert not set(res["ids"][1][l][0].tolist()) & {5, 3}
        assert not set(res["ids"][1][l][1].tolist()) & {9, 4}
        assert not set(res["ids"][2][l][0].tolist()) & {5, 3, 7}
        assert not set(res["ids"][2][l][1].tolist()) & {9, 4, 2}
    # round 2 of layer 0, query 0, attends over [doc 5 ; doc 3 ; doc 7 ; query tokens]
    lay = lays[0]
    coff = lay["doc_chunk_off"]
    cpd = int(np.max(np.diff(coff)))
    gi, cl = oracle.gather(res["ids"][2][0], coff, w.k * cpd)
    parts = [dk(0, doc) for doc in (5, 3, 7)]
    K_loc = np.concatenate([p[0] for p in parts] + [lay["K_q"][0]])[None]
    V_loc = np.concatenate([p[1] for p in parts] + [lay["V_q"][0]])[None]
    O = oracle.attend(lay["Q"][:1], K_loc, V_loc, lay["Kbar"], lay["Vbar"], gi[:1], cl[:1], w.k,
                      w.rope_base)
    assert np.array_equal(O[0], res["O64"][2][0][0])


def test_oracle_interleave_attends_to_appended_text():
    """Round 1 equals attention over [memory ; round-0 docs' raw K/V ; query tokens]."""
    w, lays = _case(B=1, layers=1, seed=9)
    dk = lambda l, d: synth.appended_doc_kv(w, l, d)  # noqa: E731
    res = oracle.interleave(lays, w.k, 2, w.rope_base, dk)
    lay = lays[0]
    app = res["appended"][0][:w.k]
    K_loc = np.concatenate([dk(0, d)[0] for d in app] + [lay["K_q"][0]])[None]
    V_loc = np.concatenate([dk(0, d)[1] for d in app] + [lay["V_q"][0]])[None]
    assert K_loc.shape[1] == w.T + w.k * w.doc_len
    gi, cl = oracle.gather(res["ids"][1][0], lay["doc_chunk_off"], w.k * w.cpd)
    O = oracle.attend(lay["Q"], K_loc, V_loc, lay["Kbar"], lay["Vbar"], gi, cl, w.k, w.rope_base)
    assert np.max(np.abs(O - res["O64"][1][0])) == 0.0


@pytest.mark.gpu
def test_interleave_engine_matches_oracle(gpu):
    import torch

    import long_context_doc_b200 as msa
    from long_context_doc_b200 import engine
    w, lays = _case()
    dk_np = lambda l, d: synth.appended_doc_kv(w, l, d)  # noqa: E731
    ref = oracle.interleave(lays, w.k, 3, w.rope_base, dk_np)
    layers = []
    for lay in lays:
        Krb = to_dev(lay["Kbar_r"], gpu)
        layers.append(engine.RoutedLayer(
            Kbar_r=Krb, kr_inv_norm=msa.kr_inv_norm(Krb), Kbar=to_dev(lay["Kbar"], gpu),
            Vbar=to_dev(lay["Vbar"], gpu),
            doc_chunk_off=torch.from_numpy(lay["doc_chunk_off"]).to(gpu),
            Q_r=to_dev(lay["Q_r"], gpu), Q=to_dev(lay["Q"], gpu), K_q=to_dev(lay["K_q"], gpu),
            V_q=to_dev(lay["V_q"], gpu), Kbar_r_hat=msa.kr_normalize(Krb)))
    cache = {}

    def dk_dev(l, d):
        if (l, d) not in cache:
            kk, vv = dk_np(l, d)
            cache[(l, d)] = (to_dev(kk, gpu), to_dev(vv, gpu))
        return cache[(l, d)]

    ids, scores, O, appended = engine.interleave_rounds(layers, w.k, 3, w.rope_base, dk_dev)
    torch.cuda.synchronize()
    assert len(ids) == 3
    followed = _check_rounds_on_engine_selection(w, lays, ids, scores, O, dk_np)
    assert appended == followed
    if all(np.array_equal(ids[r][l].cpu().numpy(), ref["ids"][r][l])
           for r in range(3) for l in range(len(lays))):
        assert appended == ref["appended"]
        for r in range(3):
            for l in range(len(lays)):
                check_attention(O[r][l], ref["O64"][r][l], "bf16")


@pytest.mark.gpu
def test_interleave_engine_with_selected_docs_matches_oracle(gpu):
    """The engine's loop with the appended documents chosen by a caller (here: the first routed
    layer's two best documents, best first) and an early stop, against the oracle's loop."""
    import torch

    import long_context_doc_b200 as msa
    from long_context_doc_b200 import engine
    w, lays = _case(seed=9)
    dk_np = lambda l, d: synth.appended_doc_kv(w, l, d)  # noqa: E731

    def sel(r, ids_r):
        if r == 2:
            return None
        return [[int(x) for x in ids_r[0][b][:2]] for b in range(w.B)]

    ref = oracle.interleave(lays, w.k, 4, w.rope_base, dk_np, select=sel)
    assert ref["rounds"] == 3
    layers = []
    for lay in lays:
        Krb = to_dev(lay["Kbar_r"], gpu)
        layers.append(engine.RoutedLayer(
            Kbar_r=Krb, kr_inv_norm=msa.kr_inv_norm(Krb), Kbar=to_dev(lay["Kbar"], gpu),
            Vbar=to_dev(lay["Vbar"], gpu),
            doc_chunk_off=torch.from_numpy(lay["doc_chunk_off"]).to(gpu),
            Q_r=to_dev(lay["Q_r"], gpu), Q=to_dev(lay["Q"], gpu), K_q=to_dev(lay["K_q"], gpu),
            V_q=to_dev(lay["V_q"], gpu), Kbar_r_hat=msa.kr_normalize(Krb)))
    cache = {}

    def dk_dev(l, d):
        if (l, d) not in cache:
            kk, vv = dk_np(l, d)
            cache[(l, d)] = (to_dev(kk, gpu), to_dev(vv, gpu))
        return cache[(l, d)]

    ids, scores, O, appended = engine.interleave_rounds(layers, w.k, 4, w.rope_base, dk_dev,
                                                        select=sel)
    torch.cuda.synchronize()
    assert len(ids) == 3
    followed = _check_rounds_on_engine_selection(w, lays, ids, scores, O, dk_np, select=sel)
    assert appended == followed
    if all(np.array_equal(ids[r][l].cpu().numpy(), ref["ids"][r][l])
           for r in range(3) for l in range(len(lays))):
        assert appended == ref["appended"]


def _check_rounds_on_engine_selection(w, lays, ids, scores, O, dk_np, select=None):
    """Every round and routed layer of the engine's loop against the oracle, on the engine's
    own selections: the oracle routes with the documents the engine appended so far excluded
    and the engine's top-k must be a valid one under the gap rule; the oracle then gathers the
    engine's ids and attends over [appended documents' raw K/V ; query tokens], and the
    engine's output must match it. Near-ties therefore never skip a comparison. Returns the
    appended documents per query that this replay of the loop arrives at."""
    B = w.B
    n_docs = len(lays[0]["doc_chunk_off"]) - 1
    words = (n_docs + 31) // 32
    tol = SCORE_TOL["bf16"]
    appended = [[] for _ in range(B)]
    for r in range(len(ids)):
        ex = None
        if r > 0:
            ex = np.zeros((B, words), np.uint32)
            for b in range(B):
                for doc in appended[b]:
                    ex[b, doc // 32] |= np.uint32(1 << (doc % 32))
        g_round = []
        for l, lay in enumerate(lays):
            coff = lay["doc_chunk_off"]
            r_ids, r_sc, r_ds = oracle.route(lay["Q_r"], lay["Kbar_r"], coff, w.k, ex)
            masked = r_ds.copy()
            for b in range(B):
                masked[b, appended[b]] = -np.inf
            g_ids = ids[r][l].cpu().numpy()
            check_topk(g_ids, scores[r][l].cpu().numpy().astype(np.float64), r_ids, r_sc, masked,
                       tol)
            for b in range(B):
                assert not set(g_ids[b].tolist()) & set(appended[b])
            gi, cl = oracle.gather(g_ids, coff, w.k * int(np.max(np.diff(coff))))
            K_loc = np.stack([np.concatenate([dk_np(l, d)[0] for d in appended[b]] +
                                             [lay["K_q"][b]]) for b in range(B)])
            V_loc = np.stack([np.concatenate([dk_np(l, d)[1] for d in appended[b]] +
                                             [lay["V_q"][b]]) for b in range(B)])
            O_ref = oracle.attend(lay["Q"], K_loc, V_loc, lay["Kbar"], lay["Vbar"], gi, cl, w.k,
                                  w.rope_base)
            check_attention(O[r][l], O_ref, "bf16")
            g_round.append(g_ids)
        chosen = ([sorted(int(i) for i in g_round[-1][b] if i >= 0) for b in range(B)]
                  if select is None else select(r, g_round))
        if chosen is None:
            assert r == len(ids) - 1
            break
        for b in range(B):
            for doc in chosen[b]:
                if doc >= 0 and doc not in appended[b]:
                    appended[b].append(int(doc))
    return appended


@pytest.mark.gpu
@pytest.mark.parametrize("dt", ["fp32", "bf16"])
def test_assemble_local_matches_concatenation(gpu, dt):
    """msa_assemble_local writes [segments in order ; query rows] bit for bit; a query whose
    segment lengths do not add up to L_loc - T is reported through the workspace status."""
    import torch

    import long_context_doc_b200 as msa
    from long_context_doc_b200 import engine
    rng = np.random.default_rng(2)
    B, T, h, d = 3, 5, 2, 64
    lens = [[7, 3, 12], [10, 10, 2], [1, 20, 1]]  # 22 appended rows per query
    tdt = torch.float32 if dt == "fp32" else torch.bfloat16

    def mk(*shape):
        return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(gpu).to(tdt)

    parts = [[(mk(n, h, d), mk(n, h, d)) for n in row] for row in lens]
    Kq, Vq = mk(B, T, h, d), mk(B, T, h, d)
    K, V = engine.assemble_local(parts, Kq, Vq)
    torch.cuda.synchronize()
    assert K.shape == (B, 22 + T, h, d)
    for b in range(B):
        assert torch.equal(K[b], torch.cat([p[0] for p in parts[b]] + [Kq[b]]))
        assert torch.equal(V[b], torch.cat([p[1] for p in parts[b]] + [Vq[b]]))
    # one row too many in L_loc: every query mismatches, nothing is written, status is set
    kp = torch.tensor([[kv[0].data_ptr() for kv in p] for p in parts], dtype=torch.int64).to(gpu)
    vp = torch.tensor([[kv[1].data_ptr() for kv in p] for p in parts], dtype=torch.int64).to(gpu)
    ln = torch.tensor(lens, dtype=torch.int32).to(gpu)
    Ko = torch.full((B, 22 + T + 1, h, d), 7.0, dtype=tdt, device=gpu)
    Vo = torch.full_like(Ko, 7.0)
    ws = torch.zeros(256, dtype=torch.uint8, device=gpu)
    msa.msa_assemble_local(kp, vp, ln, Kq, Vq, Ko, Vo, ws)
    torch.cuda.synchronize()
    assert msa.msa_workspace_status(ws) != 0
    assert bool((Ko == 7.0).all()) and bool((Vo == 7.0).all())
