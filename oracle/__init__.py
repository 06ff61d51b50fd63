"""CPU oracle of the MSA routed-memory path (double precision).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and bench.py's CPU baseline
are the only code allowed to import this package. The CUDA library never imports it and
shares no code with it; the two meet only through the seeded inputs of ``synth``.

The per-output arithmetic lives in ``msa_oracle.c`` (plain C, double precision, one output at
a time) and this module marshals numpy arrays into it; the loops composing it (generation,
interleave rounds, the encode from hidden states with numpy's matrix product as the
projection) and the auxiliary routing loss are plain numpy here. Storage rounding of the bf16 configuration is
mirrored with the oracle's own round-to-nearest-even (``round_bf16``).

Parity unpinned: ``aux_routing_loss`` follows a reading of a loss the pages name without a
formula (its arithmetic is pinned, its agreement with the authors' loss is not).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

FP32, BF16 = 0, 1


def build(force: bool = False, src: str | None = None, out: str | None = None) -> str:
    """Compile the oracle with gcc (OpenMP). ``src``/``out`` let a test build a variant."""
    src = src or _SRC
    out = out or _SO
    if force or not os.path.exists(out) or os.path.getmtime(src) > os.path.getmtime(out):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", out, src, "-lm"])
    return out


def _declare(L):
    vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    L.orc_num_threads.restype = i32
    L.orc_round_bf16.restype = ctypes.c_uint16
    L.orc_round_bf16.argtypes = [dbl]
    L.orc_round_bf16_array.restype = None
    L.orc_round_bf16_array.argtypes = [vp, vp, i64]
    L.orc_rope.restype = None
    L.orc_rope.argtypes = [vp, i32, dbl, dbl]
    L.orc_cosine.restype = dbl
    L.orc_cosine.argtypes = [vp, vp, i32]
    L.orc_encode_pool.restype = i64
    L.orc_encode_pool.argtypes = [i32, vp, vp, vp, vp, i32, i32, i32, i32, dbl, vp, vp, vp, vp]
    L.orc_route.restype = i32
    L.orc_route.argtypes = [i32, vp, i32, i32, i32, vp, i32, i32, vp, i32, i32, vp, vp, vp, vp]
    L.orc_gather.restype = i32
    L.orc_gather.argtypes = [vp, i32, i32, vp, i32, i32, vp, vp]
    L.orc_attend.restype = i32
    L.orc_attend.argtypes = [i32, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp, i32, i32, i32,
                             i32, dbl, dbl, vp]
    L.orc_attend_backward.restype = i32
    L.orc_attend_backward.argtypes = [i32, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp, i32,
                                      i32, i32, i32, dbl, dbl, vp, vp, vp, vp, vp, vp]
    return L


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def load_variant(path: str):
    """Load a separately built copy of the oracle (used by the planted-mistake tests)."""
    return _declare(ctypes.CDLL(path))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(x: np.ndarray) -> int:
    if x.dtype == np.float32:
        return FP32
    if x.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {x.dtype}")


def _c(x):
    return np.ascontiguousarray(x)


def _same(*arrs) -> int:
    """All tensor inputs of one oracle call share one storage type; return its code."""
    codes = {_dt(a) for a in arrs}
    if len(codes) != 1:
        raise TypeError("oracle inputs of one call must share a dtype (float32 or bf16 bits)")
    return codes.pop()


def num_threads(L=None) -> int:
    return (L or lib()).orc_num_threads()


def round_bf16(x: np.ndarray, L=None) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    (L or lib()).orc_round_bf16_array(_p(x), _p(out), x.size)
    return out


def store_as(x: np.ndarray, dtype: str, L=None) -> np.ndarray:
    """Round double results to the storage type of the configuration."""
    return round_bf16(x, L) if dtype == "bf16" else np.asarray(x, dtype=np.float32)


def rope(x: np.ndarray, pos: float, base: float, L=None) -> np.ndarray:
    """RoPE of one head vector (copy, float64)."""
    v = np.array(x, dtype=np.float64, copy=True)
    (L or lib()).orc_rope(_p(v), v.shape[-1], float(pos), float(base))
    return v


def cosine(q, k, L=None) -> float:
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    return (L or lib()).orc_cosine(_p(q), _p(k), q.shape[-1])


def encode_pool(K, V, K_r, doc_tok_off, chunk: int, rope_base: float, L=None):
    """Doc-wise RoPE + chunk mean pooling. Returns (Kbar, Vbar, Krbar) float64
    [n_chunks, h_kv, d] and doc_chunk_off [n_docs+1] int64."""
    K, V, K_r = _c(K), _c(V), _c(K_r)
    off = np.ascontiguousarray(doc_tok_off, dtype=np.int64)
    n_docs = len(off) - 1
    h_kv, d = K.shape[1], K.shape[2]
    n_chunks = int(sum(-(-int(off[i + 1] - off[i]) // chunk) for i in range(n_docs)))
    Kb = np.empty((n_chunks, h_kv, d))
    Vb = np.empty_like(Kb)
    Rb = np.empty_like(Kb)
    coff = np.empty(n_docs + 1, dtype=np.int64)
    r = (L or lib()).orc_encode_pool(_same(K, V, K_r), _p(K), _p(V), _p(K_r), _p(off), n_docs, chunk, h_kv,
                                     d, float(rope_base), _p(Kb), _p(Vb), _p(Rb), _p(coff))
    if r != n_chunks:
        raise ValueError(f"orc_encode_pool returned {r}")
    return Kb, Vb, Rb, coff


def encode_hidden(H, W_k, W_v, W_r, doc_tok_off, chunk: int, rope_base: float, h_kv: int,
                  L=None):
    """Offline encode from hidden states. The pages name the projections but not where they
    sit; the reading here is that the per-token keys, values and router keys are projections
    of the hidden states, K = H W_k, V = H W_v,
    K_r = H W_r (the router K projector makes the routing keys: ruixiangma.github.io blog,
    "稀疏注意力机制"), computed here as plain matrix products in double precision; they then
    go through doc-wise RoPE and chunk mean pooling exactly as in ``encode_pool``.
    H [N_tok, D] and W_* [D, h_kv * d] in one storage type (float32, or bf16 bits as uint16).
    Returns (Kbar, Vbar, Krbar, doc_chunk_off) as ``encode_pool``."""
    def f64(x):
        x = np.ascontiguousarray(x)
        if x.dtype == np.uint16:
            return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        return x.astype(np.float64)

    H64 = f64(H)
    n = H64.shape[0]
    d = f64(W_k).shape[1] // h_kv
    # per-token projections, handed to the pooling in fp32 (the accumulation precision of the
    # product; a fused kernel never rounds them to the storage type)
    proj = [(H64 @ f64(W)).reshape(n, h_kv, d).astype(np.float32) for W in (W_k, W_v, W_r)]
    return encode_pool(proj[0], proj[1], proj[2], doc_tok_off, chunk, rope_base, L)


def route(Q_r, Kbar_r, doc_chunk_off, k: int, exclude_bits=None, L=None):
    """Cosine routing + top-k. Returns (top_ids int32 [B,k], top_scores f64 [B,k],
    doc_scores f64 [B, n_docs])."""
    Q_r, Kbar_r = _c(Q_r), _c(Kbar_r)
    B, T, h_qr, d = Q_r.shape
    h_kv = Kbar_r.shape[1]
    coff = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    n_docs = len(coff) - 1
    ids = np.empty((B, k), dtype=np.int32)
    ts = np.empty((B, k))
    ds = np.empty((B, n_docs))
    ex = None if exclude_bits is None else np.ascontiguousarray(exclude_bits, dtype=np.uint32)
    r = (L or lib()).orc_route(_same(Q_r, Kbar_r), _p(Q_r), B, T, h_qr, _p(Kbar_r), h_kv, d, _p(coff),
                               n_docs, k, _p(ex), _p(ds), _p(ids), _p(ts))
    if r != 0:
        raise ValueError("orc_route: invalid arguments")
    return ids, ts, ds


def gather(top_ids, doc_chunk_off, max_ctx: int, L=None):
    """Returns (gather_idx int32 [B, max_ctx], ctx_len int32 [B])."""
    ids = np.ascontiguousarray(top_ids, dtype=np.int32)
    B, k = ids.shape
    coff = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    gi = np.empty((B, max_ctx), dtype=np.int32)
    cl = np.empty(B, dtype=np.int32)
    r = (L or lib()).orc_gather(_p(ids), B, k, _p(coff), len(coff) - 1, max_ctx, _p(gi), _p(cl))
    if r != 0:
        raise ValueError(f"orc_gather returned {r}")
    return gi, cl


def attend(Q, K_loc, V_loc, Kbar, Vbar, gather_idx, ctx_len, pos0: int, rope_base: float,
           scale: float = 0.0, L=None):
    """Global-RoPE GQA attention over [gathered memory ; causal local]. Returns O float64."""
    Q, K_loc, V_loc, Kbar, Vbar = map(_c, (Q, K_loc, V_loc, Kbar, Vbar))
    B, T, h_q, d = Q.shape
    Lloc, h_kv = K_loc.shape[1], K_loc.shape[2]
    gi = np.ascontiguousarray(gather_idx, dtype=np.int32)
    cl = np.ascontiguousarray(ctx_len, dtype=np.int32)
    O = np.empty((B, T, h_q, d))
    r = (L or lib()).orc_attend(_same(Q, K_loc, V_loc, Kbar, Vbar), _p(Q), B, T, h_q, _p(K_loc), _p(V_loc), Lloc, _p(Kbar),
                                _p(Vbar), _p(gi), _p(cl), gi.shape[1], h_kv, d, int(pos0),
                                float(rope_base), float(scale), _p(O))
    if r != 0:
        raise ValueError("orc_attend: invalid arguments")
    return O


def attend_backward(Q, K_loc, V_loc, Kbar, Vbar, gather_idx, ctx_len, pos0: int,
                    rope_base: float, dO, scale: float = 0.0, L=None) -> dict:
    """Gradients of ``attend`` w.r.t. its inputs for an output gradient dO [B, T, h_q, d]
    (reverse mode of the same arithmetic, double precision). Returns dict(dQ, dK_loc, dV_loc,
    dK_ctx, dV_ctx, dKbar, dVbar): dK_ctx/dV_ctx [B, max_ctx, h_kv, d] per gathered row,
    dKbar/dVbar the same scattered into the bank rows (summed over the queries that gathered
    them). Routing itself (top-k) has no gradient."""
    Q, K_loc, V_loc, Kbar, Vbar = map(_c, (Q, K_loc, V_loc, Kbar, Vbar))
    B, T, h_q, d = Q.shape
    Lloc, h_kv = K_loc.shape[1], K_loc.shape[2]
    gi = np.ascontiguousarray(gather_idx, dtype=np.int32)
    cl = np.ascontiguousarray(ctx_len, dtype=np.int32)
    max_ctx = gi.shape[1]
    g_o = np.ascontiguousarray(dO, dtype=np.float64)
    out = dict(dQ=np.empty((B, T, h_q, d)), dK_loc=np.empty((B, Lloc, h_kv, d)),
               dV_loc=np.empty((B, Lloc, h_kv, d)), dK_ctx=np.empty((B, max_ctx, h_kv, d)),
               dV_ctx=np.empty((B, max_ctx, h_kv, d)))
    r = (L or lib()).orc_attend_backward(
        _same(Q, K_loc, V_loc, Kbar, Vbar), _p(Q), B, T, h_q, _p(K_loc), _p(V_loc), Lloc,
        _p(Kbar), _p(Vbar), _p(gi), _p(cl), max_ctx, h_kv, d, int(pos0), float(rope_base),
        float(scale), _p(g_o), _p(out["dQ"]), _p(out["dK_loc"]), _p(out["dV_loc"]),
        _p(out["dK_ctx"]), _p(out["dV_ctx"]))
    if r != 0:
        raise ValueError("orc_attend_backward: invalid arguments")
    dKb = np.zeros(Kbar.shape)
    dVb = np.zeros(Vbar.shape)
    for b in range(B):
        for j in range(int(cl[b])):
            dKb[gi[b, j]] += out["dK_ctx"][b, j]
            dVb[gi[b, j]] += out["dV_ctx"][b, j]
    out.update(dKbar=dKb, dVbar=dVb)
    return out


def aux_routing_loss(Q_r, Kbar_r, positive, tau: float = 0.1):
    """Auxiliary routing loss (a reading: the pages name a supervised
    contrastive loss that separates relevant from irrelevant document chunks but give no
    formula, so this function's parity with the authors' loss is unpinned).

    Chunk scores as in routing before the document maximum: s[b, c] = max over query tokens t of
    the mean over router heads h of cos(Q_r[b, t, h], Kbar_r[c, g(h)]), g(h) = h // (h_qr/h_kv).
    Positives positive[b, c] (bool): the chunks of the query's relevant documents. Loss per query
    = -mean over positives c of log softmax_c(s[b, :] / tau); averaged over the queries that
    have positives. Returns (loss, dQ_r, dKbar_r) in float64; the maximum over tokens passes its
    gradient to the first maximising token."""
    Q = np.asarray(Q_r, dtype=np.float64)
    K = np.asarray(Kbar_r, dtype=np.float64)
    pos = np.asarray(positive, dtype=bool)
    B, T, h_qr, d = Q.shape
    n, h_kv = K.shape[0], K.shape[1]
    grp = h_qr // h_kv
    qn = np.linalg.norm(Q, axis=-1, keepdims=True)
    kn = np.linalg.norm(K, axis=-1, keepdims=True)
    qh = np.where(qn > 0, Q / np.where(qn > 0, qn, 1), 0.0)      # [B, T, h_qr, d]
    kh = np.where(kn > 0, K / np.where(kn > 0, kn, 1), 0.0)      # [n, h_kv, d]
    kg = kh[:, np.arange(h_qr) // grp]                          # [n, h_qr, d]
    cos = np.einsum("bthd,chd->btch", qh, kg)                   # [B, T, n, h_qr]
    s_t = cos.mean(-1)                                          # [B, T, n]
    arg = s_t.argmax(1)                                         # [B, n] first maximising token
    s = np.take_along_axis(s_t, arg[:, None, :], 1)[:, 0]       # [B, n]
    loss, dQ, dK = 0.0, np.zeros_like(Q), np.zeros_like(K)
    rows = [b for b in range(B) if pos[b].any()]
    for b in rows:
        z = s[b] / tau
        z = z - z.max()
        p = np.exp(z) / np.exp(z).sum()
        P = pos[b]
        loss += -np.mean(np.log(p[P]))
        ds = (p - P / P.sum()) / tau / len(rows)                # d loss / d s[b, c]
        for c in range(n):
            t = arg[b, c]
            for h in range(h_qr):
                g = h // grp
                # d cos(q, k) / d q = (k_hat - cos q_hat) / |q|, and symmetrically for k
                w = ds[c] / h_qr
                if qn[b, t, h, 0] > 0 and kn[c, g, 0] > 0:
                    cq = cos[b, t, c, h]
                    dQ[b, t, h] += w * (kg[c, h] - cq * qh[b, t, h]) / qn[b, t, h, 0]
                    dK[c, g] += w * (qh[b, t, h] - cq * kh[c, g]) / kn[c, g, 0]
    return loss / max(len(rows), 1), dQ, dK


def pipeline(w, inp: dict, L=None) -> dict:
    """Oracle of one routed layer: (encode →) route → gather → attend, with the storage
    rounding of the configuration between steps. ``inp`` comes from synth."""
    out = {}
    dt = w.dtype
    if "K" in inp:  # per-token inputs: offline encode first
        Kb, Vb, Rb, coff = encode_pool(inp["K"], inp["V"], inp["K_r"], inp["doc_tok_off"],
                                       w.chunk, w.rope_base, L)
        out.update(Kbar64=Kb, Vbar64=Vb, Krbar64=Rb)
        Kbar, Vbar, Krbar = (store_as(a, dt, L) for a in (Kb, Vb, Rb))
        out.update(Kbar=Kbar, Vbar=Vbar, Kbar_r=Krbar, doc_chunk_off=coff)
    else:
        Kbar, Vbar, Krbar, coff = inp["Kbar"], inp["Vbar"], inp["Kbar_r"], inp["doc_chunk_off"]
    ids, ts, ds = route(inp["Q_r"], Krbar, coff, w.k, inp.get("exclude_bits"), L)
    out.update(top_ids=ids, top_scores=ts, doc_scores=ds)
    cpd_max = int(np.max(np.diff(coff))) if len(coff) > 1 else 0
    max_ctx = inp.get("max_ctx", w.k * cpd_max)
    gi, cl = gather(ids, coff, max_ctx, L)
    out.update(gather_idx=gi, ctx_len=cl)
    O = attend(inp["Q"], inp["K_loc"], inp["V_loc"], Kbar, Vbar, gi, cl, pos0=w.k,
               rope_base=w.rope_base, L=L)
    out["O64"] = O
    out["O"] = store_as(O, dt, L)
    return out


def interleave(layers: list, k: int, rounds: int, rope_base: float, doc_kv, L=None,
               select=None) -> dict:
    """Oracle of Memory Interleaving rounds. The pages describe the loop (retrieve, append the
    retrieved documents' text, repeat) but not which routed layer's selection is appended
    without a model; the reading here takes the last routed layer's selection, keeps pos0 = k
    in every round and excludes appended documents from later routing.

    layers[l]: dict with Kbar_r, Kbar, Vbar (stored dtype), doc_chunk_off, Q_r, Q and the query
    tokens' own K_q, V_q [B, T, h_kv, d]. doc_kv(l, doc) -> raw (K, V) [len, h_kv, d] of a
    retrieved document. Round 0 attends to the query tokens alone; after each round the docs
    selected by the LAST routed layer are appended (ascending id) for every later round,
    before the query tokens, and excluded from routing. pos0 = k in every round.
    ``select(r, ids_r)``, if given, stands for the model's generative retrieval: it receives the
    round's selections (ids_r[l] int32 [B, k] per routed layer) and returns, per query, the doc
    ids to append in order (already appended ids and ids < 0 are skipped), or None when the
    accumulated documents suffice, which ends the loop (ai-papers.net summary, "MSAの提案手法";
    ruixiangma.github.io blog, "Memory Interleaving": the model generates document ids, their
    text is appended, and the loop repeats until the model judges the documents sufficient).
    Returns dict(ids=[r][l] int32 [B,k], scores=[r][l], doc_scores=[r][l], O64=[r][l],
    appended=[b] list, rounds=rounds run)."""
    B = layers[0]["Q"].shape[0]
    n_docs = len(layers[0]["doc_chunk_off"]) - 1
    words = (n_docs + 31) // 32
    appended = [[] for _ in range(B)]
    res = dict(ids=[], scores=[], doc_scores=[], O64=[])
    for r in range(rounds):
        ex = np.zeros((B, words), dtype=np.uint32)
        for b in range(B):
            for doc in appended[b]:
                ex[b, doc // 32] |= np.uint32(1) << np.uint32(doc % 32)
        ids_r, sc_r, ds_r, O_r = [], [], [], []
        for li, lay in enumerate(layers):
            coff = lay["doc_chunk_off"]
            ids, sc, ds = route(lay["Q_r"], lay["Kbar_r"], coff, k, ex if r > 0 else None, L)
            cpd = int(np.max(np.diff(coff)))
            gi, cl = gather(ids, coff, k * cpd, L)
            K_loc = np.stack([np.concatenate([doc_kv(li, doc)[0] for doc in appended[b]] +
                                             [lay["K_q"][b]]) for b in range(B)])
            V_loc = np.stack([np.concatenate([doc_kv(li, doc)[1] for doc in appended[b]] +
                                             [lay["V_q"][b]]) for b in range(B)])
            O = attend(lay["Q"], K_loc, V_loc, lay["Kbar"], lay["Vbar"], gi, cl, pos0=k,
                       rope_base=rope_base, L=L)
            ids_r.append(ids)
            sc_r.append(sc)
            ds_r.append(ds)
            O_r.append(O)
        res["ids"].append(ids_r)
        res["scores"].append(sc_r)
        res["doc_scores"].append(ds_r)
        res["O64"].append(O_r)
        chosen = ([sorted(int(i) for i in ids_r[-1][b] if i >= 0) for b in range(B)]
                  if select is None else select(r, ids_r))
        if chosen is None:
            break
        for b in range(B):
            for doc in chosen[b]:
                if doc >= 0 and doc not in appended[b]:
                    appended[b].append(int(doc))
    res["appended"] = appended
    res["rounds"] = len(res["ids"])
    return res


def generate(Q_steps, Kn_steps, Vn_steps, K_prompt, V_prompt, Kbar, Vbar, gather_idx, ctx_len,
             pos0: int, rope_base: float, scale: float = 0.0, L=None):
    """Oracle of sparse generation over an assembled context. The pages route once, when the
    context is constructed, and generate over it; the reading here keeps the routed memory fixed
    for every generated token and appends each token's K/V to the local context.

    Routing and context assembly come first and the routed memory then stays fixed while the
    model generates autoregressively over the assembled context [news.neo-ai.one article,
    "推論パイプライン"; ruixiangma.github.io blog, "三阶段推理流程"]. Step s brings the K/V of
    its new tokens, Kn_steps[s], Vn_steps[s] [B, T, h_kv, d]: they join the end of the local
    context [K_prompt ; tokens of steps 0 .. s-1], and the step's queries Q_steps[s]
    [B, T, h_q, d] attend over [gathered memory ; that local context] exactly as ``attend``
    (query token t is the local row L - T + t). Returns O64 [S, B, T, h_q, d]."""
    K_loc, V_loc = np.asarray(K_prompt), np.asarray(V_prompt)
    out = []
    for s in range(len(Q_steps)):
        K_loc = np.concatenate([K_loc, np.asarray(Kn_steps[s])], axis=1)
        V_loc = np.concatenate([V_loc, np.asarray(Vn_steps[s])], axis=1)
        out.append(attend(Q_steps[s], K_loc, V_loc, Kbar, Vbar, gather_idx, ctx_len, pos0,
                          rope_base, scale, L))
    return np.stack(out)
