"""Routed-layer loops over the libmsa entry points: the decode step over a tiered memory bank
(``RoutedDecode``) and Memory Interleaving rounds (``interleave_rounds``).

Decode over a tiered bank: the router keys of every routed layer stay resident on the GPU
while the content K̄/V̄ sit in host memory and only the selected documents' rows are fetched,
asynchronously, when routing has chosen them [ruixiangma.github.io blog, "Memory Parallel /
分层内存存储"; news.neo-ai.one article, "推論パイプライン"]. ``RoutedDecode`` schedules one
decode step of all routed layers so that each layer's fetch runs on a side stream while the
next layer's routing scan streams its bank.

Memory Interleaving alternates generative retrieval, context extension and generation: the
documents a round retrieves have their original text appended to the query for the next
round, and routing repeats until the model judges the accumulated documents sufficient
[ai-papers.net summary, "MSAの提案手法"; ruixiangma.github.io blog, "Memory Interleaving"].
Without a model to generate document ids, a round's retrieval is read from the routing
itself: the documents selected by the last routed layer of round r are appended (their raw
per-token K/V, in ascending doc id, after the documents of earlier rounds and before the
query tokens) and excluded from routing in later rounds. Every round uses pos0 = k.

Only the loop lives here; every step of every round runs in libmsa's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import numpy as np
import torch

from . import (Fetcher, LocalCache, gather, msa_assemble_local, msa_decode_step,
               msa_decode_step_workspace, msa_gather, msa_route_topk, msa_route_topk_workspace,
               msa_sparse_attend, msa_sparse_attend_workspace, route_topk, sparse_attend)


@dataclass
class RoutedLayer:
    """One routed layer's memory bank and the query's per-layer tensors."""
    Kbar_r: torch.Tensor        # [n_chunks, h_kv, d]
    kr_inv_norm: torch.Tensor   # [n_chunks, h_kv] fp32
    Kbar: torch.Tensor          # [n_chunks, h_kv, d] (device or pinned host memory)
    Vbar: torch.Tensor
    doc_chunk_off: torch.Tensor  # [n_docs + 1] int64, device
    Q_r: torch.Tensor           # [B, T, h_qr, d]
    Q: torch.Tensor             # [B, T, h_q, d]
    K_q: torch.Tensor           # [B, T, h_kv, d] the query tokens' own keys (before RoPE)
    V_q: torch.Tensor           # [B, T, h_kv, d]
    Kbar_r_hat: Optional[torch.Tensor] = None  # normalised bank for the tensor-core scan


def exclusion_bits(appended: Sequence[Sequence[int]], n_docs: int, device) -> torch.Tensor:
    """[B, ceil(n_docs/32)] int32 bitsets of the documents already appended per query."""
    words = (n_docs + 31) // 32
    bits = torch.zeros((len(appended), words), dtype=torch.int64)
    for b, docs in enumerate(appended):
        for doc in docs:
            bits[b, doc // 32] |= 1 << (doc % 32)
    bits = torch.where(bits >= 2 ** 31, bits - 2 ** 32, bits)
    return bits.to(torch.int32).to(device)


def assemble_local(parts, K_q, V_q):
    """parts[b] = [(K, V) [len, h_kv, d] device tensors of the appended documents, in order];
    returns the local K/V [B, sum(len) + T, h_kv, d] built by msa_assemble_local."""
    B, T = K_q.shape[0], K_q.shape[1]
    n_seg = len(parts[0])
    if any(len(p) != n_seg for p in parts):
        raise ValueError("every query appends the same number of documents")
    L = {sum(kv[0].shape[0] for kv in p) + T for p in parts}
    if len(L) != 1:
        raise ValueError("interleaved local contexts must have one length per batch")
    L = L.pop()
    dev = K_q.device
    kp = torch.tensor([[kv[0].data_ptr() for kv in p] for p in parts], dtype=torch.int64).to(dev)
    vp = torch.tensor([[kv[1].data_ptr() for kv in p] for p in parts], dtype=torch.int64).to(dev)
    ln = torch.tensor([[kv[0].shape[0] for kv in p] for p in parts], dtype=torch.int32).to(dev)
    K_out = torch.empty((B, L) + tuple(K_q.shape[2:]), dtype=K_q.dtype, device=dev)
    V_out = torch.empty_like(K_out)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    msa_assemble_local(kp, vp, ln, K_q, V_q, K_out, V_out, ws)
    return K_out, V_out


def routed_layer(layer: RoutedLayer, k: int, K_loc: torch.Tensor, V_loc: torch.Tensor,
                 rope_base: float, exclude_bits: Optional[torch.Tensor] = None):
    """Route -> gather -> sparse attention for one routed layer.
    Returns (top_ids, top_scores, O)."""
    ids, scores, _ = route_topk(layer.Q_r, layer.Kbar_r, layer.kr_inv_norm, layer.doc_chunk_off, k,
                                exclude_bits=exclude_bits, Kbar_r_hat=layer.Kbar_r_hat)
    cpd = int((layer.doc_chunk_off[1:] - layer.doc_chunk_off[:-1]).max().item())
    _, ctx_len, ctxK, ctxV = gather(ids, layer.doc_chunk_off, layer.Kbar, layer.Vbar, k * cpd)
    O = sparse_attend(layer.Q, K_loc, V_loc, ctxK, ctxV, ctx_len, k, rope_base)
    return ids, scores, O


def interleave_rounds(layers: List[RoutedLayer], k: int, rounds: int, rope_base: float,
                      doc_kv: Callable[[int, int], tuple], select=None):
    """Memory Interleaving over up to ``rounds`` rounds of all routed layers.

    ``doc_kv(layer, doc)`` returns the raw per-token (K, V) [len, h_kv, d] device tensors of a
    retrieved document at that layer. ``select(r, ids_r)``, if given, takes the place of the
    model's generative retrieval: it gets the round's selections (numpy int32 [B, k] per routed
    layer) and returns per query the doc ids to append, in order, or None to end the loop (the
    documents suffice); without it the last routed layer's selection is appended. Returns
    (ids[r][l] [B, k], scores[r][l] [B, k], O[r][l] [B, T, h_q, d], appended[b] = the
    documents appended per query, in order).
    """
    B = layers[0].Q.shape[0]
    n_docs = layers[0].doc_chunk_off.shape[0] - 1
    appended: List[List[int]] = [[] for _ in range(B)]
    all_ids, all_sc, all_O = [], [], []
    for r in range(rounds):
        ex = exclusion_bits(appended, n_docs, layers[0].Q.device) if r > 0 else None
        ids_r, sc_r, O_r = [], [], []
        for li, layer in enumerate(layers):
            if r == 0:
                K_loc, V_loc = layer.K_q, layer.V_q
            else:  # [appended documents' raw K/V, in the order appended ; query tokens]
                K_loc, V_loc = assemble_local(
                    [[doc_kv(li, doc) for doc in appended[b]] for b in range(B)],
                    layer.K_q, layer.V_q)
            ids, sc, O = routed_layer(layer, k, K_loc, V_loc, rope_base, ex)
            ids_r.append(ids)
            sc_r.append(sc)
            O_r.append(O)
        all_ids.append(ids_r)
        all_sc.append(sc_r)
        all_O.append(O_r)
        if select is None:
            last = ids_r[-1].cpu().tolist()
            chosen = [sorted(i for i in last[b] if i >= 0) for b in range(B)]
        else:
            chosen = select(r, [x.cpu().numpy() for x in ids_r])
        if chosen is None:
            break
        for b in range(B):
            for doc in chosen[b]:
                if doc >= 0 and doc not in appended[b]:
                    appended[b].append(int(doc))
    return all_ids, all_sc, all_O, appended


# ----------------------------------------------------------------------------- decode step
@dataclass
class DecodeLayer:
    """One routed layer of a decode step: its memory bank and the batch's per-layer inputs.

    Routing reads ``Kbar_r_hat`` (bf16 per-head unit rows, the tensor-core scan) when given,
    else ``Kbar_r`` with ``kr_inv_norm`` (the CUDA-core scan). ``Kbar``/``Vbar`` are either
    device tensors or pinned host tensors [n_chunks, h_kv, d]; several layers may share one
    host bank.

    The local context is either ``K_loc``/``V_loc`` (keys before RoPE, rotated by the attention
    on every call) or a ``cache`` (a ``LocalCache`` whose keys are stored rotated at their global
    positions pos0 + j, pos0 = k) into which the step first appends the query tokens' own
    ``K_new``/``V_new`` (before RoPE) and then attends: the decode loop of a model, where every
    key is rotated once, when it is appended."""
    Q_r: torch.Tensor                  # [B, T, h_qr, d]
    Q: torch.Tensor                    # [B, T, h_q, d]
    K_loc: Optional[torch.Tensor]      # [B, L_loc, h_kv, d] (before RoPE), or None with a cache
    V_loc: Optional[torch.Tensor]      # [B, L_loc, h_kv, d]
    Kbar: torch.Tensor                 # [n_chunks, h_kv, d], device or pinned host memory
    Vbar: torch.Tensor
    Kbar_r_hat: Optional[torch.Tensor] = None
    Kbar_r: Optional[torch.Tensor] = None
    kr_inv_norm: Optional[torch.Tensor] = None
    cache: Optional[LocalCache] = None  # rotated local cache (pos0 = k, the same RoPE base)
    K_new: Optional[torch.Tensor] = None  # [B, T, h_kv, d] appended to the cache by the step
    V_new: Optional[torch.Tensor] = None


class RoutedDecode:
    """One decode step over all routed layers: per layer route + top-k over the whole bank,
    context assembly from the (device or host) bank, sparse attention of the query tokens.

    Schedule (all on ``self.stream`` except the fetch): route(0), fetch(0); then for each
    layer l: route(l+1), fetch(l+1), attend(l). With a host bank the fetch of layer l+1 runs on
    ``self.copy_stream`` as soon as its routing has finished, beside the attention of layer l
    and the routing scan of layer l+2, so the host-link transfer hides behind HBM-bound work.
    ``fetch``:

    * ``"device"``: K̄/V̄ in device memory, msa_gather on the main stream.
    * ``"zerocopy"``: K̄/V̄ in pinned host memory; msa_gather reads the selected rows over the
      host link on the copy stream, ordered after the layer's routing and before its attention
      by CUDA events (no host round trip, so a step can be captured as one CUDA graph).
    * ``"memcpy"``: K̄/V̄ in pinned host memory; msa_fetch_begin/finish copy the selected chunk
      runs with cudaMemcpyAsync on the copy stream (one host wait per layer for the ids: not
      capturable).

    Per-layer outputs persist after a step: ``ids``/``scores`` [L, B, k], ``gather_idx``
    [L, B, max_ctx], ``ctx_len`` [L, B], ``O`` [L, B, T, h_q, d]. The gathered K/V rows and the
    workspaces rotate through ``nbuf`` buffer sets (2 suffice: the fetch of layer l+1 is ordered
    after the attention of layer l-1, which read the same set).
    """

    def __init__(self, layers: List[DecodeLayer], doc_chunk_off_host: np.ndarray, k: int,
                 rope_base: float, fetch: str = "auto", nbuf: int = 2, scale: float = 0.0,
                 device=None, stream=None, copy_stream=None, fetch_timeout_ms: int = 10_000):
        if not layers:
            raise ValueError("RoutedDecode needs at least one routed layer")
        self.layers = layers
        self.L = len(layers)
        self.k, self.rope_base, self.scale = int(k), float(rope_base), float(scale)
        self.dev = torch.device(device) if device is not None else layers[0].Q.device
        host = not layers[0].Kbar.is_cuda
        if any((not la.Kbar.is_cuda) != host or (not la.Vbar.is_cuda) != host for la in layers):
            raise ValueError("every layer's K̄/V̄ must be on the same side (device or host)")
        if fetch == "auto":
            fetch = "zerocopy" if host else "device"
        if fetch not in ("device", "zerocopy", "memcpy"):
            raise ValueError(f"unknown fetch mode {fetch!r}")
        if (fetch == "device") == host:
            raise ValueError(f"fetch={fetch!r} does not match a {'host' if host else 'device'} bank")
        if host and not all(la.Kbar.is_pinned() and la.Vbar.is_pinned() for la in layers):
            raise ValueError("a host bank must be in pinned memory")
        self.fetch = fetch
        self.timeout_ms = int(fetch_timeout_ms)
        self.coff_host = np.ascontiguousarray(doc_chunk_off_host, dtype=np.int64)
        self.coff = torch.from_numpy(self.coff_host).to(self.dev)
        self.n_docs = len(self.coff_host) - 1
        self.n_chunks = int(self.coff_host[-1])
        la0 = layers[0]
        B, T, h_q, d = la0.Q.shape
        h_qr = la0.Q_r.shape[2]
        self.cached = la0.cache is not None
        if any((la.cache is not None) != self.cached for la in layers):
            raise ValueError("either every layer has a local cache or none has")
        for la in layers:
            if la.cache is not None and (la.cache.pos0 != int(k) or la.K_new is None or
                                         la.V_new is None):
                raise ValueError("a cached layer needs pos0 = k and the step's K_new/V_new")
        h_kv = (la0.cache.K if self.cached else la0.K_loc).shape[2]
        L_loc = la0.cache.K.shape[1] if self.cached else la0.K_loc.shape[1]
        self.B, self.T, self.h_q, self.h_kv, self.d = B, T, h_q, h_kv, d
        cpd = int(np.max(np.diff(self.coff_host))) if self.n_docs else 0
        self.max_ctx = self.k * cpd
        self.stream = stream or torch.cuda.Stream(self.dev)
        self.copy_stream = copy_stream or torch.cuda.Stream(self.dev)
        bank_dtype = 1  # the routing workspace is sized for the largest (tensor-core) plan
        ws_r = max(msa_route_topk_workspace(B, T, h_qr, h_kv, d, bank_dtype, self.n_docs,
                                            self.n_chunks, self.k),
                   msa_route_topk_workspace(B, T, h_qr, h_kv, d, 0, self.n_docs, self.n_chunks,
                                            self.k))
        ws_a = (msa_decode_step_workspace(B, T, h_q, h_kv, d, self.max_ctx, L_loc) if self.cached
                else msa_sparse_attend_workspace(B, T, h_q, h_kv, d, self.max_ctx, L_loc))
        dt = la0.Q.dtype
        dev = self.dev
        self.ids = torch.empty((self.L, B, self.k), dtype=torch.int32, device=dev)
        self.scores = torch.empty((self.L, B, self.k), dtype=torch.float32, device=dev)
        self.gather_idx = torch.empty((self.L, B, self.max_ctx), dtype=torch.int32, device=dev)
        self.ctx_len = torch.empty((self.L, B), dtype=torch.int32, device=dev)
        self.O = torch.empty((self.L, B, T, h_q, d), dtype=dt, device=dev)
        self.nbuf = max(1, min(int(nbuf), self.L))
        if self.fetch != "device" and self.L > 1:
            self.nbuf = max(self.nbuf, 2)
        self.buf = []
        for _ in range(self.nbuf):
            self.buf.append(dict(
                ws_r=torch.empty(max(ws_r, 256), dtype=torch.uint8, device=dev),
                ws_a=torch.empty(max(ws_a, 256), dtype=torch.uint8, device=dev),
                ws_g=torch.zeros(256, dtype=torch.uint8, device=dev),
                cK=torch.empty((B, self.max_ctx, h_kv, d), dtype=dt, device=dev),
                cV=torch.empty((B, self.max_ctx, h_kv, d), dtype=dt, device=dev)))
        if self.fetch == "zerocopy":
            self.ev_route = [torch.cuda.Event() for _ in range(self.nbuf)]
            self.ev_fetch = [torch.cuda.Event() for _ in range(self.nbuf)]
        if self.fetch == "memcpy":
            self.fetchers = [Fetcher(B, self.k) for _ in range(2)]
        self.route_events = None  # optional [(start, end)] * L CUDA events around each routing

    # ----------------------------------------------------------------- per-layer pieces
    def _route(self, l: int):
        la, bf = self.layers[l], self.buf[l % self.nbuf]
        if self.route_events is not None:
            self.route_events[l][0].record(self.stream)
        msa_route_topk(la.Q_r, la.Kbar_r, la.kr_inv_norm, self.coff, self.k, None, self.ids[l],
                       self.scores[l], None, bf["ws_r"], self.stream, la.Kbar_r_hat)
        if self.route_events is not None:
            self.route_events[l][1].record(self.stream)

    def _fetch_begin(self, l: int):
        la, bf, j = self.layers[l], self.buf[l % self.nbuf], l % self.nbuf
        if self.fetch == "device":
            msa_gather(self.ids[l], self.coff, la.Kbar, la.Vbar, self.max_ctx,
                       self.gather_idx[l], self.ctx_len[l], bf["cK"], bf["cV"], bf["ws_g"],
                       self.stream)
        elif self.fetch == "zerocopy":
            self.ev_route[j].record(self.stream)
            self.copy_stream.wait_event(self.ev_route[j])
            msa_gather(self.ids[l], self.coff, la.Kbar, la.Vbar, self.max_ctx,
                       self.gather_idx[l], self.ctx_len[l], bf["cK"], bf["cV"], bf["ws_g"],
                       self.copy_stream)
            self.ev_fetch[j].record(self.copy_stream)
        else:
            self.fetchers[l % 2].begin(self.ids[l], self.coff, self.max_ctx, self.gather_idx[l],
                                       self.ctx_len[l], bf["ws_g"], self.stream)

    def _fetch_finish(self, l: int):
        la, bf, j = self.layers[l], self.buf[l % self.nbuf], l % self.nbuf
        if self.fetch == "zerocopy":
            self.stream.wait_event(self.ev_fetch[j])
        elif self.fetch == "memcpy":
            self.fetchers[l % 2].finish(self.coff_host, la.Kbar, la.Vbar, self.max_ctx, bf["cK"],
                                        bf["cV"], self.stream, self.copy_stream, self.timeout_ms)

    def _attend(self, l: int):
        la, bf = self.layers[l], self.buf[l % self.nbuf]
        if self.cached:  # append the step's tokens (rotated), then attend over the cache
            c = la.cache
            msa_decode_step(la.Q, la.K_new, la.V_new, c.K, c.V, c.length, bf["cK"], bf["cV"],
                            self.ctx_len[l], self.k, self.rope_base, self.scale, self.O[l],
                            bf["ws_a"], self.stream)
        else:
            msa_sparse_attend(la.Q, la.K_loc, la.V_loc, bf["cK"], bf["cV"], self.ctx_len[l],
                              self.k, self.rope_base, self.scale, self.O[l], bf["ws_a"],
                              self.stream)

    # ----------------------------------------------------------------- the step
    def step(self, local_ready: "torch.cuda.Event" = None):
        """Enqueue one decode step of every routed layer on ``self.stream``.

        ``local_ready``: optional CUDA event that the stream waits on before the first
        attention, for attention inputs (the local K/V, a cache's new token) that another stream
        writes while the first layers route; routing reads none of them."""
        self._route(0)
        self._fetch_begin(0)
        for l in range(self.L):
            if l + 1 < self.L:
                self._route(l + 1)
                self._fetch_begin(l + 1)
            self._fetch_finish(l)
            if l == 0 and local_ready is not None:
                self.stream.wait_event(local_ready)
            self._attend(l)

    @property
    def capturable(self) -> bool:
        return self.fetch != "memcpy"

    def capture(self) -> "torch.cuda.CUDAGraph":
        """Capture one step as a CUDA graph on ``self.stream`` (run ``step`` once before, so
        that every lazily created library state exists). Replay with ``replay``."""
        if not self.capturable:
            raise RuntimeError("fetch='memcpy' waits on the host per layer: not capturable")
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self.step()
        self.graph = g
        return g

    def replay(self):
        with torch.cuda.stream(self.stream):
            self.graph.replay()

    def kernels_per_step(self) -> int:
        """Launches of libmsa kernels per step (memsets and copies excluded): per layer the
        routing call (tensor-core scan: query fold + scan with fused top-k; CUDA-core scan: one
        kernel per pass of up to 16 query rows), the gather (none with fetch='memcpy': the
        gather indices kernel only), the decode attention (with a cache, the token's append
        is fused into it) and the merge of its splits."""
        n = 0
        for la in self.layers:
            tc = la.Kbar_r_hat is not None and la.Q_r.dtype == torch.bfloat16
            route = 2 if tc else -(-self.B * self.T // 16)
            n += route + 1 + 2
        return n
