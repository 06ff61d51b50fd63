"""Routed-layer loop and Memory Interleaving rounds over the libmsa entry points.

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

import torch

from . import gather, msa_assemble_local, route_topk, sparse_attend


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
