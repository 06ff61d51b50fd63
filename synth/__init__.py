"""Seeded synthetic workloads for the MSA routed-memory path.

This module builds inputs only. It holds none of the method's arithmetic, so both the CPU
oracle (``oracle/``) and the CUDA library (``long_context_doc_b200``) may take their inputs
from it. The generator is defined at the top of ``synth.c``: SplitMix64 words, a
sum-of-twelve-uniforms normal that is exact in fp32, bf16 by round-to-nearest-even, and
multiply-shift uniform integers. ``synth_dev.cu`` is its bit-identical device twin, used to
create multi-gigabyte banks in place.

The workloads follow the five configurations of the routed-memory hot path (tiny fp32 layer,
1M-token bank prefill, 10M-token bank decode, 100M-token bank decode over 18 routed layers,
batched interleaved routing). Planted documents follow the stated recipe
"0.6 * mean-query-direction + 0.4 * N(0,1)": the unit mean query direction of each router
head is scaled by sqrt(d) so that its norm matches an N(0,1) row.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SO_DEV = os.path.join(_HERE, "libsynth_dev.so")

# tensor ids used in generator tags
K, V, KR, Q, QR, KLOC, VLOC, KBAR, VBAR, KRBAR, APPK, APPV = range(1, 13)
PLANT_DOCS, PLANT_EPS, DOC_LEN, EXTRA = 20, 21, 22, 23
GEN_Q, GEN_K, GEN_V = 30, 31, 32  # a generated token's query and K/V


def tag(tid: int, layer: int = 0, sub: int = 0) -> int:
    """64-bit generator tag of a tensor: (tensor id, routed layer, sub-stream)."""
    return (int(tid) << 48) | ((int(layer) & 0xFFFF) << 32) | (int(sub) & 0xFFFFFFFF)


def _stale(so: str, srcs) -> bool:
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    return any(os.path.getmtime(s) > t for s in srcs)


def build(device: bool = True, force: bool = False) -> None:
    """Compile libsynth.so (gcc) and, if ``device``, libsynth_dev.so (nvcc, sm_100a)."""
    src = os.path.join(_HERE, "synth.c")
    if force or _stale(_SO, [src]):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", _SO, src])
    if device:
        dsrc = os.path.join(_HERE, "synth_dev.cu")
        if force or _stale(_SO_DEV, [dsrc]):
            subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                                   "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                                   "-o", _SO_DEV, dsrc])


_lib = None
_lib_dev = None


def lib():
    global _lib
    if _lib is None:
        build(device=False)
        L = ctypes.CDLL(_SO)
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        L.syn_key.restype = u64
        L.syn_key.argtypes = [u64, u64]
        L.syn_word.restype = u64
        L.syn_word.argtypes = [u64, u64]
        L.syn_fill_normal.restype = None
        L.syn_fill_normal.argtypes = [vp, i64, ctypes.c_int, u64, u64, u64, ctypes.c_float]
        L.syn_fill_normal_f64.restype = None
        L.syn_fill_normal_f64.argtypes = [vp, i64, u64, u64, u64]
        L.syn_fill_uniform.restype = None
        L.syn_fill_uniform.argtypes = [vp, i64, u64, u64, u64]
        L.syn_distinct.restype = ctypes.c_int
        L.syn_distinct.argtypes = [vp, i64, u64, u64, u64]
        L.syn_to_bf16.restype = None
        L.syn_to_bf16.argtypes = [vp, vp, i64]
        _lib = L
    return _lib


def lib_dev():
    global _lib_dev
    if _lib_dev is None:
        build(device=True)
        L = ctypes.CDLL(_SO_DEV)
        L.synth_dev_fill_normal.restype = ctypes.c_int
        L.synth_dev_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                            ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                            ctypes.c_float, ctypes.c_void_p]
        _lib_dev = L
    return _lib_dev


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------------------------------
# primitive draws
# ----------------------------------------------------------------------------------------
def normal(seed: int, tg: int, shape, dtype: str = "fp32", first: int = 0,
           scale: float = 1.0) -> np.ndarray:
    """Normals as float32 (``dtype='fp32'``) or bf16 bit patterns in uint16 (``'bf16'``)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32 if dtype == "fp32" else np.uint16)
    lib().syn_fill_normal(_ptr(out), n, 0 if dtype == "fp32" else 1, seed, tg, first, scale)
    return out.reshape(shape)


def normal_f64(seed: int, tg: int, shape, first: int = 0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float64)
    lib().syn_fill_normal_f64(_ptr(out), n, seed, tg, first)
    return out.reshape(shape)


def uniform(seed: int, tg: int, n: int, hi: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    lib().syn_fill_uniform(_ptr(out), n, seed, tg, hi)
    return out


def distinct(seed: int, tg: int, k: int, hi: int) -> np.ndarray:
    out = np.empty(k, dtype=np.int64)
    if lib().syn_distinct(_ptr(out), k, seed, tg, hi) != 0:
        raise ValueError("k > hi")
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().syn_to_bf16(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_to_f32(x) if dtype == "bf16" else np.asarray(x, dtype=np.float32)


def store(x32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16(x32) if dtype == "bf16" else np.ascontiguousarray(x32, np.float32)


# ----------------------------------------------------------------------------------------
# workload configurations
# ----------------------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    dtype: str                 # "fp32" | "bf16"
    n_docs: int
    doc_len: int               # tokens per document (all equal unless ragged=True)
    chunk: int
    h_q: int
    h_kv: int
    d: int
    h_qr: int
    B: int
    T: int
    k: int
    L_loc: int                 # local K/V rows per query (query tokens are the last T)
    n_planted: int             # planted docs (per query for pre-pooled banks)
    rope_base: float = 1e6
    prepooled: bool = False    # bank given as K̄/V̄/K̄_r directly (no encode step)
    layers: int = 1
    rounds: int = 1
    ragged: bool = False       # random doc lengths in [1, 2*doc_len)
    seed: int = 0

    @property
    def cpd(self) -> int:
        return -(-self.doc_len // self.chunk)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five configurations of the routed-memory path.
C1 = Workload("tiny_fp32_32k", "fp32", n_docs=64, doc_len=512, chunk=64, h_q=4, h_kv=2, d=64,
              h_qr=2, B=1, T=16, k=4, L_loc=16, n_planted=4)
C2 = Workload("qwen3_4b_1m_prefill", "bf16", n_docs=1024, doc_len=1024, chunk=64, h_q=32,
              h_kv=8, d=128, h_qr=8, B=1, T=128, k=16, L_loc=128, n_planted=16)
C3 = Workload("bank10m_decode_b8", "bf16", n_docs=20000, doc_len=500, chunk=64, h_q=32,
              h_kv=8, d=128, h_qr=8, B=8, T=1, k=16, L_loc=2048, n_planted=1, prepooled=True)
C4 = Workload("bank100m_decode_b4_18l", "bf16", n_docs=200000, doc_len=500, chunk=64, h_q=32,
              h_kv=8, d=128, h_qr=8, B=4, T=1, k=16, L_loc=2048, n_planted=1,
              prepooled=True, layers=18)
C5 = Workload("bank10m_interleave_b32_t256", "bf16", n_docs=20000, doc_len=500, chunk=64,
              h_q=32, h_kv=8, d=128, h_qr=8, B=32, T=256, k=8, L_loc=256, n_planted=1,
              prepooled=True, layers=18, rounds=3)
CONFIGS = {w.name: w for w in (C1, C2, C3, C4, C5)}


def doc_tok_offsets(w: Workload) -> np.ndarray:
    """[n_docs+1] token offsets of the documents in the flat token stream."""
    if w.ragged:
        lens = 1 + uniform(w.seed, tag(DOC_LEN), w.n_docs, 2 * w.doc_len - 1)
    else:
        lens = np.full(w.n_docs, w.doc_len, dtype=np.int64)
    off = np.zeros(w.n_docs + 1, dtype=np.int64)
    np.cumsum(lens, out=off[1:])
    return off


def chunk_offsets_from_lengths(lens: np.ndarray, chunk: int) -> np.ndarray:
    """[n_docs+1] chunk offsets for a bank whose documents are padded to whole chunks."""
    nch = -(-np.asarray(lens, dtype=np.int64) // chunk)
    off = np.zeros(len(nch) + 1, dtype=np.int64)
    np.cumsum(nch, out=off[1:])
    return off


def planted_direction(qr32: np.ndarray, h_kv: int) -> np.ndarray:
    """Unit mean query direction per KV head, scaled by sqrt(d). qr32: [T, h_qr, d] floats.

    Returns [h_kv, d] float64. Router heads map to KV head floor(h / (h_qr / h_kv)).
    """
    T, h_qr, d = qr32.shape
    m = h_qr // h_kv
    mean = qr32.astype(np.float64).reshape(T, h_kv, m, d).mean(axis=(0, 2))
    nrm = np.linalg.norm(mean, axis=-1, keepdims=True)
    nrm[nrm == 0] = 1.0
    return mean / nrm * math.sqrt(d)


def planted_rows(seed: int, layer: int, sub: int, u: np.ndarray, n_rows: int,
                 dtype: str) -> np.ndarray:
    """[n_rows, h_kv, d] rows 0.6 * u + 0.4 * eps (u already scaled), stored in dtype."""
    h_kv, d = u.shape
    eps = normal_f64(seed, tag(PLANT_EPS, layer, sub), (n_rows, h_kv, d))
    rows = 0.6 * u[None] + 0.4 * eps
    return store(rows.astype(np.float32), dtype)


def make_token_workload(w: Workload, layer: int = 0) -> dict:
    """Per-token inputs of the offline encode plus one routed layer's query (C1/C2 style).

    K, V, K_r: [N_tok, h_kv, d]; Q: [B, T, h_q, d]; Q_r: [B, T, h_qr, d];
    K_loc, V_loc: [B, L_loc, h_kv, d]. Planted docs get per-token K_r rows before RoPE.
    """
    s, dt = w.seed, w.dtype
    off = doc_tok_offsets(w)
    n_tok = int(off[-1])
    out = dict(doc_tok_off=off, n_tok=n_tok)
    out["K"] = normal(s, tag(K, layer), (n_tok, w.h_kv, w.d), dt)
    out["V"] = normal(s, tag(V, layer), (n_tok, w.h_kv, w.d), dt)
    Kr = normal(s, tag(KR, layer), (n_tok, w.h_kv, w.d), dt)
    out["Q"] = normal(s, tag(Q, layer), (w.B, w.T, w.h_q, w.d), dt)
    out["Q_r"] = normal(s, tag(QR, layer), (w.B, w.T, w.h_qr, w.d), dt)
    out["K_loc"] = normal(s, tag(KLOC, layer), (w.B, w.L_loc, w.h_kv, w.d), dt)
    out["V_loc"] = normal(s, tag(VLOC, layer), (w.B, w.L_loc, w.h_kv, w.d), dt)
    planted = np.sort(distinct(s, tag(PLANT_DOCS, layer), min(w.n_planted, w.n_docs),
                               w.n_docs)) if w.n_planted else np.zeros(0, np.int64)
    if len(planted):
        u = planted_direction(as_f32(out["Q_r"][0], dt), w.h_kv)
        for j, p in enumerate(planted):
            a, b = int(off[p]), int(off[p + 1])
            Kr[a:b] = planted_rows(s, layer, j, u, b - a, dt)
    out["K_r"] = Kr
    out["planted"] = planted
    return out


def make_bank_workload(w: Workload, layer: int = 0, with_bank: bool = True) -> dict:
    """Pre-pooled bank (K̄_r, K̄, V̄ ~ N(0,1)) plus one layer's decode/prefill queries.

    Every document has ceil(doc_len / chunk) chunks ("docs padded to whole chunks"). Each
    query b gets ``n_planted`` planted docs whose every K̄_r chunk row is
    0.6 * sqrt(d) * unit(mean Q_r[b]) + 0.4 * N(0,1).
    """
    s, dt = w.seed, w.dtype
    if w.ragged:
        lens = 1 + uniform(s, tag(DOC_LEN), w.n_docs, 2 * w.doc_len - 1)
    else:
        lens = np.full(w.n_docs, w.doc_len, dtype=np.int64)
    coff = chunk_offsets_from_lengths(lens, w.chunk)
    n_chunks = int(coff[-1])
    out = dict(doc_chunk_off=coff, n_chunks=n_chunks, doc_len=lens)
    out["Q"] = normal(s, tag(Q, layer), (w.B, w.T, w.h_q, w.d), dt)
    out["Q_r"] = normal(s, tag(QR, layer), (w.B, w.T, w.h_qr, w.d), dt)
    out["K_loc"] = normal(s, tag(KLOC, layer), (w.B, w.L_loc, w.h_kv, w.d), dt)
    out["V_loc"] = normal(s, tag(VLOC, layer), (w.B, w.L_loc, w.h_kv, w.d), dt)
    out["planted"] = plant_docs(w, layer)
    if with_bank:
        Krb = normal(s, tag(KRBAR, layer), (n_chunks, w.h_kv, w.d), dt)
        for (b, j), p, rows in planted_bank_rows(w, layer, out["Q_r"], coff):
            Krb[coff[p]:coff[p + 1]] = rows
        out["Kbar_r"] = Krb
        out["Kbar"] = normal(s, tag(KBAR, layer), (n_chunks, w.h_kv, w.d), dt)
        out["Vbar"] = normal(s, tag(VBAR, layer), (n_chunks, w.h_kv, w.d), dt)
    return out


def plant_docs(w: Workload, layer: int) -> np.ndarray:
    """[B, n_planted] distinct planted doc ids of one layer (distinct across the batch)."""
    n = w.B * w.n_planted
    if n == 0:
        return np.zeros((w.B, 0), np.int64)
    return distinct(w.seed, tag(PLANT_DOCS, layer), n, w.n_docs).reshape(w.B, w.n_planted)


def planted_bank_rows(w: Workload, layer: int, Q_r: np.ndarray, coff: np.ndarray):
    """Yield ((b, j), doc, rows) for every planted doc of a pre-pooled bank."""
    planted = plant_docs(w, layer)
    for b in range(w.B):
        u = planted_direction(as_f32(Q_r[b], w.dtype), w.h_kv)
        for j in range(w.n_planted):
            p = int(planted[b, j])
            n = int(coff[p + 1] - coff[p])
            yield (b, j), p, planted_rows(w.seed, layer, b * max(w.n_planted, 1) + j, u, n,
                                          w.dtype)


def appended_doc_kv(w: Workload, layer: int, doc: int, dtype: str | None = None):
    """Raw per-token K, V ([doc_len, h_kv, d]) of a retrieved document, appended to the
    query's local context by an interleave round."""
    dt = dtype or w.dtype
    n = w.doc_len * w.h_kv * w.d
    k = normal(w.seed, tag(APPK, layer), (w.doc_len, w.h_kv, w.d), dt, first=doc * n)
    v = normal(w.seed, tag(APPV, layer), (w.doc_len, w.h_kv, w.d), dt, first=doc * n)
    return k, v


# ----------------------------------------------------------------------------------------
# device-side construction (bit-identical to the host arrays above)
# ----------------------------------------------------------------------------------------
def dev_normal(t, seed: int, tg: int, first: int = 0, scale: float = 1.0, stream=None):
    """Fill the contiguous float32/bfloat16 device tensor ``t`` with normal(seed, tg, first+i)."""
    import torch
    assert t.is_contiguous() and t.dtype in (torch.float32, torch.bfloat16)
    st = (stream or torch.cuda.current_stream()).cuda_stream
    rc = lib_dev().synth_dev_fill_normal(t.data_ptr(), t.numel(),
                                         0 if t.dtype == torch.float32 else 1, seed, tg, first,
                                         scale, st)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_normal failed with cudaError {rc}")
    return t


def _tdtype(dtype: str):
    import torch
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_torch(x: np.ndarray, dev):
    import torch
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(x).to(dev)


def dev_token_workload(w: Workload, dev, layer: int = 0) -> dict:
    """Device twin of make_token_workload: the same values, generated in place on the GPU
    (queries and planted rows are small and built on the host)."""
    import torch
    s, dt = w.seed, w.dtype
    td = _tdtype(dt)
    off = doc_tok_offsets(w)
    n_tok = int(off[-1])
    out = dict(doc_tok_off=off, n_tok=n_tok)
    for name, tid in (("K", K), ("V", V), ("K_r", KR)):
        out[name] = dev_normal(torch.empty((n_tok, w.h_kv, w.d), dtype=td, device=dev), s,
                               tag(tid, layer))
    host = dict(Q_r=normal(s, tag(QR, layer), (w.B, w.T, w.h_qr, w.d), dt))
    out["Q_r"] = to_torch(host["Q_r"], dev)
    out["Q"] = dev_normal(torch.empty((w.B, w.T, w.h_q, w.d), dtype=td, device=dev), s,
                          tag(Q, layer))
    out["K_loc"] = dev_normal(torch.empty((w.B, w.L_loc, w.h_kv, w.d), dtype=td, device=dev), s,
                              tag(KLOC, layer))
    out["V_loc"] = dev_normal(torch.empty((w.B, w.L_loc, w.h_kv, w.d), dtype=td, device=dev), s,
                              tag(VLOC, layer))
    planted = np.sort(distinct(s, tag(PLANT_DOCS, layer), min(w.n_planted, w.n_docs),
                               w.n_docs)) if w.n_planted else np.zeros(0, np.int64)
    if len(planted):
        u = planted_direction(as_f32(host["Q_r"][0], dt), w.h_kv)
        for j, p in enumerate(planted):
            a, b = int(off[p]), int(off[p + 1])
            out["K_r"][a:b] = to_torch(planted_rows(s, layer, j, u, b - a, dt), dev)
    out["planted"] = planted
    return out


def host_token_rows(w: Workload, name: str, t0: int, t1: int, layer: int = 0) -> np.ndarray:
    """Host copy of token rows [t0, t1) of K / V / K_r (planted rows included)."""
    tid = {"K": K, "V": V, "K_r": KR}[name]
    row = w.h_kv * w.d
    x = normal(w.seed, tag(tid, layer), (t1 - t0, w.h_kv, w.d), w.dtype, first=t0 * row)
    if name == "K_r" and w.n_planted:
        off = doc_tok_offsets(w)
        planted = np.sort(distinct(w.seed, tag(PLANT_DOCS, layer), min(w.n_planted, w.n_docs),
                                   w.n_docs))
        qr = normal(w.seed, tag(QR, layer), (w.B, w.T, w.h_qr, w.d), w.dtype)
        u = planted_direction(as_f32(qr[0], w.dtype), w.h_kv)
        for j, p in enumerate(planted):
            a, b = int(off[p]), int(off[p + 1])
            lo, hi = max(a, t0), min(b, t1)
            if lo < hi:
                rows = planted_rows(w.seed, layer, j, u, b - a, w.dtype)
                x[lo - t0:hi - t0] = rows[lo - a:hi - a]
    return x


def dev_bank_workload(w: Workload, dev, layer: int = 0, with_kv: bool = True) -> dict:
    """Device twin of make_bank_workload (pre-pooled bank generated in place)."""
    import torch
    s, dt = w.seed, w.dtype
    td = _tdtype(dt)
    lens = (1 + uniform(s, tag(DOC_LEN), w.n_docs, 2 * w.doc_len - 1)) if w.ragged else \
        np.full(w.n_docs, w.doc_len, dtype=np.int64)
    coff = chunk_offsets_from_lengths(lens, w.chunk)
    n_chunks = int(coff[-1])
    out = dict(doc_chunk_off=coff, n_chunks=n_chunks, doc_len=lens)
    qr = normal(s, tag(QR, layer), (w.B, w.T, w.h_qr, w.d), dt)
    out["Q_r_host"] = qr
    out["Q_r"] = to_torch(qr, dev)
    out["Q"] = dev_normal(torch.empty((w.B, w.T, w.h_q, w.d), dtype=td, device=dev), s,
                          tag(Q, layer))
    out["K_loc"] = dev_normal(torch.empty((w.B, w.L_loc, w.h_kv, w.d), dtype=td, device=dev), s,
                              tag(KLOC, layer))
    out["V_loc"] = dev_normal(torch.empty((w.B, w.L_loc, w.h_kv, w.d), dtype=td, device=dev), s,
                              tag(VLOC, layer))
    Krb = dev_normal(torch.empty((n_chunks, w.h_kv, w.d), dtype=td, device=dev), s,
                     tag(KRBAR, layer))
    for _, p, rows in planted_bank_rows(w, layer, qr, coff):
        Krb[int(coff[p]):int(coff[p + 1])] = to_torch(rows, dev)
    out["Kbar_r"] = Krb
    out["planted"] = plant_docs(w, layer)
    if with_kv:
        out["Kbar"] = dev_normal(torch.empty((n_chunks, w.h_kv, w.d), dtype=td, device=dev), s,
                                 tag(KBAR, layer))
        out["Vbar"] = dev_normal(torch.empty((n_chunks, w.h_kv, w.d), dtype=td, device=dev), s,
                                 tag(VBAR, layer))
    return out


def host_bank_rows(w: Workload, name: str, c0: int, c1: int, layer: int = 0,
                   coff: np.ndarray | None = None, Q_r: np.ndarray | None = None) -> np.ndarray:
    """Host copy of bank rows [c0, c1) of K̄_r / K̄ / V̄ (planted K̄_r rows included)."""
    tid = {"Kbar_r": KRBAR, "Kbar": KBAR, "Vbar": VBAR}[name]
    row = w.h_kv * w.d
    x = normal(w.seed, tag(tid, layer), (c1 - c0, w.h_kv, w.d), w.dtype, first=c0 * row)
    if name == "Kbar_r" and w.n_planted:
        if Q_r is None:
            Q_r = normal(w.seed, tag(QR, layer), (w.B, w.T, w.h_qr, w.d), w.dtype)
        for _, p, rows in planted_bank_rows(w, layer, Q_r, coff):
            a, b = int(coff[p]), int(coff[p + 1])
            lo, hi = max(a, c0), min(b, c1)
            if lo < hi:
                x[lo - c0:hi - c0] = rows[lo - a:hi - a]
    return x
