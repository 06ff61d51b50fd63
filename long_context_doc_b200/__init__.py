"""Python binding of libmsa, the B200 (sm_100a) routed-memory hot path of Memory Sparse
Attention (MSA).

The ``msa_*`` functions mirror the C ABI of ``include/msa.h`` one to one: they marshal
torch tensors (device memory) into pointers and sizes and raise :class:`MSAError` when the
library returns a non-zero status. Every step of the path runs in the library's CUDA
kernels; torch only provides device memory and streams. There is no fallback: if
``libmsa.so`` is missing or fails to load, importing this package raises.

The lower-case helpers (``encode_pool``, ``route_topk``, ``gather``, ``sparse_attend``,
``Fetcher``) allocate outputs and workspaces with torch and call the ``msa_*`` functions.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

from . import build as _build

MSA_FP32, MSA_BF16 = 0, 1
STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_WORKSPACE",
          4: "MSA_ERR_CUDA", 5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_DEVICE"}
LIB_PATH = _build.LIB

# every symbol include/msa.h declares
SYMBOLS = ("msa_status_string", "msa_last_error", "msa_version", "msa_set_device_wait_limit",
           "msa_count_chunks",
           "msa_encode_pool", "msa_encode_pool_status", "msa_kr_inv_norm", "msa_kr_normalize", "msa_route_topk_workspace",
           "msa_route_topk", "msa_route_topk_noalloc", "msa_route_topk_noalloc_status",
           "msa_workspace_status", "msa_gather", "msa_fetch_create", "msa_fetch_destroy",
           "msa_fetch_begin", "msa_fetch_finish", "msa_sparse_attend_workspace",
           "msa_sparse_attend", "msa_assemble_local", "msa_kv_append",
           "msa_decode_step_workspace", "msa_decode_step", "msa_encode_hidden_workspace",
           "msa_encode_hidden", "msa_sparse_attend_backward_workspace",
           "msa_sparse_attend_backward", "msa_scatter_bank_grad", "msa_aux_routing_loss_workspace",
           "msa_aux_routing_loss")


class MSAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.message = message


def _load():
    if not os.path.exists(LIB_PATH) or _build.stale():
        _build.build()
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
    L.msa_status_string.restype = ctypes.c_char_p
    L.msa_status_string.argtypes = [ctypes.c_int]
    L.msa_last_error.restype = ctypes.c_char_p
    L.msa_last_error.argtypes = []
    L.msa_version.restype = ctypes.c_int
    L.msa_set_device_wait_limit.restype = i64
    L.msa_set_device_wait_limit.argtypes = [i64]
    L.msa_count_chunks.restype = i64
    L.msa_count_chunks.argtypes = [vp, i64, i32]
    L.msa_encode_pool_status.restype = ctypes.c_int
    L.msa_encode_pool_status.argtypes = [vp, vp]
    L.msa_encode_pool.restype = ctypes.c_int
    L.msa_encode_pool.argtypes = [vp, vp, vp, i64, vp, vp, i64, i32, i32, i32, i32, f32, vp, vp,
                                  vp, vp, vp, i64, vp]
    L.msa_kr_inv_norm.restype = ctypes.c_int
    L.msa_kr_inv_norm.argtypes = [vp, i64, i32, i32, i32, vp, vp]
    L.msa_kr_normalize.restype = ctypes.c_int
    L.msa_kr_normalize.argtypes = [vp, i64, i32, i32, i32, vp, vp]
    L.msa_route_topk_workspace.restype = sz
    L.msa_route_topk_workspace.argtypes = [i32, i32, i32, i32, i32, i32, i64, i64, i32]
    L.msa_route_topk.restype = ctypes.c_int
    L.msa_route_topk.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, i64, i64, i32, i32, i32, i32,
                                 vp, vp, vp, vp, vp, sz, vp]
    L.msa_route_topk_noalloc.restype = ctypes.c_int
    L.msa_route_topk_noalloc.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, i64, i64, i32, i32, i32,
                                         i32, vp, vp, vp, vp, vp]
    L.msa_route_topk_noalloc_status.restype = ctypes.c_int
    L.msa_route_topk_noalloc_status.argtypes = [vp, vp]
    L.msa_workspace_status.restype = ctypes.c_int
    L.msa_workspace_status.argtypes = [vp, vp, vp]
    L.msa_gather.restype = ctypes.c_int
    L.msa_gather.argtypes = [vp, i32, i32, vp, i64, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp,
                             vp, sz, vp]
    L.msa_fetch_create.restype = ctypes.c_int
    L.msa_fetch_create.argtypes = [i32, i32, vp]
    L.msa_fetch_destroy.restype = None
    L.msa_fetch_destroy.argtypes = [vp]
    L.msa_fetch_begin.restype = ctypes.c_int
    L.msa_fetch_begin.argtypes = [vp, vp, i32, i32, vp, i64, i32, vp, vp, vp, sz, vp]
    L.msa_fetch_finish.restype = ctypes.c_int
    L.msa_fetch_finish.argtypes = [vp, vp, i64, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, i32]
    L.msa_sparse_attend_workspace.restype = sz
    L.msa_sparse_attend_workspace.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    L.msa_sparse_attend.restype = ctypes.c_int
    L.msa_sparse_attend.argtypes = [vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32,
                                    i32, f32, f32, vp, vp, sz, vp]
    L.msa_assemble_local.restype = ctypes.c_int
    L.msa_assemble_local.argtypes = [i32, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i64, vp, vp,
                                     vp, sz, vp]
    L.msa_kv_append.restype = ctypes.c_int
    L.msa_kv_append.argtypes = [vp, vp, i32, i32, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, sz,
                                vp]
    L.msa_decode_step_workspace.restype = sz
    L.msa_decode_step_workspace.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    L.msa_encode_hidden_workspace.restype = sz
    L.msa_encode_hidden_workspace.argtypes = [i64]
    L.msa_encode_hidden.restype = ctypes.c_int
    L.msa_encode_hidden.argtypes = [vp, i64, i32, vp, vp, vp, vp, i64, i32, i32, i32, i32, f32, vp,
                                    vp, vp, vp, i64, vp, sz, vp]
    L.msa_sparse_attend_backward_workspace.restype = sz
    L.msa_sparse_attend_backward_workspace.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    L.msa_sparse_attend_backward.restype = ctypes.c_int
    L.msa_sparse_attend_backward.argtypes = [vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, i32, i32,
                                             i32, i32, i32, f32, f32, vp, vp, vp, vp, vp, vp, vp,
                                             sz, vp]
    L.msa_scatter_bank_grad.restype = ctypes.c_int
    L.msa_scatter_bank_grad.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, i64, vp, sz, vp]
    L.msa_aux_routing_loss_workspace.restype = sz
    L.msa_aux_routing_loss_workspace.argtypes = [i32, i64]
    L.msa_aux_routing_loss.restype = ctypes.c_int
    L.msa_aux_routing_loss.argtypes = [vp, i32, i32, i32, vp, i64, i32, i32, i32, vp, f32, vp, vp,
                                       vp, vp, sz, vp]
    L.msa_decode_step.restype = ctypes.c_int
    L.msa_decode_step.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp, i32, i32,
                                  i32, i32, i32, f32, f32, vp, vp, sz, vp]
    return L


lib = _load()


def _check(status: int):
    if status != 0:
        raise MSAError(status, lib.msa_last_error().decode(errors="replace"))


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MSA_FP32
    if t.dtype == torch.bfloat16:
        return MSA_BF16
    raise TypeError(f"libmsa tensors are float32 or bfloat16, got {t.dtype}")


# ----------------------------------------------------------------------------- raw ABI
def msa_count_chunks(doc_tok_off_host: np.ndarray, chunk: int) -> int:
    off = np.ascontiguousarray(doc_tok_off_host, dtype=np.int64)
    return int(lib.msa_count_chunks(off.ctypes.data, len(off) - 1, chunk))


def msa_encode_pool(K, V, K_r, doc_tok_off_host, doc_tok_off, chunk, rope_base, Kbar, Vbar,
                    Kbar_r, kr_inv_norm, doc_chunk_off, stream=None):
    off = np.ascontiguousarray(doc_tok_off_host, dtype=np.int64)
    _check(lib.msa_encode_pool(_p(K), _p(V), _p(K_r), K.shape[0], off.ctypes.data,
                               _p(doc_tok_off), len(off) - 1, chunk, K.shape[1], K.shape[2],
                               dtype_code(K), rope_base, _p(Kbar), _p(Vbar), _p(Kbar_r),
                               _p(kr_inv_norm), _p(doc_chunk_off), Kbar.shape[0], _s(stream)))


def msa_encode_hidden(H, W_k, W_v, W_r, doc_tok_off_host, chunk, rope_base, Kbar, Vbar, Kbar_r,
                      doc_chunk_off, ws, stream=None):
    """H [n_tok, D]; W_* [h_kv * 128, D]; outputs [n_chunks, h_kv, 128] and doc_chunk_off."""
    off = np.ascontiguousarray(doc_tok_off_host, dtype=np.int64)
    n_tok, D = H.shape
    _check(lib.msa_encode_hidden(_p(H), n_tok, D, _p(W_k), _p(W_v), _p(W_r), off.ctypes.data,
                                 len(off) - 1, chunk, Kbar.shape[1], Kbar.shape[2],
                                 dtype_code(H), rope_base, _p(Kbar), _p(Vbar), _p(Kbar_r),
                                 _p(doc_chunk_off), Kbar.shape[0], _p(ws),
                                 ws.numel() * ws.element_size(), _s(stream)))


def encode_hidden(H, W_k, W_v, W_r, doc_tok_off_host, chunk: int, rope_base: float, h_kv: int,
                  stream=None):
    """Projections of the hidden states fused with doc-wise RoPE + chunk pooling. Returns
    dict(Kbar, Vbar, Kbar_r, doc_chunk_off)."""
    dev = H.device
    off = np.ascontiguousarray(doc_tok_off_host, dtype=np.int64)
    n_chunks = msa_count_chunks(off, chunk)
    if n_chunks < 0:
        raise MSAError(1, "invalid document offsets")
    shape = (n_chunks, h_kv, W_k.shape[0] // h_kv)
    out = dict(Kbar=torch.empty(shape, dtype=H.dtype, device=dev),
               Vbar=torch.empty(shape, dtype=H.dtype, device=dev),
               Kbar_r=torch.empty(shape, dtype=H.dtype, device=dev),
               doc_chunk_off=torch.empty(len(off), dtype=torch.int64, device=dev))
    ws = _ws(msa_encode_hidden_workspace(n_chunks), dev)
    msa_encode_hidden(H, W_k, W_v, W_r, off, chunk, rope_base, out["Kbar"], out["Vbar"],
                      out["Kbar_r"], out["doc_chunk_off"], ws, stream)
    return out


def msa_encode_hidden_workspace(n_chunks) -> int:
    return int(lib.msa_encode_hidden_workspace(n_chunks))


def msa_kr_inv_norm(Kbar_r, out, stream=None):
    n, h_kv, d = Kbar_r.shape
    _check(lib.msa_kr_inv_norm(_p(Kbar_r), n, h_kv, d, dtype_code(Kbar_r), _p(out), _s(stream)))


def msa_kr_normalize(Kbar_r, out, stream=None):
    n, h_kv, d = Kbar_r.shape
    _check(lib.msa_kr_normalize(_p(Kbar_r), n, h_kv, d, dtype_code(Kbar_r), _p(out), _s(stream)))


def msa_route_topk_workspace(B, T, h_qr, h_kv, d, dtype, n_docs, n_chunks, k) -> int:
    return int(lib.msa_route_topk_workspace(B, T, h_qr, h_kv, d, dtype, n_docs, n_chunks, k))


def _bank(Kbar_r, Kbar_r_hat):
    """(n_chunks, h_kv, dtype code) of a routing bank; Kbar_r may be None when the normalised
    bank Kbar_r_hat is given (the tensor-core scan reads only that)."""
    ref = Kbar_r if Kbar_r is not None else Kbar_r_hat
    return ref.shape[0], ref.shape[1], dtype_code(ref)


def msa_route_topk(Q_r, Kbar_r, kr_inv_norm, doc_chunk_off, k, exclude_bits, top_ids, top_scores,
                   doc_scores, ws, stream=None, Kbar_r_hat=None):
    B, T, h_qr, d = Q_r.shape
    n_chunks, h_kv, dt = _bank(Kbar_r, Kbar_r_hat)
    _check(lib.msa_route_topk(_p(Q_r), B, T, h_qr, _p(Kbar_r), _p(kr_inv_norm), _p(Kbar_r_hat),
                              _p(doc_chunk_off),
                              doc_chunk_off.shape[0] - 1, n_chunks, h_kv, d, dt, k,
                              _p(exclude_bits), _p(top_ids), _p(top_scores), _p(doc_scores),
                              _p(ws), ws.numel() * ws.element_size(), _s(stream)))


def msa_route_topk_noalloc(Q_r, Kbar_r, kr_inv_norm, doc_chunk_off, k, exclude_bits, top_ids,
                           top_scores, doc_scores, stream=None, Kbar_r_hat=None):
    """msa_route_topk without a workspace (the library's built-in 2 MiB scratch)."""
    B, T, h_qr, d = Q_r.shape
    n_chunks, h_kv, dt = _bank(Kbar_r, Kbar_r_hat)
    _check(lib.msa_route_topk_noalloc(_p(Q_r), B, T, h_qr, _p(Kbar_r), _p(kr_inv_norm),
                                      _p(Kbar_r_hat), _p(doc_chunk_off), doc_chunk_off.shape[0] - 1,
                                      n_chunks, h_kv, d, dt, k, _p(exclude_bits),
                                      _p(top_ids), _p(top_scores), _p(doc_scores), _s(stream)))


def msa_set_device_wait_limit(cycles: int) -> int:
    """Wait limit of the tensor-core routing scan's epilogue (SM clocks; 0: default). Returns the
    previous setting."""
    return int(lib.msa_set_device_wait_limit(int(cycles)))


def msa_route_topk_noalloc_status(stream=None) -> int:
    """Status word of msa_route_topk_noalloc's built-in scratch (0 = no device error)."""
    code = ctypes.c_int32(0)
    st = lib.msa_route_topk_noalloc_status(ctypes.addressof(code), _s(stream))
    if st not in (0, 6):
        _check(st)
    return int(code.value)


def msa_workspace_status(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    st = lib.msa_workspace_status(_p(ws), ctypes.addressof(code), _s(stream))
    if st not in (0, 6):
        _check(st)
    return int(code.value)


def msa_encode_pool_status(stream=None) -> int:
    """Status word of the last msa_encode_pool call (0, or the code of an expired device
    wait); synchronises `stream`."""
    code = ctypes.c_int32(0)
    st = lib.msa_encode_pool_status(ctypes.addressof(code), _s(stream))
    if st not in (0, 6):
        _check(st)
    return int(code.value)


def msa_assemble_local(seg_k_ptrs, seg_v_ptrs, seg_len, K_q, V_q, K_out, V_out, ws, stream=None):
    """seg_k_ptrs, seg_v_ptrs: int64 device tensors [B, n_seg] of segment data pointers;
    seg_len: int32 device [B, n_seg]; K_q, V_q: [B, T, h_kv, d]; K_out, V_out: [B, L, h_kv, d]."""
    B, n_seg = seg_len.shape
    T, h_kv, d = K_q.shape[1], K_q.shape[2], K_q.shape[3]
    _check(lib.msa_assemble_local(B, n_seg, _p(seg_k_ptrs), _p(seg_v_ptrs), _p(seg_len), _p(K_q),
                                  _p(V_q), T, h_kv, d, dtype_code(K_q), K_out.shape[1], _p(K_out),
                                  _p(V_out), _p(ws), ws.numel() * ws.element_size(), _s(stream)))


def msa_kv_append(K_cache, V_cache, length, K_new, V_new, pos0, rope_base, ws, stream=None):
    """K_cache, V_cache: [B, cap, h_kv, d]; length: int32 device tensor of one element;
    K_new, V_new: [B, T_new, h_kv, d] (keys stored rotated at pos0 + row when rope_base > 0)."""
    B, cap, h_kv, d = K_cache.shape
    _check(lib.msa_kv_append(_p(K_cache), _p(V_cache), B, cap, _p(length), _p(K_new), _p(V_new),
                             K_new.shape[1], h_kv, d, dtype_code(K_cache), pos0, rope_base,
                             _p(ws), ws.numel() * ws.element_size(), _s(stream)))


def msa_decode_step_workspace(B, T, h_q, h_kv, d, max_ctx, cap) -> int:
    return int(lib.msa_decode_step_workspace(B, T, h_q, h_kv, d, max_ctx, cap))


def msa_decode_step(Q, K_new, V_new, K_cache, V_cache, length, ctxK, ctxV, ctx_len, pos0,
                    rope_base, scale, O, ws, stream=None):
    """One generation step of one routed layer (append, then attend over the cache)."""
    B, T, h_q, d = Q.shape
    cap, h_kv = K_cache.shape[1], K_cache.shape[2]
    _check(lib.msa_decode_step(_p(Q), _p(K_new), _p(V_new), B, T, h_q, _p(K_cache), _p(V_cache),
                               cap, _p(length), _p(ctxK), _p(ctxV), _p(ctx_len), ctxK.shape[1],
                               h_kv, d, dtype_code(Q), pos0, rope_base, scale, _p(O), _p(ws),
                               ws.numel() * ws.element_size(), _s(stream)))


def msa_gather(top_ids, doc_chunk_off, Kbar, Vbar, max_ctx, gather_idx, ctx_len, ctxK, ctxV, ws,
               stream=None):
    B, k = top_ids.shape
    _check(lib.msa_gather(_p(top_ids), B, k, _p(doc_chunk_off), doc_chunk_off.shape[0] - 1,
                          _p(Kbar), _p(Vbar), Kbar.shape[1], Kbar.shape[2], dtype_code(Kbar),
                          max_ctx, _p(gather_idx), _p(ctx_len), _p(ctxK), _p(ctxV), _p(ws),
                          ws.numel() * ws.element_size(), _s(stream)))


def msa_sparse_attend_workspace(B, T, h_q, h_kv, d, max_ctx, L_loc) -> int:
    return int(lib.msa_sparse_attend_workspace(B, T, h_q, h_kv, d, max_ctx, L_loc))


def msa_sparse_attend(Q, K_loc, V_loc, ctxK, ctxV, ctx_len, pos0, rope_base, scale, O, ws,
                      stream=None):
    B, T, h_q, d = Q.shape
    L_loc, h_kv = K_loc.shape[1], K_loc.shape[2]
    max_ctx = ctxK.shape[1]
    _check(lib.msa_sparse_attend(_p(Q), B, T, h_q, _p(K_loc), _p(V_loc), L_loc, _p(ctxK), _p(ctxV),
                                 _p(ctx_len), max_ctx, h_kv, d, dtype_code(Q), pos0, rope_base,
                                 scale, _p(O), _p(ws), ws.numel() * ws.element_size(), _s(stream)))


def msa_sparse_attend_backward_workspace(B, T, h_q, h_kv, d, max_ctx, L_loc) -> int:
    return int(lib.msa_sparse_attend_backward_workspace(B, T, h_q, h_kv, d, max_ctx, L_loc))


def msa_sparse_attend_backward(Q, K_loc, V_loc, ctxK, ctxV, ctx_len, pos0, rope_base, scale, dO,
                               dQ, dK_loc, dV_loc, dK_ctx, dV_ctx, ws, stream=None):
    B, T, h_q, d = Q.shape
    L_loc, h_kv = K_loc.shape[1], K_loc.shape[2]
    _check(lib.msa_sparse_attend_backward(
        _p(Q), B, T, h_q, _p(K_loc), _p(V_loc), L_loc, _p(ctxK), _p(ctxV), _p(ctx_len),
        ctxK.shape[1], h_kv, d, dtype_code(Q), pos0, rope_base, scale, _p(dO), _p(dQ),
        _p(dK_loc), _p(dV_loc), _p(dK_ctx), _p(dV_ctx), _p(ws), ws.numel() * ws.element_size(),
        _s(stream)))


def msa_scatter_bank_grad(gather_idx, ctx_len, dK_ctx, dV_ctx, dKbar, dVbar, ws, stream=None):
    B, max_ctx, h_kv, d = dK_ctx.shape
    _check(lib.msa_scatter_bank_grad(_p(gather_idx), _p(ctx_len), B, max_ctx, h_kv, d,
                                     _p(dK_ctx), _p(dV_ctx), _p(dKbar), _p(dVbar),
                                     dKbar.shape[0], _p(ws), ws.numel() * ws.element_size(),
                                     _s(stream)))


def msa_aux_routing_loss(Q_r, Kbar_r, positive_bits, tau, loss, dQ_r, dKbar_r, ws, stream=None):
    B, T, h_qr, d = Q_r.shape
    n_chunks, h_kv = Kbar_r.shape[0], Kbar_r.shape[1]
    _check(lib.msa_aux_routing_loss(_p(Q_r), B, T, h_qr, _p(Kbar_r), n_chunks, h_kv, d,
                                    dtype_code(Q_r), _p(positive_bits), tau, _p(loss), _p(dQ_r),
                                    _p(dKbar_r), _p(ws), ws.numel() * ws.element_size(),
                                    _s(stream)))


# ----------------------------------------------------------------------------- helpers
def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def encode_pool(K, V, K_r, doc_tok_off_host, chunk: int, rope_base: float, stream=None):
    """Doc-wise RoPE + chunk pooling. Returns dict(Kbar, Vbar, Kbar_r, kr_inv_norm,
    doc_chunk_off)."""
    dev = K.device
    off = np.ascontiguousarray(doc_tok_off_host, dtype=np.int64)
    n_chunks = msa_count_chunks(off, chunk)
    if n_chunks < 0:
        raise MSAError(1, "invalid document offsets")
    n, h_kv, d = K.shape
    out = dict(Kbar=torch.empty((n_chunks, h_kv, d), dtype=K.dtype, device=dev),
               Vbar=torch.empty((n_chunks, h_kv, d), dtype=K.dtype, device=dev),
               Kbar_r=torch.empty((n_chunks, h_kv, d), dtype=K.dtype, device=dev),
               kr_inv_norm=torch.empty((n_chunks, h_kv), dtype=torch.float32, device=dev),
               doc_chunk_off=torch.empty(len(off), dtype=torch.int64, device=dev))
    tok_off = torch.from_numpy(off).to(dev)
    msa_encode_pool(K, V, K_r, off, tok_off, chunk, rope_base, out["Kbar"], out["Vbar"],
                    out["Kbar_r"], out["kr_inv_norm"], out["doc_chunk_off"], stream)
    return out


def kr_normalize(Kbar_r, stream=None):
    out = torch.empty(Kbar_r.shape, dtype=torch.bfloat16, device=Kbar_r.device)
    msa_kr_normalize(Kbar_r, out, stream)
    return out


def kr_inv_norm(Kbar_r, stream=None):
    out = torch.empty(Kbar_r.shape[:2], dtype=torch.float32, device=Kbar_r.device)
    msa_kr_inv_norm(Kbar_r, out, stream)
    return out


def route_topk(Q_r, Kbar_r, kr_inv, doc_chunk_off, k: int, exclude_bits=None,
               doc_scores: bool = False, ws=None, stream=None, Kbar_r_hat=None):
    """Returns (top_ids int32 [B,k], top_scores f32 [B,k], doc_scores f32 [B,n_docs] or None)."""
    B, T, h_qr, d = Q_r.shape
    n_chunks, h_kv, dt = _bank(Kbar_r, Kbar_r_hat)
    n_docs = doc_chunk_off.shape[0] - 1
    dev = Q_r.device
    if ws is None:
        ws = _ws(msa_route_topk_workspace(B, T, h_qr, h_kv, d, dt, n_docs, n_chunks, k), dev)
    ids = torch.empty((B, k), dtype=torch.int32, device=dev)
    sc = torch.empty((B, k), dtype=torch.float32, device=dev)
    ds = torch.empty((B, n_docs), dtype=torch.float32, device=dev) if doc_scores else None
    msa_route_topk(Q_r, Kbar_r, kr_inv, doc_chunk_off, k, exclude_bits, ids, sc, ds, ws, stream,
                   Kbar_r_hat)
    return ids, sc, ds


def gather(top_ids, doc_chunk_off, Kbar, Vbar, max_ctx: int, ws=None, stream=None):
    """Returns (gather_idx [B,max_ctx], ctx_len [B], ctxK, ctxV [B,max_ctx,h_kv,d])."""
    B = top_ids.shape[0]
    dev = top_ids.device
    h_kv, d = Kbar.shape[1], Kbar.shape[2]
    gi = torch.empty((B, max_ctx), dtype=torch.int32, device=dev)
    cl = torch.empty(B, dtype=torch.int32, device=dev)
    cK = torch.empty((B, max_ctx, h_kv, d), dtype=Kbar.dtype, device=dev)
    cV = torch.empty_like(cK)
    if ws is None:
        ws = _ws(256, dev)
    msa_gather(top_ids, doc_chunk_off, Kbar, Vbar, max_ctx, gi, cl, cK, cV, ws, stream)
    return gi, cl, cK, cV


def sparse_attend(Q, K_loc, V_loc, ctxK, ctxV, ctx_len, pos0: int, rope_base: float,
                  scale: float = 0.0, ws=None, stream=None):
    B, T, h_q, d = Q.shape
    if ws is None:
        ws = _ws(msa_sparse_attend_workspace(B, T, h_q, K_loc.shape[2], d, ctxK.shape[1],
                                             K_loc.shape[1]), Q.device)
    O = torch.empty_like(Q)
    msa_sparse_attend(Q, K_loc, V_loc, ctxK, ctxV, ctx_len, pos0, rope_base, scale, O, ws, stream)
    return O


class Fetcher:
    """msa_fetch context: asynchronous fetch of selected K̄/V̄ from a pinned host bank."""

    def __init__(self, max_B: int, max_k: int):
        h = ctypes.c_void_p()
        _check(lib.msa_fetch_create(max_B, max_k, ctypes.addressof(h)))
        self.h = h
        self.ws = None

    def begin(self, top_ids, doc_chunk_off, max_ctx, gather_idx, ctx_len, ws, stream=None):
        B, k = top_ids.shape
        _check(lib.msa_fetch_begin(self.h, _p(top_ids), B, k, _p(doc_chunk_off),
                                   doc_chunk_off.shape[0] - 1, max_ctx, _p(gather_idx),
                                   _p(ctx_len), _p(ws), ws.numel() * ws.element_size(),
                                   _s(stream)))

    def finish(self, doc_chunk_off_host: np.ndarray, Kbar_host, Vbar_host, max_ctx, ctxK, ctxV,
               stream=None, copy_stream=None, timeout_ms: int = 10000):
        off = doc_chunk_off_host
        h_kv, d = Kbar_host.shape[1], Kbar_host.shape[2]
        _check(lib.msa_fetch_finish(self.h, off.ctypes.data, len(off) - 1, _p(Kbar_host),
                                    _p(Vbar_host), h_kv, d, dtype_code(Kbar_host), max_ctx,
                                    _p(ctxK), _p(ctxV), _s(stream), _s(copy_stream), timeout_ms))

    def close(self):
        if self.h:
            lib.msa_fetch_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class LocalCache:
    """Preallocated local K/V of sparse generation: [B, cap, h_kv, d] plus its length, one
    int32 in device memory that msa_kv_append / msa_decode_step read and advance. Keys are
    stored rotated at their global positions pos0 + row (RoPE base ``rope_base``)."""

    def __init__(self, B: int, cap: int, h_kv: int, d: int, pos0: int = 0,
                 rope_base: float = 0.0, dtype=torch.bfloat16, device="cuda", length=None):
        self.pos0, self.rope_base = int(pos0), float(rope_base)
        self.K = torch.empty((B, cap, h_kv, d), dtype=dtype, device=device)
        self.V = torch.empty_like(self.K)
        # ``length``: an int32 device tensor of one element to use (e.g. a view of one array
        # holding the lengths of several layers' caches); a new zero otherwise
        self.length = (torch.zeros(1, dtype=torch.int32, device=device) if length is None
                       else length)
        self.ws = _ws(256, device)

    def append(self, K_new, V_new, stream=None):
        msa_kv_append(self.K, self.V, self.length, K_new, V_new, self.pos0, self.rope_base,
                      self.ws, stream)


def decode_step(cache: LocalCache, Q, K_new, V_new, ctxK, ctxV, ctx_len, scale: float = 0.0,
                O=None, ws=None, stream=None):
    """Append the step's tokens to ``cache`` and attend (global RoPE with the cache's pos0 and
    base); returns O [B, T, h_q, d]."""
    B, T, h_q, d = Q.shape
    pos0, rope_base = cache.pos0, cache.rope_base
    if ws is None:
        ws = _ws(msa_decode_step_workspace(B, T, h_q, cache.K.shape[2], d, ctxK.shape[1],
                                           cache.K.shape[1]), Q.device)
    if O is None:
        O = torch.empty_like(Q)
    msa_decode_step(Q, K_new, V_new, cache.K, cache.V, cache.length, ctxK, ctxV, ctx_len, pos0,
                    rope_base, scale, O, ws, stream)
    return O



def sparse_attend_backward(Q, K_loc, V_loc, ctxK, ctxV, ctx_len, pos0: int, rope_base: float,
                           dO, scale: float = 0.0, ws=None, stream=None) -> dict:
    """Gradients of ``sparse_attend`` for the output gradient dO; returns fp32 dict(dQ, dK_loc,
    dV_loc, dK_ctx, dV_ctx)."""
    B, T, h_q, d = Q.shape
    L_loc, h_kv = K_loc.shape[1], K_loc.shape[2]
    max_ctx = ctxK.shape[1]
    dev = Q.device
    f32 = torch.float32
    out = dict(dQ=torch.empty((B, T, h_q, d), dtype=f32, device=dev),
               dK_loc=torch.empty((B, L_loc, h_kv, d), dtype=f32, device=dev),
               dV_loc=torch.empty((B, L_loc, h_kv, d), dtype=f32, device=dev),
               dK_ctx=torch.empty((B, max_ctx, h_kv, d), dtype=f32, device=dev),
               dV_ctx=torch.empty((B, max_ctx, h_kv, d), dtype=f32, device=dev))
    if ws is None:
        ws = _ws(msa_sparse_attend_backward_workspace(B, T, h_q, h_kv, d, max_ctx, L_loc), dev)
    msa_sparse_attend_backward(Q, K_loc, V_loc, ctxK, ctxV, ctx_len, pos0, rope_base, scale, dO,
                               out["dQ"], out["dK_loc"], out["dV_loc"], out["dK_ctx"],
                               out["dV_ctx"], ws, stream)
    return out


def scatter_bank_grad(gather_idx, ctx_len, dK_ctx, dV_ctx, n_chunks: int, dKbar=None,
                      dVbar=None, ws=None, stream=None):
    """Adds the gathered rows' gradients into fp32 bank gradients [n_chunks, h_kv, d] (zeros
    unless given); returns (dKbar, dVbar)."""
    h_kv, d = dK_ctx.shape[2], dK_ctx.shape[3]
    dev = dK_ctx.device
    if dKbar is None:
        dKbar = torch.zeros((n_chunks, h_kv, d), dtype=torch.float32, device=dev)
    if dVbar is None:
        dVbar = torch.zeros((n_chunks, h_kv, d), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _ws(256, dev)
    msa_scatter_bank_grad(gather_idx, ctx_len, dK_ctx, dV_ctx, dKbar, dVbar, ws, stream)
    return dKbar, dVbar


def aux_routing_loss(Q_r, Kbar_r, positive_bits, tau: float = 0.1, stream=None):
    """Auxiliary routing loss over the chunk scores and its gradients; positive_bits int32
    [B, ceil(n_chunks/32)] (bit c: chunk c relevant). Returns (loss [1] fp32, dQ_r, dKbar_r)."""
    B, T, h_qr, d = Q_r.shape
    n_chunks = Kbar_r.shape[0]
    dev = Q_r.device
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dQ = torch.empty((B, T, h_qr, d), dtype=torch.float32, device=dev)
    dK = torch.empty(tuple(Kbar_r.shape), dtype=torch.float32, device=dev)
    ws = _ws(int(lib.msa_aux_routing_loss_workspace(B, n_chunks)), dev)
    msa_aux_routing_loss(Q_r, Kbar_r, positive_bits, tau, loss, dQ, dK, ws, stream)
    return loss, dQ, dK
