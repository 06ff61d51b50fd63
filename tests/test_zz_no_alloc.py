"""msa_route_topk_noalloc: routing for callers that cannot allocate device memory at the call
site (a framework's memory planner owns every allocation, allocation may synchronise the
device, or the serving loop forbids allocator calls). It must return what msa_route_topk
returns with a caller workspace, call after call, although all calls share one scratch
array inside the library. Collected last on purpose: a failure here leaves every other test
already run."""
import numpy as np
import pytest
import torch

import synth
from _util import SCORE_TOL, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


def _inputs(gpu, tensor_path: bool, B=8, T=1, exclude=False):
    w = synth.C3.scaled(n_docs=1500, B=B, T=T, ragged=True, seed=31 + T)
    inp = synth.make_bank_workload(w)
    Krb = to_dev(inp["Kbar_r"], gpu)
    import long_context_doc_b200 as m
    ex = None
    if exclude:  # every third document, and each query's planted one, not eligible
        words = (w.n_docs + 31) // 32
        bits = np.zeros((B, words), np.uint32)
        for b in range(B):
            for i in list(range(0, w.n_docs, 3)) + [int(inp["planted"][b, 0])]:
                bits[b, i // 32] |= np.uint32(1 << (i % 32))
        ex = torch.from_numpy(bits.view(np.int32)).to(gpu)
    return dict(w=w, Q_r=to_dev(inp["Q_r"], gpu), Kbar_r=Krb, inv=m.kr_inv_norm(Krb),
                hat=m.kr_normalize(Krb) if tensor_path else None, ex=ex,
                coff=torch.from_numpy(inp["doc_chunk_off"]).to(gpu))


@pytest.mark.parametrize("tensor_path,B,T,exclude", [
    (False, 8, 1, False),   # decode batch, CUDA-core scan
    (True, 8, 1, False),    # decode batch, tensor-core scan
    (True, 1, 128, False),  # one long query on the tensor-core scan (folded queries in scratch)
    (True, 4, 1, True),     # exclusion bits
], ids=["cuda_core_scan", "tensor_core_scan", "tensor_core_long_query", "exclusion"])
def test_noalloc_matches_workspace_route_two_calls(msa, gpu, tensor_path, B, T, exclude):
    d = _inputs(gpu, tensor_path, B, T, exclude)
    w = d["w"]
    ref_ids, ref_sc, ref_ds = msa.route_topk(d["Q_r"], d["Kbar_r"], d["inv"], d["coff"], w.k,
                                             exclude_bits=d["ex"], doc_scores=True,
                                             Kbar_r_hat=d["hat"])
    torch.cuda.synchronize()
    n_docs = d["coff"].shape[0] - 1
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        ids = torch.full((w.B, w.k), -7, dtype=torch.int32, device=gpu)
        sc = torch.full((w.B, w.k), np.nan, dtype=torch.float32, device=gpu)
        ds = torch.full((w.B, n_docs), np.nan, dtype=torch.float32, device=gpu)
        msa.msa_route_topk_noalloc(d["Q_r"], d["Kbar_r"], d["inv"], d["coff"], w.k, d["ex"], ids,
                                   sc, ds, Kbar_r_hat=d["hat"])
        # the status word of the built-in scratch: a caller's only view of device-side errors
        assert msa.msa_route_topk_noalloc_status() == 0
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids)
        np.testing.assert_allclose(sc.cpu().numpy(), ref_sc.cpu().numpy(), rtol=0,
                                   atol=SCORE_TOL["bf16"])
        np.testing.assert_allclose(ds.cpu().numpy(), ref_ds.cpu().numpy(), rtol=0,
                                   atol=SCORE_TOL["bf16"])


def test_noalloc_rejects_calls_beyond_its_scratch(msa, gpu):
    d = _inputs(gpu, True)
    Q = torch.zeros((64, 256, 8, 128), dtype=torch.bfloat16, device=gpu)  # 32 MB of folded queries
    ids = torch.empty((64, 4), dtype=torch.int32, device=gpu)
    sc = torch.empty((64, 4), dtype=torch.float32, device=gpu)
    with pytest.raises(msa.MSAError) as e:
        msa.msa_route_topk_noalloc(Q, d["Kbar_r"], d["inv"], d["coff"], 4, None, ids, sc, None,
                                   Kbar_r_hat=d["hat"])
    assert e.value.status == 2 and "scratch" in e.value.message


def test_noalloc_status_reports_a_device_error_then_clears(msa, gpu):
    """A device wait of the built-in-scratch call that runs out (the consumer-side limit cut to
    a few dozen cycles) shows in msa_route_topk_noalloc_status; the next normal call clears it
    and routes correctly."""
    d = _inputs(gpu, True)
    w = d["w"]
    ref_ids, _, _ = msa.route_topk(d["Q_r"], d["Kbar_r"], d["inv"], d["coff"], w.k,
                                   Kbar_r_hat=d["hat"])
    ids = torch.empty((w.B, w.k), dtype=torch.int32, device=gpu)
    sc = torch.empty((w.B, w.k), dtype=torch.float32, device=gpu)
    prev = msa.msa_set_device_wait_limit(64)
    try:
        msa.msa_route_topk_noalloc(d["Q_r"], d["Kbar_r"], d["inv"], d["coff"], w.k, None, ids,
                                   sc, None, Kbar_r_hat=d["hat"])
        code = msa.msa_route_topk_noalloc_status()
    finally:
        msa.msa_set_device_wait_limit(prev)
    assert code == 1
    msa.msa_route_topk_noalloc(d["Q_r"], d["Kbar_r"], d["inv"], d["coff"], w.k, None, ids, sc,
                               None, Kbar_r_hat=d["hat"])
    assert msa.msa_route_topk_noalloc_status() == 0
    assert torch.equal(ids, ref_ids)
