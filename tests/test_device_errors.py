"""Device-side failures reach the caller, and the context stays usable.

A bounded device wait that runs out must record its error in the workspace status word (read
with msa_workspace_status, MSA_ERR_DEVICE), leave no copy or tensor-core operation in flight,
and let the next call on the same stream run normally. The failure is made by the caller, not by
a fault: msa_set_device_wait_limit shortens the consumer-side waits of the tensor-core routing
scan (its epilogue warps waiting for the tensor cores' accumulators) to a few dozen cycles,
which no tile loaded from memory and multiplied meets; the waits for copies and MMAs in flight
keep the default limit. No test here faults, traps or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import SCORE_TOL, check_topk, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


@pytest.fixture(scope="module")
def bank(gpu):
    import long_context_doc_b200 as m
    w = synth.C3.scaled(n_docs=3000, B=8, seed=41)
    inp = synth.make_bank_workload(w)
    Krb = to_dev(inp["Kbar_r"], gpu)
    return dict(w=w, inp=inp, Q_r=to_dev(inp["Q_r"], gpu), hat=m.kr_normalize(Krb),
                coff=torch.from_numpy(inp["doc_chunk_off"]).to(gpu))


def _route(msa, d, ws, st):
    w = d["w"]
    ids = torch.full((w.B, w.k), -7, dtype=torch.int32, device=ws.device)
    sc = torch.full((w.B, w.k), np.nan, dtype=torch.float32, device=ws.device)
    msa.msa_route_topk(d["Q_r"], None, None, d["coff"], w.k, None, ids, sc, None, ws, st, d["hat"])
    return ids, sc


def test_route_wait_timeout_is_reported_and_the_stream_recovers(msa, gpu, bank):
    w = bank["w"]
    st = torch.cuda.Stream()
    ws = torch.zeros(msa.msa_route_topk_workspace(w.B, 1, w.h_qr, w.h_kv, w.d, 1, w.n_docs,
                                                  bank["inp"]["n_chunks"], w.k),
                     dtype=torch.uint8, device=gpu)
    prev = msa.msa_set_device_wait_limit(64)
    try:
        _route(msa, bank, ws, st)
        code = msa.msa_workspace_status(ws, st)  # synchronises the stream
    finally:
        assert msa.msa_set_device_wait_limit(prev) == 64
    assert code == 1  # a bounded wait ran out
    # the next call on the same stream, with the default limit, is correct
    ids, sc = _route(msa, bank, ws, st)
    assert msa.msa_workspace_status(ws, st) == 0
    r_ids, r_sc, r_ds = oracle.route(bank["inp"]["Q_r"], bank["inp"]["Kbar_r"],
                                     bank["inp"]["doc_chunk_off"], w.k)
    check_topk(ids.cpu().numpy(), sc.cpu().numpy().astype(np.float64), r_ids, r_sc, r_ds,
               SCORE_TOL["bf16"])


def test_default_wait_limit_is_restored_by_zero(msa, gpu):
    prev = msa.msa_set_device_wait_limit(1000)
    assert msa.msa_set_device_wait_limit(0) == 1000
    assert msa.msa_set_device_wait_limit(prev) == 0
