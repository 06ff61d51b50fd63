"""Shared helpers of the parity tests: numpy <-> torch marshalling of the synthetic inputs
and the comparison rules of the routed-memory path.

Tolerances (stated for the method's outputs): scores 1e-5 abs (fp32) / 2e-3 abs (bf16);
attention 1e-4 rel (fp32) / 2e-2 rel (bf16), rel = max-abs error / max-abs reference per
(b, t, h) output row; top-k ids exact whenever the oracle's k-th/(k+1)-th score gap exceeds
the score tolerance; gather indices bit-exact whenever the selected set matches; pooled
tensors within one storage ulp (bf16: 2^-8 relative) plus fp32 accumulation slack.
"""
import numpy as np

SCORE_TOL = {"fp32": 1e-5, "bf16": 2e-3}
ATT_TOL = {"fp32": 1e-4, "bf16": 2e-2}


def to_dev(x, dev):
    import torch
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(x).to(dev)


def to_np(t):
    """Device tensor -> numpy float64 (bf16 decoded exactly)."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def stored_f64(x, dtype):
    """Synthetic / oracle storage array (float32 or bf16 bits) -> float64."""
    if dtype == "bf16" or x.dtype == np.uint16:
        return (np.ascontiguousarray(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def check_pooled(got, ref64, dtype, what=""):
    """got: device tensor; ref64: oracle double result before storage rounding."""
    g = to_np(got)
    if dtype == "bf16":
        tol = 2.0 ** -8 * np.abs(ref64) + 1e-6
    else:
        tol = 1e-5 * np.abs(ref64) + 2e-6
    bad = np.abs(g - ref64) > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {np.max(np.abs(g - ref64))}"


def check_topk(ids, scores, ref_ids, ref_scores, ref_doc_scores, tol):
    """The gap rule: exact set whenever the oracle's k-th/(k+1)-th gap exceeds tol; otherwise
    every selected doc's oracle score must be within tol of the k-th score. Rank order is
    compared where adjacent oracle gaps exceed tol. Returns the number of exact rows."""
    B, k = ref_ids.shape
    exact_rows = 0
    for b in range(B):
        s_sorted = np.sort(ref_doc_scores[b])[::-1]
        kth = ref_scores[b, k - 1]
        nxt = s_sorted[k] if len(s_sorted) > k else -np.inf
        got = ids[b].tolist()
        assert len(set(got)) == k, f"row {b}: repeated ids {got}"
        if kth - nxt > tol:
            assert set(got) == set(ref_ids[b].tolist()), f"row {b}: {got} vs {ref_ids[b].tolist()}"
            exact_rows += 1
            for j in range(k - 1):
                if ref_scores[b, j] - ref_scores[b, j + 1] > tol:
                    assert set(got[:j + 1]) == set(ref_ids[b, :j + 1].tolist()), f"row {b} rank {j}"
        else:
            for i in got:
                assert ref_doc_scores[b, i] >= kth - tol, f"row {b}: doc {i} not a valid choice"
        np.testing.assert_allclose(scores[b], ref_doc_scores[b, ids[b]], atol=tol, rtol=0)
    return exact_rows


def check_attention(O, ref64, dtype):
    g = to_np(O)
    err = np.abs(g - ref64).max(axis=-1)
    scale = np.abs(ref64).max(axis=-1)
    rel = err / np.maximum(scale, 1e-30)
    assert rel.max() < ATT_TOL[dtype], f"attention rel err {rel.max():.3e}"
    return float(rel.max())
