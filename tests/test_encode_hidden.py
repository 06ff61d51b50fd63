"""GPU parity of the offline encode from hidden states (msa_encode_hidden: tcgen05 projections
fused with doc-wise RoPE and chunk pooling) against the oracle's projections + encode_pool."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import check_pooled, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(gpu):
    import long_context_doc_b200 as m
    return m


@pytest.mark.parametrize("lens,D,h_kv,base", [
    ([64, 1, 130, 200, 63, 0, 17], 256, 4, 1e6),   # ragged docs, partial and empty, odd chunks
    ([700, 333, 1015], 2560, 8, 1e6),              # the backbone's hidden size, many slices
    ([5, 90], 128, 2, 0.0),                        # RoPE off, one head pair
])
def test_encode_hidden_matches_oracle(msa, gpu, lens, D, h_kv, base):
    off = np.zeros(len(lens) + 1, np.int64)
    off[1:] = np.cumsum(lens)
    n = int(off[-1])
    H = synth.normal(21, 40, (n, D), "bf16")
    Ws = [synth.normal(21, 41 + i, (h_kv * 128, D), "bf16", scale=D ** -0.5) for i in range(3)]
    # the oracle takes W as [D, h_kv * 128]
    Wt = [np.ascontiguousarray(w.T) for w in Ws]
    Kb, Vb, Rb, coff = oracle.encode_hidden(H, Wt[0], Wt[1], Wt[2], off, 64, base, h_kv)
    out = msa.encode_hidden(to_dev(H, gpu), *(to_dev(w, gpu) for w in Ws), off, 64, base, h_kv)
    torch.cuda.synchronize()
    assert out["doc_chunk_off"].cpu().numpy().tolist() == coff.tolist()
    for name, ref in (("Kbar", Kb), ("Vbar", Vb), ("Kbar_r", Rb)):
        check_pooled(out[name], ref, "bf16", name)
