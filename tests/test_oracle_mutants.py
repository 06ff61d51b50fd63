"""Planted mistakes: each mutant is a copy of the oracle with one plausible slip (a sign, an
index, a dropped term, a reversed order). It is compiled in a temporary directory and must
fail at least one pin of the battery below, which reuses the independent references of
test_oracle_pins (transformers' Qwen3 RoPE, scipy cosine, numpy sort, torch SDPA)."""
import os
import shutil
import tempfile

import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import _qwen3_rope, _route_brute, _tiny_tokens

SRC = os.path.join(os.path.dirname(oracle.__file__), "msa_oracle.c")

MUTANTS = {
    "rope_sign": ("x[i] = x1 * c - x2 * s;", "x[i] = x1 * c + x2 * s;"),
    "rope_freq": ("-2.0 * (double)i / (double)d", "-1.0 * (double)i / (double)d"),
    "rope_pairing": ("double x1 = x[i], x2 = x[i + half];", "double x1 = x[2 * (i / 2)], x2 = x[i + half];"),
    "pool_divisor": ("ro[e] /= n; }", "ro[e] /= (n + 1.0); }"),
    "pool_position_not_restarted": ("double pos = (double)(t - t_doc);", "double pos = (double)t;"),
    "pool_rotates_v": ("vo[e] += orc_at(V, dtype, base + e);", "vo[e] += kx[e];"),
    "head_mean_count": ("s /= (double)h_qr;", "s /= (double)h_kv;"),
    "kv_head_map": ("int g = h / m;", "int g = h % h_kv;"),
    "chunk_max_to_sum": ("if (mt > best) best = mt;", "best = (best == -INFINITY ? 0.0 : best) + mt;"),
    "tie_break": ("return (x->id < y->id) ? -1 : (x->id > y->id);",
                  "return (x->id > y->id) ? -1 : (x->id < y->id);"),
    "gather_unsorted": ("qsort(ids, (size_t)n, sizeof(int32_t), orc_int_cmp);", ""),
    "causal_off_by_one": ("j <= qi;", "j < qi;"),
    "query_position": ("(double)pos0 + (double)qi", "(double)pos0 + (double)t"),
    "local_key_not_shifted": ("orc_rope(r, d, (double)pos0 + (double)j, rope_base);",
                              "orc_rope(r, d, (double)j, rope_base);"),
    "softmax_scale": ("scale = 1.0 / sqrt((double)d);", "scale = 1.0 / (double)d;"),
    "softmax_unnormalised": ("o[e] /= den;", "o[e] /= 1.0;"),
    "bw_ds_sign": ("const double ds = p[n] * (dp[n] - dsum) * scale;",
                   "const double ds = p[n] * (dsum - dp[n]) * scale;"),
    "bw_query_not_rotated_back": ("orc_rope(dq, d, -pos, rope_base);",
                                  "orc_rope(dq, d, pos, rope_base);"),
    "bw_dv_unweighted": ("gv[e] += p[n] * go[e];", "gv[e] += go[e];"),
    "bw_local_key_not_rotated_back": ("orc_rope(r, d, -((double)pos0 + (double)j), rope_base);",
                                      ""),
}


def _battery(L) -> list:
    """Run the pins against oracle handle L; return the names of the failing checks."""
    fails = []
    rng = np.random.default_rng(0)

    def check(name, ok):
        if not ok:
            fails.append(name)

    # RoPE against the backbone
    pos = np.array([0, 3, 17, 200])
    x = rng.standard_normal((4, 16))
    ref = _qwen3_rope(x, pos, 1e4)
    mine = np.stack([oracle.rope(x[i], pos[i], 1e4, L) for i in range(4)])
    check("rope", np.max(np.abs(mine - ref)) < 2e-4)
    # pooling brute force on ragged docs
    lens = [1, 5, 9]
    K, V, R, off = _tiny_tokens(lens, 2, 8, seed=1)
    Kb, Vb, Rb, coff = oracle.encode_pool(K, V, R, off, 4, 1e4, L)
    c = 0
    ok = True
    for i, n in enumerate(lens):
        for j in range(0, n, 4):
            sl = slice(off[i] + j, off[i] + min(j + 4, n))
            p = np.arange(j, min(j + 4, n))
            for h in range(2):
                ok &= np.max(np.abs(Kb[c, h] - _qwen3_rope(K[sl, h].astype(np.float64), p, 1e4)
                                    .mean(0))) < 2e-4
                ok &= np.max(np.abs(Vb[c, h] - V[sl, h].astype(np.float64).mean(0))) < 1e-12
                ok &= np.max(np.abs(Rb[c, h] - _qwen3_rope(R[sl, h].astype(np.float64), p, 1e4)
                                    .mean(0))) < 2e-4
            c += 1
    check("pool", ok)
    # routing brute force + exhaustive sort with duplicate docs
    n_docs = 12
    coff = np.array([0, 1, 3, 4, 6, 7, 9, 10, 12, 13, 15, 16, 18], np.int64)
    Krb = rng.standard_normal((18, 2, 8)).astype(np.float32)
    Krb[3] = Krb[16]
    Krb[16 + 1] = Krb[16]
    Krb[coff[3]:coff[4]] = Krb[coff[10]:coff[11]]
    Qr = rng.standard_normal((2, 3, 4, 8)).astype(np.float32)
    Qr[1, 0, :2] = Krb[coff[10], 0]
    Qr[1, 0, 2:] = Krb[coff[10], 1]
    ids, ts, ds = oracle.route(Qr, Krb, coff, n_docs, None, L)
    check("route_scores", np.max(np.abs(ds - _route_brute(Qr, Krb, coff))) < 1e-12)
    check("route_order", all(np.array_equal(ids[b], np.lexsort((np.arange(n_docs), -ds[b])))
                             for b in range(2)))
    # gather order
    gi, cl = oracle.gather(np.array([[5, 1, 3]], np.int32), coff, 8, L)
    want = np.concatenate([np.arange(coff[d], coff[d + 1]) for d in (1, 3, 5)])
    check("gather", cl[0] == len(want) and np.array_equal(gi[0, :cl[0]], want))
    # attention: dense equivalence with chunk 1, k = n_docs
    import torch.nn.functional as F
    lens = [2, 3]
    K, V, R, off = _tiny_tokens(lens, 1, 8, seed=2)
    Q = rng.standard_normal((1, 2, 2, 8)).astype(np.float32)
    Kl = rng.standard_normal((1, 3, 1, 8)).astype(np.float32)
    Vl = rng.standard_normal((1, 3, 1, 8)).astype(np.float32)
    Kb, Vb, Rb, coff = oracle.encode_pool(K, V, R, off, 1, 1e4, L)
    gi = np.arange(5, dtype=np.int32)[None]
    O = oracle.attend(Q, Kl, Vl, Kb.astype(np.float32), Vb.astype(np.float32), gi,
                      np.array([5], np.int32), pos0=2, rope_base=1e4, L=L)
    mem_k = np.concatenate([_qwen3_rope(K[off[i]:off[i + 1], 0].astype(np.float64),
                                        np.arange(lens[i]), 1e4) for i in range(2)])
    loc_k = _qwen3_rope(Kl[0, :, 0].astype(np.float64), 2 + np.arange(3), 1e4)
    q = _qwen3_rope(Q[0].astype(np.float64).transpose(1, 0, 2), 2 + np.array([1, 2]), 1e4)
    keys = torch.from_numpy(np.concatenate([mem_k, loc_k]))[None].expand(2, -1, -1)
    vals = torch.from_numpy(np.concatenate([V[:, 0], Vl[0, :, 0]]).astype(np.float64))[None]
    mask = torch.ones(2, 8, dtype=torch.bool)
    mask[0, 7] = False
    ref = F.scaled_dot_product_attention(torch.from_numpy(q), keys, vals.expand(2, -1, -1),
                                         attn_mask=mask).numpy()
    check("attend", np.max(np.abs(O[0].transpose(1, 0, 2) - ref)) < 5e-4)
    # attention gradients: central differences of the forward along random directions
    Q = rng.standard_normal((1, 2, 2, 8)).astype(np.float32)
    Kl = rng.standard_normal((1, 4, 1, 8)).astype(np.float32)
    Vl = rng.standard_normal((1, 4, 1, 8)).astype(np.float32)
    Kb = rng.standard_normal((3, 1, 8)).astype(np.float32)
    Vb = rng.standard_normal((3, 1, 8)).astype(np.float32)
    gi = np.array([[2, 0]], np.int32)
    cl = np.array([2], np.int32)
    dO = rng.standard_normal((1, 2, 2, 8))
    g = oracle.attend_backward(Q, Kl, Vl, Kb, Vb, gi, cl, 3, 1e4, dO, L=L)
    args = dict(Q=Q, K_loc=Kl, V_loc=Vl, Kbar=Kb, Vbar=Vb)
    grads = dict(Q=g["dQ"], K_loc=g["dK_loc"], V_loc=g["dV_loc"], Kbar=g["dKbar"],
                 Vbar=g["dVbar"])
    ok = True
    for name, x in args.items():
        delta = rng.standard_normal(x.shape).astype(np.float32)
        o = []
        for sgn in (1, -1):
            a = dict(args, **{name: (x.astype(np.float64) + sgn * 1e-2 * delta).astype(np.float32)})
            o.append(oracle.attend(a["Q"], a["K_loc"], a["V_loc"], a["Kbar"], a["Vbar"], gi, cl,
                                   3, 1e4, L=L))
        fd = np.sum(dO * (o[0] - o[1])) / 2e-2
        an = np.sum(grads[name] * delta)
        ok &= abs(fd - an) <= 2e-3 * (1 + abs(an))
    check("attend_backward", ok)
    return fails


def test_battery_passes_on_the_real_oracle():
    assert _battery(oracle.lib()) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert old in src, f"mutation site of {name} not found"
    tmp = tempfile.mkdtemp(prefix="orc_mut_")
    try:
        path = os.path.join(tmp, "m.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        so = oracle.build(force=True, src=path, out=os.path.join(tmp, "libm.so"))
        L = oracle.load_variant(so)
        assert _battery(L), f"mutant {name} passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
