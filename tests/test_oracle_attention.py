"""Pins for the float64 chunk-attention oracle.

Source: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
Selection", Abstract (chunked prefill over the per-group tables, KV read in
place).  Pinned by: a hand-derived case, scalar brute force, torch's float64
scaled_dot_product_attention (a library routine) on dense and token-masked
problems, closed forms, page-permutation invariance, the LSE-merge identity and
chunk composition.  Two planted mistakes show the pins are sensitive.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _val(s):
    if s == "-inf":
        return -math.inf
    if s.startswith("ln"):
        return math.log(float(s[2:]))
    return float(Fraction(s))


@pytest.mark.parametrize("fixture", ["attention_hand.json", "attention_unaligned_hand.json"])
def test_hand_derived_case(fixture):
    """Hand-derived values; the unaligned fixture has prefix 3 + chunk 2 at
    block 2, so its last block holds one key and an empty slot."""
    g = json.load(open(os.path.join(GOLD, fixture)))
    a = np.array([_val(x) for x in g["a"]])
    b = np.array([_val(x) for x in g["b"]])
    T = len(a)
    assert T == g["prefix_len"] + g["chunk_len"]
    pt = np.array(g["page_table"])
    B = g["block"]
    nK = len(pt)
    assert nK == -(-T // B)
    K = np.zeros((nK * B, 2))                                # logical keys, empty slots 0
    V = np.zeros((nK * B, 2))
    K[:T] = math.sqrt(2.0) * np.stack([a, b], axis=1)
    V[:T] = np.stack([np.arange(T, dtype=float), np.ones(T)], axis=1)
    Kp = np.zeros((nK, 1, B, 2))
    Vp = np.zeros((nK, 1, B, 2))
    for kb, page in enumerate(pt):
        Kp[page, 0] = K[kb * B:(kb + 1) * B]
        Vp[page, 0] = V[kb * B:(kb + 1) * B]
    Q = np.array(g["Q"])
    for case in g["cases"]:
        tab = np.full((1, nK), -1)
        tab[0, :case["count"]] = case["table"]
        O, L = oracle.oracle_chunk_attention(Q, Kp, Vp, pt, tab, [case["count"]], g["prefix_len"])
        expL = np.array([_val(x) for x in case["LSE"]])
        expO = np.array([[_val(x) for x in r] for r in case["O"]])
        np.testing.assert_allclose(L[0], expL, rtol=0, atol=1e-12)
        np.testing.assert_allclose(O[:, 0, :], expO, rtol=0, atol=1e-12)


def _np(t):
    return t.double().numpy()


def small_case(seed=0, Hq=4, Hkv=2, d=16, B=8, P=24, Lc=16, rho=0.4, kind="bernoulli"):
    w = workloads.Workload("s", Hq, Hkv, d, "fp32", P, Lc, B, kind, rho=rho, corr=0.5,
                           window=2, seed=seed)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    t, c = oracle.oracle_tables(m, Hkv)
    return w, x, m, t, c


def sdpa_reference(Q, Kfull, Vfull, visible, G):
    """torch float64 SDPA with an explicit boolean mask, plus LSE recovered by an
    extra key of score 0 whose value is a one-hot column: its weight is
    w = 1 / (1 + exp(LSE)), so LSE = ln(1/w - 1).

    Q [L, Hq, d]; Kfull/Vfull [Hkv, T, d]; visible [Hq, L, T] bool.
    """
    L, Hq, d = Q.shape
    Hkv, T, _ = Kfull.shape
    q = torch.from_numpy(np.ascontiguousarray(Q.transpose(1, 0, 2)))          # [Hq, L, d]
    k = torch.from_numpy(np.repeat(Kfull, G, axis=0))                         # [Hq, T, d]
    v = torch.from_numpy(np.repeat(Vfull, G, axis=0))
    kz = torch.cat([k, torch.zeros(Hq, 1, d, dtype=k.dtype)], dim=1)
    vz = torch.zeros(Hq, T + 1, d + 1, dtype=v.dtype)
    vz[:, :T, :d] = v
    vz[:, T, d] = 1.0
    msk = torch.ones(Hq, L, T + 1, dtype=torch.bool)
    msk[:, :, :T] = torch.from_numpy(visible)
    # the library's default scale is 1/sqrt(last dim of q), which is 1/sqrt(d)
    out = torch.nn.functional.scaled_dot_product_attention(q, kz, vz[..., :], attn_mask=msk)
    wgt = out[..., d].numpy()
    O = (out[..., :d].numpy() / (1.0 - wgt)[..., None]).transpose(1, 0, 2)
    with np.errstate(divide="ignore"):
        LSE = np.log(1.0 / wgt - 1.0)
    return O, LSE


def token_visibility(t, c, Hq, Hkv, P, Lc, B, nKblk):
    G = Hq // Hkv
    T = nKblk * B
    j = np.arange(T)
    vis = np.zeros((Hq, Lc, T), dtype=bool)
    for h in range(Hq):
        g = h // G
        inblk = np.isin(j // B, t[g, :c[g]])
        vis[h] = inblk[None, :] & (j[None, :] <= (P + np.arange(Lc))[:, None])
    return vis


def test_brute_force_small():
    w, x, m, t, c = small_case(seed=1, Hq=4, Hkv=2, d=8, B=4, P=12, Lc=8)
    args = (_np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"]), x["page_table"].numpy(), t, c,
            w.prefix_len)
    O, L = oracle.oracle_chunk_attention(*args)
    Ob, Lb = oracle.brute_force_attention(args[0].tolist(), args[1].tolist(), args[2].tolist(),
                                          *args[3:])
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", ["bernoulli", "vslash"])
def test_token_masked_sdpa(kind):
    w, x, m, t, c = small_case(seed=2, kind=kind, rho=0.15)
    Q, Kp, Vp = _np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"])
    pt = x["page_table"].numpy()
    O, L = oracle.oracle_chunk_attention(Q, Kp, Vp, pt, t, c, w.prefix_len)
    Kf, Vf = oracle.depage(Kp, pt, w.nKblk), oracle.depage(Vp, pt, w.nKblk)
    vis = token_visibility(t, c, w.Hq, w.Hkv, w.prefix_len, w.chunk_len, w.block, w.nKblk)
    Or, Lr = sdpa_reference(Q, Kf, Vf, vis, w.G)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-10)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-10)


def test_all_ones_equals_dense_causal_tiny():
    w = workloads.get_config("tiny").with_(mask_kind="ones")
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    t, c = oracle.oracle_tables(m, w.Hkv)
    assert c.tolist() == [w.nKblk]
    Q, Kp, Vp = _np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"])
    pt = x["page_table"].numpy()
    O, L = oracle.oracle_chunk_attention(Q, Kp, Vp, pt, t, c, w.prefix_len)
    T = w.nKblk * w.block
    causal = np.arange(T)[None, :] <= (w.prefix_len + np.arange(w.chunk_len))[:, None]
    vis = np.broadcast_to(causal, (w.Hq,) + causal.shape).copy()
    Or, Lr = sdpa_reference(Q, oracle.depage(Kp, pt, w.nKblk), oracle.depage(Vp, pt, w.nKblk),
                            vis, w.G)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-10)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-10)


def test_closed_form_zero_keys():
    """K = 0: every visible score is 0, so O is the mean of the visible V and LSE = ln(#visible)."""
    w, x, m, t, c = small_case(seed=3)
    Kp = np.zeros_like(_np(x["K_pages"]))
    Vp = _np(x["V_pages"])
    pt = x["page_table"].numpy()
    O, L = oracle.oracle_chunk_attention(_np(x["Q"]), Kp, Vp, pt, t, c, w.prefix_len)
    Vf = oracle.depage(Vp, pt, w.nKblk)
    for h in range(w.Hq):
        g = h // w.G
        for i in range(w.chunk_len):
            p = w.prefix_len + i
            keys = [kb * w.block + r for kb in t[g, :c[g]] for r in range(w.block)
                    if kb * w.block + r <= p]
            assert L[h, i] == pytest.approx(math.log(len(keys)), abs=1e-12)
            np.testing.assert_allclose(O[i, h], Vf[g, keys].mean(axis=0), atol=1e-12)


def test_closed_form_constant_values():
    w, x, m, t, c = small_case(seed=4)
    Vp = np.full_like(_np(x["V_pages"]), 0.625)
    O, _ = oracle.oracle_chunk_attention(_np(x["Q"]), _np(x["K_pages"]), Vp,
                                         x["page_table"].numpy(), t, c, w.prefix_len)
    np.testing.assert_allclose(O, 0.625, atol=1e-12)


def test_empty_table_rows():
    w, x, m, t, c = small_case(seed=5)
    t = t.copy()
    c = c.copy()
    t[1] = -1
    c[1] = 0
    O, L = oracle.oracle_chunk_attention(_np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"]),
                                         x["page_table"].numpy(), t, c, w.prefix_len)
    G = w.G
    assert np.all(O[:, G:2 * G] == 0) and np.all(np.isneginf(L[G:2 * G]))
    assert np.all(np.isfinite(L[:G]))


def test_page_permutation_invariance():
    w, x, m, t, c = small_case(seed=6)
    Kp, Vp = _np(x["K_pages"]), _np(x["V_pages"])
    pt = x["page_table"].numpy()
    Kid = np.stack([Kp[pt[kb]] for kb in range(w.nKblk)])
    Vid = np.stack([Vp[pt[kb]] for kb in range(w.nKblk)])
    ident = np.arange(w.nKblk)
    O1, L1 = oracle.oracle_chunk_attention(_np(x["Q"]), Kp, Vp, pt, t, c, w.prefix_len)
    O2, L2 = oracle.oracle_chunk_attention(_np(x["Q"]), Kid, Vid, ident, t, c, w.prefix_len)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_lse_merge_identity():
    """Attention over the union of two disjoint block sets = LSE-combine of the two."""
    w, x, m, t, c = small_case(seed=7, rho=0.5)
    args = (_np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"]), x["page_table"].numpy())
    O, L = oracle.oracle_chunk_attention(*args, t, c, w.prefix_len)
    parts = []
    for sel in (lambda e: e % 2 == 0, lambda e: e % 2 == 1):
        tp = np.full_like(t, -1)
        cp = np.zeros_like(c)
        for g in range(w.Hkv):
            e = [kb for kb in t[g, :c[g]] if sel(kb)]
            tp[g, :len(e)] = e
            cp[g] = len(e)
        parts.append(oracle.oracle_chunk_attention(*args, tp, cp, w.prefix_len))
    Om, Lm = oracle.lse_combine(np.stack([p[0] for p in parts]),
                                np.stack([p[1].T for p in parts]))
    np.testing.assert_allclose(Om, O, atol=1e-12)
    np.testing.assert_allclose(Lm.T, L, atol=1e-12)


def test_lse_combine_all_empty():
    O, L = oracle.lse_combine(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(O == 0) and np.all(np.isneginf(L))


def test_chunk_composition_equals_one_shot_causal():
    """All-ones masks over 4 consecutive chunks reproduce full causal attention."""
    Hq, Hkv, d, B, Lc, n = 4, 2, 16, 8, 16, 4
    T = Lc * n
    w = workloads.Workload("comp", Hq, Hkv, d, "fp32", T - Lc, Lc, B, "ones")
    rng = np.random.default_rng(11)
    Qall = rng.standard_normal((T, Hq, d))
    pages_k = rng.standard_normal((T // B, Hkv, B, d))
    pages_v = rng.standard_normal((T // B, Hkv, B, d))
    pt_all = rng.permutation(T // B)
    Kf = oracle.depage(pages_k, pt_all, T // B)
    Vf = oracle.depage(pages_v, pt_all, T // B)
    causal = np.arange(T)[None, :] <= np.arange(T)[:, None]
    Oref, Lref = sdpa_reference(Qall, Kf, Vf, np.broadcast_to(causal, (Hq, T, T)).copy(), Hq // Hkv)
    for ci in range(n):
        P = ci * Lc
        nK = (P + Lc) // B
        m = workloads.ones_mask(Hq, P // B, Lc // B, nK)
        t, c = oracle.oracle_tables(m, Hkv)
        O, L = oracle.oracle_chunk_attention(Qall[P:P + Lc], pages_k, pages_v, pt_all[:nK], t, c, P)
        np.testing.assert_allclose(O, Oref[P:P + Lc], atol=1e-10)
        np.testing.assert_allclose(L, Lref[:, P:P + Lc], atol=1e-10)


def test_rows_helper_matches_full():
    w, x, m, t, c = small_case(seed=8)
    args = (_np(x["Q"]), x["K_pages"].double().numpy(), x["V_pages"].double().numpy(),
            x["page_table"].numpy(), t, c, w.prefix_len)
    O, L = oracle.oracle_chunk_attention(*args)
    rows = [(0, 0), (3, 15), (2, 7), (1, 9)]
    Or, Lr = oracle.oracle_rows(*args, rows)
    for r, (h, i) in enumerate(rows):
        np.testing.assert_allclose(Or[r], O[i, h], atol=1e-13)
        assert Lr[r] == pytest.approx(L[h, i], abs=1e-13)


def test_planted_wrong_scale_is_caught(monkeypatch):
    import oracle.attention as A
    w, x, m, t, c = small_case(seed=9)
    Q, Kp, Vp = _np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"])
    pt = x["page_table"].numpy()
    monkeypatch.setattr(A.math, "sqrt", lambda v: float(v))      # 1/d instead of 1/sqrt(d)
    O, L = oracle.oracle_chunk_attention(Q, Kp, Vp, pt, t, c, w.prefix_len)
    monkeypatch.undo()
    vis = token_visibility(t, c, w.Hq, w.Hkv, w.prefix_len, w.chunk_len, w.block, w.nKblk)
    Or, Lr = sdpa_reference(Q, oracle.depage(Kp, pt, w.nKblk), oracle.depage(Vp, pt, w.nKblk),
                            vis, w.G)
    assert np.abs(L - Lr).max() > 1e-3


def test_planted_dropped_key_is_caught(monkeypatch):
    import oracle.attention as A
    w, x, m, t, c = small_case(seed=10)
    Q, Kp, Vp = _np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"])
    pt = x["page_table"].numpy()
    real = A._key_ids
    monkeypatch.setattr(A, "_key_ids", lambda row, cnt, B: real(row, cnt, B)[:-1])
    O, L = oracle.oracle_chunk_attention(Q, Kp, Vp, pt, t, c, w.prefix_len)
    monkeypatch.undo()
    vis = token_visibility(t, c, w.Hq, w.Hkv, w.prefix_len, w.chunk_len, w.block, w.nKblk)
    Or, Lr = sdpa_reference(Q, oracle.depage(Kp, pt, w.nKblk), oracle.depage(Vp, pt, w.nKblk),
                            vis, w.G)
    assert np.abs(L - Lr).max() > 1e-6


# ---- unaligned prefix / chunk lengths and batches of sequences

def unaligned_case(seed, Hq=4, Hkv=2, d=16, B=8, P=21, Lc=13, rho=0.3):
    w = workloads.Workload("u", Hq, Hkv, d, "fp32", P, Lc, B, "bernoulli", rho=rho, seed=seed)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    t, c = oracle.oracle_tables(m, Hkv)
    return w, x, m, t, c


@pytest.mark.parametrize("P,Lc", [(21, 13), (0, 5), (7, 1), (8, 9), (3, 30)])
def test_unaligned_token_masked_sdpa(P, Lc):
    w, x, m, t, c = unaligned_case(seed=P + Lc, P=P, Lc=Lc)
    assert w.nKblk == -(-(P + Lc) // w.block)
    Q, Kp, Vp = _np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"])
    pt = x["page_table"].numpy()
    O, L = oracle.oracle_chunk_attention(Q, Kp, Vp, pt, t, c, P)
    Kf, Vf = oracle.depage(Kp, pt, w.nKblk), oracle.depage(Vp, pt, w.nKblk)
    vis = token_visibility(t, c, w.Hq, w.Hkv, P, Lc, w.block, w.nKblk)
    Or, Lr = sdpa_reference(Q, Kf, Vf, vis, w.G)
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-10)
    np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-10)


def test_unaligned_brute_force():
    w, x, m, t, c = unaligned_case(seed=3, Hq=2, Hkv=1, d=4, B=4, P=6, Lc=5)
    args = (_np(x["Q"]), _np(x["K_pages"]), _np(x["V_pages"]), x["page_table"].numpy(), t, c, 6)
    O, L = oracle.oracle_chunk_attention(*args)
    Ob, Lb = oracle.brute_force_attention(args[0].tolist(), args[1].tolist(), args[2].tolist(),
                                          *args[3:])
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


def test_unaligned_masks_select_the_last_live_block():
    """Q-block qb of a chunk at prefix P reaches block (P + last token of qb) // B."""
    last = workloads.last_live_block(21, 13, 8)        # Q-blocks: tokens 0-7, 8-12
    assert last.tolist() == [(21 + 7) // 8, (21 + 12) // 8]
    live = workloads.causal_live(0, 2, 5, last)
    assert live.sum(axis=1).tolist() == [4, 5]


def test_unaligned_chunk_composition_equals_one_shot_causal():
    """All-ones masks over chunks of ragged lengths reproduce full causal attention."""
    Hq, Hkv, d, B = 4, 2, 16, 8
    lens = [5, 13, 1, 9, 20]
    T = sum(lens)
    rng = np.random.default_rng(12)
    Qall = rng.standard_normal((T, Hq, d))
    nKall = -(-T // B)
    pages_k = rng.standard_normal((nKall + 2, Hkv, B, d))
    pages_v = rng.standard_normal((nKall + 2, Hkv, B, d))
    pt_all = rng.permutation(nKall + 2)[:nKall]
    Kf = oracle.depage(pages_k, pt_all, nKall)[:, :T]
    Vf = oracle.depage(pages_v, pt_all, nKall)[:, :T]
    causal = np.arange(T)[None, :] <= np.arange(T)[:, None]
    Oref, Lref = sdpa_reference(Qall, Kf, Vf, np.broadcast_to(causal, (Hq, T, T)).copy(), Hq // Hkv)
    P = 0
    for Lc in lens:
        nQ, nK = -(-Lc // B), -(-(P + Lc) // B)
        m = workloads.ones_mask(Hq, P // B, nQ, nK, workloads.last_live_block(P, Lc, B))
        t, c = oracle.oracle_tables(m, Hkv)
        O, L = oracle.oracle_chunk_attention(Qall[P:P + Lc], pages_k, pages_v, pt_all[:nK], t, c, P)
        np.testing.assert_allclose(O, Oref[P:P + Lc], atol=1e-10)
        np.testing.assert_allclose(L, Lref[:, P:P + Lc], atol=1e-10)
        P += Lc


def test_varlen_equals_independent_sequences():
    """A batch over one page pool = each sequence on its own (SDPA per sequence)."""
    Hq, Hkv, d, B = 4, 2, 8, 8
    seqs = [(19, 6), (0, 17), (40, 1), (8, 8)]          # (prefix, chunk)
    rng = np.random.default_rng(5)
    nKs = [-(-(P + L) // B) for P, L in seqs]
    num_pages = sum(nKs) + 3
    perm = rng.permutation(num_pages)
    Kp = rng.standard_normal((num_pages, Hkv, B, d))
    Vp = rng.standard_normal((num_pages, Hkv, B, d))
    cu_q = np.concatenate([[0], np.cumsum([L for _, L in seqs])])
    cu_pages = np.concatenate([[0], np.cumsum(nKs)])
    Q = rng.standard_normal((cu_q[-1], Hq, d))
    tables, counts = [], []
    for s, (P, L) in enumerate(seqs):
        m = workloads.bernoulli_mask(Hq, P // B, -(-L // B), nKs[s], 0.4, seed=s,
                                     last=workloads.last_live_block(P, L, B))
        t, c = oracle.oracle_tables(m, Hkv)
        tables.append(t.reshape(-1))
        counts.append(c)
    O, LSE = oracle.oracle_varlen(Q, Kp, Vp, cu_q, [P for P, _ in seqs], perm[:cu_pages[-1]],
                                  cu_pages, np.concatenate(tables), np.stack(counts))
    for s, (P, L) in enumerate(seqs):
        pt = perm[cu_pages[s]:cu_pages[s + 1]]
        t = tables[s].reshape(Hkv, nKs[s])
        Kf, Vf = oracle.depage(Kp, pt, nKs[s]), oracle.depage(Vp, pt, nKs[s])
        vis = token_visibility(t, counts[s], Hq, Hkv, P, L, B, nKs[s])
        Or, Lr = sdpa_reference(Q[cu_q[s]:cu_q[s + 1]], Kf, Vf, vis, Hq // Hkv)
        np.testing.assert_allclose(O[cu_q[s]:cu_q[s + 1]], Or, atol=1e-10)
        np.testing.assert_allclose(LSE[:, cu_q[s]:cu_q[s + 1]], Lr, atol=1e-10)
