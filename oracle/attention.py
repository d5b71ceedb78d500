"""Chunk attention over the selected KV blocks of a paged cache, float64.

Source: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
Selection", Abstract — chunked prefill; the per-group block tables decide
which KV blocks every query of the group reads; selected blocks are accessed
in place (here: through the page table) without compacting the KV.

For head h (group g = h // G), chunk query i at absolute position p = P + i:
  J      = { j : j // B in tables[g][:counts[g]],  j <= p }
  s_j    = (Q[i, h] . K[g, j]) / sqrt(d)
  LSE    = ln sum_{j in J} exp(s_j)                  (natural log)
  O[i,h] = sum_{j in J} exp(s_j - LSE) V[g, j]
where K[g, j] = K_pages[page_table[j // B], g, j % B].  An empty J gives
O = 0 and LSE = -inf.  Every query of the group reads every block of its
group's table (the table is a selection of KV, not a per-query plan), and the
token-level causal rule j <= p removes keys past the query.
"""
import math

import numpy as np


def depage(pages, page_table, nKblk):
    """[num_pages, Hkv, B, d] pages + page table -> contiguous [Hkv, nKblk*B, d] float64."""
    pages = np.asarray(pages, dtype=np.float64)
    _, Hkv, B, d = pages.shape
    out = np.empty((Hkv, nKblk * B, d), dtype=np.float64)
    for kb in range(nKblk):
        out[:, kb * B:(kb + 1) * B, :] = pages[int(page_table[kb])]
    return out


def _page(pages, p, g):
    """One [B, d] page as float64; accepts numpy arrays or torch CPU tensors (e.g. bf16)."""
    x = pages[p, g]
    if hasattr(x, "double"):
        return x.double().numpy()
    return np.asarray(x, dtype=np.float64)


def _key_ids(table_row, count, B):
    blocks = np.asarray(table_row[:count], dtype=np.int64)
    return (blocks[:, None] * B + np.arange(B)[None, :]).reshape(-1)


def _attend(q, Kj, Vj, key_pos, pos, d):
    """q [n, d] rows at absolute positions pos [n] against gathered keys Kj/Vj [T, d]
    whose absolute positions are key_pos [T] (ascending)."""
    n = q.shape[0]
    O = np.zeros((n, Vj.shape[1]))
    LSE = np.full(n, -np.inf)
    if key_pos.size == 0:
        return O, LSE
    s = (q @ Kj.T) / math.sqrt(d)                    # [n, T]
    visible = key_pos[None, :] <= pos[:, None]
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=1)
    live = np.isfinite(m)
    msafe = np.where(live, m, 0.0)
    e = np.exp(s - msafe[:, None])                   # exp(-inf) = 0 for hidden keys
    l = e.sum(axis=1)
    LSE[live] = msafe[live] + np.log(l[live])
    O[live] = (e[live] / l[live][:, None]) @ Vj
    return O, LSE


def oracle_chunk_attention(Q, K_pages, V_pages, page_table, tables, counts, prefix_len,
                           rows_per_step=256):
    """Q [L_c, Hq, d]; pages [num_pages, Hkv, B, d] -> O [L_c, Hq, d], LSE [Hq, L_c] (float64)."""
    Q = np.asarray(Q, dtype=np.float64)
    L_c, Hq, d = Q.shape
    Hkv, B = np.asarray(K_pages).shape[1], np.asarray(K_pages).shape[2]
    nKblk = -(-(prefix_len + L_c) // B)  # blocks holding positions 0 .. P + L_c - 1
    G = Hq // Hkv
    K = depage(K_pages, page_table, nKblk)
    V = depage(V_pages, page_table, nKblk)
    O = np.zeros((L_c, Hq, d))
    LSE = np.full((Hq, L_c), -np.inf)
    for h in range(Hq):
        g = h // G
        J = _key_ids(tables[g], int(counts[g]), B)
        Kj, Vj = K[g][J], V[g][J]
        for i0 in range(0, L_c, rows_per_step):
            i1 = min(L_c, i0 + rows_per_step)
            pos = prefix_len + np.arange(i0, i1)
            o, lse = _attend(Q[i0:i1, h, :], Kj, Vj, J, pos, d)
            O[i0:i1, h, :] = o
            LSE[h, i0:i1] = lse
    return O, LSE


def oracle_varlen(Q, K_pages, V_pages, cu_q, prefix_len, page_table, cu_pages, tables, counts):
    """A batch of sequences sharing one page pool: sequence s has chunk rows
    cu_q[s] .. cu_q[s+1] of Q, prefix prefix_len[s], page table
    page_table[cu_pages[s] ...] and tables [Hkv, nKblk_s] stored flat from
    Hkv * cu_pages[s]; each is exactly the single-sequence definition.
    Returns O [total_q, Hq, d] and LSE [Hq, total_q]."""
    Q = np.asarray(Q, dtype=np.float64)
    total_q, Hq, d = Q.shape
    Hkv, B = np.asarray(K_pages).shape[1], np.asarray(K_pages).shape[2]
    tables = np.asarray(tables)
    counts = np.asarray(counts).reshape(-1, Hkv)
    O = np.zeros((total_q, Hq, d))
    LSE = np.full((Hq, total_q), -np.inf)
    for s in range(len(prefix_len)):
        q0, q1, P = int(cu_q[s]), int(cu_q[s + 1]), int(prefix_len[s])
        if q1 == q0:
            continue
        nK = -(-(P + q1 - q0) // B)
        p0 = int(cu_pages[s])
        pt = np.asarray(page_table)[p0:p0 + nK]
        tab = tables[Hkv * p0:Hkv * p0 + Hkv * nK].reshape(Hkv, nK)
        o, lse = oracle_chunk_attention(Q[q0:q1], K_pages, V_pages, pt, tab, counts[s], P)
        O[q0:q1] = o
        LSE[:, q0:q1] = lse
    return O, LSE


def oracle_rows(Q, K_pages, V_pages, page_table, tables, counts, prefix_len, rows):
    """The same definition for a sample of (h, i) rows only.

    Reads just the pages of one group's selected blocks at a time, so it stays
    cheap at full 128K size.  Returns O [len(rows), d] and LSE [len(rows)].
    """
    Q = np.asarray(Q)
    L_c, Hq, d = Q.shape
    Hkv, B = K_pages.shape[1], K_pages.shape[2]
    G = Hq // Hkv
    O = np.zeros((len(rows), d))
    LSE = np.full(len(rows), -np.inf)
    by_group = {}
    for r, (h, i) in enumerate(rows):
        by_group.setdefault(h // G, []).append(r)
    for g, idx in by_group.items():
        cnt = int(counts[g])
        blocks = np.asarray(tables[g][:cnt], dtype=np.int64)
        if cnt:
            Kg = np.concatenate([_page(K_pages, int(page_table[kb]), g) for kb in blocks], axis=0)
            Vg = np.concatenate([_page(V_pages, int(page_table[kb]), g) for kb in blocks], axis=0)
        else:
            Kg = Vg = np.zeros((0, d))
        J = _key_ids(tables[g], cnt, B)
        for r in idx:
            h, i = rows[r]
            q = np.asarray(Q[i, h], dtype=np.float64)[None]
            o, lse = _attend(q, Kg, Vg, J, np.array([prefix_len + i]), d)
            O[r] = o[0]
            LSE[r] = lse[0]
    return O, LSE


def brute_force_attention(Q, K_pages, V_pages, page_table, tables, counts, prefix_len):
    """Scalar loops over (h, i, j) with Python floats; tiny inputs only."""
    L_c, Hq, d = len(Q), len(Q[0]), len(Q[0][0])
    Hkv, B = len(K_pages[0]), len(K_pages[0][0])
    G = Hq // Hkv
    O = [[[0.0] * d for _ in range(Hq)] for _ in range(L_c)]
    LSE = [[-math.inf] * L_c for _ in range(Hq)]
    for h in range(Hq):
        g = h // G
        for i in range(L_c):
            p = prefix_len + i
            scores, vals = [], []
            for t in range(int(counts[g])):
                kb = int(tables[g][t])
                page = int(page_table[kb])
                for r in range(B):
                    j = kb * B + r
                    if j > p:
                        continue
                    k = K_pages[page][g][r]
                    scores.append(math.fsum(float(Q[i][h][c]) * float(k[c]) for c in range(d))
                                  / math.sqrt(d))
                    vals.append(V_pages[page][g][r])
            if not scores:
                continue
            m = max(scores)
            z = math.fsum(math.exp(s - m) for s in scores)
            lse = m + math.log(z)
            LSE[h][i] = lse
            for c in range(d):
                O[i][h][c] = math.fsum(math.exp(s - lse) * float(v[c]) for s, v in zip(scores, vals))
    return np.array(O), np.array(LSE)


def lse_combine(O_parts, LSE_parts):
    """Merge attention results over disjoint key sets.

    O_parts [S, ..., d], LSE_parts [S, ...]:  LSE = ln sum_s exp(LSE_s),
    O = sum_s exp(LSE_s - LSE) O_s.  All-empty rows stay O = 0, LSE = -inf.
    """
    O_parts = np.asarray(O_parts, dtype=np.float64)
    LSE_parts = np.asarray(LSE_parts, dtype=np.float64)
    m = LSE_parts.max(axis=0)
    live = np.isfinite(m)
    msafe = np.where(live, m, 0.0)
    w = np.exp(LSE_parts - msafe[None])
    tot = w.sum(axis=0)
    LSE = np.where(live, msafe + np.log(np.where(live, tot, 1.0)), -np.inf)
    scale = np.where(live, 1.0, 0.0)[None] * np.exp(LSE_parts - np.where(live, LSE, 0.0)[None])
    O = (scale[..., None] * O_parts).sum(axis=0)
    return O, LSE


def oracle_append_kv(K_pages, V_pages, page_table, K_new, V_new, prefix_len):
    """Writing a chunk into the paged cache: token i of the chunk, at position
    p = prefix_len + i, lands in row p mod B of page page_table[p // B]; the
    rows of that last block after the chunk's last position are cleared to 0
    (empty slots of the sequence's last block).

    Works on numpy arrays or torch CPU tensors (any dtype: a pure copy) and
    returns updated copies of the two page arrays.
    """
    def _copy(x):
        return x.clone() if hasattr(x, "clone") else np.array(x, copy=True)

    K, V = _copy(K_pages), _copy(V_pages)
    B = K.shape[2]
    L = K_new.shape[0]
    for i in range(L):
        p = prefix_len + i
        page = int(page_table[p // B])
        K[page, :, p % B, :] = K_new[i]
        V[page, :, p % B, :] = V_new[i]
    if L > 0:
        last = prefix_len + L - 1
        page = int(page_table[last // B])
        for r in range(last % B + 1, B):
            K[page, :, r, :] = 0
            V[page, :, r, :] = 0
    return K, V
