"""Work and traffic accounting for throughput reporting (host side, numpy).

FLOPs count 4 * B^2 * d per live (query head, Q-block, KV block) pair: two
B x B x d contractions (Q K^T and P V) at 2 FLOPs per multiply-add.  A pair
is live when the KV block can hold a key visible to the Q-block
(kb <= nPblk + qb); diagonal blocks are counted in full.  "Selected" keeps
only the pairs whose KV block is in the group's table.
"""
import numpy as np


def selected_pairs(tables, counts, Hq, nPblk, nQblk):
    tables = np.asarray(tables)
    counts = np.asarray(counts)
    Hkv = tables.shape[0]
    G = Hq // Hkv
    total = 0
    diag = nPblk + np.arange(nQblk)
    for g in range(Hkv):
        row = np.sort(tables[g, :int(counts[g])])
        live = np.searchsorted(row, diag, side="right")  # entries <= diagonal, per Q-block
        total += G * int(live.sum())
    return total


def selected_pairs_pl(tables, counts, Hq, P, L, B):
    """selected_pairs for any prefix P and chunk length L: Q-block qb (chunk
    tokens [qb B, min(qb B + B, L))) is live against the table entries up to
    block (P + its last token) // B."""
    tables = np.asarray(tables)
    counts = np.asarray(counts)
    Hkv = tables.shape[0]
    G = Hq // Hkv
    nQ = -(-L // B)
    last = (P + np.minimum(np.arange(nQ) * B + B - 1, L - 1)) // B
    total = 0
    for g in range(Hkv):
        row = np.sort(tables[g, :int(counts[g])])
        total += G * int(np.searchsorted(row, last, side="right").sum())
    return total


def selected_flops_pl(tables, counts, Hq, P, L, B, head_dim):
    return 4.0 * B * B * head_dim * selected_pairs_pl(tables, counts, Hq, P, L, B)


def dense_pairs(Hq, nPblk, nQblk):
    return Hq * int(sum(nPblk + qb + 1 for qb in range(nQblk)))


def selected_flops(tables, counts, Hq, nPblk, nQblk, block, head_dim):
    return 4.0 * block * block * head_dim * selected_pairs(tables, counts, Hq, nPblk, nQblk)


def dense_flops(Hq, nPblk, nQblk, block, head_dim):
    return 4.0 * block * block * head_dim * dense_pairs(Hq, nPblk, nQblk)


def builder_bytes(nb, Hq, Hkv, nQblk, nKblk, bits=False):
    """Algorithmic bytes of one table-builder launch: mask read (one byte per block, or
    one bit packed in 32-bit words) + tables + counts written."""
    mask = Hq * nQblk * (4 * ((nKblk + 31) // 32) if bits else nKblk)
    return nb * (mask + Hkv * nKblk * 4 + Hkv * 4)
