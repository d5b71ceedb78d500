"""Block-Union KV selection, written as its set definition (float-free).

Source: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
Selection", Abstract — masks are turned into per-group KV block tables by a
Q-block union and an intra-group union, producing the minimal tables that keep
every KV block the masks select.

Definition used here:
  U[g]      = { kb : exists h with h // G == g, exists qb : M[h, qb, kb] != 0 }
  tables[g] = sorted(U[g]) followed by -1 up to nKblk entries
  counts[g] = |U[g]|
"""
import numpy as np


def oracle_tables(mask, Hkv):
    """mask uint8/bool [Hq, nQblk, nKblk] -> (tables int32 [Hkv, nKblk], counts int32 [Hkv])."""
    mask = np.asarray(mask)
    Hq, nQblk, nKblk = mask.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    tables = np.full((Hkv, nKblk), -1, dtype=np.int32)
    counts = np.zeros(Hkv, dtype=np.int32)
    for g in range(Hkv):
        heads = mask[g * G:(g + 1) * G]                 # the group's heads
        selected = (heads != 0).any(axis=(0, 1))        # exists (h, qb)
        U = np.flatnonzero(selected)                    # ascending block ids
        counts[g] = U.size
        tables[g, :U.size] = U
    return tables, counts


def brute_force_tables(mask, Hkv):
    """Triple loop over (h, qb, kb) with Python sets; tiny inputs only."""
    Hq, nQblk, nKblk = np.asarray(mask).shape
    G = Hq // Hkv
    sets = [set() for _ in range(Hkv)]
    for h in range(Hq):
        for qb in range(nQblk):
            for kb in range(nKblk):
                if mask[h][qb][kb]:
                    sets[h // G].add(kb)
    tables = [[-1] * nKblk for _ in range(Hkv)]
    counts = [0] * Hkv
    for g in range(Hkv):
        s = sorted(sets[g])
        counts[g] = len(s)
        tables[g][:len(s)] = s
    return np.array(tables, dtype=np.int32), np.array(counts, dtype=np.int32)


def unpack_mask_bits(bits, nKblk):
    """uint32 words [..., W] -> uint8 mask [..., nKblk]: block kb is bit (kb mod 32),
    least significant first, of word kb // 32; bits at or past nKblk are ignored."""
    words = np.asarray(bits, dtype=np.uint32)
    out = np.zeros(words.shape[:-1] + (nKblk,), dtype=np.uint8)
    for kb in range(nKblk):
        out[..., kb] = (words[..., kb // 32] >> np.uint32(kb % 32)) & np.uint32(1)
    return out


def oracle_tables_bits(bits, Hkv, nKblk):
    """Tables from bit-packed masks: the same set definition on the unpacked mask."""
    return oracle_tables(unpack_mask_bits(bits, nKblk), Hkv)
