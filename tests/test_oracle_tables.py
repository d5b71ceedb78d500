"""Pins for the float-free table oracle (Q-block union + intra-group union).

Source: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
Selection", Abstract.  Pinned by a hand-derived case, brute force, the
coverage / minimality invariants and the special cases the definition reduces
to.
"""
import json
import os

import numpy as np
import pytest

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_derived_case():
    g = json.load(open(os.path.join(GOLD, "tables_hand.json")))
    t, c = oracle.oracle_tables(np.array(g["mask"], dtype=np.uint8), g["Hkv"])
    assert t.tolist() == g["tables"]
    assert c.tolist() == g["counts"]


SHAPES = [(4, 1, 4, 20), (4, 2, 3, 33), (8, 8, 5, 7), (6, 2, 1, 64), (8, 2, 2, 1),
          (1, 1, 1, 1), (16, 4, 7, 100)]


@pytest.mark.parametrize("Hq,Hkv,nQ,nK", SHAPES)
@pytest.mark.parametrize("rho", [0.0, 0.02, 0.3, 1.0])
def test_against_brute_force(Hq, Hkv, nQ, nK, rho):
    rng = np.random.default_rng(Hq * 1000 + nK + int(rho * 100))
    m = (rng.random((Hq, nQ, nK)) < rho).astype(np.uint8)
    t, c = oracle.oracle_tables(m, Hkv)
    tb, cb = oracle.brute_force_tables(m.tolist(), Hkv)
    assert np.array_equal(t, tb) and np.array_equal(c, cb)


def check_invariants(m, Hkv, t, c):
    Hq, nQ, nK = m.shape
    G = Hq // Hkv
    for g in range(Hkv):
        n = int(c[g])
        row = t[g]
        assert np.all(row[n:] == -1)
        ent = row[:n]
        assert np.all(np.diff(ent) > 0), "strictly increasing"
        assert np.all((ent >= 0) & (ent < nK))
        sel = m[g * G:(g + 1) * G] != 0
        # coverage: every selected (h, qb, kb) has kb in the group table
        need = np.flatnonzero(sel.any(axis=(0, 1)))
        assert set(need.tolist()) <= set(ent.tolist())
        # minimality: every entry is selected by some (h, qb) of its group
        for kb in ent.tolist():
            assert sel[:, :, kb].any()
        assert n == len(need)


@pytest.mark.parametrize("name", ["tiny", "llama16k", "ctx128k"])
def test_invariants_on_configs(name):
    w = workloads.get_config(name)
    m = workloads.mask_for(w)
    t, c = oracle.oracle_tables(m, w.Hkv)
    check_invariants(m, w.Hkv, t, c)


def test_invariants_unclipped_mask():
    w = workloads.get_config("tiny")
    m = workloads.mask_for(w, clip=False)
    assert (m & ~workloads.causal_live(w.nPblk, w.nQblk, w.nKblk)[None]).any()
    t, c = oracle.oracle_tables(m, w.Hkv)
    check_invariants(m, w.Hkv, t, c)


def test_all_ones_gives_every_block():
    m = np.ones((8, 3, 45), np.uint8)
    t, c = oracle.oracle_tables(m, 2)
    assert c.tolist() == [45, 45]
    assert np.array_equal(t, np.tile(np.arange(45, dtype=np.int32), (2, 1)))


def test_all_zeros_gives_empty_tables():
    t, c = oracle.oracle_tables(np.zeros((4, 2, 9), np.uint8), 2)
    assert c.tolist() == [0, 0] and np.all(t == -1)


def test_single_bit():
    m = np.zeros((8, 4, 77), np.uint8)
    m[5, 2, 70] = 1
    t, c = oracle.oracle_tables(m, 4)       # G = 2: head 5 -> group 2
    assert c.tolist() == [0, 0, 1, 0]
    assert t[2, 0] == 70 and np.all(t[2, 1:] == -1)


def test_group_of_one_is_q_union_only():
    rng = np.random.default_rng(3)
    m = (rng.random((5, 6, 40)) < 0.1).astype(np.uint8)
    t, c = oracle.oracle_tables(m, 5)
    for h in range(5):
        expect = sorted({kb for qb in range(6) for kb in range(40) if m[h, qb, kb]})
        assert t[h, :c[h]].tolist() == expect


def test_one_q_block_is_group_union_only():
    rng = np.random.default_rng(4)
    m = (rng.random((8, 1, 40)) < 0.1).astype(np.uint8)
    t, c = oracle.oracle_tables(m, 2)
    for g in range(2):
        expect = sorted({kb for h in range(4 * g, 4 * g + 4) for kb in range(40) if m[h, 0, kb]})
        assert t[g, :c[g]].tolist() == expect


def test_nonzero_bytes_count_as_selected():
    m = np.zeros((2, 1, 4), np.uint8)
    m[0, 0, 1] = 255
    m[1, 0, 3] = 2
    t, c = oracle.oracle_tables(m, 1)
    assert t[0].tolist() == [1, 3, -1, -1] and c.tolist() == [2]


def test_planted_dropped_group_head_is_caught(monkeypatch):
    """A union that forgets the last head of each group must fail the brute-force pin."""
    import oracle.tables as T
    real = T.oracle_tables

    def wrong(mask, Hkv):
        mask = np.array(mask)
        G = mask.shape[0] // Hkv
        mask[G - 1::G] = 0
        return real(mask, Hkv)

    rng = np.random.default_rng(9)
    m = (rng.random((8, 2, 30)) < 0.2).astype(np.uint8)
    tw, cw = wrong(m, 2)
    tb, cb = oracle.brute_force_tables(m.tolist(), 2)
    assert not (np.array_equal(tw, tb) and np.array_equal(cw, cb))


def test_unpack_bits_hand_example():
    """Word 0x00000005 selects blocks 0 and 2; word 1 bit 1 (0x2) selects block 33;
    a set bit past nKblk = 35 (block 34+) is ignored."""
    bits = np.array([[[0x00000005, 0x00000002 | 0x00000008]]], dtype=np.uint32)  # bit 3 of w1 = block 35
    m = oracle.unpack_mask_bits(bits, 35)
    assert np.flatnonzero(m[0, 0]).tolist() == [0, 2, 33]


@pytest.mark.parametrize("nK", [1, 31, 32, 33, 100, 2048])
def test_pack_unpack_roundtrip(nK):
    rng = np.random.default_rng(nK)
    m = (rng.random((3, 2, nK)) < 0.3).astype(np.uint8)
    bits = workloads.pack_mask_bits(m)
    assert bits.shape == (3, 2, (nK + 31) // 32) and bits.dtype == np.uint32
    assert np.array_equal(oracle.unpack_mask_bits(bits, nK), m)
    t1, c1 = oracle.oracle_tables_bits(bits, 1, nK)
    t2, c2 = oracle.oracle_tables(m, 1)
    assert np.array_equal(t1, t2) and np.array_equal(c1, c2)


@pytest.mark.parametrize("name", ["tiny", "llama16k", "ctx128k"])
def test_aligned_configs_last_live_block_is_the_diagonal(name):
    """For block-aligned prefix and chunk the general rule gives the diagonal
    block nPblk + qb, so the aligned configs' masks are what they always were."""
    w = workloads.get_config(name)
    last = workloads.last_live_block(w.prefix_len, w.chunk_len, w.block)
    assert last.tolist() == (w.nPblk + np.arange(w.nQblk)).tolist()
    live = workloads.causal_live(w.nPblk, w.nQblk, w.nKblk)
    assert np.array_equal(live, workloads.causal_live(w.nPblk, w.nQblk, w.nKblk, last))
