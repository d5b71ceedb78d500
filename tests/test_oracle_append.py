"""Pins for the paged-cache append oracle (chunked prefill writes the chunk's
keys and values into the accumulated, paged KV cache).

Source: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
Selection", Abstract (chunked prefill over a paged KV cache read in place).
Pinned by a hand-placed case, by reading the result back through the
independent page-to-sequence map (``depage``) and by an untouched-rows check.
"""
import numpy as np
import pytest

import oracle


def test_hand_placed_case():
    # B = 2, three pages, logical block kb -> page [2, 0, 1][kb]; prefix 1, chunk 3:
    # position 1 -> page 2 row 1, position 2 -> page 0 row 0, position 3 -> page 0 row 1.
    K = np.zeros((3, 1, 2, 1))
    V = np.zeros((3, 1, 2, 1))
    kn = np.array([[[10.0]], [[20.0]], [[30.0]]])
    K2, V2 = oracle.oracle_append_kv(K, V, [2, 0, 1], kn, -kn, 1)
    assert K2[:, 0, :, 0].tolist() == [[20.0, 30.0], [0.0, 0.0], [0.0, 10.0]]
    assert V2[:, 0, :, 0].tolist() == [[-20.0, -30.0], [0.0, 0.0], [0.0, -10.0]]
    assert K.sum() == 0  # inputs not modified


@pytest.mark.parametrize("prefix,L,B", [(0, 7, 4), (5, 9, 4), (8, 8, 4), (3, 0, 2), (0, 1, 1),
                                        (63, 130, 64)])
def test_readback_through_depage(prefix, L, B):
    rng = np.random.default_rng(prefix * 131 + L)
    Hkv, d = 2, 3
    nK = max(1, -(-(prefix + L) // B))
    num_pages = nK + 3
    pt = rng.permutation(num_pages)[:nK]
    K = rng.standard_normal((num_pages, Hkv, B, d))
    V = rng.standard_normal((num_pages, Hkv, B, d))
    kn = rng.standard_normal((L, Hkv, d))
    vn = rng.standard_normal((L, Hkv, d))
    K2, V2 = oracle.oracle_append_kv(K, V, pt, kn, vn, prefix)
    seqK, seqV = oracle.depage(K2, pt, nK), oracle.depage(V2, pt, nK)
    oldK = oracle.depage(K, pt, nK)
    for i in range(L):
        assert np.array_equal(seqK[:, prefix + i], kn[i])
        assert np.array_equal(seqV[:, prefix + i], vn[i])
    assert np.array_equal(seqK[:, :prefix], oldK[:, :prefix])  # the prefix is kept
    # pages outside the table are untouched
    other = np.setdiff1d(np.arange(num_pages), pt)
    assert np.array_equal(K2[other], K[other]) and np.array_equal(V2[other], V[other])
    # the rest of the last block is cleared; exactly L + tail rows per head changed
    tail = (B - (prefix + L) % B) % B if L else 0
    if tail:
        seqK0 = oracle.depage(K2, pt, nK)
        assert np.all(seqK0[:, prefix + L:prefix + L + tail] == 0)
    assert int((K2 != K).any(axis=-1).sum()) == (L + tail) * Hkv


def test_hand_placed_tail_is_cleared():
    # B = 4, one page; prefix 1, chunk 2: positions 1, 2 written, position 3 cleared,
    # position 0 (the prefix) kept.
    K = np.full((1, 1, 4, 1), 7.0)
    K2, _ = oracle.oracle_append_kv(K, K, [0], np.array([[[1.0]], [[2.0]]]),
                                    np.array([[[1.0]], [[2.0]]]), 1)
    assert K2[0, 0, :, 0].tolist() == [7.0, 1.0, 2.0, 0.0]


def test_planted_off_by_one_is_caught():
    """Writing at position prefix + i + 1 must fail the depage read-back."""
    rng = np.random.default_rng(1)
    K = rng.standard_normal((4, 1, 4, 2))
    kn = rng.standard_normal((5, 1, 2))
    pt = [3, 1, 0, 2]
    Kw, _ = oracle.oracle_append_kv(K, K, pt, kn, kn, 3)   # correct position 3
    Kp, _ = oracle.oracle_append_kv(K, K, pt, kn, kn, 4)   # planted shift by one
    seq_ok, seq_bad = oracle.depage(Kw, pt, 4), oracle.depage(Kp, pt, 4)
    assert np.array_equal(seq_ok[:, 3], kn[0])
    assert not np.array_equal(seq_bad[:, 3], kn[0])
