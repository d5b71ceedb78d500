"""The seeded input recipe (host only): the vertical-slash masks carry their
sink, local window and column statistics, the page table is a permutation,
and bit packing is the little-endian word layout the builder reads."""
import numpy as np

import workloads


def test_vslash_structure_and_column_density():
    w = workloads.Workload("v", 32, 8, 128, "bf16", 8192 * 4, 2048, 64, "vslash", rho=0.05,
                           corr=0.7, window=8, seed=3)
    m = workloads.mask_for(w)
    last = workloads.last_live_block(w.prefix_len, w.chunk_len, w.block)
    for qb in range(w.nQblk):
        assert m[:, qb, 0].all()                                   # sink block
        lo = max(0, last[qb] - w.window + 1)
        assert m[:, qb, lo:last[qb] + 1].all()                     # local window to the diagonal
        assert not m[:, qb, last[qb] + 1:].any()                   # nothing past the diagonal
    # columns outside sink and window: per-head density close to rho_col
    cols = m[:, 0, 1:last[0] - w.window + 1].astype(float)
    assert abs(cols.mean() - w.rho) < 0.01


def test_vslash_full_correlation_shares_columns_within_a_group():
    w = workloads.Workload("v", 8, 2, 64, "bf16", 4096, 256, 64, "vslash", rho=0.1, corr=1.0,
                           window=2, seed=1)
    m = workloads.mask_for(w)
    G = w.Hq // w.Hkv
    for g in range(w.Hkv):
        heads = m[g * G:(g + 1) * G]
        assert all(np.array_equal(heads[0], heads[i]) for i in range(1, G))


def test_page_table_is_a_permutation_prefix():
    w = workloads.get_config("llama16k")
    x = workloads.make_qkv_pages(w, num_pages=w.nKblk + 50)
    pt = x["page_table"].numpy()
    assert len(pt) == w.nKblk and len(set(pt.tolist())) == w.nKblk
    assert pt.min() >= 0 and pt.max() < w.nKblk + 50


def test_pack_bits_little_endian_words():
    m = np.zeros((1, 1, 40), np.uint8)
    m[0, 0, [0, 5, 31, 32, 39]] = 1
    b = workloads.pack_mask_bits(m)
    assert b.shape == (1, 1, 2)
    assert int(b[0, 0, 0]) == (1 << 0) | (1 << 5) | (1 << 31)
    assert int(b[0, 0, 1]) == (1 << 0) | (1 << 7)
