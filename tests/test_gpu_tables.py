"""GPU parity of the table builder (ca_build_tables*) against the oracle:
bit-exact on the configs' masks and on edge cases (empty, full, single bit,
ragged nKblk, G = 1, nQblk = 1, unclipped masks, unaligned mask pointers,
batched launches)."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsc():
    import block_sparse_chunked_b200
    return block_sparse_chunked_b200


def run(bsc, m_np, Hkv, dtype=torch.uint8):
    m = torch.from_numpy(np.ascontiguousarray(m_np)).to(dtype).cuda()
    t, c = bsc.build_tables(m, Hkv)
    torch.cuda.synchronize()
    return t.cpu().numpy(), c.cpu().numpy()


def assert_exact(bsc, m_np, Hkv, dtype=torch.uint8):
    t, c = run(bsc, m_np, Hkv, dtype)
    to, co = oracle.oracle_tables(m_np, Hkv)
    assert np.array_equal(c, co)
    assert np.array_equal(t, to)


@pytest.mark.parametrize("name", ["tiny", "llama16k", "ctx128k"])
def test_configs_bit_exact(bsc, name):
    w = workloads.get_config(name)
    assert_exact(bsc, workloads.mask_for(w), w.Hkv)


@pytest.mark.parametrize("c", [0, 1, 7, 31])
def test_sweep_chunks_bit_exact(bsc, c):
    w = workloads.sweep_chunk(c)
    assert_exact(bsc, workloads.mask_for(w), w.Hkv)


@pytest.mark.parametrize("block,rho,corr", [(64, 0.05, 0.0), (64, 0.2, 1.0), (128, 0.1, 0.5)])
def test_density_cells_bit_exact(bsc, block, rho, corr):
    w = workloads.density_cell(rho, corr, block=block)
    assert_exact(bsc, workloads.mask_for(w), w.Hkv)


SHAPES = [(4, 1, 4, 20), (4, 2, 3, 33), (8, 8, 5, 7), (6, 2, 1, 64), (8, 2, 2, 1), (1, 1, 1, 1),
          (16, 4, 7, 100), (32, 8, 32, 1023), (32, 8, 32, 1025), (8, 1, 3, 4097),
          (4, 2, 2, 65536), (2, 1, 1, 8191), (12, 3, 9, 300)]


@pytest.mark.parametrize("Hq,Hkv,nQ,nK", SHAPES)
@pytest.mark.parametrize("rho", [0.0, 0.01, 0.3, 1.0])
def test_random_shapes_bit_exact(bsc, Hq, Hkv, nQ, nK, rho):
    rng = np.random.default_rng(Hq * 7919 + nK * 31 + nQ + int(rho * 1000))
    m = (rng.random((Hq, nQ, nK)) < rho).astype(np.uint8)
    assert_exact(bsc, m, Hkv)


def test_single_bit_everywhere(bsc):
    Hq, Hkv, nQ, nK = 8, 2, 3, 300
    rng = np.random.default_rng(5)
    for _ in range(20):
        m = np.zeros((Hq, nQ, nK), np.uint8)
        m[rng.integers(Hq), rng.integers(nQ), rng.integers(nK)] = rng.integers(1, 256)
        assert_exact(bsc, m, Hkv)


def test_bool_input_and_nonunit_bytes(bsc):
    rng = np.random.default_rng(6)
    m = (rng.random((8, 4, 96)) < 0.1)
    assert_exact(bsc, m, 2, dtype=torch.bool)
    mb = (rng.integers(0, 256, (8, 4, 96)) * (rng.random((8, 4, 96)) < 0.1)).astype(np.uint8)
    assert_exact(bsc, mb, 4)


def test_unaligned_mask_pointer(bsc):
    """A view starting one byte into a buffer forces the byte-load path."""
    rng = np.random.default_rng(7)
    m = (rng.random((8, 4, 128)) < 0.05).astype(np.uint8)
    buf = torch.zeros(m.size + 1, dtype=torch.uint8, device="cuda")
    buf[1:] = torch.from_numpy(m.reshape(-1)).cuda()
    view = buf[1:].view(8, 4, 128)
    t, c = bsc.build_tables(view, 2)
    to, co = oracle.oracle_tables(m, 2)
    assert np.array_equal(t.cpu().numpy(), to) and np.array_equal(c.cpu().numpy(), co)


def test_unclipped_mask(bsc):
    w = workloads.get_config("llama16k")
    assert_exact(bsc, workloads.mask_for(w, clip=False), w.Hkv)


def test_batched_matches_per_mask(bsc):
    w = workloads.get_config("ctx128k")
    masks = np.stack([workloads.mask_for(w, seed=s) for s in range(5)])
    mt = torch.from_numpy(masks).cuda()
    t, c = bsc.build_tables_batched(mt, w.Hkv)
    t, c = t.cpu().numpy(), c.cpu().numpy()
    for s in range(5):
        to, co = oracle.oracle_tables(masks[s], w.Hkv)
        assert np.array_equal(t[s], to) and np.array_equal(c[s], co)


def test_repeatable_and_overwrites_stale_output(bsc):
    w = workloads.get_config("llama16k")
    m = torch.from_numpy(workloads.mask_for(w)).cuda()
    t = torch.full((w.Hkv, w.nKblk), 12345, dtype=torch.int32, device="cuda")
    c = torch.full((w.Hkv,), 777, dtype=torch.int32, device="cuda")
    bsc.build_tables(m, w.Hkv, t, c)
    t1, c1 = t.clone(), c.clone()
    bsc.build_tables(m, w.Hkv, t, c)
    assert torch.equal(t, t1) and torch.equal(c, c1)
    to, co = oracle.oracle_tables(workloads.mask_for(w), w.Hkv)
    assert np.array_equal(t.cpu().numpy(), to)


@pytest.mark.parametrize("nb,Hq,Hkv,nQ,nK,rho", [
    (16, 32, 8, 32, 2048, None),      # 128 (mask, group) units of the 128K config
    (40, 8, 4, 3, 1000, 0.05),        # ragged width: 4-byte loads
    (130, 4, 1, 2, 37, 0.3),          # odd width: 1-byte loads
    (32, 8, 4, 2, 20000, 0.01),       # many units and a wide table: 3 slabs per cluster
    (64, 2, 2, 1, 33000, 0.001),      # wider than 4 slabs: the cluster grows to 5
])
def test_batched_many_masks_and_wide_tables(bsc, nb, Hq, Hkv, nQ, nK, rho):
    if rho is None:
        w = workloads.get_config("ctx128k")
        masks = np.stack([workloads.mask_for(w, seed=s) for s in range(nb)])
    else:
        rng = np.random.default_rng(nb + nK)
        masks = (rng.random((nb, Hq, nQ, nK)) < rho).astype(np.uint8)
    t, c = bsc.build_tables_batched(torch.from_numpy(masks).cuda(), Hkv)
    t, c = t.cpu().numpy(), c.cpu().numpy()
    for s in range(nb):
        to, co = oracle.oracle_tables(masks[s], Hkv)
        assert np.array_equal(t[s], to) and np.array_equal(c[s], co), s
