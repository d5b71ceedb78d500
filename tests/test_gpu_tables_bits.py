"""GPU parity of the bit-packed table builder (ca_build_tables_bits) against
the oracle: bit-exact on the configs' masks, ragged widths, stray bits past
nKblk, unaligned word buffers and batches."""
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


def run_bits(bsc, bits_np, Hkv, nK):
    b = torch.from_numpy(np.ascontiguousarray(bits_np).view(np.int32)).cuda()
    if b.dim() == 3:
        b = b.unsqueeze(0)
    t, c = bsc.build_tables_bits(b, Hkv, nK)
    return t.cpu().numpy(), c.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "llama16k", "ctx128k"])
def test_configs_bit_exact(bsc, name):
    w = workloads.get_config(name)
    m = workloads.mask_for(w)
    t, c = run_bits(bsc, workloads.pack_mask_bits(m), w.Hkv, w.nKblk)
    to, co = oracle.oracle_tables(m, w.Hkv)
    assert np.array_equal(t[0], to) and np.array_equal(c[0], co)


@pytest.mark.parametrize("Hq,Hkv,nQ,nK", [(4, 1, 4, 20), (8, 2, 3, 33), (8, 8, 5, 7),
                                          (32, 8, 32, 1023), (4, 2, 2, 65536), (12, 3, 9, 300),
                                          (2, 1, 1, 1), (16, 4, 7, 129)])
@pytest.mark.parametrize("rho", [0.0, 0.01, 0.3, 1.0])
def test_random_shapes_bit_exact(bsc, Hq, Hkv, nQ, nK, rho):
    rng = np.random.default_rng(Hq * 131 + nK + int(rho * 100))
    m = (rng.random((Hq, nQ, nK)) < rho).astype(np.uint8)
    bits = workloads.pack_mask_bits(m)
    if nK % 32:  # stray bits past nKblk must be ignored
        bits[..., -1] |= np.uint32(0xFFFFFFFF) << np.uint32(nK % 32)
    t, c = run_bits(bsc, bits, Hkv, nK)
    to, co = oracle.oracle_tables(m, Hkv)
    assert np.array_equal(t[0], to) and np.array_equal(c[0], co)


def test_batched_and_unaligned(bsc):
    w = workloads.get_config("ctx128k")
    masks = np.stack([workloads.mask_for(w, seed=s) for s in range(3)])
    bits = workloads.pack_mask_bits(masks)
    t, c = run_bits(bsc, bits, w.Hkv, w.nKblk)
    for s in range(3):
        to, co = oracle.oracle_tables(masks[s], w.Hkv)
        assert np.array_equal(t[s], to) and np.array_equal(c[s], co)
    # a word buffer starting 4 bytes into an allocation takes the 4-byte load path
    flat = torch.from_numpy(bits.reshape(-1).view(np.int32)).cuda()
    buf = torch.zeros(flat.numel() + 1, dtype=torch.int32, device="cuda")
    buf[1:] = flat
    view = buf[1:].view(bits.shape)
    t2, c2 = bsc.build_tables_bits(view, w.Hkv, w.nKblk)
    assert np.array_equal(t2.cpu().numpy(), t) and np.array_equal(c2.cpu().numpy(), c)
