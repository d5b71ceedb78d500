"""GPU parity of the fused builder + attention (ca_chunk_attention_masked):
bit-identical O / LSE to the two-launch path on the 128K chunk (same tables,
same schedule), tables written on the side bit-exact against the oracle, and
oracle parity on medium, small-unit (KV-split), unaligned and fp32 shapes."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def bsc():
    import block_sparse_chunked_b200
    return block_sparse_chunked_b200


def bits_of(m):
    return torch.from_numpy(workloads.pack_mask_bits(m).view(np.int32)).cuda()


def fused(bsc, w, x, m, n_splits=0):
    d = {k: v.cuda() for k, v in x.items()}
    t = torch.full((w.Hkv, w.nKblk), 7, dtype=torch.int32, device="cuda")
    c = torch.full((w.Hkv,), 7, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, L = bsc.chunk_attention_masked(d["Q"], d["K_pages"], d["V_pages"], d["page_table"],
                                      bits_of(m), w.prefix_len, n_splits=n_splits, err_flag=err,
                                      tables_out=t, counts_out=c)
    bsc.check(err)
    return O, L, t.cpu().numpy(), c.cpu().numpy()


def compare(O, L, Oo, Lo):
    assert np.array_equal(np.isneginf(L), np.isneginf(Lo))
    fin = np.isfinite(Lo)
    if fin.any():
        assert np.abs(L[fin] - Lo[fin]).max() <= LSE_TOL
    assert np.abs(O - Oo).max() <= O_TOL


@pytest.mark.parametrize("n_splits", [0, 1])
def test_fused_bit_identical_to_two_step_128k(bsc, n_splits):
    """Same kernel, same plan (n_splits 0: the last partial wave in KV pieces;
    1: one CTA per unit), tables built in the CTAs instead of read: bit-identical."""
    w = workloads.get_config("ctx128k")
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, L, t, c = fused(bsc, w, x, m, n_splits=n_splits)
    to, co = oracle.oracle_tables(m, w.Hkv)
    assert np.array_equal(t, to) and np.array_equal(c, co)
    d = {k: v.cuda() for k, v in x.items()}
    tt, cc = bsc.build_tables(torch.from_numpy(m).cuda(), w.Hkv)
    O2, L2 = bsc.chunk_attention(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], tt, cc,
                                 w.prefix_len, n_splits=n_splits)
    assert torch.equal(O, O2) and torch.equal(L, L2)


CASES = [
    # Hq, Hkv, d, B, P, L, dtype, n_splits
    (8, 2, 128, 64, 1024, 512, "bf16", 0),     # 16 units: automatic KV splits
    (8, 2, 128, 64, 1024, 512, "bf16", 1),
    (8, 2, 64, 128, 512, 256, "bf16", 0),
    (8, 2, 128, 64, 1000, 100, "bf16", 0),     # unaligned
    (4, 1, 64, 64, 1024, 256, "fp32", 0),      # tiny shape, fp32
    (32, 8, 128, 64, 63488, 2048, "bf16", 0),  # 64K density-sweep shape
]


@pytest.mark.parametrize("Hq,Hkv,d,B,P,L,dtype,S", CASES)
def test_fused_against_oracle(bsc, Hq, Hkv, d, B, P, L, dtype, S):
    w = workloads.Workload("f", Hq, Hkv, d, dtype, P, L, B, "vslash", rho=0.1, corr=0.5,
                           window=4, seed=P + L)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, Lse, t, c = fused(bsc, w, x, m, S)
    to, co = oracle.oracle_tables(m, Hkv)
    assert np.array_equal(t, to) and np.array_equal(c, co)
    if P + L > 20000:   # large: sampled rows
        rng = np.random.default_rng(1)
        rows = [(int(h), int(i)) for h, i in zip(rng.integers(0, Hq, 48), rng.integers(0, L, 48))]
        Oo, Lo = oracle.oracle_rows(x["Q"].double().numpy(), x["K_pages"], x["V_pages"],
                                    x["page_table"].numpy(),
                                    to, co, P, rows)
        On, Ln = O.float().cpu().numpy(), Lse.cpu().numpy()
        compare(np.stack([On[i, h] for h, i in rows]), np.array([Ln[h, i] for h, i in rows]),
                Oo, Lo)
    else:
        Oo, Lo = oracle.oracle_chunk_attention(x["Q"].double().numpy(),
                                               x["K_pages"].double().numpy(),
                                               x["V_pages"].double().numpy(),
                                               x["page_table"].numpy(), to, co, P)
        compare(O.float().cpu().numpy(), Lse.cpu().numpy(), Oo, Lo)


def test_counts_out_without_tables_out(bsc):
    w = workloads.Workload("c", 8, 2, 128, "bf16", 1024, 256, 64, "vslash", rho=0.1, corr=0.5,
                           window=4, seed=5)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    d = {k: v.cuda() for k, v in x.items()}
    c = torch.full((w.Hkv,), 7, dtype=torch.int32, device="cuda")
    bsc.chunk_attention_masked(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], bits_of(m),
                               w.prefix_len, counts_out=c)
    _, co = oracle.oracle_tables(m, w.Hkv)
    assert np.array_equal(c.cpu().numpy(), co)
