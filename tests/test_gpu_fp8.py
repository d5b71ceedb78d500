"""GPU parity of the E4M3 paged-cache attention (ca_chunk_attention_fp8)
against the float64 oracle on the decoded cache: full comparison at medium,
small-unit (KV split), unaligned and d = 64 shapes, sampled rows at the 128K
chunk.  Tolerances as for bf16 pages: |O| <= 1e-2, |LSE| <= 1e-3 (the
kernel's operands are the exact decoded values; its f16 P and Q carry more
bits than the bf16 path's)."""
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


def compare(O, L, Oo, Lo):
    assert np.array_equal(np.isneginf(L), np.isneginf(Lo))
    fin = np.isfinite(Lo)
    if fin.any():
        assert np.abs(L[fin] - Lo[fin]).max() <= LSE_TOL
    assert np.abs(O - Oo).max() <= O_TOL


def run(bsc, w, x, m, n_splits=0, scale_spread=0.0, seed=0):
    fk = fv = None
    if scale_spread:  # scales up to 2^spread coarser than amax / 448, per (page, head)
        rng = np.random.default_rng(seed)
        shape = x["K_pages"].shape[:2]
        fk = torch.from_numpy(np.exp2(rng.uniform(0, scale_spread, shape))).float()
        fv = torch.from_numpy(np.exp2(rng.uniform(0, scale_spread, shape))).float()
    K8, sK = workloads.quantize_pages_e4m3(x["K_pages"], fk)
    V8, sV = workloads.quantize_pages_e4m3(x["V_pages"], fv)
    t, c = oracle.oracle_tables(m, w.Hkv)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, L = bsc.chunk_attention_fp8(x["Q"].cuda(), K8.cuda(), V8.cuda(), sK.cuda(), sV.cuda(),
                                   x["page_table"].cuda(), torch.from_numpy(t).cuda(),
                                   torch.from_numpy(c).cuda(), w.prefix_len, n_splits=n_splits,
                                   err_flag=err)
    bsc.check(err)
    return O.float().cpu().numpy(), L.cpu().numpy(), (K8, sK, V8, sV, t, c)


CASES = [
    # Hq, Hkv, d, B, P, L, n_splits, scale spread (log2)
    (8, 2, 128, 64, 1024, 512, 1, 0.0),
    (8, 2, 128, 64, 1024, 512, 0, 3.0),      # 16 units: automatic KV splits; spread scales
    (8, 2, 64, 64, 640, 256, 1, 2.0),
    (8, 2, 128, 128, 1024, 512, 1, 1.0),
    (8, 2, 128, 64, 1000, 100, 0, 2.0),      # unaligned
    (4, 4, 128, 64, 512, 256, 1, 0.0),       # G = 1
]


@pytest.mark.parametrize("Hq,Hkv,d,B,P,L,S,spread", CASES)
def test_fp8_against_oracle(bsc, Hq, Hkv, d, B, P, L, S, spread):
    w = workloads.Workload("e", Hq, Hkv, d, "bf16", P, L, B, "vslash", rho=0.15, corr=0.5,
                           window=4, seed=P + L + d)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, Lse, (K8, sK, V8, sV, t, c) = run(bsc, w, x, m, S, spread, seed=P)
    Oo, Lo = oracle.oracle_chunk_attention_fp8(x["Q"].double().numpy(), K8.numpy(), V8.numpy(),
                                               sK.numpy(), sV.numpy(), x["page_table"].numpy(),
                                               t, c, P)
    compare(O, Lse, Oo, Lo)


def test_fp8_ctx128k_sampled_rows(bsc):
    w = workloads.get_config("ctx128k")
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, Lse, (K8, sK, V8, sV, t, c) = run(bsc, w, x, m)
    rng = np.random.default_rng(4)
    rows = [(int(h), int(i)) for h, i in zip(rng.integers(0, w.Hq, 40),
                                             rng.integers(0, w.chunk_len, 40))]
    rows += [(0, 0), (31, w.chunk_len - 1)]
    Oo, Lo = oracle.oracle_rows_fp8(x["Q"].double().numpy(), K8.numpy(), V8.numpy(), sK.numpy(),
                                    sV.numpy(), x["page_table"].numpy(), t, c, w.prefix_len,
                                    rows)
    compare(np.stack([O[i, h] for h, i in rows]), np.array([Lse[h, i] for h, i in rows]), Oo, Lo)
