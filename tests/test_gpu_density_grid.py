"""GPU parity over the whole 64K density / within-group-correlation sweep, and
one element-wise comparison of the full 128K chunk.

The sweep: prefix 63488 + chunk 2048, 32 query / 8 KV heads, d 128, bf16,
blocks of 64 and 128; column density rho in {1, 0.5, 0.2, 0.1, 0.05} (rho = 1
is the all-ones mask, once per block size) x correlation c in {0, 0.5, 1}:
26 cells.  rho is the vertical-slash generator's column density (the sink
block and the local window come on top of it).

Every cell: the tables are bit-exact against the oracle, and O / LSE match it
on sampled rows (all heads, ~10 tokens including both ends of the chunk and
of the first and last query spans).  One cell per block size is compared
element by element, as is the whole 128K last chunk (65,536 query rows).
Tolerances as everywhere: max |O - O_oracle| <= 1e-2, max |LSE - LSE_oracle|
<= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
LSE_TOL = 1e-3

RHOS = [0.5, 0.2, 0.1, 0.05]
CORRS = [0.0, 0.5, 1.0]
CELLS = [(1.0, 0.0, b) for b in (64, 128)] + \
    [(r, c, b) for b in (64, 128) for r in RHOS for c in CORRS]
FULL = {(0.05, 0.0, 64), (0.1, 0.5, 128)}   # compared element by element


@pytest.fixture(scope="module")
def bsc():
    import block_sparse_chunked_b200
    return block_sparse_chunked_b200


_DATA = {}


def _data(block):
    """Q / K / V pages of the 64K cell shape (they do not depend on rho or c), on
    the host and on the device, made once per block size."""
    if block not in _DATA:
        _DATA.clear()
        w = workloads.density_cell(1.0, 0.0, block=block)
        x = workloads.make_qkv_pages(w)
        _DATA[block] = (x, {k: v.cuda() for k, v in x.items()})
    return _DATA[block]


def _rows(w, seed):
    rng = np.random.default_rng(seed)
    L = w.chunk_len
    toks = sorted(set([0, 63, 64, L // 2, L - 64, L - 1] + rng.integers(0, L, 4).tolist()))
    return [(h, i) for h in range(w.Hq) for i in toks]


def _compare(O, L, Oo, Lo, what):
    assert np.array_equal(np.isneginf(L), np.isneginf(Lo)), what
    fin = np.isfinite(Lo)
    oerr = float(np.abs(O - Oo).max())
    lerr = float(np.abs(L[fin] - Lo[fin]).max()) if fin.any() else 0.0
    assert oerr <= O_TOL, f"{what}: O max err {oerr}"
    assert lerr <= LSE_TOL, f"{what}: LSE max err {lerr}"


@pytest.mark.parametrize("rho,corr,block", CELLS)
def test_density_grid_cell(bsc, rho, corr, block):
    w = workloads.density_cell(rho, corr, block=block)
    x, d = _data(block)
    m = workloads.mask_for(w)
    tables, counts = bsc.build_tables(torch.from_numpy(m).cuda(), w.Hkv)
    t, c = tables.cpu().numpy(), counts.cpu().numpy()
    to, co = oracle.oracle_tables(m, w.Hkv)
    assert np.array_equal(t, to) and np.array_equal(c, co), "tables differ from the oracle"
    if rho >= 1.0:  # the all-ones cell: exactly the density-100% path's tables
        assert c.tolist() == [w.nKblk] * w.Hkv
        assert np.array_equal(t, np.tile(np.arange(w.nKblk, dtype=t.dtype), (w.Hkv, 1)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, L = bsc.chunk_attention(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], tables,
                               counts, w.prefix_len, err_flag=err)
    bsc.check(err)
    O, L = O.float().cpu().numpy(), L.cpu().numpy()
    assert np.all(np.isfinite(L))
    what = f"rho {rho} c {corr} B {block}"
    if (rho, corr, block) in FULL:
        Oo, Lo = oracle.oracle_chunk_attention(x["Q"].double().numpy(),
                                               x["K_pages"].double().numpy(),
                                               x["V_pages"].double().numpy(),
                                               x["page_table"].numpy(), t, c, w.prefix_len)
        _compare(O, L, Oo, Lo, what + " (every element)")
    else:
        rows = _rows(w, seed=int(rho * 100) + int(corr * 10) + block)
        Oo, Lo = oracle.oracle_rows(x["Q"].double().numpy(), x["K_pages"], x["V_pages"],
                                    x["page_table"].numpy(), t, c, w.prefix_len, rows)
        _compare(np.stack([O[i, h] for h, i in rows]), np.array([L[h, i] for h, i in rows]),
                 Oo, Lo, what + " (sampled rows)")


def test_ctx128k_every_element(bsc):
    """The 128K last chunk in the benchmark's launch configuration, all 65,536
    (head, token) rows against the full oracle."""
    _DATA.clear()
    w = workloads.get_config("ctx128k")
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    d = {k: v.cuda() for k, v in x.items()}
    tables, counts = bsc.build_tables(torch.from_numpy(m).cuda(), w.Hkv)
    ws = torch.empty(max(1, bsc.workspace_size(torch.bfloat16, w.Hq, w.Hkv, w.head_dim, w.block,
                                               w.chunk_len, w.prefix_len, w.num_pages)),
                     dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, L = bsc.chunk_attention(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], tables,
                               counts, w.prefix_len, err_flag=err, workspace=ws)
    bsc.check(err)
    del d
    t, c = tables.cpu().numpy(), counts.cpu().numpy()
    Oo, Lo = oracle.oracle_chunk_attention(x["Q"].double().numpy(), x["K_pages"].double().numpy(),
                                           x["V_pages"].double().numpy(),
                                           x["page_table"].numpy(), t, c, w.prefix_len)
    _compare(O.float().cpu().numpy(), L.cpu().numpy(), Oo, Lo, "ctx128k (every element)")
