"""GPU parity of ca_chunk_attention against the float64 oracle.

Tolerances (fixed by the acceptance bar): max |O - O_oracle| <= 1e-2 and
max |LSE - LSE_oracle| <= 1e-3.  The oracle sees the exact input values
(bf16 inputs are exact in float64; fp32 inputs are used as fp32, while the
kernel rounds them to bf16, which the tiny-config bound absorbs).

Small and medium cases compare every element; the LLaMA-shape configs
compare sampled rows that the oracle computes one by one, in the same launch
configuration the benchmark times.
"""
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


def to_dev(x):
    return {k: v.cuda() for k, v in x.items()}


def gpu_run(bsc, w, x, mask, n_splits=0, tables=None, counts=None):
    d = to_dev(x)
    if tables is None:
        tables, counts = bsc.build_tables(torch.from_numpy(mask).cuda(), w.Hkv)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, L = bsc.chunk_attention(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], tables,
                               counts, w.prefix_len, n_splits=n_splits, err_flag=err)
    bsc.check(err)
    return O.float().cpu().numpy(), L.cpu().numpy(), tables.cpu().numpy(), counts.cpu().numpy()


def full_oracle(w, x, t, c):
    return oracle.oracle_chunk_attention(x["Q"].double().numpy(), x["K_pages"].double().numpy(),
                                         x["V_pages"].double().numpy(), x["page_table"].numpy(),
                                         t, c, w.prefix_len)


def compare(O, L, Oo, Lo):
    assert np.array_equal(np.isneginf(L), np.isneginf(Lo))
    fin = np.isfinite(Lo)
    lerr = np.abs(L[fin] - Lo[fin]).max() if fin.any() else 0.0
    oerr = np.abs(O - Oo).max()
    assert oerr <= O_TOL, f"O max err {oerr}"
    assert lerr <= LSE_TOL, f"LSE max err {lerr}"
    return oerr, lerr


def test_tiny_config(bsc):
    w = workloads.get_config("tiny")
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, L, t, c = gpu_run(bsc, w, x, m)
    to, co = oracle.oracle_tables(m, w.Hkv)
    assert np.array_equal(t, to) and np.array_equal(c, co)
    compare(O, L, *full_oracle(w, x, t, c))


MEDIUM = [
    # Hq, Hkv, d, B, P, L, kind, rho
    (8, 2, 128, 64, 1024, 512, "vslash", 0.1),
    (8, 2, 128, 64, 960, 320, "bernoulli", 0.05),
    (8, 2, 64, 64, 640, 256, "vslash", 0.2),
    (8, 2, 128, 128, 1024, 512, "vslash", 0.15),
    (8, 2, 64, 128, 512, 256, "bernoulli", 0.1),
    (4, 4, 128, 64, 512, 256, "vslash", 0.1),     # G = 1
    (8, 4, 128, 64, 512, 256, "vslash", 0.1),     # G = 2
    (16, 2, 128, 64, 512, 256, "vslash", 0.1),    # G = 8
    (6, 2, 128, 64, 512, 192, "vslash", 0.1),     # G = 3
    (8, 2, 128, 64, 0, 256, "ones", 1.0),         # first chunk, no prefix
    (8, 2, 128, 64, 1024, 64, "vslash", 0.1),     # one query span
]


@pytest.mark.parametrize("Hq,Hkv,d,B,P,L,kind,rho", MEDIUM)
@pytest.mark.parametrize("n_splits", [0, 1, 3])
def test_medium_cases_full(bsc, Hq, Hkv, d, B, P, L, kind, rho, n_splits):
    w = workloads.Workload("m", Hq, Hkv, d, "bf16", P, L, B, kind, rho=rho, corr=0.5,
                           window=4, seed=Hq + P + L + B)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, Lg, t, c = gpu_run(bsc, w, x, m, n_splits=n_splits)
    compare(O, Lg, *full_oracle(w, x, t, c))


def test_odd_table_lengths_use_half_stage(bsc):
    """Tables whose live prefix has odd length end with a 64-key MMA stage."""
    w = workloads.Workload("odd", 8, 2, 128, "bf16", 1024, 256, 64, "vslash", rho=0.1)
    x = workloads.make_qkv_pages(w)
    m = np.zeros((w.Hq, w.nQblk, w.nKblk), np.uint8)
    m[:, :, [0, 3, 5]] = 1                       # 3 prefix blocks
    for qb in range(w.nQblk):
        m[:, qb, w.nPblk + qb] = 1               # diagonal
    O, Lg, t, c = gpu_run(bsc, w, x, m)
    assert c.tolist() == [3 + w.nQblk] * w.Hkv
    compare(O, Lg, *full_oracle(w, x, t, c))


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("n_splits", [0, 3])
def test_row_max_jumps_mid_row(bsc, d, n_splits):
    """The running max of the rows jumps by more than 2^8 (log2 units) at
    three later stages, in either key half of a 128-key stage, so the stage
    is redone and O rescaled mid-row.  Every query leans on coordinate 0
    (+4); the keys of prefix blocks 4, 7 and 10 are lam * e_0, with q.k /
    sqrt(d) = (q_0 + 4) * (10, 25, 40) / 4 against O(1) for the other keys."""
    w = workloads.Workload("jump", 8, 2, d, "bf16", 1024, 256, 64, "ones", rho=1.0)
    x = workloads.make_qkv_pages(w)
    Q = x["Q"].float()
    Q[..., 0] += 4.0
    K = x["K_pages"].float()
    pt = x["page_table"].numpy()
    for kb, target in ((4, 10.0), (7, 25.0), (10, 40.0)):
        K[pt[kb]] = 0.0
        K[pt[kb], :, :, 0] = target * d ** 0.5 / 4.0
    x = dict(x, Q=Q.to(torch.bfloat16), K_pages=K.to(torch.bfloat16))
    m = workloads.mask_for(w)
    O, Lg, t, c = gpu_run(bsc, w, x, m, n_splits=n_splits)
    Oo, Lo = full_oracle(w, x, t, c)
    assert np.isfinite(Lo).all() and (Lo > 20.0).mean() > 0.9  # the spikes dominate the rows
    compare(O, Lg, Oo, Lo)


def test_diagonal_missing_and_future_blocks(bsc):
    """No diagonal block selected, plus blocks above the causal diagonal (unclipped)."""
    w = workloads.Workload("nodiag", 8, 2, 128, "bf16", 512, 256, 64, "bernoulli", rho=0.2)
    x = workloads.make_qkv_pages(w)
    rng = np.random.default_rng(3)
    m = (rng.random((w.Hq, w.nQblk, w.nKblk)) < 0.2).astype(np.uint8)
    m[:, :, w.nPblk:] = 0
    m[0, 0, w.nKblk - 1] = 1                     # future block for most spans
    O, Lg, t, c = gpu_run(bsc, w, x, m)
    compare(O, Lg, *full_oracle(w, x, t, c))


def test_empty_group_table(bsc):
    w = workloads.Workload("empty", 8, 2, 128, "bf16", 512, 256, 64, "vslash", rho=0.1)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    m[4:] = 0                                    # group 1 selects nothing
    O, Lg, t, c = gpu_run(bsc, w, x, m)
    assert c[1] == 0
    assert np.all(O[:, 4:] == 0) and np.all(np.isneginf(Lg[4:]))
    compare(O, Lg, *full_oracle(w, x, t, c))


def test_page_permutation_invariance_bitwise(bsc):
    w = workloads.Workload("perm", 8, 2, 128, "bf16", 1024, 256, 64, "vslash", rho=0.1)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    pt = x["page_table"].numpy()
    xi = dict(x)
    xi["K_pages"] = x["K_pages"][torch.from_numpy(pt).long()].contiguous()
    xi["V_pages"] = x["V_pages"][torch.from_numpy(pt).long()].contiguous()
    xi["page_table"] = torch.arange(w.nKblk, dtype=torch.int32)
    O1, L1, _, _ = gpu_run(bsc, w, x, m)
    O2, L2, _, _ = gpu_run(bsc, w, xi, m)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_split_equals_unsplit(bsc):
    w = workloads.Workload("split", 8, 2, 128, "bf16", 2048, 256, 64, "vslash", rho=0.2)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O1, L1, t, c = gpu_run(bsc, w, x, m, n_splits=1)
    for s in (2, 5, 16):
        O2, L2, _, _ = gpu_run(bsc, w, x, m, n_splits=s)
        assert np.abs(O1 - O2).max() <= 4e-3
        assert np.abs(L1 - L2).max() <= 1e-4


def sample_rows(w, seed=0, ntok=12):
    rng = np.random.default_rng(seed)
    L = w.chunk_len
    toks = sorted(set([0, 1, 63, 64, L // 2, L - 65, L - 64, L - 1] +
                      rng.integers(0, L, ntok).tolist()))
    return [(h, i) for h in range(w.Hq) for i in toks]


@pytest.mark.parametrize("name", ["llama16k", "ctx128k"])
def test_llama_configs_sampled_rows(bsc, name):
    w = workloads.get_config(name)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, Lg, t, c = gpu_run(bsc, w, x, m)
    to, co = oracle.oracle_tables(m, w.Hkv)
    assert np.array_equal(t, to) and np.array_equal(c, co)
    rows = sample_rows(w)
    Oo, Lo = oracle.oracle_rows(x["Q"].double().numpy(), x["K_pages"], x["V_pages"],
                                x["page_table"].numpy(), t, c, w.prefix_len, rows)
    Os = np.stack([O[i, h] for h, i in rows])
    Ls = np.array([Lg[h, i] for h, i in rows])
    compare(Os, Ls, Oo, Lo)
    # properties at every row: finite LSE, |O| bounded by max |V|
    assert np.all(np.isfinite(Lg))
    assert np.abs(O).max() <= float(x["V_pages"].float().abs().max()) + 1e-2


def test_all_ones_equals_dense_path_128k_sampled(bsc):
    """Density 100%: the table is every block; the result is dense causal attention."""
    w = workloads.get_config("ctx128k").with_(mask_kind="ones")
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, Lg, t, c = gpu_run(bsc, w, x, m)
    assert c.tolist() == [w.nKblk] * w.Hkv
    rows = sample_rows(w, seed=1, ntok=4)[:: 4]
    Oo, Lo = oracle.oracle_rows(x["Q"].double().numpy(), x["K_pages"], x["V_pages"],
                                x["page_table"].numpy(), t, c, w.prefix_len, rows)
    compare(np.stack([O[i, h] for h, i in rows]), np.array([Lg[h, i] for h, i in rows]), Oo, Lo)


def test_bad_page_id_sets_bounds_error(bsc):
    w = workloads.Workload("bad", 8, 2, 128, "bf16", 512, 256, 64, "vslash", rho=0.1)
    x = workloads.make_qkv_pages(w)
    x["page_table"][3] = 10 ** 6
    m = workloads.mask_for(w)
    m[:, :, 3] = 1
    d = to_dev(x)
    t, c = bsc.build_tables(torch.from_numpy(m).cuda(), w.Hkv)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsc.chunk_attention(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], t, c, w.prefix_len,
                        err_flag=err)
    with pytest.raises(bsc.CompactAttnError) as e:
        bsc.check(err)
    assert e.value.code == bsc.CA_ERR_BOUNDS
    bsc.check(err)  # cleared


def test_bad_count_sets_bounds_error(bsc):
    w = workloads.Workload("badc", 8, 2, 128, "bf16", 512, 256, 64, "vslash", rho=0.1)
    x = to_dev(workloads.make_qkv_pages(w))
    t, c = bsc.build_tables(torch.from_numpy(workloads.mask_for(w)).cuda(), w.Hkv)
    c[0] = w.nKblk + 5
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsc.chunk_attention(x["Q"], x["K_pages"], x["V_pages"], x["page_table"], t, c, w.prefix_len,
                        err_flag=err)
    with pytest.raises(bsc.CompactAttnError) as e:
        bsc.check(err)
    assert e.value.code == bsc.CA_ERR_BOUNDS


def test_bounded_wait_times_out_cleanly(bsc):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsc.wait_probe(err, 2000)
    with pytest.raises(bsc.CompactAttnError) as e:
        bsc.check(err)
    assert e.value.code == bsc.CA_ERR_TIMEOUT
    # the context is still usable afterwards
    w = workloads.get_config("tiny")
    x = workloads.make_qkv_pages(w)
    O, L, t, c = gpu_run(bsc, w, x, workloads.mask_for(w))
    compare(O, L, *full_oracle(w, x, t, c))


@pytest.mark.parametrize("c", [0, 12, 31])
def test_sweep_chunks_sampled_rows(bsc, c):
    """Chunk c of the 131072-token chunked prefill (4096-token chunks, growing paged KV)."""
    w = workloads.sweep_chunk(c)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    O, Lg, t, cn = gpu_run(bsc, w, x, m)
    to, co = oracle.oracle_tables(m, w.Hkv)
    assert np.array_equal(t, to) and np.array_equal(cn, co)
    rows = sample_rows(w, seed=c, ntok=6)[::2]
    Oo, Lo = oracle.oracle_rows(x["Q"].double().numpy(), x["K_pages"], x["V_pages"],
                                x["page_table"].numpy(), t, cn, w.prefix_len, rows)
    compare(np.stack([O[i, h] for h, i in rows]), np.array([Lg[h, i] for h, i in rows]), Oo, Lo)
    assert np.all(np.isfinite(Lg))
