"""ca_chunk_attention_noalloc: the entry point for callers that cannot allocate
device memory (an engine that owns every byte of the GPU through its own
allocator, or a loop where cudaMalloc is not allowed).  Its split partials live
in a fixed scratch array inside the library instead of caller workspace.

Checked through the C ABI on two calls in a row, both against the regular entry
point (same split mode, caller workspace) and against the float64 oracle.  The
second call has another shape and other inputs, so its split partials land on
scratch bytes the first call left behind: a stale partial leaking into the
result would show.  Both split modes run: n_splits = 0 (the automatic plan,
here the persistent schedule's partial slots) and n_splits = 3 (every unit's
KV range in three pieces, merged by the split combine).  This file is collected
last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

O_TOL = 1e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def bsc():
    import block_sparse_chunked_b200
    return block_sparse_chunked_b200


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_oversized_split_is_rejected_before_launch(bsc):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the size check comes first
    rc = bsc.lib.ca_chunk_attention_noalloc(fake, fake, fake, 2048, fake, fake, fake, 32, 8, 128,
                                            64, 2048, 129024, fake, fake, 4, None, None)
    assert rc == bsc.CA_ERR_WORKSPACE
    assert "scratch" in bsc.last_error()
    assert bsc.lib.ca_noalloc_scratch_bytes() == 32 << 20


# two calls in a row: (workload, seed); the second is a different shape
CALLS = [
    (workloads.Workload("na0", 8, 2, 128, "bf16", 1024, 512, 64, "vslash", rho=0.15, corr=0.5,
                        window=4), 0),
    (workloads.Workload("na1", 8, 2, 128, "bf16", 1600, 448, 64, "vslash", rho=0.2, corr=0.3,
                        window=4), 1),
]


@pytest.mark.gpu
@pytest.mark.parametrize("n_splits", [0, 3])
def test_noalloc_matches_regular_entry_point_and_oracle_twice(bsc, n_splits):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (w, seed) in enumerate(CALLS):
        need = bsc.workspace_size(torch.bfloat16, w.Hq, w.Hkv, w.head_dim, w.block, w.chunk_len,
                                  w.prefix_len, w.num_pages, n_splits=n_splits)
        assert 0 < need <= bsc.lib.ca_noalloc_scratch_bytes()   # the split uses the scratch
        xh = workloads.make_qkv_pages(w, seed=seed)
        x = {k: v.cuda() for k, v in xh.items()}
        m = workloads.mask_for(w, seed=seed)
        t, c = bsc.build_tables(torch.from_numpy(m).cuda(), w.Hkv)
        O_ref, L_ref = bsc.chunk_attention(x["Q"], x["K_pages"], x["V_pages"], x["page_table"],
                                           t, c, w.prefix_len, n_splits=n_splits)
        O = torch.full_like(x["Q"], float("nan"))
        L = torch.full((w.Hq, w.chunk_len), float("nan"), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = bsc.lib.ca_chunk_attention_noalloc(
            _p(x["Q"]), _p(x["K_pages"]), _p(x["V_pages"]), w.num_pages, _p(x["page_table"]),
            _p(t), _p(c), w.Hq, w.Hkv, w.head_dim, w.block, w.chunk_len, w.prefix_len, _p(O),
            _p(L), n_splits, _p(err), stream)
        assert rc == bsc.CA_OK, bsc.last_error()
        bsc.check(err)
        o, o_ref = O.float().cpu().numpy(), O_ref.float().cpu().numpy()
        l, l_ref = L.cpu().numpy(), L_ref.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(l).all(), f"call {call}"
        assert np.abs(o - o_ref).max() <= O_TOL, f"call {call}"
        assert np.abs(l - l_ref).max() <= LSE_TOL, f"call {call}"
        tn, cn = t.cpu().numpy(), c.cpu().numpy()
        Oo, Lo = oracle.oracle_chunk_attention(xh["Q"].double().numpy(),
                                               xh["K_pages"].double().numpy(),
                                               xh["V_pages"].double().numpy(),
                                               xh["page_table"].numpy(), tn, cn, w.prefix_len)
        assert np.abs(o - Oo).max() <= O_TOL, f"call {call} vs oracle"
        assert np.abs(l - Lo).max() <= LSE_TOL, f"call {call} vs oracle"
