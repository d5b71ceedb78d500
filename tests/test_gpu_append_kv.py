"""GPU parity of the paged-cache append (ca_append_kv) against the oracle:
bit-exact (a pure copy) for bf16 and fp32, block-aligned and unaligned
prefixes, an empty chunk, the 128K configuration at full size, and a page id
out of range (reported through the error word, nothing written)."""
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsc():
    import block_sparse_chunked_b200
    return block_sparse_chunked_b200


def _case(Hkv, d, B, prefix, L, dtype, seed, extra_pages=3):
    g = torch.Generator().manual_seed(seed)
    nK = max(1, -(-(prefix + L) // B))
    num_pages = nK + extra_pages
    pt = torch.randperm(num_pages, generator=g)[:nK].to(torch.int32)
    K = torch.randn(num_pages, Hkv, B, d, generator=g).to(dtype)
    V = torch.randn(num_pages, Hkv, B, d, generator=g).to(dtype)
    kn = torch.randn(L, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(L, Hkv, d, generator=g).to(dtype)
    return K, V, pt, kn, vn


def _run(bsc, K, V, pt, kn, vn, prefix):
    Kd, Vd = K.cuda(), V.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsc.append_kv(kn.cuda(), vn.cuda(), Kd, Vd, pt.cuda(), prefix, err_flag=err)
    bsc.check(err)
    return Kd.cpu(), Vd.cpu()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("Hkv,d,B,prefix,L", [
    (8, 128, 64, 1024, 512), (8, 128, 64, 1000, 517), (2, 64, 128, 0, 300), (1, 8, 64, 5, 1),
    (4, 64, 16, 33, 250), (3, 128, 64, 64, 0),
])
def test_append_bit_exact(bsc, dtype, Hkv, d, B, prefix, L):
    K, V, pt, kn, vn = _case(Hkv, d, B, prefix, L, dtype, seed=prefix + L + d)
    Ko, Vo = oracle.oracle_append_kv(K, V, pt, kn, vn, prefix)
    Kg, Vg = _run(bsc, K, V, pt, kn, vn, prefix)
    assert torch.equal(Kg, Ko) and torch.equal(Vg, Vo)


def test_append_ctx128k_full_size(bsc):
    w = workloads.get_config("ctx128k")
    x = workloads.make_qkv_pages(w)
    g = torch.Generator().manual_seed(7)
    kn = torch.randn(w.chunk_len, w.Hkv, w.head_dim, generator=g).to(torch.bfloat16)
    vn = torch.randn(w.chunk_len, w.Hkv, w.head_dim, generator=g).to(torch.bfloat16)
    Ko, Vo = oracle.oracle_append_kv(x["K_pages"], x["V_pages"], x["page_table"], kn, vn,
                                     w.prefix_len)
    Kg, Vg = _run(bsc, x["K_pages"], x["V_pages"], x["page_table"], kn, vn, w.prefix_len)
    assert torch.equal(Kg, Ko) and torch.equal(Vg, Vo)


def test_page_id_out_of_range_is_reported(bsc):
    K, V, pt, kn, vn = _case(2, 64, 64, 64, 128, torch.bfloat16, seed=3)
    bad = pt.clone()
    bad[2] = K.shape[0] + 5          # block 2 (positions 128..191) points past the cache
    Kd, Vd = K.cuda(), V.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsc.append_kv(kn.cuda(), vn.cuda(), Kd, Vd, bad.cuda(), 64, err_flag=err)
    with pytest.raises(bsc.CompactAttnError):
        bsc.check(err)
    # block 1 (positions 64..127) is still written; nothing else changes
    Ko, Vo = oracle.oracle_append_kv(K, V, pt, kn[:64], vn[:64], 64)
    assert torch.equal(Kd.cpu(), Ko) and torch.equal(Vd.cpu(), Vo)
