"""Host-side tests of the C ABI (no GPU): the library builds, loads, exports
every symbol include/compactattn.h declares, and rejects bad arguments before
launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bsc():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_bsc_build", os.path.join(ROOT, "block_sparse_chunked_b200", "_build.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    m.build_library()
    import block_sparse_chunked_b200
    return block_sparse_chunked_b200


def header_symbols():
    src = open(os.path.join(ROOT, "include", "compactattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t)\s+(ca_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_expected_calls():
    syms = header_symbols()
    for s in ["ca_build_tables", "ca_build_tables_batched", "ca_workspace_size",
              "ca_chunk_attention", "ca_check", "ca_last_error"]:
        assert s in syms


def test_library_exports_every_declared_symbol(bsc):
    lib = ctypes.CDLL(bsc.LIB_PATH)
    for s in header_symbols():
        assert hasattr(lib, s), s
    assert set(header_symbols()) <= set(bsc.EXPORTS)


def header_prototypes():
    """name -> (return type, [parameter C types]) for every declaration."""
    src = open(os.path.join(ROOT, "include", "compactattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*(int|size_t)\s+(ca_\w+)\s*\(([^)]*)\)\s*;", src, flags=re.M):
        params = [x.strip() for x in m.group(3).split(",") if x.strip() and x.strip() != "void"]
        out[m.group(2)] = (m.group(1), params)
    return out


def test_binding_signatures_match_header(bsc):
    """Each ctypes declaration has the header's arity and, parameter by
    parameter, a matching kind: pointer -> c_void_p / c_char_p, int -> c_int,
    size_t -> c_size_t.  (A drift here would pass wrong values to the GPU.)"""
    protos = header_prototypes()
    assert set(protos) == set(header_symbols())
    for name, (ret, params) in protos.items():
        res, args = bsc.EXPORTS[name]
        assert res is (ctypes.c_int if ret == "int" else ctypes.c_size_t), name
        assert len(args) == len(params), (name, len(args), len(params))
        for a, ctype in zip(args, params):
            if "*" in ctype:
                assert a in (ctypes.c_void_p, ctypes.c_char_p), (name, ctype)
            elif re.match(r"(const\s+)?size_t\b", ctype):
                assert a is ctypes.c_size_t, (name, ctype)
            else:
                assert re.match(r"(const\s+)?int\b", ctype) and a is ctypes.c_int, (name, ctype)


def test_version(bsc):
    assert bsc.version() == 100


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first


@pytest.mark.parametrize("Hq,Hkv,nQ,nK,nb", [(6, 4, 2, 10, 1), (4, 0, 2, 10, 1), (4, 2, 0, 10, 1),
                                              (4, 2, 2, 0, 1), (4, 2, 2, 65537, 1),
                                              (4, 2, 2, 10, 0), (4, 8, 2, 10, 1)])
def test_build_tables_rejects_bad_shapes(bsc, Hq, Hkv, nQ, nK, nb):
    rc = bsc.lib.ca_build_tables_batched(FAKE, nb, Hq, Hkv, nQ, nK, FAKE, FAKE, None)
    assert rc == bsc.CA_ERR_ARG
    assert "ca_build_tables" in bsc.last_error()


def test_build_tables_rejects_null(bsc):
    assert bsc.lib.ca_build_tables(None, 4, 2, 2, 10, FAKE, FAKE, None) == bsc.CA_ERR_ARG


def _attn(bsc, **kw):
    a = dict(Q=FAKE, K=FAKE, V=FAKE, dtype=0, num_pages=20, pt=FAKE, tables=FAKE, counts=FAKE,
             Hq=4, Hkv=1, d=64, B=64, L=256, P=1024, O=FAKE, LSE=FAKE, ws=None, wsn=0, S=1,
             err=None)
    a.update(kw)
    return bsc.lib.ca_chunk_attention(a["Q"], a["K"], a["V"], a["dtype"], a["num_pages"], a["pt"],
                                      a["tables"], a["counts"], a["Hq"], a["Hkv"], a["d"], a["B"],
                                      a["L"], a["P"], a["O"], a["LSE"], a["ws"], a["wsn"], a["S"],
                                      a["err"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(Q=None), -1), (dict(dtype=7), -3), (dict(P=-5), -1), (dict(L=0), -1),
    (dict(B=32), -1), (dict(d=96), -1), (dict(Hq=6, Hkv=4), -1), (dict(num_pages=19), -1),
    (dict(Q=ctypes.c_void_p(0x1001)), -1), (dict(dtype=1), -7), (dict(S=4), -7), (dict(S=0), -7),
])
def test_chunk_attention_rejects_bad_arguments(bsc, kw, code):
    assert _attn(bsc, **kw) == code
    assert bsc.last_error()


def test_workspace_size_rules(bsc):
    ws = bsc.lib.ca_workspace_size
    # bf16, one CTA per unit: no workspace
    assert ws(0, 32, 8, 128, 64, 2048, 129024, 2048, 1) == 0
    # automatic mode at 128K: 512 one-tile units on 148 SMs; the 68 units of
    # the last partial wave run as 2 KV pieces each (fp32 partials of 128 rows)
    tail = 68 * 2 * 128
    assert ws(0, 32, 8, 128, 64, 2048, 129024, 2048, 0) == tail * 128 * 4 + tail * 4
    # automatic mode, 2 groups x 2 head pairs x 8 spans = 32 units (< 148 SMs):
    # every unit in floor(148 / 32) = 4 KV pieces, fp32 partials of every row
    n = ws(0, 8, 2, 128, 64, 512, 1024, 24, 0)
    assert n == 4 * 512 * 8 * 128 * 4 + 4 * 8 * 512 * 4
    # fp32 inputs keep the two-tile kernel: its persistent grid of
    # min(148, 16*12/4) = 48 CTAs with <= 2 partial pieces per CTA
    n = ws(1, 8, 4, 128, 64, 512, 1024, 24, 0)
    assert n >= 2 * 48 * 256 * 128 * 4
    # explicit split: fp32 partials + LSE partials
    n = ws(0, 32, 8, 128, 64, 2048, 129024, 2048, 2)
    assert n >= 2 * 2048 * 32 * 128 * 4 + 2 * 32 * 2048 * 4
    # fp32 input adds bf16 copies of Q, K and V
    assert ws(1, 4, 1, 64, 64, 256, 1024, 20, 1) >= (256 * 4 * 64 + 2 * 20 * 64 * 64) * 2
    assert ws(0, 4, 3, 64, 64, 256, 1024, 20, 1) == ctypes.c_size_t(-1).value


def test_workspace_size_unaligned_and_batched(bsc):
    ws = bsc.lib.ca_workspace_size
    # unaligned prefix / chunk: accepted (any alignment), bf16 with one split -> 0
    assert ws(0, 32, 8, 128, 64, 100, 1000, 20, 1) == 0
    # the chunk's blocks exceed the pages: rejected
    assert ws(0, 32, 8, 128, 64, 100, 1000, 17, 1) == ctypes.c_size_t(-1).value
    wv = bsc.lib.ca_workspace_size_varlen
    # batched: descriptors always need workspace
    n = wv(0, 32, 8, 128, 64, 5, 500, 5000, 200, 1)
    assert 0 < n < 65536
    # two KV splits add fp32 partials for every row
    assert wv(0, 32, 8, 128, 64, 5, 500, 5000, 200, 2) >= 2 * 500 * 32 * 128 * 4
    assert wv(0, 32, 8, 128, 64, 0, 500, 5000, 200, 1) == ctypes.c_size_t(-1).value


def _varlen(bsc, **kw):
    a = dict(Q=FAKE, K=FAKE, V=FAKE, dtype=0, num_pages=20, S=2, total_q=10, cu_q=FAKE, P=FAKE,
             max_kv=100, pt=FAKE, cu_pages=FAKE, tables=FAKE, counts=FAKE, Hq=4, Hkv=1, d=64,
             B=64, O=FAKE, LSE=FAKE, ws=None, wsn=0, splits=1)
    a.update(kw)
    return bsc.lib.ca_chunk_attention_varlen(
        a["Q"], a["K"], a["V"], a["dtype"], a["num_pages"], a["S"], a["total_q"], a["cu_q"],
        a["P"], a["max_kv"], a["pt"], a["cu_pages"], a["tables"], a["counts"], a["Hq"], a["Hkv"],
        a["d"], a["B"], a["O"], a["LSE"], a["ws"], a["wsn"], a["splits"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(cu_q=None), -1), (dict(dtype=2), -3), (dict(S=0), -1), (dict(B=32), -1),
    (dict(d=96), -1), (dict(Hq=6, Hkv=4), -1), (dict(total_q=-1), -1),
    (dict(Q=ctypes.c_void_p(0x1004)), -1), (dict(), -7),
])
def test_varlen_rejects_bad_arguments(bsc, kw, code):
    assert _varlen(bsc, **kw) == code
    assert "ca_chunk_attention_varlen" in bsc.last_error()


def test_check_and_probe_reject_null(bsc):
    assert bsc.lib.ca_check(None, None) == bsc.CA_ERR_ARG
    assert bsc.lib.ca_wait_probe(None, 10, None) == bsc.CA_ERR_ARG
    with pytest.raises(ValueError):
        bsc.check(None)
    with pytest.raises(ValueError):
        bsc.wait_probe(None, 10)


def test_binding_device_check(bsc):
    """Every tensor of a call must sit on the device the call runs on (the
    kernels take raw pointers); a tensor elsewhere is refused before any launch."""
    import torch
    from block_sparse_chunked_b200 import _capi
    dev = torch.device("cuda", 0)
    _capi._same_device(torch.device("cpu"), a=torch.zeros(1), b=None)
    with pytest.raises(ValueError, match="K_pages is on cpu"):
        _capi._same_device(dev, K_pages=torch.zeros(1))
    with pytest.raises(ValueError, match="err_flag"):
        _capi._errp(torch.zeros(1, dtype=torch.int32), dev)   # not a CUDA tensor


def test_accounting_dense_128k(bsc):
    # 32 heads x sum_{qb<32} (2016 + qb + 1) pairs x 4 * 64^2 * 128 FLOPs
    assert bsc.dense_flops(32, 2016, 32, 64, 128) == 4 * 64 * 64 * 128 * 32 * (32 * 2017 + 496)


def _append(bsc, **kw):
    a = dict(K=FAKE, V=FAKE, dtype=0, KP=FAKE, VP=FAKE, num_pages=40, pt=FAKE, Hkv=2, d=128, B=64,
             P=100, L=64, err=None)
    a.update(kw)
    return bsc.lib.ca_append_kv(a["K"], a["V"], a["dtype"], a["KP"], a["VP"], a["num_pages"],
                                a["pt"], a["Hkv"], a["d"], a["B"], a["P"], a["L"], a["err"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(K=None), -1), (dict(pt=None), -1), (dict(dtype=5), -3), (dict(d=4), -1),
    (dict(d=6, dtype=1), -1), (dict(Hkv=0), -1), (dict(P=-1), -1), (dict(B=0), -1),
    (dict(num_pages=2), -1), (dict(KP=ctypes.c_void_p(0x1008)), -1),
])
def test_append_kv_rejects_bad_arguments(bsc, kw, code):
    assert _append(bsc, **kw) == code
    assert "ca_append_kv" in bsc.last_error()


def _masked(bsc, **kw):
    a = dict(Q=FAKE, K=FAKE, V=FAKE, dtype=0, num_pages=40, pt=FAKE, bits=FAKE, Hq=8, Hkv=2,
             d=128, B=64, L=256, P=1024, t=None, c=None, O=FAKE, LSE=FAKE, ws=None, wsn=0,
             splits=1)
    a.update(kw)
    return bsc.lib.ca_chunk_attention_masked(
        a["Q"], a["K"], a["V"], a["dtype"], a["num_pages"], a["pt"], a["bits"], a["Hq"],
        a["Hkv"], a["d"], a["B"], a["L"], a["P"], a["t"], a["c"], a["O"], a["LSE"], a["ws"],
        a["wsn"], a["splits"], None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(bits=None), -1), (dict(dtype=9), -3), (dict(P=200000, num_pages=5000), -1),
    (dict(num_pages=10), -1), (dict(bits=ctypes.c_void_p(0x1002)), -1), (dict(L=0), -1),
    (dict(splits=4), -7),
])
def test_masked_rejects_bad_arguments(bsc, kw, code):
    assert _masked(bsc, **kw) == code
    assert "ca_chunk_attention_masked" in bsc.last_error()


def test_workspace_size_masked(bsc):
    wm = bsc.lib.ca_workspace_size_masked
    # bf16, head_dim 128, G = 4: the CTA-pair kernel; at 128K the last partial
    # wave (68 of 512 units) runs as 2 KV pieces each
    tail = 68 * 2 * 128
    assert wm(0, 32, 8, 128, 64, 2048, 129024, 2048, 0) == tail * 128 * 4 + tail * 4
    assert wm(0, 8, 2, 128, 64, 512, 1024, 24, 0) > 0                  # 32 units: KV splits
    # fp32 inputs keep the two-tile kernel: 256 units, one CTA each
    assert wm(1, 32, 8, 128, 64, 2048, 129024, 2048, 0) > 0            # (bf16 copies of Q/K/V)
    assert wm(0, 32, 8, 128, 64, 2048, 129024 + 64, 2049, 0) == ctypes.c_size_t(-1).value


def test_fp8_entry_rejects_bad_arguments(bsc):
    f = bsc.lib.ca_chunk_attention_fp8
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 40, FAKE, FAKE, FAKE, 8, 2, 128, 64, 256, 1024, FAKE,
            FAKE, None, 0, 1, None, None]
    assert f(*args) == bsc.CA_ERR_WORKSPACE          # the fp8 path always needs workspace
    bad = list(args)
    bad[3] = None                                    # no K scales
    assert f(*bad) == bsc.CA_ERR_ARG
    bad = list(args)
    bad[11] = 96                                     # head_dim
    assert f(*bad) == bsc.CA_ERR_ARG
    assert bsc.lib.ca_workspace_size_fp8(8, 2, 128, 64, 256, 1024, 40, 1) > 0
    assert bsc.lib.ca_workspace_size_fp8(8, 2, 128, 64, 256, 1024, 10, 1) == ctypes.c_size_t(-1).value


def test_accounting_general_lengths_match_aligned(bsc):
    import numpy as np
    import oracle
    import workloads
    w = workloads.get_config("llama16k")
    t, c = oracle.oracle_tables(workloads.mask_for(w), w.Hkv)
    a = bsc.selected_pairs(t, c, w.Hq, w.nPblk, w.nQblk)
    b = bsc.selected_pairs_pl(t, c, w.Hq, w.prefix_len, w.chunk_len, w.block)
    assert a == b
    # unaligned: brute force over (h, qb, entry)
    P, L, B, Hq, Hkv = 100, 70, 64, 4, 2
    nK = -(-(P + L) // B)
    rng = np.random.default_rng(0)
    m = (rng.random((Hq, -(-L // B), nK)) < 0.5).astype(np.uint8)
    t, c = oracle.oracle_tables(m, Hkv)
    brute = 0
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for qb in range(-(-L // B)):
            last_tok = min(qb * B + B - 1, L - 1)
            brute += sum(1 for e in t[g, :c[g]] if e * B <= P + last_tok)
    assert bsc.selected_pairs_pl(t, c, Hq, P, L, B) == brute

