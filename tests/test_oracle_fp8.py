"""Pins for the E4M3 page decode and the fp8-cache attention oracle.

The decode is pinned by hand-checked codes from the format definition (sign,
4-bit exponent with bias 7, 3-bit mantissa, subnormals, NaN) and by torch's
float8_e4m3fn conversion (a library routine) over all 256 codes; the
attention over decoded pages by equality with the bf16/fp64 oracle on the
decoded values and by the scale's linearity.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


@pytest.mark.parametrize("code,value", [
    (0x38, 1.0), (0xB8, -1.0), (0x7E, 448.0), (0xFE, -448.0), (0x01, 2.0 ** -9),
    (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x40, 2.0), (0x3C, 1.5), (0x00, 0.0),
    (0x30, 0.5), (0x3F, 1.875),
])
def test_decode_hand_codes(code, value):
    assert oracle.decode_e4m3([code])[0] == value


def test_decode_nan_codes():
    v = oracle.decode_e4m3([0x7F, 0xFF])
    assert np.isnan(v).all()


def test_decode_matches_library_on_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    ours = oracle.decode_e4m3(codes)
    both_nan = np.isnan(lib) & np.isnan(ours)
    assert np.array_equal(np.where(both_nan, 0, lib), np.where(both_nan, 0, ours))


def test_quantizer_round_trip_error_bound():
    """Generator check: decode(codes) * scale is within half an E4M3 step of the input."""
    w = workloads.Workload("q", 4, 2, 16, "fp32", 64, 64, 16, "ones")
    x = workloads.make_qkv_pages(w)["K_pages"]
    codes, scale = workloads.quantize_pages_e4m3(x)
    deq = oracle.dequantize_pages(codes.numpy(), scale.numpy())
    err = np.abs(deq - x.double().numpy())
    # relative step of E4M3 is 2^-3; subnormal step 2^-9 * scale
    bound = np.maximum(np.abs(x.double().numpy()) * 2.0 ** -4,
                       2.0 ** -10 * scale.double().numpy()[:, :, None, None]) * 1.0001
    assert np.all(err <= bound)


def test_fp8_oracle_is_the_oracle_on_decoded_pages():
    w = workloads.Workload("q", 4, 2, 16, "fp32", 48, 16, 16, "bernoulli", rho=0.4, seed=3)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    t, c = oracle.oracle_tables(m, w.Hkv)
    K8, sK = workloads.quantize_pages_e4m3(x["K_pages"])
    V8, sV = workloads.quantize_pages_e4m3(x["V_pages"])
    O, L = oracle.oracle_chunk_attention_fp8(x["Q"].numpy(), K8.numpy(), V8.numpy(), sK.numpy(),
                                             sV.numpy(), x["page_table"].numpy(), t, c,
                                             w.prefix_len)
    Kd = oracle.decode_e4m3(K8.numpy()) * sK.numpy()[:, :, None, None]
    Vd = oracle.decode_e4m3(V8.numpy()) * sV.numpy()[:, :, None, None]
    O2, L2 = oracle.oracle_chunk_attention(x["Q"].numpy(), Kd, Vd, x["page_table"].numpy(), t,
                                           c, w.prefix_len)
    assert np.array_equal(O, O2) and np.array_equal(L, L2)
    # doubling every V scale doubles O and leaves LSE unchanged
    O3, L3 = oracle.oracle_chunk_attention_fp8(x["Q"].numpy(), K8.numpy(), V8.numpy(),
                                               sK.numpy(), 2 * sV.numpy(),
                                               x["page_table"].numpy(), t, c, w.prefix_len)
    np.testing.assert_allclose(O3, 2 * O, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(L3, L, rtol=0, atol=1e-12)


def _fp8_case():
    """A small E4M3 cache with scales spread over (page, head) so that a wrong
    tile or a dropped scale moves the result: 3 KV heads, 11 pages."""
    w = workloads.Workload("qr", 6, 3, 16, "fp32", 144, 32, 16, "bernoulli", rho=0.35, seed=5)
    x = workloads.make_qkv_pages(w)
    m = workloads.mask_for(w)
    t, c = oracle.oracle_tables(m, w.Hkv)
    K8, sK = workloads.quantize_pages_e4m3(x["K_pages"])
    V8, sV = workloads.quantize_pages_e4m3(x["V_pages"])
    rng = np.random.default_rng(7)
    sK = sK.numpy() * rng.uniform(0.5, 4.0, sK.shape)
    sV = sV.numpy() * rng.uniform(0.5, 4.0, sV.shape)
    rows = [(h, i) for h in range(w.Hq) for i in range(w.chunk_len)]
    return w, x, t, c, K8.numpy(), V8.numpy(), sK, sV, rows


def test_rows_fp8_matches_full_fp8_oracle_row_by_row():
    """oracle_rows_fp8 (pages decoded one (page, head) tile at a time, the
    checker of the full-size E4M3 GPU test) equals oracle_chunk_attention_fp8 on
    every (head, token) row of a small cache."""
    w, x, t, c, K8, V8, sK, sV, rows = _fp8_case()
    Q = x["Q"].double().numpy()
    pt = x["page_table"].numpy()
    O, L = oracle.oracle_chunk_attention_fp8(Q, K8, V8, sK, sV, pt, t, c, w.prefix_len)
    Or, Lr = oracle.oracle_rows_fp8(Q, K8, V8, sK, sV, pt, t, c, w.prefix_len, rows)
    np.testing.assert_allclose(Or, np.stack([O[i, h] for h, i in rows]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lr, np.array([L[h, i] for h, i in rows]), rtol=0, atol=1e-12)


class _SwappedTile(oracle.fp8._DecodedPages):
    def __getitem__(self, idx):  # planted mistake: (head, page) instead of (page, head)
        p, g = idx
        return oracle.decode_e4m3(self.codes[g % self.shape[0], p % self.shape[1]]) * \
            self.scale[p, g]


class _DroppedScale(oracle.fp8._DecodedPages):
    def __getitem__(self, idx):  # planted mistake: the tile's scale left out
        p, g = idx
        return oracle.decode_e4m3(self.codes[p, g])


class _WrongScale(oracle.fp8._DecodedPages):
    def __getitem__(self, idx):  # planted mistake: another head's scale
        p, g = idx
        return oracle.decode_e4m3(self.codes[p, g]) * self.scale[p, (g + 1) % self.shape[1]]


@pytest.mark.parametrize("planted", [_SwappedTile, _DroppedScale, _WrongScale])
def test_rows_fp8_pin_catches_planted_mistakes(planted):
    w, x, t, c, K8, V8, sK, sV, rows = _fp8_case()
    Q = x["Q"].double().numpy()
    pt = x["page_table"].numpy()
    O, L = oracle.oracle_chunk_attention_fp8(Q, K8, V8, sK, sV, pt, t, c, w.prefix_len)
    Ob, Lb = oracle.oracle_rows(Q, planted(K8, sK), planted(V8, sV), pt, t, c, w.prefix_len,
                                rows)
    Of = np.stack([O[i, h] for h, i in rows])
    Lf = np.array([L[h, i] for h, i in rows])
    assert np.abs(Ob - Of).max() > 1e-3 or np.abs(Lb - Lf).max() > 1e-3
