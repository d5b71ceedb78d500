"""FP8 (E4M3) KV pages: the decode of the stored bytes and attention over the
decoded cache (TEST INFRASTRUCTURE ONLY, like the rest of this package).

Storage format of a quantised page (the reading used for the fp8 cache of
the chunked-prefill path): each K (or V) element is one E4M3 byte (1 sign
bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds
subnormals m * 2^-9; 0x7F / 0xFF are NaN, there is no infinity), and every
(page, KV head) tile has one float32 scale: value = decode(byte) * scale.
The attention is then exactly the single-sequence definition of
``attention.oracle_chunk_attention`` on the decoded pages.
"""
import numpy as np

from .attention import oracle_chunk_attention, oracle_rows


def decode_e4m3(codes):
    """uint8 codes -> float64 values, written out from the bit layout."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = sign * (m / 8.0) * np.exp2(-6.0)
    out = np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


def dequantize_pages(codes, scale):
    """codes uint8 [num_pages, Hkv, B, d], scale float32 [num_pages, Hkv] -> float64 pages."""
    return decode_e4m3(codes) * np.asarray(scale, dtype=np.float64)[:, :, None, None]


def oracle_chunk_attention_fp8(Q, K8, V8, K_scale, V_scale, page_table, tables, counts,
                               prefix_len):
    return oracle_chunk_attention(np.asarray(Q, dtype=np.float64), dequantize_pages(K8, K_scale),
                                  dequantize_pages(V8, V_scale), page_table, tables, counts,
                                  prefix_len)


class _DecodedPages:
    """Pages decoded one (page, head) tile at a time, for the row sampler on a
    large cache (the whole cache in float64 would not fit)."""

    def __init__(self, codes, scale):
        self.codes = np.asarray(codes)
        self.scale = np.asarray(scale, dtype=np.float64)
        self.shape = self.codes.shape

    def __getitem__(self, idx):
        p, g = idx
        return decode_e4m3(self.codes[p, g]) * self.scale[p, g]


def oracle_rows_fp8(Q, K8, V8, K_scale, V_scale, page_table, tables, counts, prefix_len, rows):
    return oracle_rows(Q, _DecodedPages(K8, K_scale), _DecodedPages(V8, V_scale), page_table,
                       tables, counts, prefix_len, rows)
