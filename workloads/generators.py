"""Seeded generators: Q/K/V pages, page permutation, 2D block-sparse masks.

Everything here is drawn from ``numpy.random.default_rng(seed)`` so that the
CUDA path and the oracle see identical inputs.  Nothing here computes a table
or an attention output.

Layouts (shared by both sides):
  Q           [L_c, Hq, d]                 fp32 or bf16 (torch CPU tensor)
  K/V pages   [num_pages, Hkv, B, d]       same dtype as Q
  page_table  [nKblk] int32                logical KV block -> physical page
  mask        [Hq, nQblk, nKblk] uint8     nonzero = block selected
"""
import numpy as np
import torch

_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


def _normal(rng, shape):
    return torch.from_numpy(rng.standard_normal(size=shape, dtype=np.float32))


def make_qkv_pages(w, seed=None, num_pages=None, identity_pages=False):
    """Q ~ N(0,1) [L_c,Hq,d]; K/V pages ~ N(0,1); a random page permutation.

    The page table maps logical block kb to physical page
    ``perm[kb]`` with ``perm = rng.permutation(num_pages)[:nKblk]``.
    """
    seed = w.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    num_pages = w.num_pages if num_pages is None else num_pages
    assert num_pages >= w.nKblk
    dt = _DT[w.dtype]
    q = _normal(rng, (w.chunk_len, w.Hq, w.head_dim)).to(dt)
    k = _normal(rng, (num_pages, w.Hkv, w.block, w.head_dim)).to(dt)
    v = _normal(rng, (num_pages, w.Hkv, w.block, w.head_dim)).to(dt)
    if identity_pages:
        pt = np.arange(w.nKblk, dtype=np.int32)
    else:
        pt = rng.permutation(num_pages)[: w.nKblk].astype(np.int32)
    return {"Q": q, "K_pages": k, "V_pages": v, "page_table": torch.from_numpy(pt)}


def last_live_block(P, L, B):
    """int [nQblk]: the last KV block holding a position visible to Q-block qb
    (chunk tokens [qb B, min(qb B + B, L)) at positions P + t).  For block-aligned
    P and L it is the diagonal block nPblk + qb."""
    nQ = -(-L // B)
    qb = np.arange(nQ)
    return (P + np.minimum(qb * B + B - 1, L - 1)) // B


def _last(nPblk, nQblk, last):
    return nPblk + np.arange(nQblk) if last is None else np.asarray(last)


def causal_live(nPblk, nQblk, nKblk, last=None):
    """bool [nQblk, nKblk]: KV block kb can hold a key visible to Q-block qb."""
    kb = np.arange(nKblk)[None, :]
    return kb <= _last(nPblk, nQblk, last)[:, None]


def _sink_diag(nPblk, nQblk, nKblk, last=None):
    kb = np.arange(nKblk)[None, :]
    return (kb == 0) | (kb == _last(nPblk, nQblk, last)[:, None])


def bernoulli_mask(Hq, nPblk, nQblk, nKblk, rho, seed, clip=True, last=None):
    """i.i.d. Bernoulli(rho) blocks, plus the sink block and the diagonal block
    (the last live block of each Q-block)."""
    rng = np.random.default_rng(seed)
    m = rng.random((Hq, nQblk, nKblk)) < rho
    m |= _sink_diag(nPblk, nQblk, nKblk, last)[None]
    if clip:
        m &= causal_live(nPblk, nQblk, nKblk, last)[None]
    return m.astype(np.uint8)


def vertical_slash_mask(Hq, Hkv, nPblk, nQblk, nKblk, rho_col, corr, window, seed, clip=True,
                        last=None):
    """Vertical columns shared within a GQA group with probability ``corr``,
    a sink block, and a local window of ``window`` blocks ending at the diagonal.

    Head h of group g = h // (Hq/Hkv) takes column kb from the group's shared
    draw with probability corr, else from its own draw; both are
    Bernoulli(rho_col), so the per-head column density is rho_col.
    """
    rng = np.random.default_rng(seed)
    G = Hq // Hkv
    shared = rng.random((Hkv, nKblk)) < rho_col
    own = rng.random((Hq, nKblk)) < rho_col
    pick = rng.random((Hq, nKblk)) < corr
    cols = np.where(pick, np.repeat(shared, G, axis=0), own)
    kb = np.arange(nKblk)[None, :]
    lastc = _last(nPblk, nQblk, last)[:, None]
    slash = (kb == 0) | ((kb > lastc - window) & (kb <= lastc))
    m = cols[:, None, :] | slash[None]
    if clip:
        m &= causal_live(nPblk, nQblk, nKblk, last)[None]
    return m.astype(np.uint8)


def ones_mask(Hq, nPblk, nQblk, nKblk, last=None):
    """Every causally live block selected (the density-100% case)."""
    live = causal_live(nPblk, nQblk, nKblk, last)
    return np.broadcast_to(live[None], (Hq, nQblk, nKblk)).astype(np.uint8).copy()


def mask_for(w, seed=None, clip=True):
    seed = w.seed if seed is None else seed
    last = last_live_block(w.prefix_len, w.chunk_len, w.block)
    if w.mask_kind == "bernoulli":
        return bernoulli_mask(w.Hq, w.nPblk, w.nQblk, w.nKblk, w.rho, seed, clip, last)
    if w.mask_kind == "vslash":
        return vertical_slash_mask(w.Hq, w.Hkv, w.nPblk, w.nQblk, w.nKblk, w.rho, w.corr,
                                   w.window, seed, clip, last)
    if w.mask_kind == "ones":
        return ones_mask(w.Hq, w.nPblk, w.nQblk, w.nKblk, last)
    raise ValueError(w.mask_kind)


def pack_mask_bits(mask):
    """uint8 mask [..., nKblk] -> uint32 words [..., ceil(nKblk/32)], bit j of word w
    (least significant first) = mask[..., 32w + j] != 0; bits past nKblk are 0."""
    m = (np.asarray(mask) != 0)
    nK = m.shape[-1]
    W = (nK + 31) // 32
    pad = np.zeros(m.shape[:-1] + (W * 32 - nK,), dtype=bool)
    b = np.packbits(np.concatenate([m, pad], axis=-1), axis=-1, bitorder="little")
    return np.ascontiguousarray(b).view("<u4").astype(np.uint32)


def quantize_pages_e4m3(pages, scale_factor=None):
    """float pages [num_pages, Hkv, B, d] (torch) -> (uint8 E4M3 codes, float32 scales
    [num_pages, Hkv]): one scale per (page, KV head) tile, amax / 448 (448 being the
    largest E4M3 value) times an optional factor >= 1 per tile (coarser codes, so
    that scales differ more between pages), codes by torch's round-to-nearest cast.
    Input generation only: the decode belongs to each side."""
    x = pages.float()
    amax = x.abs().amax(dim=(2, 3))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    if scale_factor is not None:
        scale = scale * scale_factor
    codes = (x / scale[:, :, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()
