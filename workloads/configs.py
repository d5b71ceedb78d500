"""Workload shapes for CompactAttention chunked prefill.

Shapes follow the LLaMA-3.1-8B attention geometry the CompactAttention
abstract evaluates on (32 query heads, 8 KV heads, head_dim 128) at the
context lengths it names (up to 128K, chunked prefill).  Mask recipes are
synthetic stand-ins for the output of a pattern-search method (the pages
publish no masks); their constants are stated here and nowhere else.
"""
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    Hq: int
    Hkv: int
    head_dim: int
    dtype: str          # "fp32" or "bf16": dtype of Q, K and V
    prefix_len: int     # P: tokens already in the paged KV cache
    chunk_len: int      # L_c: tokens of this chunk
    block: int          # B: KV block size == page size == Q-block size
    mask_kind: str      # "bernoulli" | "vslash" | "ones"
    rho: float = 0.0    # bernoulli density, or per-column density for vslash
    corr: float = 0.0   # vslash: within-group head correlation c
    window: int = 8     # vslash: local window in blocks, ending at the diagonal
    seed: int = 0

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def nPblk(self):
        return self.prefix_len // self.block

    @property
    def nQblk(self):  # Q-block qb = chunk tokens [qb B, qb B + B); the last may be partial
        return -(-self.chunk_len // self.block)

    @property
    def nKblk(self):  # KV block kb = positions [kb B, kb B + B); the last may be partial
        return -(-(self.prefix_len + self.chunk_len) // self.block)

    @property
    def num_pages(self):
        return self.nKblk

    def with_(self, **kw):
        return replace(self, **kw)


CONFIGS = {
    # small case: 4 q heads sharing one KV head, fp32 inputs
    "tiny": Workload("tiny", 4, 1, 64, "fp32", 1024, 256, 64, "bernoulli", rho=0.3),
    # LLaMA-3.1-8B attention shape, 16K prefix + 2K chunk
    "llama16k": Workload("llama16k", 32, 8, 128, "bf16", 16384, 2048, 64, "bernoulli", rho=0.2),
    # last 2K chunk of a 128K prompt, vertical-slash masks at ~10% density
    "ctx128k": Workload("ctx128k", 32, 8, 128, "bf16", 129024, 2048, 64, "vslash",
                        rho=0.05, corr=0.7, window=8),
}


def get_config(name):
    return CONFIGS[name]


def sweep_chunk(c, chunk_len=4096, total=131072):
    """Chunk c of the full chunked-prefill sweep (131072 tokens in chunks of 4096)."""
    assert 0 <= c < total // chunk_len
    return Workload(f"sweep{c}", 32, 8, 128, "bf16", c * chunk_len, chunk_len, 64, "vslash",
                    rho=0.05, corr=0.7, window=8, seed=c)


def density_cell(rho_col, corr, block=64, seed=0):
    """One cell of the 64K density / correlation sweep (prefix 63488 + chunk 2048)."""
    kind = "ones" if rho_col >= 1.0 else "vslash"
    return Workload(f"d64k_b{block}_r{rho_col}_c{corr}", 32, 8, 128, "bf16", 63488, 2048, block,
                    kind, rho=rho_col, corr=corr, window=8 if block == 64 else 4, seed=seed)
