"""Seeded synthetic inputs for MLA decode over a paged latent KV cache.

This module is shared by the fp64 oracle (``oracle/``) and by the CUDA path's
tests and benchmark.  It holds none of the method's arithmetic: it only draws
random numbers, rounds them to the storage dtype (bf16 round-to-nearest-even,
a plain dtype conversion) and lays out page tables.  Everything the method
computes -- projections, RoPE, absorption, softmax, quantisation -- happens on
either side of it, independently.

Workloads (shapes from the DeepSeek-V2 page, "MLA architecture" section,
table of configuration parameters: h=128, d=128, d_c=512, d_r=64):

``tiny_fp32``        batch 1, H=8, d_model=256, d_c=64, d_r=16, d_nope=d_v=32,
                     context 128, contiguous pages, fp32; the cache contents
                     come from x through W_DKV / W_KR (drawn here, projected by
                     the method's own code).
``v2_b32_l2048``     batch 32, context 2048 each, bf16, identity page table.
``v2_b32_l2048_shuf`` the same data with the pool's pages permuted.
``v2_ragged64``      64 sequences, history length uniform in [1, 8192], pages
                     shuffled in a shared pool with 5% spare pages; one token
                     appended per sequence at position len, decode over len+1.
``v2_b4_l32k``       batch 4, context 32768.
``v2_b2_l128k_fp8``  batch 2, context 131072, e4m3 cache with per-token scale.

Every sequence b has ``hist_len[b]`` cached history tokens at positions
0..hist_len[b]-1 and one new token at position ``hist_len[b]`` that the decode
step appends before attending over ``hist_len[b] + 1`` tokens.  For the fixed
context workloads hist_len = L - 1, so the query sits at position L-1 and
attends to all L tokens.

bf16 arrays are returned as ``uint16`` bit patterns; ``bf16_to_f32`` /
``bf16_to_f64`` convert them exactly.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

BLOCK_SIZE = 64

V2_DIMS = dict(num_heads=128, d_model=5120, d_c=512, d_r=64, d_nope=128, d_v=128)
TINY_DIMS = dict(num_heads=8, d_model=256, d_c=64, d_r=16, d_nope=32, d_v=32)

WORKLOADS = (
    "tiny_fp32",
    "v2_b32_l2048",
    "v2_b32_l2048_shuf",
    "v2_ragged64",
    "v2_b4_l32k",
    "v2_b2_l128k_fp8",
)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    r = r.astype(np.uint16)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_to_f32(b).astype(np.float64)


@dataclasses.dataclass
class Workload:
    name: str
    dims: Dict[str, int]
    act_dtype: str            # "bf16" | "fp32"
    cache_dtype: str          # "bf16" | "fp8_e4m3" | "fp32"
    batch: int
    hist_len: np.ndarray      # int32 [B]
    block_table: np.ndarray   # int32 [B, max_blocks]; unused entries are 0
    num_blocks: int
    # history tokens, grouped by sequence in order, positions 0..hist_len-1
    hist_seq: np.ndarray      # int32 [T]
    hist_pos: np.ndarray      # int32 [T]
    # activations: bf16 bits (uint16) for bf16 workloads, float32 for fp32
    hist_c_kv: Optional[np.ndarray]   # [T, d_c]
    hist_k_r: Optional[np.ndarray]    # [T, d_r]  (before RoPE)
    new_c_kv: Optional[np.ndarray]    # [B, d_c]
    new_k_r: Optional[np.ndarray]     # [B, d_r]  (before RoPE)
    q_nope: np.ndarray                # [B, H, d_nope]
    q_pe: np.ndarray                  # [B, H, d_r]  (before RoPE)
    w_uk: np.ndarray                  # [H, d_nope, d_c]
    w_uv: np.ndarray                  # [H, d_v, d_c]
    w_o: np.ndarray                   # [d_model, H*d_v]
    # tiny workload only: token inputs and down projections
    hist_x: Optional[np.ndarray] = None   # [T, d_model]
    new_x: Optional[np.ndarray] = None    # [B, d_model]
    w_dkv: Optional[np.ndarray] = None    # [d_c, d_model]
    w_kr: Optional[np.ndarray] = None     # [d_r, d_model]
    rope_base: float = 10000.0

    @property
    def seq_lens(self) -> np.ndarray:
        return (self.hist_len + 1).astype(np.int32)

    @property
    def new_pos(self) -> np.ndarray:
        return self.hist_len.astype(np.int32)

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.sum())

    def to_f64(self, a: np.ndarray) -> np.ndarray:
        """Exact float64 view of an activation or weight array of this workload."""
        if a.dtype == np.uint16:
            return bf16_to_f64(a)
        return np.asarray(a, dtype=np.float64)


def _normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def _normal_f32(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _page_table(rng: Optional[np.random.Generator], hist_len: np.ndarray, spare_frac: float,
                shuffle: bool):
    """Blocks for each sequence's hist_len+1 tokens, drawn from one pool."""
    need = (hist_len + 1 + BLOCK_SIZE - 1) // BLOCK_SIZE
    used = int(need.sum())
    num_blocks = used + int(np.ceil(used * spare_frac))
    pool = np.arange(num_blocks, dtype=np.int32)
    if shuffle:
        pool = rng.permutation(num_blocks).astype(np.int32)
    max_blocks = int(need.max())
    table = np.zeros((len(hist_len), max_blocks), dtype=np.int32)
    k = 0
    for b, n in enumerate(need):
        table[b, :n] = pool[k:k + n]
        k += n
    return table, num_blocks


def _hist_index(hist_len: np.ndarray):
    seq = np.repeat(np.arange(len(hist_len), dtype=np.int32), hist_len)
    starts = np.concatenate([[0], np.cumsum(hist_len)[:-1]])
    pos = (np.arange(int(hist_len.sum()), dtype=np.int64) - np.repeat(starts, hist_len)).astype(np.int32)
    return seq, pos


def make(name: str, *, seed: Optional[int] = None, batch: Optional[int] = None,
         context: Optional[int] = None, with_weights: bool = True) -> Workload:
    """Build one named workload.  ``batch``/``context`` override the sizes (small cases
    for fast tests); ``seed`` overrides the default seed of the workload."""
    if name == "tiny_fp32":
        return _make_tiny(seed=0 if seed is None else seed, batch=batch or 1, context=context or 128)
    if name not in WORKLOADS:
        raise KeyError(name)
    defaults = {
        "v2_b32_l2048": (1, 32, 2048, "bf16", False),
        "v2_b32_l2048_shuf": (1, 32, 2048, "bf16", True),
        "v2_ragged64": (2, 64, None, "bf16", True),
        "v2_b4_l32k": (3, 4, 32768, "bf16", False),
        "v2_b2_l128k_fp8": (4, 2, 131072, "fp8_e4m3", False),
    }
    dseed, dbatch, dctx, cache_dtype, shuffle = defaults[name]
    seed = dseed if seed is None else seed
    B = batch or dbatch
    rng = np.random.default_rng(seed)
    if name == "v2_ragged64":
        maxlen = context or 8192
        hist_len = rng.integers(1, maxlen + 1, B).astype(np.int32)
        spare = 0.05
    else:
        L = context or dctx
        hist_len = np.full(B, L - 1, dtype=np.int32)
        spare = 0.0
    # the page permutation has its own stream, so a shuffled workload holds the same data
    page_rng = np.random.default_rng(seed + 1000) if shuffle else None
    return _make_v2(name, rng, page_rng, hist_len, cache_dtype, spare, with_weights)


def _make_v2(name, rng, page_rng, hist_len, cache_dtype, spare, with_weights) -> Workload:
    d = V2_DIMS
    H, dc, dr, dn, dv, dm = d["num_heads"], d["d_c"], d["d_r"], d["d_nope"], d["d_v"], d["d_model"]
    B = len(hist_len)
    table, num_blocks = _page_table(page_rng, hist_len, spare, page_rng is not None)
    seq, pos = _hist_index(hist_len)
    T = int(hist_len.sum())
    hist_c = _normal_bf16(rng, (T, dc))
    hist_k = _normal_bf16(rng, (T, dr))
    new_c = _normal_bf16(rng, (B, dc))
    new_k = _normal_bf16(rng, (B, dr))
    q_nope = _normal_bf16(rng, (B, H, dn))
    q_pe = _normal_bf16(rng, (B, H, dr))
    if with_weights:
        w_uk = _normal_bf16(rng, (H, dn, dc), 1.0 / np.sqrt(dc))
        w_uv = _normal_bf16(rng, (H, dv, dc), 1.0 / np.sqrt(dc))
        w_o = _normal_bf16(rng, (dm, H * dv), 1.0 / np.sqrt(H * dv))
    else:
        w_uk = w_uv = w_o = None
    return Workload(name=name, dims=dict(d), act_dtype="bf16", cache_dtype=cache_dtype, batch=B,
                    hist_len=hist_len, block_table=table, num_blocks=num_blocks,
                    hist_seq=seq, hist_pos=pos, hist_c_kv=hist_c, hist_k_r=hist_k,
                    new_c_kv=new_c, new_k_r=new_k, q_nope=q_nope, q_pe=q_pe,
                    w_uk=w_uk, w_uv=w_uv, w_o=w_o)


def _make_tiny(seed: int, batch: int, context: int) -> Workload:
    d = TINY_DIMS
    H, dc, dr, dn, dv, dm = d["num_heads"], d["d_c"], d["d_r"], d["d_nope"], d["d_v"], d["d_model"]
    rng = np.random.default_rng(seed)
    hist_len = np.full(batch, context - 1, dtype=np.int32)
    table, num_blocks = _page_table(None, hist_len, 0.0, False)
    seq, pos = _hist_index(hist_len)
    T = int(hist_len.sum())
    hist_x = _normal_f32(rng, (T, dm))
    new_x = _normal_f32(rng, (batch, dm))
    w_dkv = _normal_f32(rng, (dc, dm), 1.0 / np.sqrt(dm))
    w_kr = _normal_f32(rng, (dr, dm), 1.0 / np.sqrt(dm))
    q_nope = _normal_f32(rng, (batch, H, dn))
    q_pe = _normal_f32(rng, (batch, H, dr))
    w_uk = _normal_f32(rng, (H, dn, dc), 1.0 / np.sqrt(dc))
    w_uv = _normal_f32(rng, (H, dv, dc), 1.0 / np.sqrt(dc))
    w_o = _normal_f32(rng, (dm, H * dv), 1.0 / np.sqrt(H * dv))
    return Workload(name="tiny_fp32", dims=dict(d), act_dtype="fp32", cache_dtype="fp32",
                    batch=batch, hist_len=hist_len, block_table=table, num_blocks=num_blocks,
                    hist_seq=seq, hist_pos=pos, hist_c_kv=None, hist_k_r=None,
                    new_c_kv=None, new_k_r=None, q_nope=q_nope, q_pe=q_pe,
                    w_uk=w_uk, w_uv=w_uv, w_o=w_o, hist_x=hist_x, new_x=new_x,
                    w_dkv=w_dkv, w_kr=w_kr)


def random_tokens(rng: np.random.Generator, n: int, d_c: int, d_r: int, bf16: bool = True):
    """n standalone (c_KV, k_R) token rows, N(0,1); used by append-only tests."""
    if bf16:
        return _normal_bf16(rng, (n, d_c)), _normal_bf16(rng, (n, d_r))
    return _normal_f32(rng, (n, d_c)), _normal_f32(rng, (n, d_r))
