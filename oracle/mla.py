"""MLA decode over a latent KV cache, in float64 on the CPU (test infrastructure).

Notation follows the DeepSeek-V2 page (snabindia.com, sections 2.1-2.3):
per token the cache keeps the joint latent ``c_KV = W_DKV x`` (width d_c) and
one decoupled RoPE key ``k_R = RoPE(W_KR x, pos)`` (width d_r) shared by all
heads.  Per head i the full key and value would be ``K_i = W_UK_i c_KV (+) k_R``
and ``V_i = W_UV_i c_KV``; the query of head i is ``q_nope_i (+) RoPE(q_pe_i)``.

Two forms are implemented and must agree (associativity pin):

* ``decode_unabsorbed`` -- the primary form: rebuild K and V per head, then
  softmax(q K^T * scale) V  (CSDN guide, section 2.1; V2 page, section 2.3
  formula Softmax((Q_c (+) Q_R)(K_c^T (+) K_R^T) / sqrt(d))).
* ``decode_absorbed`` -- W_UK folded into the query and W_UV into the output
  (V2 page, section 2.3 "硬件友好设计" and section 4.1
  ``optimize_for_inference``): all heads attend directly over the latent rows
  ``row_j = c_KV_j (+) k_R_j`` (width D = d_c + d_r), with V = row[:d_c].

Readings of points the pages leave open:

* softmax scale = 1/sqrt(d_nope + d_r), the width of the un-absorbed dot
  product, in both forms;
* RoPE pairs dimension i with i + d_r/2 (rotate-half), theta_i = base^(-2i/d_r),
  applied at each key's own position and at the query's position;
* W_UK and W_UV are stored [H][d_nope or d_v][d_c] so that K_nope = W_UK_h c;
* the query of a decode step sits at the position of the token appended in that
  step and attends to every cached token of its sequence, itself included.

No blocking, fusion or reordering beyond the definitions: numpy matrix
products serve as the contraction steps.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

from .e4m3 import e4m3_encode, E4M3_MAX


# ---------------------------------------------------------------------------
# configuration-level quantities
# ---------------------------------------------------------------------------

def softmax_scale(d_nope: int, d_r: int) -> float:
    """1/sqrt(d) with d the width of the un-absorbed per-head dot product
    (V2 page section 2.3 attention formula; d = d_nope + d_r)."""
    return 1.0 / np.sqrt(float(d_nope + d_r))


def cache_bytes_per_token(d_c: int, d_r: int, dtype: str) -> float:
    """Bytes one token occupies in one layer's latent cache (V2 page section 2.3:
    only KV_comp and k_R are stored).  fp8 adds the per-token fp32 scale."""
    width = d_c + d_r
    if dtype == "bf16":
        return 2.0 * width
    if dtype == "fp32":
        return 4.0 * width
    if dtype == "fp8_e4m3":
        return 1.0 * width + 4.0
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# RoPE (V2 page section 2.2 apply_rope / mla_rope; CSDN RotaryEmbedding)
# ---------------------------------------------------------------------------

def rope_inv_freq(d_r: int, base: float = 10000.0) -> np.ndarray:
    """theta_i = 1 / base^(2i/d_r), i = 0 .. d_r/2-1 (``arange(0, d, 2) / d``)."""
    i = np.arange(0, d_r, 2, dtype=np.float64)
    return 1.0 / np.power(float(base), i / float(d_r))


def rope(x: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate the last axis of ``x`` (width d_r) by angle pos*theta_i on the pairs
    (i, i + d_r/2):  y = x*cos + rotate_half(x)*sin  with rotate_half(x) =
    (-x[h:], x[:h]).  ``pos`` broadcasts against x's leading axes."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(d, base)
    cos, sin = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


# ---------------------------------------------------------------------------
# joint compression and the cache (V2 page sections 2.1-2.3; V3 page MLA sketch)
# ---------------------------------------------------------------------------

def down_project(x: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray):
    """KV_comp = W_DKV x and the pre-RoPE key W_KR x, for token rows x [T, d_model]."""
    x = np.asarray(x, dtype=np.float64)
    return x @ np.asarray(w_dkv, np.float64).T, x @ np.asarray(w_kr, np.float64).T


def cache_row(c_kv: np.ndarray, k_raw: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """The cached latent row of a token: c_KV followed by RoPE(k_raw, pos)."""
    return np.concatenate([np.asarray(c_kv, np.float64), rope(k_raw, pos, base)], axis=-1)


def paged_slot(block_table: np.ndarray, seq: np.ndarray, pos: np.ndarray,
               block_size: int) -> np.ndarray:
    """Physical row of token (seq, pos) in a paged cache: the page
    block_table[seq][pos // block_size], row pos % block_size inside it."""
    seq = np.asarray(seq, dtype=np.int64)
    pos = np.asarray(pos, dtype=np.int64)
    page = np.asarray(block_table, dtype=np.int64)[seq, pos // block_size]
    return page * block_size + pos % block_size


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), as float64."""
    x = np.asarray(x, dtype=np.float64)
    _, k = np.frexp(np.where(x != 0, x, 1.0))
    quantum = np.ldexp(1.0, (k - 8).astype(np.int64))   # 8 significant bits
    return np.where(x != 0, np.rint(x / quantum) * quantum, 0.0)


def fp8_quantize_row(row32: np.ndarray):
    """Per-token e4m3 quantisation of cache rows [..., D] given in float32.

    amax = max |row|; scale = amax / 448 and inv = 448 / amax, both float32;
    codes = e4m3(row * inv) with round-to-nearest-even and saturation.  A zero
    row gets scale 1 and zero codes.  (Config "one fp32 scale per token
    (absmax/448)"; V3 page FP8 KV cache.)"""
    r = np.asarray(row32, dtype=np.float32)
    amax = np.max(np.abs(r), axis=-1).astype(np.float32)
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    scale = np.where(zero, np.float32(1.0), (safe / np.float32(E4M3_MAX)).astype(np.float32))
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    scaled = (r * inv[..., None]).astype(np.float32)
    codes = e4m3_encode(scaled)
    codes[zero] = 0
    return codes, scale.astype(np.float32)


def append_tokens(cache: np.ndarray, block_table: np.ndarray, seq: np.ndarray, pos: np.ndarray,
                  c_kv: np.ndarray, k_raw: np.ndarray, block_size: int,
                  base: float = 10000.0) -> np.ndarray:
    """Write each token's row c_KV (+) RoPE(k_raw, pos) into ``cache`` (a float64
    array [num_blocks * block_size, D]) at its paged slot; returns the slots."""
    slots = paged_slot(block_table, seq, pos, block_size)
    cache[slots] = cache_row(c_kv, k_raw, pos, base)
    return slots


# ---------------------------------------------------------------------------
# absorbed query (V2 page section 2.3; section 4.1 optimize_for_inference)
# ---------------------------------------------------------------------------

def absorb_q(q_nope: np.ndarray, q_pe: np.ndarray, w_uk: np.ndarray, pos,
             base: float = 10000.0) -> np.ndarray:
    """q_lat[b,h] = (W_UK_h^T q_nope[b,h]) (+) RoPE(q_pe[b,h], pos_b).

    With K_nope_j = W_UK_h c_j, the nope score q_nope . K_nope_j equals
    (W_UK_h^T q_nope) . c_j, which is what the absorbed query carries."""
    q_nope = np.asarray(q_nope, np.float64)          # [B, H, dn]
    w_uk = np.asarray(w_uk, np.float64)              # [H, dn, dc]
    lat = np.einsum("bhk,hkc->bhc", q_nope, w_uk)
    pos = np.asarray(pos, np.float64)[:, None]       # [B, 1] broadcast over heads
    return np.concatenate([lat, rope(q_pe, pos, base)], axis=-1)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _softmax_lse(s: np.ndarray):
    """Row softmax of scores s [..., L] with max subtraction; returns (p, lse)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=-1, keepdims=True)
    return e / z, (m + np.log(z))[..., 0]


def decode_unabsorbed(q_nope: np.ndarray, q_pe_rot: np.ndarray, c_kv: np.ndarray,
                      k_r_rot: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray,
                      scale: float, heads: Optional[Sequence[int]] = None,
                      return_p: bool = False):
    """One sequence, the un-absorbed form.

    q_nope [H, dn], q_pe_rot [H, dr] (already rotated at the query position),
    c_kv [L, dc], k_r_rot [L, dr] (rotated at each key's position),
    w_uk [H, dn, dc], w_uv [H, dv, dc].  For each head h:
    K_h = [c W_UK_h^T | k_R] (L x (dn+dr)), V_h = c W_UV_h^T (L x dv),
    s = scale * K_h q_h, p = softmax(s), o_h = p V_h, lse_h = log sum exp s.
    Returns o [len(heads), dv], lse [len(heads)] (and p if asked)."""
    c = np.asarray(c_kv, np.float64)
    kr = np.asarray(k_r_rot, np.float64)
    heads = range(q_nope.shape[0]) if heads is None else heads
    outs, lses, ps = [], [], []
    for h in heads:
        k_nope = c @ np.asarray(w_uk[h], np.float64).T          # [L, dn]
        v = c @ np.asarray(w_uv[h], np.float64).T               # [L, dv]
        k = np.concatenate([k_nope, kr], axis=1)                # [L, dn+dr]
        q = np.concatenate([np.asarray(q_nope[h], np.float64),
                            np.asarray(q_pe_rot[h], np.float64)])
        s = scale * (k @ q)
        p, lse = _softmax_lse(s)
        outs.append(p @ v)
        lses.append(lse)
        ps.append(p)
    res = (np.stack(outs), np.array(lses))
    return res + (np.stack(ps),) if return_p else res


def decode_absorbed(q_lat: np.ndarray, rows: np.ndarray, scale: float, d_c: int,
                    row_scale: Optional[np.ndarray] = None, return_p: bool = False):
    """One sequence, the absorbed form: all heads attend over the latent rows.

    q_lat [H, D], rows [L, D] (D = d_c + d_r).  s_hj = scale * q_lat_h . row_j,
    p = softmax_j(s), o_lat_h = sum_j p_hj row_j[:d_c], lse_h = log sum_j exp s_hj.
    ``row_scale`` [L] multiplies each row (a dequantised fp8 cache: row = scale_j * code_j).
    With L = 0 the output is zero and lse is -inf."""
    q = np.asarray(q_lat, np.float64)
    r = np.asarray(rows, np.float64)
    if row_scale is not None:
        r = r * np.asarray(row_scale, np.float64)[:, None]
    if r.shape[0] == 0:
        o = np.zeros((q.shape[0], d_c))
        lse = np.full(q.shape[0], -np.inf)
        return (o, lse, np.zeros((q.shape[0], 0))) if return_p else (o, lse)
    s = scale * (q @ r.T)                                       # [H, L]
    p, lse = _softmax_lse(s)
    o = p @ r[:, :d_c]
    return (o, lse, p) if return_p else (o, lse)


def split_partials(q_lat: np.ndarray, rows: np.ndarray, scale: float, d_c: int,
                   bounds: Sequence[int]):
    """Attention restricted to each token range [bounds[s], bounds[s+1]): the
    per-split normalised output and log-sum-exp (the flash-decoding partials)."""
    outs, lses = [], []
    for s in range(len(bounds) - 1):
        o, lse = decode_absorbed(q_lat, rows[bounds[s]:bounds[s + 1]], scale, d_c)
        outs.append(o)
        lses.append(lse)
    return np.stack(outs), np.stack(lses)


def combine(o_parts: np.ndarray, lse_parts: np.ndarray):
    """Merge S partials: lse = log sum_s exp(lse_s);
    o = sum_s exp(lse_s - lse) o_s.  Splits with lse_s = -inf carry no weight;
    if every split is empty the result is o = 0, lse = -inf."""
    o_parts = np.asarray(o_parts, np.float64)       # [S, ..., dc]
    lse_parts = np.asarray(lse_parts, np.float64)   # [S, ...]
    m = np.max(lse_parts, axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe), 0.0)
    z = np.sum(w, axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, z, 1.0)), -np.inf)
    o = np.sum(w[..., None] * o_parts, axis=0) / np.where(finite, z, 1.0)[..., None]
    o = np.where(finite[..., None], o, 0.0)
    return o, lse


# ---------------------------------------------------------------------------
# output side (V2 page section 2.3: W_UV absorbed into W_O)
# ---------------------------------------------------------------------------

def up_project_out(o_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """o[b,h] = W_UV_h o_lat[b,h]:  [B,H,dc] x [H,dv,dc] -> [B,H,dv]."""
    return np.einsum("bhc,hvc->bhv", np.asarray(o_lat, np.float64), np.asarray(w_uv, np.float64))


def out_project(o: np.ndarray, w_o: np.ndarray) -> np.ndarray:
    """y[b] = W_O concat_h o[b,h]:  [B, H*dv] x [dm, H*dv]^T -> [B, dm]."""
    o = np.asarray(o, np.float64)
    return o.reshape(o.shape[0], -1) @ np.asarray(w_o, np.float64).T


# ---------------------------------------------------------------------------
# a whole decode step on a workload (absorbed form, every sequence)
# ---------------------------------------------------------------------------

def _rows_of_sequence(wl, b: int, base: float):
    """float64 latent rows of sequence b (history + the appended token), in order."""
    d = wl.dims
    if wl.hist_x is not None:
        sel = wl.hist_seq == b
        c_h, k_h = down_project(wl.hist_x[sel], wl.w_dkv, wl.w_kr)
        c_n, k_n = down_project(wl.new_x[b:b + 1], wl.w_dkv, wl.w_kr)
    else:
        sel = wl.hist_seq == b
        c_h, k_h = wl.to_f64(wl.hist_c_kv[sel]), wl.to_f64(wl.hist_k_r[sel])
        c_n, k_n = wl.to_f64(wl.new_c_kv[b:b + 1]), wl.to_f64(wl.new_k_r[b:b + 1])
    pos_h = wl.hist_pos[sel]
    c = np.concatenate([c_h, c_n])
    k = np.concatenate([k_h, k_n])
    pos = np.concatenate([pos_h, [wl.hist_len[b]]])
    assert c.shape == (wl.hist_len[b] + 1, d["d_c"])
    return c, k, pos


def step_outputs(wl, seqs: Optional[List[int]] = None, fp8_dequant: bool = False) -> Dict[str, np.ndarray]:
    """All outputs of one decode step for the sequences ``seqs`` (default: all):
    q_lat [n,H,D], o_lat [n,H,dc], lse [n,H], o [n,H,dv], y [n,dm].

    ``fp8_dequant``: attend over the oracle's own e4m3-quantised rows (codes times
    per-token scale) instead of the exact rows -- the reference for the FP8
    cache on its dequantised values."""
    d = wl.dims
    base = wl.rope_base
    scale = softmax_scale(d["d_nope"], d["d_r"])
    seqs = list(range(wl.batch)) if seqs is None else list(seqs)
    q_nope = wl.to_f64(wl.q_nope[seqs])
    q_pe = wl.to_f64(wl.q_pe[seqs])
    q_lat = absorb_q(q_nope, q_pe, wl.to_f64(wl.w_uk), wl.new_pos[seqs], base)
    o_lat, lse = [], []
    for i, b in enumerate(seqs):
        c, k, pos = _rows_of_sequence(wl, b, base)
        rows = cache_row(c, k, pos, base)
        if fp8_dequant:
            from .e4m3 import e4m3_decode
            deq = np.empty_like(rows)
            for r0 in range(0, rows.shape[0], 8192):     # rows are quantised independently
                codes, sc = fp8_quantize_row(rows[r0:r0 + 8192].astype(np.float32))
                deq[r0:r0 + 8192] = e4m3_decode(codes) * sc[:, None].astype(np.float64)
            o, l = decode_absorbed(q_lat[i], deq, scale, d["d_c"])
        else:
            o, l = decode_absorbed(q_lat[i], rows, scale, d["d_c"])
        o_lat.append(o)
        lse.append(l)
    o_lat = np.stack(o_lat)
    lse = np.stack(lse)
    o = up_project_out(o_lat, wl.to_f64(wl.w_uv))
    y = out_project(o, wl.to_f64(wl.w_o))
    return dict(q_lat=q_lat, o_lat=o_lat, lse=lse, o=o, y=y)


def step_outputs_unabsorbed(wl, b: int, heads: Optional[Sequence[int]] = None):
    """The un-absorbed form for sequence b: per-head o [n, dv] and lse [n]."""
    d = wl.dims
    base = wl.rope_base
    scale = softmax_scale(d["d_nope"], d["d_r"])
    c, k, pos = _rows_of_sequence(wl, b, base)
    k_rot = rope(k, pos, base)
    q_pe_rot = rope(wl.to_f64(wl.q_pe[b]), wl.new_pos[b], base)
    return decode_unabsorbed(wl.to_f64(wl.q_nope[b]), q_pe_rot, c, k_rot,
                             wl.to_f64(wl.w_uk), wl.to_f64(wl.w_uv), scale, heads)
