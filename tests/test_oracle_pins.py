"""Pins of the fp64 oracle against things other than itself.

Each test names what it pins and which plausible mistake it would catch.
None of these tests needs a GPU.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads
from oracle import mla as om


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# RoPE: closed forms worked by hand, norm, identity, relative-position property
# ---------------------------------------------------------------------------

def test_rope_closed_forms(golden_dir):
    """Hand-derived values: catch a wrong sign, a swapped pairing
    (interleaved instead of rotate-half) or a wrong frequency exponent."""
    g = json.load(open(os.path.join(golden_dir, "rope_closed_forms.json")))
    for c in g["cases"]:
        y = oracle.rope(np.array(c["x"], float), c["pos"], c["base"])
        np.testing.assert_allclose(y, c["y"], rtol=0, atol=1e-15)


def test_rope_inv_freq_endpoints(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "page_figures.json")))
    d = g["rope_dim"]["qk_rope_head_dim"]
    base = g["rope_base"]["base"]
    th = oracle.rope_inv_freq(d, base)
    assert th.shape == (d // 2,)
    assert th[0] == 1.0
    # last frequency: base^(-(d-2)/d) = 10000^(-62/64)
    assert th[-1] == pytest.approx(10000.0 ** (-62.0 / 64.0), rel=1e-15)
    assert np.all(np.diff(th) < 0)


def test_rope_norm_identity_relative():
    rng = _rng(1)
    x = rng.standard_normal((50, 64))
    pos = rng.integers(0, 200000, 50)
    y = oracle.rope(x, pos)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_array_equal(oracle.rope(x, 0), x)
    # <R(m) q, R(n) k> depends on m - n only
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n, t in [(5, 3, 17), (1000, 20, 4096), (131071, 0, 7)]:
        a = oracle.rope(q, m) @ oracle.rope(k, n)
        b = oracle.rope(q, m + t) @ oracle.rope(k, n + t)
        assert a == pytest.approx(b, rel=1e-9, abs=1e-9)


# ---------------------------------------------------------------------------
# paging and cache size
# ---------------------------------------------------------------------------

def test_paged_slot_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "paging_small.json")))
    bt = np.array(g["block_table"], np.int32)
    seq = [t["seq"] for t in g["tokens"]]
    pos = [t["pos"] for t in g["tokens"]]
    slots = oracle.paged_slot(bt, seq, pos, g["block_size"])
    assert list(slots) == [t["slot"] for t in g["tokens"]]


def test_append_tokens_writes_only_its_slots():
    rng = _rng(2)
    bt = np.array([[3, 1], [0, 2]], np.int32)
    cache = np.full((4 * 64, 10), 7.0)
    seq = np.array([0, 1, 1])
    pos = np.array([70, 0, 127])
    c = rng.standard_normal((3, 8))
    k = rng.standard_normal((3, 2))
    slots = oracle.append_tokens(cache, bt, seq, pos, c, k, 64)
    assert list(slots) == [1 * 64 + 6, 0 * 64 + 0, 2 * 64 + 63]
    np.testing.assert_array_equal(cache[slots, :8], c)
    np.testing.assert_allclose(cache[slots, 8:], oracle.rope(k, pos))
    untouched = np.setdiff1d(np.arange(256), slots)
    assert np.all(cache[untouched] == 7.0)


def test_cache_bytes_per_token(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "page_figures.json")))
    t = g["v2_config_table"]
    lat = g["latent_cache_per_token"]
    assert oracle.cache_bytes_per_token(t["d_c"], t["d_r"], "bf16") == lat["bf16_bytes"]
    assert oracle.cache_bytes_per_token(t["d_c"], t["d_r"], "fp8_e4m3") == lat["fp8_bytes_with_scale"]
    assert oracle.cache_bytes_per_token(t["d_c"], t["d_r"], "fp32") == lat["fp32_bytes"]
    # against the MHA figure of the CSDN guide: the per-head K and V of an MHA layer
    # at the V2 head count and width, 2 bytes each, versus the latent row
    mha = g["mha_cache_per_token"]
    assert 2 * mha["heads"] * mha["head_dim"] * mha["elem_bytes"] == mha["bytes"]
    mha_v2 = 2 * t["num_heads"] * t["head_dim"] * 2
    assert mha_v2 / oracle.cache_bytes_per_token(t["d_c"], t["d_r"], "bf16") == pytest.approx(56.888, rel=1e-3)


def test_workload_dims_match_page_table(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "page_figures.json")))
    t = g["v2_config_table"]
    d = workloads.V2_DIMS
    assert (d["num_heads"], d["d_nope"], d["d_v"], d["d_c"], d["d_r"]) == (
        t["num_heads"], t["head_dim"], t["head_dim"], t["d_c"], t["d_r"])
    assert oracle.softmax_scale(d["d_nope"], d["d_r"]) == 1.0 / math.sqrt(192.0)


# ---------------------------------------------------------------------------
# attention: brute force, closed forms, invariants, library routine
# ---------------------------------------------------------------------------

def _loop_attention(q, K, V, scale):
    """Pure-python scaled dot-product attention for one query (tiny sizes)."""
    s = [scale * sum(qi * ki for qi, ki in zip(q, krow)) for krow in K]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    z = sum(e)
    o = [sum(e[j] / z * V[j][c] for j in range(len(K))) for c in range(len(V[0]))]
    return o, m + math.log(z)


def test_unabsorbed_brute_force_tiny():
    """H=2, d_c=4, d_r=2, d_nope=d_v=3, L=3: rebuild K_h, V_h with explicit loops
    (catches a transposed W_UK / W_UV, a dropped RoPE term, a wrong scale)."""
    rng = _rng(3)
    H, dc, dr, dn, L = 2, 4, 2, 3, 3
    c = rng.standard_normal((L, dc))
    kr = rng.standard_normal((L, dr))
    w_uk = rng.standard_normal((H, dn, dc))
    w_uv = rng.standard_normal((H, dn, dc))
    qn = rng.standard_normal((H, dn))
    qr = rng.standard_normal((H, dr))
    scale = 1.0 / math.sqrt(dn + dr)
    o, lse = oracle.decode_unabsorbed(qn, qr, c, kr, w_uk, w_uv, scale)
    for h in range(H):
        K = [[sum(w_uk[h, k, cc] * c[j, cc] for cc in range(dc)) for k in range(dn)] + list(kr[j])
             for j in range(L)]
        V = [[sum(w_uv[h, v, cc] * c[j, cc] for cc in range(dc)) for v in range(dn)] for j in range(L)]
        q = list(qn[h]) + list(qr[h])
        o_ref, lse_ref = _loop_attention(q, K, V, scale)
        np.testing.assert_allclose(o[h], o_ref, rtol=1e-13, atol=1e-14)
        assert lse[h] == pytest.approx(lse_ref, rel=1e-13)


def test_absorbed_closed_forms():
    rng = _rng(4)
    dc, dr, H = 4, 2, 2
    scale = 0.7
    # L = 1: output is the single value row, lse is its score
    q = rng.standard_normal((H, dc + dr))
    row = rng.standard_normal((1, dc + dr))
    o, lse = oracle.decode_absorbed(q, row, scale, dc)
    np.testing.assert_allclose(o, np.repeat(row[:, :dc], H, 0), rtol=1e-15)
    np.testing.assert_allclose(lse, scale * q @ row[0], rtol=1e-14)
    # q = 0: uniform average of the value rows, lse = log L
    rows = rng.standard_normal((3, dc + dr))
    o, lse = oracle.decode_absorbed(np.zeros((H, dc + dr)), rows, scale, dc)
    np.testing.assert_allclose(o, np.repeat(rows[:, :dc].mean(0, keepdims=True), H, 0), rtol=1e-14)
    np.testing.assert_allclose(lse, np.log(3.0), rtol=1e-15)
    # equal scores (rows differing only orthogonally to q): again the mean
    qv = np.zeros((1, dc + dr)); qv[0, 0] = 1.0
    rows2 = rows.copy(); rows2[:, 0] = 0.5
    o, lse = oracle.decode_absorbed(qv, rows2, scale, dc)
    np.testing.assert_allclose(o[0], rows2[:, :dc].mean(0), rtol=1e-14)
    assert lse[0] == pytest.approx(scale * 0.5 + np.log(3.0), rel=1e-14)
    # one score larger by 1e3: that row alone
    rows3 = rows.copy(); rows3[:, 0] = 0.0; rows3[1, 0] = 1e3 / scale
    o, lse = oracle.decode_absorbed(qv, rows3, scale, dc)
    np.testing.assert_allclose(o[0], rows3[1, :dc], rtol=1e-14)
    # empty sequence
    o, lse = oracle.decode_absorbed(q, np.zeros((0, dc + dr)), scale, dc)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_softmax_invariants():
    rng = _rng(5)
    q = rng.standard_normal((16, 40)) * 3
    rows = rng.standard_normal((300, 40))
    o, lse, p = oracle.decode_absorbed(q, rows, 0.4, 32, return_p=True)
    assert np.max(np.abs(p.sum(1) - 1.0)) <= 1e-12
    s = 0.4 * q @ rows.T
    assert np.all(lse >= s.max(1))
    assert np.all(p >= 0)


def test_absorbed_equals_sdpa_fp64_cpu():
    """Absorbed MLA is multi-query attention with one KV head: K = latent rows
    (width D), V = rows[:, :d_c].  torch's scaled_dot_product_attention on the
    CPU in float64 is the textbook routine it must reproduce."""
    rng = _rng(6)
    H, dc, dr, L = 16, 64, 16, 333
    q = rng.standard_normal((H, dc + dr))
    rows = rng.standard_normal((L, dc + dr))
    scale = 1.0 / math.sqrt(32 + 16)
    o, lse = oracle.decode_absorbed(q, rows, scale, dc)
    tq = torch.from_numpy(q)[None, :, None, :]                   # [1, H, 1, D]
    tk = torch.from_numpy(rows)[None, None].expand(1, H, L, dc + dr)
    tv = torch.from_numpy(rows[:, :dc])[None, None].expand(1, H, L, dc)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-14)
    ref_lse = torch.logsumexp(scale * (tq[0, :, 0] @ torch.from_numpy(rows).T), dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=1e-13)


def test_associativity_absorbed_equals_unabsorbed():
    """The weight-absorption identities of the V2 page (section 2.3): the
    absorbed form reproduces the un-absorbed one (relative error <= 1e-12)."""
    wl = workloads.make("v2_b32_l2048", batch=2, context=150)
    out = oracle.step_outputs(wl)
    for b in range(wl.batch):
        heads = [0, 5, 77, 127]
        o_un, lse_un = om.step_outputs_unabsorbed(wl, b, heads)
        o_ab = out["o"][b, heads]
        assert np.max(np.abs(o_un - o_ab)) <= 1e-12 * np.max(np.abs(o_un))
        assert np.max(np.abs(lse_un - out["lse"][b, heads])) <= 1e-12 * np.max(np.abs(lse_un))
    # tiny fp32 workload: every head
    wl = workloads.make("tiny_fp32")
    out = oracle.step_outputs(wl)
    o_un, lse_un = om.step_outputs_unabsorbed(wl, 0)
    assert np.max(np.abs(o_un - out["o"][0])) <= 1e-12 * np.max(np.abs(o_un))


def test_absorb_q_pieces():
    """The absorbed query: nope part contracts q_nope with W_UK over d_nope (loop
    check), rope part is RoPE(q_pe) at the query's position."""
    rng = _rng(7)
    B, H, dn, dc, dr = 2, 3, 4, 5, 4
    qn = rng.standard_normal((B, H, dn))
    qp = rng.standard_normal((B, H, dr))
    w = rng.standard_normal((H, dn, dc))
    pos = np.array([3, 1000])
    ql = oracle.absorb_q(qn, qp, w, pos)
    for b in range(B):
        for h in range(H):
            for cc in range(dc):
                ref = sum(w[h, k, cc] * qn[b, h, k] for k in range(dn))
                assert ql[b, h, cc] == pytest.approx(ref, rel=1e-13, abs=1e-14)
            np.testing.assert_allclose(ql[b, h, dc:], oracle.rope(qp[b, h], pos[b]), rtol=1e-15)


def test_output_projections_loops():
    rng = _rng(8)
    B, H, dv, dc, dm = 2, 3, 2, 4, 5
    ol = rng.standard_normal((B, H, dc))
    wuv = rng.standard_normal((H, dv, dc))
    wo = rng.standard_normal((dm, H * dv))
    o = oracle.up_project_out(ol, wuv)
    y = oracle.out_project(o, wo)
    for b in range(B):
        flat = []
        for h in range(H):
            for v in range(dv):
                ref = sum(wuv[h, v, cc] * ol[b, h, cc] for cc in range(dc))
                assert o[b, h, v] == pytest.approx(ref, rel=1e-13, abs=1e-14)
                flat.append(ref)
        for m in range(dm):
            assert y[b, m] == pytest.approx(sum(wo[m, i] * flat[i] for i in range(H * dv)), rel=1e-12, abs=1e-13)


def test_combine_reassembles_full_attention():
    """Merging split partials by log-sum-exp gives the unsplit result, for any
    split points, empty splits included."""
    rng = _rng(9)
    H, dc, dr, L = 8, 32, 8, 257
    q = rng.standard_normal((H, dc + dr))
    rows = rng.standard_normal((L, dc + dr))
    ref_o, ref_lse = oracle.decode_absorbed(q, rows, 0.3, dc)
    for bounds in ([0, L], [0, 64, 128, 192, 257], [0, 0, 100, 100, 257], [0, 1, 2, 257, 257]):
        op, lp = oracle.split_partials(q, rows, 0.3, dc, bounds)
        o, lse = oracle.combine(op, lp)
        np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse, ref_lse, rtol=1e-13)
    o, lse = oracle.combine(np.zeros((3, H, dc)), np.full((3, H), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_round_bf16_matches_torch():
    """The oracle's fp64 -> bf16 rounding against torch's CPU conversion of
    float32 inputs (exact in fp64, so single rounding on both sides)."""
    rng = _rng(10)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(om.round_bf16(x.astype(np.float64)), ref)


def test_down_project_loops():
    rng = _rng(11)
    x = rng.standard_normal((3, 6))
    wd = rng.standard_normal((4, 6))
    wk = rng.standard_normal((2, 6))
    c, k = oracle.down_project(x, wd, wk)
    for t in range(3):
        for i in range(4):
            assert c[t, i] == pytest.approx(sum(wd[i, j] * x[t, j] for j in range(6)), rel=1e-13, abs=1e-14)
        for i in range(2):
            assert k[t, i] == pytest.approx(sum(wk[i, j] * x[t, j] for j in range(6)), rel=1e-13, abs=1e-14)
