"""GPU parity of the paged row write (mla_cache_append, mla_kv_project_append)
against the oracle: slot indices and c_KV bytes bit-exact, rotated k_R within
one bf16 step, fp8 codes bit-exact where the row is exact in fp32, untouched
rows unchanged, out-of-range pages reported and skipped."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import bf16_ulp

pytestmark = pytest.mark.gpu

V2 = workloads.V2_DIMS


def _handle(dims, act="bf16", cache="bf16", max_position=131072 + 64):
    from mla_latent_kv_19_b200 import Handle
    from mla_latent_kv_19_b200.step import softmax_scale
    return Handle(num_heads=dims["num_heads"], d_c=dims["d_c"], d_r=dims["d_r"],
                  d_nope=dims["d_nope"], d_v=dims["d_v"], d_model=dims["d_model"], block_size=64,
                  act_dtype=act, cache_dtype=cache,
                  softmax_scale=softmax_scale(dims["d_nope"], dims["d_r"]), max_position=max_position)


def _tokens_with_unique_slots(rng, n, batch, max_blocks, table):
    seq, pos, seen = [], [], set()
    while len(seq) < n:
        b = int(rng.integers(0, batch))
        p = int(rng.integers(0, max_blocks * 64))
        slot = int(oracle.paged_slot(table, [b], [p], 64)[0])
        if slot in seen:
            continue
        seen.add(slot)
        seq.append(b)
        pos.append(p)
    return np.array(seq, np.int32), np.array(pos, np.int32)


def _dev(a):
    from mla_latent_kv_19_b200.step import to_device
    return to_device(a, "cuda")


def _page_setup(rng, batch=3, max_blocks=2048, pool=48):
    # every table entry points into a small pool, so long positions stay cheap
    table = rng.integers(0, pool, size=(batch, max_blocks)).astype(np.int32)
    return table, pool


def test_append_bf16_bit_exact():
    from mla_latent_kv_19_b200 import mla_cache_append, mla_last_device_error
    rng = np.random.default_rng(100)
    table, pool = _page_setup(rng)
    T = 600
    seq, pos = _tokens_with_unique_slots(rng, T, 3, table.shape[1], table)
    pos[:5] = [0, 1, 63, 64, 131071]
    seq[:5] = [0, 0, 1, 2, 2]
    keep = np.unique(oracle.paged_slot(table, seq, pos, 64), return_index=True)[1]
    seq, pos = seq[keep], pos[keep]
    T = len(seq)
    c, k = workloads.random_tokens(rng, T, V2["d_c"], V2["d_r"])
    h = _handle(V2)
    D = V2["d_c"] + V2["d_r"]
    cache = torch.full((pool * 64, D), 0x7F7F, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    mla_cache_append(h, _dev(c), _dev(k), _dev(pos), _dev(table), cache, None, seq_idx=_dev(seq),
                     batch=3)
    assert mla_last_device_error(h) == 0
    got = cache.view(torch.int16).cpu().numpy().view(np.uint16)
    slots = oracle.paged_slot(table, seq, pos, 64)
    # c_KV bytes bit-exact at the oracle's slots
    np.testing.assert_array_equal(got[slots, :V2["d_c"]], c)
    # rotated k_R within one bf16 step of the exact value
    exact = oracle.rope(workloads.bf16_to_f64(k), pos)
    g = workloads.bf16_to_f64(got[slots, V2["d_c"]:])
    assert np.all(np.abs(g - exact) <= bf16_ulp(exact))
    # almost all of them are the correctly rounded value
    assert np.mean(g == oracle.round_bf16(exact)) > 0.99
    # every other row untouched
    mask = np.ones(pool * 64, bool)
    mask[slots] = False
    assert np.all(got[mask] == 0x7F7F)
    h.close()


def test_append_fp8_codes_and_scales():
    from mla_latent_kv_19_b200 import mla_cache_append, mla_last_device_error
    rng = np.random.default_rng(101)
    B, first, pool = 40, 40, 88
    # page 0 of every sequence is its own page; later pages come from a shared range
    table = rng.integers(first, pool, size=(B, 2048)).astype(np.int32)
    table[:, 0] = np.arange(B)
    seq0 = np.arange(B, dtype=np.int32)
    pos0 = np.zeros(B, np.int32)                 # position 0: RoPE is the identity
    seq1, pos1 = _tokens_with_unique_slots(rng, 400, B, table.shape[1], table)
    ok = pos1 >= 64                               # keep the others off the page-0 pages
    seq = np.concatenate([seq0, seq1[ok]])
    pos = np.concatenate([pos0, pos1[ok]])
    T = len(seq)
    c, k = workloads.random_tokens(rng, T, V2["d_c"], V2["d_r"])
    c[7] = 0
    k[7] = 0            # an all-zero row: scale 1, zero codes
    h = _handle(V2, cache="fp8_e4m3")
    D = V2["d_c"] + V2["d_r"]
    cache = torch.full((pool * 64, D), 0x55, dtype=torch.uint8, device="cuda")
    scale = torch.full((pool * 64,), -1.0, dtype=torch.float32, device="cuda")
    mla_cache_append(h, _dev(c), _dev(k), _dev(pos), _dev(table), cache, scale, seq_idx=_dev(seq),
                     batch=B)
    assert mla_last_device_error(h) == 0
    got = cache.cpu().numpy()
    gsc = scale.cpu().numpy()
    slots = oracle.paged_slot(table, seq, pos, 64)
    assert len(np.unique(slots)) == T
    rows = oracle.cache_row(workloads.bf16_to_f64(c), workloads.bf16_to_f64(k), pos)
    codes, sc = oracle.fp8_quantize_row(rows.astype(np.float32))
    at0 = pos == 0
    # where the rotation is the identity the fp32 row is exact on both sides:
    # codes and scales bit-exact
    np.testing.assert_array_equal(got[slots[at0]], codes[at0])
    np.testing.assert_array_equal(gsc[slots[at0]], sc[at0])
    assert gsc[slots[7]] == 1.0 and np.all(got[slots[7]] == 0)
    # elsewhere the fp32 rotation may differ from the fp64 one by an ulp: the
    # dequantised rows agree within one e4m3 step at the top binade of the row
    deq_g = oracle.e4m3_decode(got[slots]) * gsc[slots, None]
    deq_o = oracle.e4m3_decode(codes) * sc[:, None]
    step = np.abs(rows).max(1, keepdims=True) / 448.0 * 32.0
    assert np.all(np.abs(deq_g - deq_o) <= step)
    assert np.mean(got[slots] == codes) > 0.99
    mask = np.ones(pool * 64, bool)
    mask[slots] = False
    assert np.all(got[mask] == 0x55) and np.all(gsc[mask] == -1.0)
    h.close()


def test_project_append_fp32_tiny():
    from mla_latent_kv_19_b200 import mla_kv_project_append, mla_last_device_error
    wl = workloads.make("tiny_fp32")
    d = wl.dims
    h = _handle(d, act="fp32", cache="fp32", max_position=256)
    D = d["d_c"] + d["d_r"]
    cache = torch.zeros((wl.num_blocks * 64, D), dtype=torch.float32, device="cuda")
    mla_kv_project_append(h, _dev(wl.hist_x), _dev(wl.w_dkv), _dev(wl.w_kr), _dev(wl.hist_pos),
                          _dev(wl.block_table), cache, None, seq_idx=_dev(wl.hist_seq), batch=1)
    assert mla_last_device_error(h) == 0
    got = cache.cpu().numpy().astype(np.float64)
    c, kraw = oracle.down_project(wl.hist_x, wl.w_dkv, wl.w_kr)
    rows = oracle.cache_row(c, kraw, wl.hist_pos)
    slots = oracle.paged_slot(wl.block_table, wl.hist_seq, wl.hist_pos, 64)
    assert np.max(np.abs(got[slots] - rows)) <= 1e-5 * np.max(np.abs(rows))
    h.close()


def test_append_out_of_range_page_is_reported_and_skipped():
    from mla_latent_kv_19_b200 import mla_cache_append, mla_last_device_error
    rng = np.random.default_rng(102)
    pool = 8
    table = np.array([[0, 1], [2, pool], [-3, 4]], np.int32)    # pool and -3 are invalid pages
    seq = np.array([0, 1, 1, 2, 2], np.int32)
    pos = np.array([5, 3, 70, 10, 70], np.int32)                # tokens 2 and 3 hit invalid pages
    c, k = workloads.random_tokens(rng, 5, V2["d_c"], V2["d_r"])
    h = _handle(V2)
    D = V2["d_c"] + V2["d_r"]
    cache = torch.full((pool * 64, D), 0x1234, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    mla_cache_append(h, _dev(c), _dev(k), _dev(pos), _dev(table), cache, None, seq_idx=_dev(seq),
                     batch=3)
    assert mla_last_device_error(h) == -6          # MLA_ERR_BAD_INDEX
    assert mla_last_device_error(h) == 0           # cleared by the read
    got = cache.view(torch.int16).cpu().numpy().view(np.uint16)
    good = [0, 1, 4]
    slots = oracle.paged_slot(np.where(table < 0, 0, np.minimum(table, pool - 1)), seq[good], pos[good], 64)
    np.testing.assert_array_equal(got[slots, :V2["d_c"]], c[good])
    mask = np.ones(pool * 64, bool)
    mask[slots] = False
    assert np.all(got[mask] == 0x1234)
    # a position beyond the table row is rejected the same way
    mla_cache_append(h, _dev(c[:1]), _dev(k[:1]), _dev(np.array([128], np.int32)), _dev(table),
                     cache, None, seq_idx=_dev(np.array([0], np.int32)), batch=3)
    assert mla_last_device_error(h) == -6
    h.close()
