"""GPU parity of a whole decode step (append -> absorb -> split-KV decode ->
merge -> output projection) through the C ABI, against the fp64 oracle on the
same seeded inputs.

Small cases span several 64-token pages, several splits and a ragged tail;
the full-size cases run the workloads at their benchmark sizes in the launch
configuration the benchmark times and compare sampled sequences (all of them
where the oracle is cheap)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import BF16_MAE, BF16_MAX_REL, FP8_MAX_REL, assert_close, errors

pytestmark = pytest.mark.gpu

KEYS = ("q_lat", "o_lat", "lse", "o", "y")


def _run(wl, num_splits=0, stage_hook=None):
    from mla_latent_kv_19_b200.step import DecodeStep
    st = DecodeStep(wl, num_splits=num_splits)
    if stage_hook:
        stage_hook(st)
    st.run()
    out = st.outputs()
    splits = st.num_splits
    st.close()
    return out, splits


def _compare(wl, g, seqs, tag=""):
    r = oracle.step_outputs(wl, seqs)
    fp8 = wl.cache_dtype == "fp8_e4m3"
    rq = oracle.step_outputs(wl, seqs, fp8_dequant=True) if fp8 else None
    for k in KEYS:
        lim, mae = BF16_MAX_REL, BF16_MAE
        if fp8 and k != "q_lat":
            # against exact values the e4m3 rounding of the cache itself counts:
            # 3e-2 (and the bf16 mean error), or 1.1x the oracle's own fp8 error
            # where that is larger (short contexts average the rounding noise
            # over few tokens)
            own_rel, own_mae = errors(rq[k], r[k])
            lim, mae = max(FP8_MAX_REL, 1.1 * own_rel), max(BF16_MAE, 1.1 * own_mae)
        assert_close(f"{tag}{k}", g[k][seqs], r[k], max_rel=lim, mae=mae)
    if fp8:
        # against the oracle run on its own e4m3 rows: the bf16 tolerance
        for k in ("o_lat", "lse", "o", "y"):
            assert_close(f"{tag}{k}(dequant)", g[k][seqs], rq[k])
    return r


SMALL = [
    ("tiny_fp32", {}),
    ("v2_b32_l2048", dict(batch=3, context=333)),
    ("v2_b32_l2048_shuf", dict(batch=5, context=1000)),
    ("v2_ragged64", dict(batch=7, context=900)),
    ("v2_b4_l32k", dict(batch=2, context=4097)),
    ("v2_b2_l128k_fp8", dict(batch=2, context=1500)),
]


@pytest.mark.parametrize("name,kw", SMALL, ids=[s[0] + "-small" for s in SMALL])
def test_step_small(name, kw):
    wl = workloads.make(name, **kw)
    g, _ = _run(wl)
    _compare(wl, g, list(range(wl.batch)))


@pytest.mark.parametrize("splits", [1, 2, 5, 16])
def test_split_count_does_not_change_the_result(splits):
    wl = workloads.make("v2_b32_l2048", batch=2, context=1100)
    g, s = _run(wl, num_splits=splits)
    assert s == splits
    _compare(wl, g, [0, 1], tag=f"S={splits} ")


@pytest.mark.parametrize("splits", [1, 3, 8])
def test_fp8_split_count_does_not_change_the_result(splits):
    wl = workloads.make("v2_b2_l128k_fp8", batch=2, context=1500)
    g, s = _run(wl, num_splits=splits)
    assert s == splits
    _compare(wl, g, [0, 1], tag=f"S={splits} ")


def _oracle_decode_inputs(wl, dev="cuda"):
    """The decode's inputs made by the oracle alone: q~ rounded to bf16, and
    a pool whose sequences' rows hold the oracle's own cache values (bf16
    rows, or e4m3 codes and fp32 scales) -- every other row holds NaN.
    Returns the device tensors and the float64 rows/q~ the kernel sees."""
    from mla_latent_kv_19_b200.step import to_device
    d = wl.dims
    D = d["d_c"] + d["d_r"]
    fp8 = wl.cache_dtype == "fp8_e4m3"
    q = oracle.absorb_q(wl.to_f64(wl.q_nope), wl.to_f64(wl.q_pe), wl.to_f64(wl.w_uk), wl.new_pos,
                        wl.rope_base)
    q_bits = workloads.f32_to_bf16_bits(q.astype(np.float32))
    rows_seen = []
    if fp8:
        codes = np.full((wl.num_blocks * 64, D), 0x7F, np.uint8)           # e4m3 NaN
        scales = np.full(wl.num_blocks * 64, np.inf, np.float32)
    else:
        cache = np.full((wl.num_blocks * 64, D), 0x7FC0, np.uint16)         # bf16 NaN
    for b in range(wl.batch):
        c, k, pos = oracle.mla._rows_of_sequence(wl, b, wl.rope_base)
        rows = oracle.cache_row(c, k, pos, wl.rope_base)
        slots = oracle.paged_slot(wl.block_table, np.full(len(pos), b), pos, 64)
        if fp8:
            cd, sc = oracle.fp8_quantize_row(rows.astype(np.float32))
            codes[slots], scales[slots] = cd, sc
            rows_seen.append(oracle.e4m3_decode(cd) * sc[:, None].astype(np.float64))
        else:
            r16 = workloads.f32_to_bf16_bits(rows.astype(np.float32))
            cache[slots] = r16
            rows_seen.append(workloads.bf16_to_f64(r16))
    if fp8:
        cache_t = torch.from_numpy(codes).to(dev)
        scale_t = torch.from_numpy(scales).to(dev)
    else:
        cache_t = to_device(cache, dev)
        scale_t = None
    return (to_device(q_bits, dev), cache_t, scale_t, workloads.bf16_to_f64(q_bits), rows_seen)


@pytest.mark.parametrize("name", ["v2_b32_l2048", "v2_b2_l128k_fp8"])
@pytest.mark.parametrize("splits", [1, 2, 3])
def test_decode_alone_on_oracle_inputs_ignores_rows_past_the_end(name, splits):
    """The split-KV decode by itself, fed only with oracle-made inputs (q~ in
    bf16, cache rows as the oracle writes them), against the oracle's absorbed
    decode on exactly those values.  Every cache row that belongs to no token
    holds NaN (bf16 NaN, or the e4m3 NaN code with an infinite scale); the last
    page of each sequence shares its tile with such rows."""
    from mla_latent_kv_19_b200 import (Handle, mla_decode, mla_decode_workspace_bytes,
                                       mla_last_device_error)
    from mla_latent_kv_19_b200.step import softmax_scale, to_device
    wl = workloads.make(name, batch=3, context=201)
    d = wl.dims
    scale = softmax_scale(d["d_nope"], d["d_r"])
    h = Handle(num_heads=d["num_heads"], d_c=d["d_c"], d_r=d["d_r"], d_nope=d["d_nope"],
               d_v=d["d_v"], d_model=d["d_model"], cache_dtype=wl.cache_dtype,
               softmax_scale=scale, max_position=4096)
    q, cache, cache_scale, q64, rows = _oracle_decode_inputs(wl)
    table = to_device(wl.block_table.astype(np.int32), "cuda")
    lens = to_device(wl.seq_lens.astype(np.int32), "cuda")
    L = int(wl.seq_lens.max())
    ws = torch.empty(mla_decode_workspace_bytes(h, wl.batch, splits, L), dtype=torch.uint8, device="cuda")
    o_lat = torch.empty(wl.batch, d["num_heads"], d["d_c"], dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(wl.batch, d["num_heads"], dtype=torch.float32, device="cuda")
    mla_decode(h, q, cache, cache_scale, table, lens, L, splits, ws, o_lat, lse)
    assert mla_last_device_error(h) == 0
    g_o = o_lat.float().cpu().numpy()
    g_l = lse.cpu().numpy()
    h.close()
    assert np.all(np.isfinite(g_o)) and np.all(np.isfinite(g_l))
    r_o, r_l = zip(*[oracle.decode_absorbed(q64[b], rows[b], scale, d["d_c"]) for b in range(wl.batch)])
    assert_close("o_lat", g_o, np.stack(r_o))
    assert_close("lse", g_l, np.stack(r_l))


def test_page_permutation_does_not_change_the_result():
    a = workloads.make("v2_b32_l2048", batch=4, context=700)
    b = workloads.make("v2_b32_l2048_shuf", batch=4, context=700)
    assert not np.array_equal(a.block_table, b.block_table)
    ga, _ = _run(a, num_splits=3)
    gb, _ = _run(b, num_splits=3)
    for k in KEYS:
        np.testing.assert_array_equal(ga[k], gb[k], err_msg=k)


def test_append_then_decode_equals_prefilled_cache():
    """The decode step's own append (one token per sequence) writes exactly
    what writing that token together with the history would have written."""
    from mla_latent_kv_19_b200 import mla_cache_append
    from mla_latent_kv_19_b200.step import to_device
    wl = workloads.make("v2_b32_l2048", batch=3, context=200)
    ga, _ = _run(wl, num_splits=2)

    def prefill_new_tokens(st):
        seq = to_device(np.arange(wl.batch, dtype=np.int32), "cuda")
        mla_cache_append(st.h, st.new_c_kv, st.new_k_r, st.new_pos, st.block_table, st.cache,
                         st.cache_scale, seq_idx=seq, batch=wl.batch)
        st.append = lambda stream=None: None      # the step itself appends nothing
    gb, _ = _run(wl, num_splits=2, stage_hook=prefill_new_tokens)
    for k in KEYS:
        np.testing.assert_array_equal(ga[k], gb[k], err_msg=k)


def test_empty_sequence_gives_zero_and_minus_inf():
    wl = workloads.make("v2_b32_l2048", batch=3, context=300)

    def empty_middle(st):
        lens = st.seq_lens.cpu().numpy()
        lens[1] = 0
        st.seq_lens.copy_(torch.from_numpy(lens))
    g, _ = _run(wl, num_splits=2, stage_hook=empty_middle)
    assert np.all(g["o_lat"][1] == 0)
    assert np.all(np.isneginf(g["lse"][1]))
    r = oracle.step_outputs(wl, [0, 2])
    for k in ("o_lat", "lse"):
        assert_close(k, g[k][[0, 2]], r[k])


def test_combine_against_oracle_merge():
    from mla_latent_kv_19_b200 import (Handle, mla_decode_combine, mla_decode_workspace_bytes)
    from mla_latent_kv_19_b200.step import softmax_scale
    d = workloads.V2_DIMS
    h = Handle(num_heads=d["num_heads"], d_c=d["d_c"], d_r=d["d_r"], d_nope=d["d_nope"],
               d_v=d["d_v"], d_model=d["d_model"], softmax_scale=softmax_scale(128, 64),
               max_position=4096)
    B, S, H, dc = 3, 6, d["num_heads"], d["d_c"]
    rng = np.random.default_rng(7)
    o = rng.standard_normal((B, S, H, dc)).astype(np.float32)
    lse = (rng.standard_normal((B, S, H)) * 4).astype(np.float32)
    lse[0, 2] = -np.inf
    lse[1, :, 5] = -np.inf           # every split of (b=1, h=5) empty
    o[0, 2] = 0
    o[1, :, 5] = 0
    nbytes = mla_decode_workspace_bytes(h, B, S, 64 * S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    n_o = B * S * H * dc * 2
    # workspace layout (bf16 activations): fp16 o_part[b][s][c/8][h][c%8]
    packed = o.astype(np.float16).reshape(B, S, H, dc // 8, 8).transpose(0, 1, 3, 2, 4)
    ws[:n_o].view(torch.float16).copy_(torch.from_numpy(np.ascontiguousarray(packed).reshape(-1)))
    off = (n_o + 255) // 256 * 256
    ws[off:off + B * S * H * 4].view(torch.float32).copy_(torch.from_numpy(lse.reshape(-1)))
    o_lat = torch.empty(B, H, dc, dtype=torch.bfloat16, device="cuda")
    g_lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    mla_decode_combine(h, B, 64 * S, S, ws, o_lat, g_lse)
    ro, rl = oracle.combine(np.moveaxis(o, 1, 0), np.moveaxis(lse, 1, 0))
    assert_close("o_lat", o_lat.float().cpu().numpy(), ro)
    gl = g_lse.cpu().numpy()
    assert np.isneginf(gl[1, 5]) and np.all(o_lat[1, 5].float().cpu().numpy() == 0)
    assert_close("lse", gl, rl)
    h.close()


# ---------------------------------------------------------------------------
# full sizes, launch configuration of the benchmark (automatic split count)
# ---------------------------------------------------------------------------

FULL = ["v2_b32_l2048", "v2_ragged64", "v2_b4_l32k", "v2_b2_l128k_fp8"]


def _sample(wl):
    if wl.name == "v2_ragged64":
        lens = wl.hist_len
        return sorted({int(lens.argmax()), int(lens.argmin()), 0, 17, 42, 63})
    return list(range(wl.batch))


@pytest.mark.parametrize("name", FULL)
def test_step_full_size(name):
    wl = workloads.make(name)
    g, _ = _run(wl)
    seqs = _sample(wl)
    _compare(wl, g, seqs)
    # the un-absorbed (primary) form directly, on a few heads of one sequence
    b = seqs[-1]
    heads = [0, 77] if wl.seq_lens[b] > 40000 else [0, 31, 77, 127]
    o_un, lse_un = oracle.mla.step_outputs_unabsorbed(wl, b, heads)
    lim = FP8_MAX_REL if wl.cache_dtype == "fp8_e4m3" else BF16_MAX_REL
    assert_close("o(unabsorbed)", g["o"][b, heads], o_un, max_rel=lim)
    assert_close("lse(unabsorbed)", g["lse"][b, heads], lse_un, max_rel=lim)


def test_tiny_fp32_every_output_unabsorbed():
    wl = workloads.make("tiny_fp32")
    g, _ = _run(wl)
    o_un, lse_un = oracle.mla.step_outputs_unabsorbed(wl, 0)
    assert_close("o", g["o"][0], o_un)
    assert_close("lse", g["lse"][0], lse_un)


def test_cuda_graph_replay_matches_eager_calls():
    """The C-ABI calls neither allocate nor synchronise, so a decode step can be
    captured in a CUDA graph; replaying it gives the same bits as the calls."""
    from mla_latent_kv_19_b200.step import DecodeStep
    wl = workloads.make("v2_b32_l2048", batch=3, context=500)
    st = DecodeStep(wl, num_splits=2)
    st.run()
    eager = st.outputs()
    st.capture()
    for k in ("o_lat", "y"):
        getattr(st, k).zero_()
    st.replay()
    replay = st.outputs()
    st.close()
    for k in KEYS:
        np.testing.assert_array_equal(eager[k], replay[k], err_msg=k)


@pytest.mark.parametrize("name,kw", [("v2_b32_l2048", {}), ("v2_b32_l2048", dict(batch=7, context=900)),
                                     ("v2_b2_l128k_fp8", dict(batch=2, context=5000))])
def test_launch_overlap_gives_the_same_bits(name, kw):
    """With launch overlap on, each kernel starts its set-up and weight loads
    while the previous one runs and waits for it before touching its outputs.
    The results are bit for bit those of plain stream-ordered launches, in eager
    calls and in repeated replays of the captured step."""
    from mla_latent_kv_19_b200.step import DecodeStep
    wl = workloads.make(name, **kw)
    ref = DecodeStep(wl, overlap=False)
    ref.run()
    want = ref.outputs()
    splits = ref.num_splits
    ref.close()
    st = DecodeStep(wl, num_splits=splits, overlap=True)
    st.run()
    got = st.outputs()
    for k in KEYS:
        np.testing.assert_array_equal(got[k], want[k], err_msg=k)
    st.capture()
    for _ in range(3):
        for k in ("q_lat", "o_lat", "lse", "o", "y"):
            getattr(st, k).fill_(float("nan"))
        st.replay()
        got = st.outputs()
        for k in KEYS:
            np.testing.assert_array_equal(got[k], want[k], err_msg=k)
    st.close()
