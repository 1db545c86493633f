"""GPU parity of the two projection calls at batch sizes that exercise the
tensor-core GEMM's padding of the batch (the UMMA N dimension, a multiple of
16), its box-depth choice for the W_O stream (deeper boxes for small batches,
shallower ones from ~96 tokens) and the largest supported batch (256), against
the fp64 oracle:

* mla_absorb_q:  q~[b,h] = W_UK_h^T q_nope[b,h] (+) RoPE(q_pe[b,h], pos_b)
  (DeepSeek V2 MLA page, sections 2.2 and 2.3);
* mla_out_proj:  o[b,h] = W_UV_h o_lat[b,h], y[b] = W_O concat_h o[b,h]
  (section 2.3, W_UV absorbed into the output side)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import assert_close

pytestmark = pytest.mark.gpu

BATCHES = [1, 17, 100, 256]


def _handle(d):
    from mla_latent_kv_19_b200 import Handle
    from mla_latent_kv_19_b200.step import softmax_scale
    return Handle(num_heads=d["num_heads"], d_c=d["d_c"], d_r=d["d_r"], d_nope=d["d_nope"],
                  d_v=d["d_v"], d_model=d["d_model"], softmax_scale=softmax_scale(d["d_nope"], d["d_r"]),
                  max_position=4096)


@pytest.mark.parametrize("batch", BATCHES)
def test_absorb_against_oracle(batch):
    from mla_latent_kv_19_b200 import mla_absorb_q, mla_last_device_error
    from mla_latent_kv_19_b200.step import to_device
    wl = workloads.make("v2_b32_l2048", batch=batch, context=64)
    d = wl.dims
    rng = np.random.default_rng(1000 + batch)
    pos = rng.integers(0, 4096, size=batch).astype(np.int32)
    h = _handle(d)
    q_lat = torch.empty(batch, d["num_heads"], d["d_c"] + d["d_r"], dtype=torch.bfloat16, device="cuda")
    mla_absorb_q(h, to_device(wl.q_nope, "cuda"), to_device(wl.q_pe, "cuda"), to_device(pos, "cuda"),
                 to_device(wl.w_uk, "cuda"), q_lat)
    assert mla_last_device_error(h) == 0
    g = q_lat.float().cpu().numpy()
    h.close()
    r = oracle.absorb_q(wl.to_f64(wl.q_nope), wl.to_f64(wl.q_pe), wl.to_f64(wl.w_uk), pos, wl.rope_base)
    assert_close("q_lat", g, r)


@pytest.mark.parametrize("batch", BATCHES)
def test_out_proj_against_oracle(batch):
    from mla_latent_kv_19_b200 import mla_last_device_error, mla_out_proj, mla_out_proj_workspace_bytes
    from mla_latent_kv_19_b200.step import to_device
    wl = workloads.make("v2_b32_l2048", batch=1, context=64)
    d = wl.dims
    rng = np.random.default_rng(2000 + batch)
    o_lat = workloads.f32_to_bf16_bits(
        rng.standard_normal((batch, d["num_heads"], d["d_c"])).astype(np.float32))
    h = _handle(d)
    ws = torch.empty(max(mla_out_proj_workspace_bytes(h, batch), 256), dtype=torch.uint8, device="cuda")
    y = torch.empty(batch, d["d_model"], dtype=torch.bfloat16, device="cuda")
    o = torch.empty(batch, d["num_heads"], d["d_v"], dtype=torch.bfloat16, device="cuda")
    mla_out_proj(h, to_device(o_lat, "cuda"), to_device(wl.w_uv, "cuda"), to_device(wl.w_o, "cuda"), ws, y, o)
    assert mla_last_device_error(h) == 0
    g_y, g_o = y.float().cpu().numpy(), o.float().cpu().numpy()
    h.close()
    r_o = oracle.up_project_out(workloads.bf16_to_f64(o_lat), wl.to_f64(wl.w_uv))
    r_y = oracle.out_project(r_o, wl.to_f64(wl.w_o))
    assert_close("o", g_o, r_o)
    assert_close("y", g_y, r_y)


@pytest.mark.parametrize("name,kw,splits", [
    ("v2_b32_l2048", dict(batch=5, context=700), 3),
    ("v2_b32_l2048", dict(batch=32, context=300), 2),
    ("v2_b2_l128k_fp8", dict(batch=2, context=3000), 8),
    ("v2_b32_l2048", dict(batch=100, context=64), 1),      # beyond the fused path: two calls
])
def test_fused_merge_out_proj_equals_the_two_calls(name, kw, splits):
    """mla_combine_out_proj (the split merge built inside the W_UV kernel) gives
    bit for bit what mla_decode_combine followed by mla_out_proj gives, and
    both match the oracle."""
    from mla_latent_kv_19_b200 import mla_combine_out_proj, mla_last_device_error
    from mla_latent_kv_19_b200.step import DecodeStep
    wl = workloads.make(name, **kw)
    st = DecodeStep(wl, num_splits=splits)
    st.append()
    st.absorb()
    st.decode_partial()
    st.decode_combine()
    st.out_proj()
    sep = {k: getattr(st, k).clone() for k in ("o_lat", "lse", "o", "y")}
    out = {k: torch.full_like(v, float("nan")) for k, v in sep.items()}
    mla_combine_out_proj(st.h, st.B, st.max_seq_len, st.num_splits, st.dec_ws, st.w_uv, st.w_o, st.op_ws,
                         out["o_lat"], out["y"], lse=out["lse"], o_out=out["o"])
    assert mla_last_device_error(st.h) == 0
    torch.cuda.synchronize()
    for k in sep:
        assert torch.equal(out[k].view(torch.int16) if out[k].dtype == torch.bfloat16 else out[k],
                           sep[k].view(torch.int16) if sep[k].dtype == torch.bfloat16 else sep[k]), k
    st.close()
    fp8 = wl.cache_dtype == "fp8_e4m3"
    r = oracle.step_outputs(wl, fp8_dequant=fp8)
    g = {k: v.float().cpu().numpy() for k, v in out.items()}
    for k in ("o_lat", "lse", "y"):
        assert_close(k, g[k], r[k])


@pytest.mark.parametrize("name", ["v2_b32_l2048", "tiny_fp32"])
def test_pack_w_o_is_the_tile_major_relayout(name):
    """mla_pack_w_o writes W_O[m][k] to [m/128][k/64][m%128][k%64], bit for bit
    (bf16 and fp32 elements)."""
    from mla_latent_kv_19_b200 import mla_pack_w_o
    from mla_latent_kv_19_b200.step import to_device
    wl = workloads.make(name, batch=1, context=64)
    h = _handle_for(wl)
    w = to_device(wl.w_o, "cuda")
    t = torch.full_like(w, float("nan"))
    mla_pack_w_o(h, w, t)
    torch.cuda.synchronize()
    h.close()
    M, K = wl.w_o.shape
    want = wl.w_o.reshape(M // 128, 128, K // 64, 64).transpose(0, 2, 1, 3).reshape(M, K)
    got = t.view(torch.int16).cpu().numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.cpu().numpy()
    np.testing.assert_array_equal(got, want)


def _handle_for(wl):
    from mla_latent_kv_19_b200 import Handle
    from mla_latent_kv_19_b200.step import softmax_scale
    d = wl.dims
    return Handle(num_heads=d["num_heads"], d_c=d["d_c"], d_r=d["d_r"], d_nope=d["d_nope"], d_v=d["d_v"],
                  d_model=d["d_model"], act_dtype=wl.act_dtype, cache_dtype=wl.cache_dtype,
                  softmax_scale=softmax_scale(d["d_nope"], d["d_r"]), max_position=4096)


@pytest.mark.parametrize("batch", BATCHES + [300])
def test_out_proj_with_tile_major_w_o_against_oracle(batch):
    """The output projection reading the tile-major W_O (tensor-core path up to
    256 tokens, CUDA-core path beyond) matches the oracle."""
    from mla_latent_kv_19_b200 import (mla_last_device_error, mla_out_proj, mla_out_proj_workspace_bytes,
                                       mla_pack_w_o, mla_set_w_o_layout)
    from mla_latent_kv_19_b200.step import to_device
    wl = workloads.make("v2_b32_l2048", batch=1, context=64)
    d = wl.dims
    rng = np.random.default_rng(3000 + batch)
    o_lat = workloads.f32_to_bf16_bits(
        rng.standard_normal((batch, d["num_heads"], d["d_c"])).astype(np.float32))
    h = _handle(d)
    w_o = to_device(wl.w_o, "cuda")
    w_t = torch.empty_like(w_o)
    mla_pack_w_o(h, w_o, w_t)
    del w_o
    mla_set_w_o_layout(h, True)
    ws = torch.empty(max(mla_out_proj_workspace_bytes(h, batch), 256), dtype=torch.uint8, device="cuda")
    y = torch.empty(batch, d["d_model"], dtype=torch.bfloat16, device="cuda")
    o = torch.empty(batch, d["num_heads"], d["d_v"], dtype=torch.bfloat16, device="cuda")
    mla_out_proj(h, to_device(o_lat, "cuda"), to_device(wl.w_uv, "cuda"), w_t, ws, y, o)
    assert mla_last_device_error(h) == 0
    g_y, g_o = y.float().cpu().numpy(), o.float().cpu().numpy()
    h.close()
    r_o = oracle.up_project_out(workloads.bf16_to_f64(o_lat), wl.to_f64(wl.w_uv))
    r_y = oracle.out_project(r_o, wl.to_f64(wl.w_o))
    assert_close("o", g_o, r_o)
    assert_close("y", g_y, r_y)
