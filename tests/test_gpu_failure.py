"""Failure handling on the GPU without a GPU fault.

Every mbarrier wait in the tensor-core kernels is bounded.  With the debug
knob mla_set_wait_limit set to one poll per wait, waits give up almost at
once: the kernels must record MLA_ERR_TIMEOUT in the handle's error word,
drain what they have in flight, release TMEM and return -- and the context
must stay usable (a normal decode right after matches the oracle)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["v2_b32_l2048", "v2_b2_l128k_fp8"])
def test_bounded_waits_report_timeout_and_context_survives(name):
    from mla_latent_kv_19_b200 import mla_last_device_error, mla_set_wait_limit
    from mla_latent_kv_19_b200.step import DecodeStep
    wl = workloads.make(name, batch=2, context=700)
    st = DecodeStep(wl, num_splits=2)
    st.append()
    st.absorb()
    assert mla_last_device_error(st.h) == 0
    mla_set_wait_limit(st.h, 1)                 # one poll per wait: waits give up
    st.decode_partial()
    assert mla_last_device_error(st.h) == -7    # MLA_ERR_TIMEOUT, reported and cleared
    mla_set_wait_limit(st.h, 0)                 # back to the default limit
    st.decode_partial()
    st.decode_combine()
    st.out_proj()
    assert mla_last_device_error(st.h) == 0
    g = st.outputs()
    st.close()
    # an e4m3 cache is compared with the oracle run on its own e4m3 rows
    r = oracle.step_outputs(wl, fp8_dequant=wl.cache_dtype == "fp8_e4m3")
    for k in ("o_lat", "lse", "y"):
        assert_close(k, g[k], r[k])


@pytest.mark.parametrize("name", ["v2_b32_l2048", "v2_b2_l128k_fp8"])
def test_out_of_range_page_in_decode_is_reported_not_read(name):
    """A page-table entry outside the pool is skipped (masked, read from page 0)
    and reported; the other sequences are unaffected."""
    from mla_latent_kv_19_b200 import mla_last_device_error
    from mla_latent_kv_19_b200.step import DecodeStep
    wl = workloads.make(name, batch=3, context=600)
    st = DecodeStep(wl, num_splits=1)
    st.run()
    assert mla_last_device_error(st.h) == 0
    bt = st.block_table.cpu().numpy()
    bt[1, 3] = wl.num_blocks + 5               # beyond the pool
    st.block_table.copy_(torch.from_numpy(bt))
    st.decode_partial()
    st.decode_combine()
    assert mla_last_device_error(st.h) == -6   # MLA_ERR_BAD_INDEX
    g = st.outputs()
    st.close()
    r = oracle.step_outputs(wl, [0, 2], fp8_dequant=wl.cache_dtype == "fp8_e4m3")
    assert_close("o_lat", g["o_lat"][[0, 2]], r["o_lat"])
    assert np.all(np.isfinite(g["o_lat"][1]))


def test_partial_beyond_fp16_range_is_reported():
    """With bf16 activations the split partials are kept in fp16.  A latent
    output beyond +-65504 (here: every cached row of one sequence set to 1e5,
    so that o_lat is 1e5 whatever the softmax) records MLA_ERR_RANGE rather
    than passing an infinity on; the other sequence and the next call are
    unaffected."""
    from mla_latent_kv_19_b200 import mla_last_device_error
    from mla_latent_kv_19_b200.step import DecodeStep
    wl = workloads.make("v2_b32_l2048", batch=2, context=300)
    st = DecodeStep(wl, num_splits=2)
    st.run()
    assert mla_last_device_error(st.h) == 0
    bt = st.block_table.cpu().numpy()
    rows = [int(p) * 64 + j for p in bt[1, :(int(wl.seq_lens[1]) + 63) // 64] for j in range(64)]
    saved = st.cache[rows].clone()
    st.cache[rows] = 1e5
    st.decode_partial()
    st.decode_combine()
    assert mla_last_device_error(st.h) == -9    # MLA_ERR_RANGE
    st.cache[rows] = saved
    st.decode_partial()
    st.decode_combine()
    assert mla_last_device_error(st.h) == 0
    g = st.outputs()
    st.close()
    r = oracle.step_outputs(wl)
    assert_close("o_lat", g["o_lat"], r["o_lat"])
