"""mla_decode_noalloc against mla_decode.

mla_decode_noalloc serves callers that cannot allocate device memory (a
plugin whose host framework owns all device buffers, a loop that must not
risk cudaMalloc's implicit device synchronisation): it keeps the split
partials in a fixed array inside the library instead of a caller workspace.
These tests call it through the C ABI twice in a row, on two different
decodes, and hold each result to the existing entry point's result on the
same inputs, within the parity tolerance of the other tests.  The second call
shows that what the first call left in the shared array does not leak.
"""
import numpy as np
import pytest
import torch

import workloads
from helpers import assert_close

pytestmark = pytest.mark.gpu


def _prepared_step(name, **kw):
    """A decode layer with its cache filled and the absorbed queries computed."""
    from mla_latent_kv_19_b200.step import DecodeStep
    wl = workloads.make(name, **kw)
    st = DecodeStep(wl)
    st.append()
    st.absorb()
    torch.cuda.synchronize()
    return st


def _decode_both(st, num_splits):
    from mla_latent_kv_19_b200 import (mla_decode, mla_decode_noalloc, mla_decode_workspace_bytes,
                                       mla_last_device_error)
    B, H, dc = st.B, st.H, st.d_c
    ws = torch.empty(mla_decode_workspace_bytes(st.h, B, num_splits, st.max_seq_len),
                     dtype=torch.uint8, device="cuda")
    ref_o = torch.empty(B, H, dc, dtype=st.act, device="cuda")
    ref_l = torch.empty(B, H, dtype=torch.float32, device="cuda")
    mla_decode(st.h, st.q_lat, st.cache, st.cache_scale, st.block_table, st.seq_lens,
               st.max_seq_len, num_splits, ws, ref_o, ref_l)
    got_o = torch.full((B, H, dc), float("nan"), dtype=st.act, device="cuda")
    got_l = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
    mla_decode_noalloc(st.h, st.q_lat, st.cache, st.cache_scale, st.block_table, st.seq_lens,
                       st.max_seq_len, num_splits, got_o, got_l)
    assert mla_last_device_error(st.h) == 0
    f = lambda t: t.float().cpu().numpy().astype(np.float64)
    return f(got_o), f(got_l), f(ref_o), f(ref_l)


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    first = _prepared_step("v2_b32_l2048", batch=4, context=1500)
    second = _prepared_step("v2_ragged64", batch=6, context=700)
    for st, splits in ((first, 3), (second, 2)):
        go, gl, ro, rl = _decode_both(st, splits)
        assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
        assert_close("o_lat", go, ro)
        assert_close("lse", gl, rl)
    first.close()
    second.close()


def test_noalloc_rejects_a_workspace_beyond_its_array():
    from mla_latent_kv_19_b200 import MLAError, mla_decode_noalloc
    st = _prepared_step("v2_b32_l2048", batch=2, context=200)
    # 2 sequences x 200 splits x 128 heads x 513 fp32 values is ~105 MB > 32 MiB
    with pytest.raises(MLAError) as e:
        mla_decode_noalloc(st.h, st.q_lat, st.cache, st.cache_scale, st.block_table, st.seq_lens,
                           200 * 64, 200, st.o_lat, st.lse)
    assert e.value.status == -4          # MLA_ERR_WORKSPACE
    st.close()
