"""One MLA decode layer held on the GPU, driven through the C ABI.

``DecodeStep`` uploads a workload's weights, page table and cached history,
then runs decode steps -- append the new tokens, absorb the query, split-KV
decode, merge, output projection -- each as one call into libmla.  PyTorch only
provides device memory and the stream.

A workload is any object with the attributes of ``workloads.Workload`` (dims,
dtypes, page table, token arrays as numpy; bf16 as uint16 bit patterns).
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
import torch

from . import (Handle, mla_absorb_q, mla_cache_append, mla_combine_out_proj, mla_decode_auto_splits,
               mla_decode_combine, mla_decode_partial, mla_decode_workspace_bytes,
               mla_kv_project_append, mla_out_proj, mla_out_proj_workspace_bytes, mla_pack_w_o,
               mla_set_launch_overlap, mla_set_w_o_layout)

BLOCK_SIZE = 64


def to_device(a: np.ndarray, device, pin: bool = False) -> torch.Tensor:
    """numpy -> torch on ``device``; uint16 arrays are bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    if device is None or device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device, non_blocking=False)


def softmax_scale(d_nope: int, d_r: int) -> float:
    """1/sqrt(d_nope + d_r): the width of the per-head dot product before absorption."""
    return 1.0 / math.sqrt(d_nope + d_r)


class DecodeStep:
    def __init__(self, wl, device="cuda", num_splits: int = 0, max_position: Optional[int] = None,
                 overlap: bool = False, w_o_tiled: bool = True):
        """overlap: launch each kernel as a programmatic dependent of the one
        before it (its set-up and first weight loads overlap that kernel's end);
        the step never writes a weight, which is what that asks of the caller.
        w_o_tiled: keep W_O in the library's tile-major order (packed once here)
        where the shape allows; ``self.w_o`` is then that copy."""
        d = wl.dims
        self.wl = wl
        self.device = torch.device(device)
        self.H, self.d_c, self.d_r = d["num_heads"], d["d_c"], d["d_r"]
        self.d_nope, self.d_v, self.d_model = d["d_nope"], d["d_v"], d["d_model"]
        self.D = self.d_c + self.d_r
        self.B = wl.batch
        self.fp8 = wl.cache_dtype == "fp8_e4m3"
        self.tiny = wl.hist_x is not None
        self.max_seq_len = int(wl.seq_lens.max())
        if max_position is None:
            max_position = max(self.max_seq_len, 64)
        with torch.cuda.device(self.device):
            self.h = Handle(num_heads=self.H, d_c=self.d_c, d_r=self.d_r, d_nope=self.d_nope,
                            d_v=self.d_v, d_model=self.d_model, block_size=BLOCK_SIZE,
                            act_dtype=wl.act_dtype, cache_dtype=wl.cache_dtype,
                            softmax_scale=softmax_scale(self.d_nope, self.d_r),
                            rope_base=wl.rope_base, max_position=max_position)
        mla_set_launch_overlap(self.h, overlap)
        dev = self.device
        act = torch.float32 if wl.act_dtype == "fp32" else torch.bfloat16
        self.act = act
        # page table and lengths
        self.block_table = to_device(wl.block_table.astype(np.int32), dev)
        self.seq_lens = to_device(wl.seq_lens.astype(np.int32), dev)
        self.new_pos = to_device(wl.new_pos.astype(np.int32), dev)
        self.num_blocks = int(wl.num_blocks)
        # cache
        rows = self.num_blocks * BLOCK_SIZE
        if self.fp8:
            self.cache = torch.zeros(rows, self.D, dtype=torch.uint8, device=dev)
            self.cache_scale = torch.zeros(rows, dtype=torch.float32, device=dev)
        else:
            self.cache = torch.zeros(rows, self.D, dtype=act, device=dev)
            self.cache_scale = None
        # weights
        self.w_uk = to_device(wl.w_uk, dev)
        self.w_uv = to_device(wl.w_uv, dev)
        self.w_o = to_device(wl.w_o, dev)
        self.w_o_tiled = w_o_tiled and self.d_model % 128 == 0 and (self.H * self.d_v) % 64 == 0
        if self.w_o_tiled:
            packed = torch.empty_like(self.w_o)
            mla_pack_w_o(self.h, self.w_o, packed)
            torch.cuda.synchronize(dev)
            self.w_o = packed
            mla_set_w_o_layout(self.h, True)
        if self.tiny:
            self.w_dkv = to_device(wl.w_dkv, dev)
            self.w_kr = to_device(wl.w_kr, dev)
        # step inputs
        self.q_nope = to_device(wl.q_nope, dev)
        self.q_pe = to_device(wl.q_pe, dev)
        if self.tiny:
            self.new_x = to_device(wl.new_x, dev)
        else:
            self.new_c_kv = to_device(wl.new_c_kv, dev)
            self.new_k_r = to_device(wl.new_k_r, dev)
        # outputs and workspaces
        B, H = self.B, self.H
        self.q_lat = torch.empty(B, H, self.D, dtype=act, device=dev)
        self.o_lat = torch.empty(B, H, self.d_c, dtype=act, device=dev)
        self.lse = torch.empty(B, H, dtype=torch.float32, device=dev)
        self.o = torch.empty(B, H, self.d_v, dtype=act, device=dev)
        self.y = torch.empty(B, self.d_model, dtype=act, device=dev)
        self.set_splits(num_splits)
        nb = mla_out_proj_workspace_bytes(self.h, B)
        self.op_ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
        # run(): the append on a side stream beside the absorb
        self.side = torch.cuda.Stream(device=dev)
        self._fork = torch.cuda.Event()
        self._join = torch.cuda.Event()
        self.prefill()

    def set_splits(self, num_splits: int) -> None:
        self.num_splits = num_splits if num_splits > 0 else mla_decode_auto_splits(
            self.h, self.B, self.max_seq_len)
        nb = mla_decode_workspace_bytes(self.h, self.B, self.num_splits, self.max_seq_len)
        self.dec_ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=self.device)

    def prefill(self) -> None:
        """Write every sequence's history tokens into the paged cache (one call)."""
        wl = self.wl
        if len(wl.hist_seq) == 0:
            return
        seq = to_device(wl.hist_seq.astype(np.int32), self.device)
        pos = to_device(wl.hist_pos.astype(np.int32), self.device)
        if self.tiny:
            x = to_device(wl.hist_x, self.device)
            mla_kv_project_append(self.h, x, self.w_dkv, self.w_kr, pos, self.block_table,
                                  self.cache, self.cache_scale, seq_idx=seq, batch=self.B)
        else:
            c = to_device(wl.hist_c_kv, self.device)
            k = to_device(wl.hist_k_r, self.device)
            mla_cache_append(self.h, c, k, pos, self.block_table, self.cache, self.cache_scale,
                             seq_idx=seq, batch=self.B)
        torch.cuda.synchronize(self.device)

    # -- the five stages of a decode step ---------------------------------
    def append(self, stream=None) -> None:
        if self.tiny:
            mla_kv_project_append(self.h, self.new_x, self.w_dkv, self.w_kr, self.new_pos,
                                  self.block_table, self.cache, self.cache_scale, stream=stream)
        else:
            mla_cache_append(self.h, self.new_c_kv, self.new_k_r, self.new_pos, self.block_table,
                             self.cache, self.cache_scale, stream=stream)

    def absorb(self, stream=None) -> None:
        mla_absorb_q(self.h, self.q_nope, self.q_pe, self.new_pos, self.w_uk, self.q_lat,
                     stream=stream)

    def decode_partial(self, stream=None) -> None:
        mla_decode_partial(self.h, self.q_lat, self.cache, self.cache_scale, self.block_table,
                           self.seq_lens, self.max_seq_len, self.num_splits, self.dec_ws,
                           stream=stream)

    def decode_combine(self, stream=None) -> None:
        mla_decode_combine(self.h, self.B, self.max_seq_len, self.num_splits, self.dec_ws,
                           self.o_lat, self.lse, stream=stream)

    def out_proj(self, stream=None) -> None:
        mla_out_proj(self.h, self.o_lat, self.w_uv, self.w_o, self.op_ws, self.y, self.o,
                     stream=stream)

    def combine_out_proj(self, stream=None) -> None:
        """The split merge and the output projection in one call (the merge runs
        inside the W_UV kernel where the library can)."""
        mla_combine_out_proj(self.h, self.B, self.max_seq_len, self.num_splits, self.dec_ws, self.w_uv,
                             self.w_o, self.op_ws, self.o_lat, self.y, lse=self.lse, o_out=self.o,
                             stream=stream)

    def stages(self):
        """(name, call) of the C-ABI calls of one decode step, in order."""
        return [("append", self.append), ("absorb", self.absorb), ("decode_partial", self.decode_partial),
                ("combine_out_proj", self.combine_out_proj)]

    def run(self, stream=None) -> None:
        """One decode step.  The append and the absorbed query are independent
        (one writes the cache, the other reads q and W_UK), so the append runs on
        a side stream beside the absorb; the decode waits for both."""
        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._fork.record(main)
        self.side.wait_event(self._fork)
        self.append(self.side)
        self._join.record(self.side)
        self.absorb(main)
        main.wait_event(self._join)
        self.decode_partial(main)
        self.combine_out_proj(main)

    def run_in_order(self, stream=None) -> None:
        """The step's calls one after another on one stream."""
        for _, fn in self.stages():
            fn(stream)

    # -- CUDA graphs of the step (the C-ABI calls neither allocate nor sync) --
    def capture(self) -> None:
        """Record one CUDA graph per stage and one for the whole step.  Call after
        an ordinary run() (first calls configure kernels).  Replays reuse the
        buffers of this object: refresh inputs in place (copy_) between replays."""
        torch.cuda.synchronize(self.device)
        self.stage_graphs = []
        for _, fn in self.stages():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            self.stage_graphs.append(g)
        self.step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.step_graph):
            self.run()
        torch.cuda.synchronize(self.device)

    def replay(self) -> None:
        self.step_graph.replay()

    def outputs(self) -> Dict[str, np.ndarray]:
        torch.cuda.synchronize(self.device)
        f = lambda t: t.float().cpu().numpy().astype(np.float64)
        return dict(q_lat=f(self.q_lat), o_lat=f(self.o_lat), lse=f(self.lse), o=f(self.o),
                    y=f(self.y))

    def close(self) -> None:
        self.h.close()
