"""Helpers shared by the GPU parity tests: move seeded workloads to the device,
run the CUDA path through the C ABI, run the oracle on the same inputs, and
measure the difference.  Marshalling only -- no attention arithmetic here.

Parity gate (from the stated target: max-abs 2e-2, max-rel 1e-2 on bf16
outputs computed with fp32 accumulation):
  * |gpu - oracle| <= 2e-2 + half a bf16 ulp of |oracle|, per element (below)
  * max_rel  = max over (token, head) rows of
               max_d |gpu - oracle| / max(max_d |oracle|, 1e-2)     <= 1e-2
    i.e. the error of each head's output vector relative to that vector's
    magnitude (a per-element ratio is meaningless for outputs near zero);
  * lse: max |gpu - oracle| <= 1e-3.
The abs gate is applied per element as 2e-2 plus half a bf16 ulp of that
element's exact value: the output itself is rounded to bf16, which alone can
move an element by half an ulp (2^-6 for |O| in [4, 8), more than 2e-2 would
leave for the arithmetic), and an element below 2 gets at most 2e-2 + 2^-8.
The per-element relative error |gpu - oracle| / max(|oracle|, 1e-2) is also
measured and reported (max_rel_elem); it is not gated, since near-zero outputs
make it a ratio of rounding noise to nothing.  With PA_PARITY_LOG set to a
file path, every checked case appends one JSON line with these statistics.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle
from paged_kv_cache_461_b200 import api
from paged_kv_cache_461_b200 import workloads as W

ATOL = 2e-2
RTOL = 1e-2
LSE_TOL = 1e-3


def to_dev_bf16(a: np.ndarray, dev="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def to_nhd(cache: torch.Tensor) -> torch.Tensor:
    """[NB, Hkv, 16, D] (HND) -> contiguous [NB, 16, Hkv, D] (NHD): the same values, token-major blocks."""
    return cache.transpose(1, 2).contiguous()


def to_hnd(cache: torch.Tensor) -> torch.Tensor:
    return cache.transpose(1, 2).contiguous()


class DevStep:
    """Device copies of one step (metadata + values).  kv_layout "NHD" stores the caches
    token-major ([NB, 16, Hkv, D]); the host values are always HND."""

    def __init__(self, layout: W.StepLayout, vals: W.StepValues, dev="cuda", kv_layout="HND"):
        self.layout = layout
        self.kv_layout = kv_layout
        self.qsl = torch.from_numpy(layout.query_start_loc).to(dev)
        self.seq_lens = torch.from_numpy(layout.seq_lens).to(dev)
        self.bt = torch.from_numpy(layout.block_table).to(dev)
        self.slots = torch.from_numpy(layout.slot_mapping).to(dev)
        if isinstance(vals.q, np.ndarray):
            self.q, self.k_new, self.v_new = (to_dev_bf16(x, dev) for x in (vals.q, vals.k_new, vals.v_new))
            self.k_cache, self.v_cache = to_dev_bf16(vals.k_cache, dev), to_dev_bf16(vals.v_cache, dev)
        else:
            self.q, self.k_new, self.v_new = vals.q, vals.k_new, vals.v_new
            self.k_cache, self.v_cache = vals.k_cache, vals.v_cache
        if kv_layout == "NHD":
            self.k_cache, self.v_cache = to_nhd(self.k_cache), to_nhd(self.v_cache)

    def write(self):
        api.kv_write(self.k_new, self.v_new, self.slots, self.k_cache, self.v_cache, layout=self.kv_layout)

    def _ws(self, workspace, kv_split_tokens, decode_max_query_len):
        lay = self.layout
        if workspace is None:
            workspace = api.alloc_workspace(lay.num_seqs, lay.num_tokens, lay.num_q_heads, self.k_cache,
                                            lay.max_seq_len, kv_split_tokens, decode_max_query_len,
                                            layout=self.kv_layout)
        return workspace

    def _outs(self, with_lse):
        lay = self.layout
        lse = torch.full((lay.num_tokens, lay.num_q_heads), float("nan"), dtype=torch.float32,
                         device=self.q.device) if with_lse else None
        return torch.full_like(self.q, float("nan")), lse

    def attend(self, kv_split_tokens=0, with_lse=True, scale=None, workspace=None, decode_max_query_len=0):
        lay = self.layout
        out, lse = self._outs(with_lse)
        workspace = self._ws(workspace, kv_split_tokens, decode_max_query_len)
        api.attention_mixed(self.q, self.k_cache, self.v_cache, self.qsl, self.seq_lens, self.bt,
                            lay.max_query_len, lay.max_seq_len, softmax_scale=scale, out=out, lse=lse,
                            workspace=workspace, kv_split_tokens=kv_split_tokens,
                            decode_max_query_len=decode_max_query_len, layout=self.kv_layout)
        self.workspace = workspace
        return out, lse

    def write_and_attend_fused(self, kv_split_tokens=0, with_lse=True, scale=None, workspace=None,
                               decode_max_query_len=0):
        """pa_attention_decode_fused: this step's K/V written by the decode kernel itself."""
        lay = self.layout
        out, lse = self._outs(with_lse)
        workspace = self._ws(workspace, kv_split_tokens, decode_max_query_len)
        api.attention_decode_fused(self.q, self.k_new, self.v_new, self.k_cache, self.v_cache, self.qsl,
                                   self.seq_lens, self.bt, lay.max_query_len, lay.max_seq_len, softmax_scale=scale,
                                   out=out, lse=lse, workspace=workspace, kv_split_tokens=kv_split_tokens,
                                   decode_max_query_len=decode_max_query_len, layout=self.kv_layout)
        self.workspace = workspace
        return out, lse


def write_and_attend_mixed(st: "DevStep", kv_split_tokens=0, with_lse=True, scale=None, workspace=None,
                           decode_max_query_len=0):
    """pa_attention_mixed_write on a DevStep: its K/V written (through its slot mapping) by the launch that
    also plans the step, then attention as attention_mixed does."""
    lay = st.layout
    out, lse = st._outs(with_lse)
    workspace = st._ws(workspace, kv_split_tokens, decode_max_query_len)
    api.attention_mixed_write(st.q, st.k_new, st.v_new, st.slots, st.k_cache, st.v_cache, st.qsl, st.seq_lens,
                              st.bt, lay.max_query_len, lay.max_seq_len, softmax_scale=scale, out=out, lse=lse,
                              workspace=workspace, kv_split_tokens=kv_split_tokens,
                              decode_max_query_len=decode_max_query_len, layout=st.kv_layout)
    st.workspace = workspace
    return out, lse


def work_counts(workspace: torch.Tensor):
    """(decode units, prefill work items, split requests) the plan kernel wrote into the workspace header."""
    h = workspace[:16].view(torch.int32).cpu().tolist()
    return h[1], h[2], h[3]


def oracle_for_step(layout: W.StepLayout, vals: W.StepValues, scale=None, token_list=None):
    """Oracle on the host copy of the inputs (KV written by the oracle's own write)."""
    kc, vc = oracle.kv_write(vals.k_new, vals.v_new, layout.slot_mapping, vals.k_cache, vals.v_cache)
    if scale is None:
        scale = 1.0 / math.sqrt(layout.head_dim)
    return oracle.attention_for(layout, kc, vc, vals.q, scale=scale, token_list=token_list)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits): 2^(e - 9) for |x| = m * 2^e, m in [0.5, 1)."""
    _, e = np.frexp(np.abs(x))
    return np.where(x == 0, 0.0, np.ldexp(1.0, e - 9))


def errors(gpu_out: torch.Tensor, ref: np.ndarray, rows=None) -> dict:
    g = bf16_to_f64(gpu_out)
    if rows is not None:
        g = g[rows]
    d = np.abs(g - ref)
    if d.size == 0:
        return {"max_abs": 0.0, "max_rel": 0.0, "max_rel_elem": 0.0, "abs_over_gate": 0.0, "nan": False}
    nan = bool(np.isnan(g).any())
    row_err = d.max(axis=-1)
    row_mag = np.maximum(np.abs(ref).max(axis=-1), 1e-2)
    rel = row_err / row_mag
    rel_elem = d / np.maximum(np.abs(ref), 1e-2)
    gate = ATOL + bf16_half_ulp(ref)
    i = np.unravel_index(int(np.nanargmax(d)), d.shape)
    return {"max_abs": float(np.nanmax(d)), "max_rel": float(np.nanmax(rel)),
            "max_rel_elem": float(np.nanmax(rel_elem)), "abs_over_gate": float(np.nanmax(d / gate)),
            "argmax": tuple(int(x) for x in i), "nan": nan}


def _log(what: str, e: dict):
    path = os.environ.get("PA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": what, **{k: v for k, v in e.items() if k != "argmax"}}) + "\n")


def assert_parity(gpu_out, ref, gpu_lse=None, ref_lse=None, rows=None, what=""):
    e = errors(gpu_out, ref, rows)
    _log(what, e)
    assert not e["nan"], f"{what}: NaN in GPU output"
    assert e["abs_over_gate"] <= 1.0, f"{what}: |err| above 2e-2 + half a bf16 ulp somewhere: {e}"
    assert e["max_rel"] <= RTOL, f"{what}: max_rel {e}"
    if gpu_lse is not None and ref_lse is not None:
        gl = gpu_lse.cpu().numpy().astype(np.float64)
        if rows is not None:
            gl = gl[rows]
        dl = np.abs(gl - ref_lse)
        assert not np.isnan(gl).any(), f"{what}: NaN in GPU lse"
        assert dl.max() <= LSE_TOL, f"{what}: lse err {dl.max()}"
    return e
