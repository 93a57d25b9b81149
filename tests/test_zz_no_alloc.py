"""The allocation-free entry point (dflash2_draft_step_static) against the workspace entry point.

Some callers cannot give the library a workspace (their device memory belongs to a
host framework's own pool, or an allocation's possible device synchronisation is not
acceptable on their path).  For them the library carries its own scratch array; this
test runs two steps in a row through each entry point, from identical starting states,
and checks that paths, scores, appended cache rows and sequence lengths agree.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from block_diffusion_drafter_dflash2_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _clone_state(st):
    return {k: ([t.clone() for t in v] if isinstance(v, list) else (v.clone() if isinstance(v, torch.Tensor) else v))
            for k, v in st.items()}


@pytest.mark.parametrize("name", ["tiny", "full_b1"])
def test_static_scratch_step_matches_workspace_step(name):
    wl = inputs.WORKLOADS[name]
    d = wl.dims
    torch.cuda.set_device(0)
    w = inputs.make_weights(d, wl.wseed, "cuda")
    dr = binding.Drafter(d, w, wl.batch)
    st_a = inputs.make_state(wl, "cuda", extra_tokens=2 * d.block)
    st_b = _clone_state(st_a)
    B, D = wl.batch, d.block - 1
    for call in range(2):
        outs = []
        for st, static in ((st_a, False), (st_b, True)):
            ins = {"taps": st["taps"], "n_new": st["n_new"], "block_tokens": st["block_tokens"]}
            path = torch.full((B, D), -1, dtype=torch.int32, device="cuda")
            scores = torch.full((B, D), float("nan"), dtype=torch.float32, device="cuda")
            if static:
                derr = torch.full((1,), -1, dtype=torch.int32, device="cuda")
                dr.draft_step_static(ins, st, path, scores, dev_err=derr)
                torch.cuda.synchronize()
                assert int(derr.item()) == 0
            else:
                dr.draft_step(ins, st, path, scores)
                torch.cuda.synchronize()
                assert dr.device_error() == 0
            outs.append((path.cpu(), scores.cpu()))
        (pa, sa), (pb, sb) = outs
        assert torch.equal(pa, pb), (call, pa, pb)
        # same kernels, same data, deterministic split-K fix-ups: the scores agree bit for bit
        assert torch.equal(sa.view(torch.int32), sb.view(torch.int32)), (call, sa, sb)
        assert torch.equal(st_a["seq_len"], st_b["seq_len"])
        for l in range(d.layers):
            assert torch.equal(st_a["k_cache"][l], st_b["k_cache"][l])
            assert torch.equal(st_a["v_cache"][l], st_b["v_cache"][l])
        # next call: the first drafted token becomes the block's first token
        for st in (st_a, st_b):
            st["block_tokens"][:, 0] = pa[:, 0].to("cuda")


def test_static_scratch_rejects_requests_beyond_its_size():
    lib = binding.load()
    cfg = binding.config(inputs.FULL)
    need = lib.dflash2_workspace_size(C.byref(cfg), 8)
    assert need > binding.STATIC_SCRATCH_BYTES
    w, ins, kv = binding.Weights(), binding.Inputs(), binding.KV()
    rc = lib.dflash2_draft_step_static(C.byref(cfg), C.byref(w), C.byref(ins), C.byref(kv), 8, None, None, None, None,
                                       None)
    assert rc == -7
