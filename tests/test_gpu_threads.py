"""Two host threads stepping two drafters on one device, each on its own stream, give exactly the
results of the same steps run one after the other (the library keeps no per-call global state;
kernel attributes are recorded per device)."""
import threading

import pytest
import torch

from block_diffusion_drafter_dflash2_b200 import inputs
from block_diffusion_drafter_dflash2_b200.binding import Drafter

pytestmark = pytest.mark.gpu


def _clone(st):
    return {k: ([t.clone() for t in v] if isinstance(v, list) else (v.clone() if isinstance(v, torch.Tensor) else v))
            for k, v in st.items()}


def _steps(dr, st, n, stream=None):
    B, D = dr.batch, dr.dims.block - 1
    out = []
    with torch.cuda.stream(stream) if stream is not None else torch.cuda.stream(torch.cuda.current_stream()):
        for _ in range(n):
            path = torch.full((B, D), -1, dtype=torch.int32, device="cuda")
            scores = torch.full((B, D), float("nan"), dtype=torch.float32, device="cuda")
            ins = {"taps": st["taps"], "n_new": st["n_new"], "block_tokens": st["block_tokens"]}
            dr.draft_step(ins, st, path, scores, stream=stream)
            st["block_tokens"][:, 0] = path[:, 0]
            out.append((path, scores))
    return out


def test_two_threads_two_drafters_match_serial_steps():
    import dataclasses
    torch.cuda.set_device(0)
    wls = [inputs.WORKLOADS["tiny"],
           dataclasses.replace(inputs.WORKLOADS["tiny"], batch=4, ctx_lo=5, ctx_hi=300, shuffled_pages=True)]
    w = inputs.make_weights(wls[0].dims, wls[0].wseed, "cuda")
    states = [inputs.make_state(wl, "cuda", extra_tokens=3 * wl.dims.block) for wl in wls]
    serial_states = [_clone(s) for s in states]
    # serial reference on the current stream
    ref = []
    for wl, st in zip(wls, serial_states):
        ref.append(_steps(Drafter(wl.dims, w, wl.batch), st, 3))
    torch.cuda.synchronize()
    # concurrent: one thread, one drafter (own workspace) and one stream each
    drs = [Drafter(wl.dims, w, wl.batch) for wl in wls]
    torch.cuda.synchronize()
    res = [None, None]
    errs = []

    def run(i):
        try:
            torch.cuda.set_device(0)
            s = torch.cuda.Stream()
            res[i] = _steps(drs[i], states[i], 3, stream=s)
            s.synchronize()
        except Exception as e:  # surfaced below
            errs.append(e)

    th = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    torch.cuda.synchronize()
    assert not errs, errs
    for i in range(2):
        assert drs[i].device_error() == 0
        for (pa, sa), (pb, sb) in zip(ref[i], res[i]):
            assert torch.equal(pa, pb)
            assert torch.equal(sa.view(torch.int32), sb.view(torch.int32))
        assert torch.equal(states[i]["seq_len"], serial_states[i]["seq_len"])
        for l in range(wls[i].dims.layers):
            assert torch.equal(states[i]["k_cache"][l], serial_states[i]["k_cache"][l])
            assert torch.equal(states[i]["v_cache"][l], serial_states[i]["v_cache"][l])
