"""CUDA path (through the C ABI) against the fp64 oracle on seeded synthetic inputs."""
import numpy as np
import pytest
import torch

import oracle
from block_diffusion_drafter_dflash2_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu

_weights = {}


def weights_for(wl):
    key = (wl.dims, wl.wseed)
    if key not in _weights:
        _weights.clear()
        torch.cuda.empty_cache()
        w = inputs.make_weights(wl.dims, wl.wseed, "cuda")
        _weights[key] = (w, *parity.host_weights(w))
    return _weights[key]


def test_tiny_step_matches_oracle():
    wl = inputs.WORKLOADS["tiny"]
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, [0])
    rep = parity.check_request(run, hw_t, hw, 0)
    print(rep)
    parity.check_accept(run)


def test_tiny_single_request_runs_as_one_persistent_kernel(monkeypatch):
    monkeypatch.setenv("DFLASH2_PERSISTENT", "1")
    wl = inputs.WORKLOADS["tiny"]
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, [0])
    assert run["drafter"].step_kernels() == 1
    parity.check_request(run, hw_t, hw, 0)


def test_tiny_kernel_sequence_matches_oracle(monkeypatch):
    """The same single request through the multi-kernel sequence (persistent kernel switched off)."""
    monkeypatch.setenv("DFLASH2_PERSISTENT", "0")
    wl = inputs.WORKLOADS["tiny"]
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, [0])
    assert run["drafter"].step_kernels() > 1
    parity.check_request(run, hw_t, hw, 0)
    parity.check_accept(run)


def test_tiny_bf16_layers_single_request_block5(monkeypatch):
    """bf16 layer matrices in the persistent kernel (block 5: 4 drafted rows, ragged query tile)."""
    import dataclasses
    monkeypatch.setenv("DFLASH2_PERSISTENT", "1")
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], dims=dataclasses.replace(inputs.TINY, wfmt=1, block=5),
                             batch=1, ctx_lo=77, ctx_hi=77)
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, [0])
    parity.check_request(run, hw_t, hw, 0)


@pytest.mark.parametrize("n_new", [[0], [1], [3], [8]])
def test_tiny_ragged_new_rows(n_new):
    """0, 1, some or all block rows carry new context tokens (ragged appends)."""
    wl = inputs.WORKLOADS["tiny"]
    w, hw_t, hw = weights_for(wl)
    st = inputs.make_state(wl, "cuda", n_new=n_new)
    run = parity.run_gpu(wl, w, [0], state=st)
    parity.check_request(run, hw_t, hw, 0)


@pytest.mark.parametrize("ctx", [0, 1, 15, 16, 57, 63, 64, 65, 200])
def test_tiny_context_lengths_around_the_window(ctx):
    """Empty cache, page boundaries, shorter than / equal to / longer than the 64-token window."""
    wl = inputs.WORKLOADS["tiny"]
    w, hw_t, hw = weights_for(wl)
    st = inputs.make_state(wl, "cuda", seq_len=[ctx])
    run = parity.run_gpu(wl, w, [0], state=st)
    parity.check_request(run, hw_t, hw, 0)


def test_tiny_batch_of_requests_is_independent():
    """Five requests with different context lengths and ragged new rows in one call."""
    import dataclasses
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=5, ctx_lo=0, ctx_hi=300, shuffled_pages=True)
    w, hw_t, hw = weights_for(wl)
    st = inputs.make_state(wl, "cuda", n_new=[8, 1, 0, 5, 8])
    run = parity.run_gpu(wl, w, range(5), state=st)
    for b in range(5):
        parity.check_request(run, hw_t, hw, b)
    parity.check_accept(run)


def test_tiny_bf16_layers_block5():
    import dataclasses
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], dims=dataclasses.replace(inputs.TINY, wfmt=1, block=5),
                             batch=3, ctx_lo=1, ctx_hi=500, window_pages_only=True, tap_outliers=True)
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, range(3))
    for b in range(3):
        parity.check_request(run, hw_t, hw, b)


def test_steps_chain_and_device_state_advances():
    """Two steps in a row: the second sees the first one's appends through the cache."""
    wl = inputs.WORKLOADS["tiny"]
    w, hw_t, hw = weights_for(wl)
    st = inputs.make_state(wl, "cuda", extra_tokens=64)
    run1 = parity.run_gpu(wl, w, [0], state=st)
    parity.check_request(run1, hw_t, hw, 0)
    st["block_tokens"][0, 0] = run1["path"][0, 2]
    st["n_new"][0] = 3
    run2 = parity.run_gpu(wl, w, [0], state=st)
    parity.check_request(run2, hw_t, hw, 0)


@pytest.mark.parametrize("pinned", [True, False])
def test_host_buffer_round_matches_device_step(pinned):
    """The host-buffer round returns the device step's path and scores bit for bit and the oracle's
    acceptance: page-locked buffers (read and written in place by the kernels) and pageable ones
    (copied)."""
    import dataclasses
    from block_diffusion_drafter_dflash2_b200.binding import Drafter
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=3, ctx_lo=1, ctx_hi=200, target_mode="first_mismatch")
    w, _, _ = weights_for(wl)
    B, D = wl.batch, wl.dims.block - 1
    dr = Drafter(wl.dims, w, B)
    st_dev, st_host = inputs.make_state(wl, "cuda"), inputs.make_state(wl, "cuda")
    path = torch.full((B, D), -7, dtype=torch.int32, device="cuda")
    scores = torch.full((B, D), float("nan"), dtype=torch.float32, device="cuda")
    dr.draft_step({"taps": st_dev["taps"], "n_new": st_dev["n_new"], "block_tokens": st_dev["block_tokens"]}, st_dev,
                  path, scores)
    torch.cuda.synchronize()
    assert dr.device_error() == 0
    target = inputs.make_targets(wl, path).cpu()

    def host(t):
        t = t.cpu().clone()
        return t.pin_memory() if pinned else t

    ins = [host(st_host[k]) for k in ("taps", "n_new", "block_tokens")] + [host(target)]
    outs = [host(torch.full(shape, -5, dtype=dt)) for shape, dt in
            (((B, D), torch.int32), ((B, D), torch.float32), ((B,), torch.int32), ((B, wl.dims.block), torch.int32))]
    assert all(t.is_pinned() == pinned for t in ins + outs)
    derr = dr.spec_step_host(st_host, *ins, *outs)
    assert derr == 0
    assert torch.equal(outs[0], path.cpu())
    assert torch.equal(outs[1].view(torch.int32), scores.cpu().view(torch.int32))
    o_acc, o_em = oracle.accept(path.cpu(), target)
    assert np.array_equal(outs[2].numpy(), o_acc) and np.array_equal(outs[3].numpy(), o_em)
    assert torch.equal(st_host["seq_len"], st_dev["seq_len"])


@pytest.mark.slow
def test_full_b1_persistent(monkeypatch):
    """The full single-request step as one persistent kernel."""
    monkeypatch.setenv("DFLASH2_PERSISTENT", "1")
    wl = inputs.WORKLOADS["full_b1"]
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, [0])
    assert run["drafter"].step_kernels() == 1
    print("full_b1 persistent", parity.check_request(run, hw_t, hw, 0))


@pytest.mark.slow
@pytest.mark.parametrize("name,sample", [("full_b1", [0]), ("full_b8_paged", [0, 5]), ("full_b64", [3, 60]),
                                         ("full_bf16_b16", [2, 11])])
def test_full_size_configs(name, sample):
    """Full drafter shapes; the oracle recomputes sampled requests (requests are independent)."""
    wl = inputs.WORKLOADS[name]
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, sample)
    for b in sample:
        rep = parity.check_request(run, hw_t, hw, b)
        print(name, b, rep)
    parity.check_accept(run)
