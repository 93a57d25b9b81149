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


def test_tiny_kernel_sequence_matches_oracle():
    """The single request as the kernel sequence the library reports."""
    wl = inputs.WORKLOADS["tiny"]
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, [0])
    assert run["drafter"].step_kernels() > 1
    parity.check_request(run, hw_t, hw, 0)
    parity.check_accept(run)


def test_tiny_bf16_layers_single_request_block5():
    """bf16 layer matrices, one request, block 5 (4 drafted rows, ragged query tile)."""
    import dataclasses
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


def test_tiny_many_requests_stream_the_window():
    """Ten requests (the streaming attention kernel's range): context lengths at page and window
    boundaries, an empty cache, ragged appends and shuffled physical pages in one call."""
    import dataclasses
    ctx = [0, 1, 15, 16, 57, 63, 64, 65, 200, 130]
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=10, shuffled_pages=True)
    w, hw_t, hw = weights_for(wl)
    st = inputs.make_state(wl, "cuda", seq_len=ctx, n_new=[8, 1, 0, 5, 8, 3, 8, 0, 2, 8])
    run = parity.run_gpu(wl, w, range(10), state=st)
    for b in range(10):
        parity.check_request(run, hw_t, hw, b)
    parity.check_accept(run)


def test_tiny_many_requests_window_pages_only_block5():
    """Eight bf16-layer requests of block 5 (ragged 20-vector query tiles) whose pages before the
    window are unbacked."""
    import dataclasses
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], dims=dataclasses.replace(inputs.TINY, wfmt=1, block=5),
                             batch=8, ctx_lo=1, ctx_hi=500, window_pages_only=True, shuffled_pages=True)
    w, hw_t, hw = weights_for(wl)
    run = parity.run_gpu(wl, w, range(8))
    for b in range(8):
        parity.check_request(run, hw_t, hw, b)


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


@pytest.mark.parametrize("mode,batch", [("pinned", 3), ("pageable", 3), ("mixed", 3), ("pinned", 40)])
def test_host_buffer_round_matches_device_step(mode, batch):
    """The host-buffer round returns the device step's path and scores bit for bit and the oracle's
    acceptance: page-locked buffers (read and written in place by the kernels), pageable ones
    (copied), and a mix (one pageable output makes the call fall back to copies); batch 40 has
    more block rows (320) than the staging kernel's 256 threads."""
    import dataclasses
    from block_diffusion_drafter_dflash2_b200.binding import Drafter
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=batch, ctx_lo=1, ctx_hi=200, target_mode="first_mismatch")
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

    def host(t, pin):
        t = t.cpu().clone()
        return t.pin_memory() if pin else t

    pinned = mode != "pageable"
    ins = [host(st_host[k], pinned) for k in ("taps", "n_new", "block_tokens")] + [host(target, pinned)]
    outs = [host(torch.full(shape, -5, dtype=dt), pinned and not (mode == "mixed" and i == 2)) for i, (shape, dt) in
            enumerate((((B, D), torch.int32), ((B, D), torch.float32), ((B,), torch.int32),
                       ((B, wl.dims.block), torch.int32)))]
    assert sum(not t.is_pinned() for t in ins + outs) == {"pinned": 0, "pageable": 8, "mixed": 1}[mode]
    derr = dr.spec_step_host(st_host, *ins, *outs)
    assert derr == 0
    assert torch.equal(outs[0], path.cpu())
    assert torch.equal(outs[1].view(torch.int32), scores.cpu().view(torch.int32))
    o_acc, o_em = oracle.accept(path.cpu(), target)
    assert np.array_equal(outs[2].numpy(), o_acc) and np.array_equal(outs[3].numpy(), o_em)
    assert torch.equal(st_host["seq_len"], st_dev["seq_len"])


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


@pytest.mark.slow
def test_full_size_320_rows_run_as_paired_tiles():
    """40 requests (320 block rows, 640 for k/v): the 4-bit layer products run as tensor-core tiles
    of two 256-row halves whose second half is partly filled (rows 256-319; for k/v 512-639 with
    an empty second half)."""
    import dataclasses
    wl = dataclasses.replace(inputs.WORKLOADS["full_b64"], batch=40)
    w, hw_t, hw = weights_for(wl)
    sample = [0, 33, 39]
    run = parity.run_gpu(wl, w, sample)
    for b in sample:
        parity.check_request(run, hw_t, hw, b)
    parity.check_accept(run)


def test_tied_candidates_are_distinct_and_in_id_order():
    """Exact logit ties in the output head: the head row of one drafted position's best token is
    copied onto 23 other ids (in its own 16-row tile, in other tiles of its 256-id record, and in
    records that other CTAs stream), so 24 ids tie at that position.  The GPU's list must hold 16
    distinct ids from the tied set, ordered by logit then smaller id (check_topk_row), and the
    oracle, fed the GPU's own final rows, must agree up to the near-tie rule."""
    wl = inputs.WORKLOADS["tiny"]
    w, _, _ = weights_for(wl)
    run = parity.run_gpu(wl, w, [0], state=inputs.make_state(wl, "cuda"))
    t_row = 2
    top = int(run["dbg"]["cand"][t_row, 0])
    V = wl.dims.vocab
    base = top // 16 * 16
    near = [base + k for k in range(16) if base + k != top][:5]            # same tile
    rec = top // 256 * 256
    same_rec = [rec + 16 * k + 3 for k in range(1, 16) if (rec + 16 * k + 3) // 16 != top // 16][:6]
    far = [(top + V // 2 + 37 * k) % V for k in range(12)]                   # other records, other CTAs
    dups = sorted(set(near + same_rec + far) - {top, V - 1})[:23]
    assert len(dups) == 23
    w2 = dict(w)
    w2["lm_head"] = w["lm_head"].clone()
    w2["lm_head"][torch.as_tensor(dups, device="cuda")] = w["lm_head"][top]
    hw_t, hw = parity.host_weights(w2)
    run2 = parity.run_gpu(wl, w2, [0], state=inputs.make_state(wl, "cuda"))
    parity.check_request(run2, hw_t, hw, 0)
    ids = run2["dbg"]["cand"][t_row].cpu().numpy()
    assert set(ids.tolist()) <= set(dups) | {top}, ids


@pytest.mark.parametrize("wfmt,block,batch", [(0, 8, 4), (0, 8, 6), (0, 8, 12), (1, 5, 20), (0, 8, 40)])
def test_tiny_many_rows_run_on_tensor_cores(wfmt, block, batch):
    """32 or more block rows: every layer product runs as a tcgen05 contraction (TMEM
    accumulators, dequantised weight tiles, TMA-staged activations; the tile's N is the rows
    rounded up to 16: 32, 48, 96, 112) followed by its fix-up kernel; Q4_K and bf16 layers, ragged
    new rows (0 included), shuffled pages, and 320 rows (two 256-row tiles, 640 rows for the k/v
    projections)."""
    import dataclasses
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], dims=dataclasses.replace(inputs.TINY, wfmt=wfmt, block=block),
                             batch=batch, ctx_lo=0, ctx_hi=300, shuffled_pages=True)
    w, hw_t, hw = weights_for(wl)
    n_new = [(3 * b) % (block + 1) for b in range(batch)]
    st = inputs.make_state(wl, "cuda", n_new=n_new)
    sample = sorted({0, 1, batch // 2, batch - 1})
    run = parity.run_gpu(wl, w, sample, state=st)
    base = 3 + 6 * wl.dims.layers + 3
    assert run["drafter"].step_kernels() == base + 6 * wl.dims.layers  # five layer products + fc, each + fix-up
    for b in sample:
        parity.check_request(run, hw_t, hw, b)
    parity.check_accept(run)


@pytest.mark.parametrize("wfmt,batch", [(2, 1), (2, 12), (3, 1), (3, 12)])
def test_tiny_alternate_codecs(wfmt, batch):
    """MLX-style 4-bit group-64 layers (decoded inside the products, streaming engine at one request,
    tensor cores at 96 rows) and Q8_0 layers (decoded once into bf16 records when the weights are
    prepared) against the oracle, which decodes both formats exactly."""
    import dataclasses
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], dims=dataclasses.replace(inputs.TINY, wfmt=wfmt),
                             batch=batch, ctx_lo=3, ctx_hi=150, shuffled_pages=batch > 1)
    w, hw_t, hw = weights_for(wl)
    sample = sorted({0, batch - 1})
    run = parity.run_gpu(wl, w, sample)
    for b in sample:
        parity.check_request(run, hw_t, hw, b)
    parity.check_accept(run)
