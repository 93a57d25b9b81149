"""Device-side error reporting: inputs that the kernels' own checks reject set bits in the
device error word (no trap, no fault), and host-side validation rejects bad arguments."""
import ctypes as C

import pytest
import torch

from block_diffusion_drafter_dflash2_b200 import binding, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    wl = inputs.WORKLOADS["tiny"]
    w = inputs.make_weights(wl.dims, wl.wseed, "cuda")
    return wl, binding.Drafter(wl.dims, w, 1)


def _step(wl, dr, st):
    D = wl.dims.block - 1
    path = torch.zeros((1, D), dtype=torch.int32, device="cuda")
    scores = torch.zeros((1, D), dtype=torch.float32, device="cuda")
    dr.draft_step({"taps": st["taps"], "n_new": st["n_new"], "block_tokens": st["block_tokens"]}, st, path, scores)
    torch.cuda.synchronize()
    return dr.device_error()


def test_clean_step_reports_no_error(tiny):
    wl, dr = tiny
    assert _step(wl, dr, inputs.make_state(wl, "cuda")) == 0


def test_out_of_range_token_sets_token_bit(tiny):
    wl, dr = tiny
    st = inputs.make_state(wl, "cuda")
    st["block_tokens"][0, 3] = wl.dims.vocab + 5
    assert _step(wl, dr, st) & binding.DEV_TOKEN
    # the word is cleared by the next step
    assert _step(wl, dr, inputs.make_state(wl, "cuda")) == 0


def test_unmapped_page_in_window_sets_page_bit(tiny):
    wl, dr = tiny
    st = inputs.make_state(wl, "cuda")
    L = int(st["seq_len"][0])
    st["page_table"][0, (L - 5) // 16] = -1  # a page the window must read
    assert _step(wl, dr, st) & binding.DEV_PAGE


def test_unmapped_append_page_sets_page_bit(tiny):
    wl, dr = tiny
    st = inputs.make_state(wl, "cuda")
    L = int(st["seq_len"][0])
    st["page_table"][0, (L + 2) // 16] = -1  # where this step appends
    assert _step(wl, dr, st) & binding.DEV_PAGE


def test_unmapped_page_in_window_sets_page_bit_many_requests():
    """Same check in the streaming attention kernel (eight requests)."""
    import dataclasses
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=8)
    w = inputs.make_weights(wl.dims, wl.wseed, "cuda")
    dr = binding.Drafter(wl.dims, w, 8)
    D = wl.dims.block - 1

    def step(st):
        path = torch.zeros((8, D), dtype=torch.int32, device="cuda")
        scores = torch.zeros((8, D), dtype=torch.float32, device="cuda")
        dr.draft_step({"taps": st["taps"], "n_new": st["n_new"], "block_tokens": st["block_tokens"]}, st, path,
                      scores)
        torch.cuda.synchronize()
        return dr.device_error()

    assert step(inputs.make_state(wl, "cuda")) == 0
    st = inputs.make_state(wl, "cuda")
    L = int(st["seq_len"][5])
    st["page_table"][5, (L - 5) // 16] = -1
    assert step(st) & binding.DEV_PAGE


def test_misaligned_taps_are_rejected(tiny):
    wl, dr = tiny
    st = inputs.make_state(wl, "cuda")
    n = st["taps"].numel()
    bad = torch.zeros(n + 8, dtype=torch.bfloat16, device="cuda")[1:1 + n].view(st["taps"].shape)  # 2-byte offset
    with pytest.raises(binding.DFlash2Error, match="ALIGN"):
        dr.draft_step({"taps": bad, "n_new": st["n_new"], "block_tokens": st["block_tokens"]}, st,
                      torch.zeros((1, 7), dtype=torch.int32, device="cuda"),
                      torch.zeros((1, 7), dtype=torch.float32, device="cuda"))
