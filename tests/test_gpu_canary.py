"""Out-of-bounds writes: every buffer the library writes (the workspace, the path and scores, the
acceptance outputs, the debug outputs) is allocated with a canary margin after its declared size,
filled with a known byte pattern; after a step and an acceptance (and a tensor-core step with many
rows) the margins must be untouched.  The cache pages outside the appended rows are checked
bit-exact by the parity tests."""
import ctypes as C
import dataclasses

import pytest
import torch

from block_diffusion_drafter_dflash2_b200 import binding, inputs

pytestmark = pytest.mark.gpu

MARGIN = 4096  # bytes of canary after every buffer
PATTERN = 0xA5


def _canaried(nbytes, dev="cuda"):
    buf = torch.full((nbytes + MARGIN,), PATTERN, dtype=torch.uint8, device=dev)
    return buf


def _check(buf, nbytes, what):
    tail = buf[nbytes:]
    bad = (tail != PATTERN).nonzero()
    assert bad.numel() == 0, f"{what}: {bad.numel()} canary bytes overwritten, first at +{int(bad[0])}"


@pytest.mark.parametrize("batch", [1, 12])
def test_no_writes_past_any_buffer(batch):
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=batch, ctx_lo=5, ctx_hi=200)
    d = wl.dims
    B, Bk, D, H = batch, d.block, d.block - 1, d.hidden
    torch.cuda.set_device(0)
    w = inputs.make_weights(d, wl.wseed, "cuda")
    st = inputs.make_state(wl, "cuda")
    dr = binding.Drafter(d, w, B)
    lib = dr.lib
    ws = _canaried(dr.ws_bytes + 256)
    off = (-ws.data_ptr()) % 256  # the workspace is 256-byte aligned
    sizes = {"path": B * D * 4, "scores": B * D * 4, "acc": B * 4, "em": B * Bk * 4, "hidden": (d.layers + 1) * B * Bk * H * 4,
             "ctx": B * Bk * H * 2, "final_h": B * D * H * 2, "cand": B * D * 64, "cand_logit": B * D * 64,
             "z": B * D * d.rank * 4}
    bufs = {k: _canaried(v) for k, v in sizes.items()}
    dbg = binding.Debug()
    for k in ("hidden", "ctx", "final_h", "cand", "cand_logit", "z"):
        setattr(dbg, k, bufs[k].data_ptr())
    ins = binding.Inputs(st["taps"].data_ptr(), st["n_new"].data_ptr(), st["block_tokens"].data_ptr())
    kv = binding.kv_struct(st)
    rc = lib.dflash2_draft_step(C.byref(dr.cfg), C.byref(dr.w), C.byref(ins), C.byref(kv), B, bufs["path"].data_ptr(),
                                bufs["scores"].data_ptr(), ws.data_ptr() + off, dr.ws_bytes, C.byref(dbg),
                                binding._stream())
    assert rc == 0
    tgt = torch.randint(0, d.vocab, (B, Bk), dtype=torch.int32, device="cuda")
    rc = lib.dflash2_accept(bufs["path"].data_ptr(), tgt.data_ptr(), B, Bk, bufs["acc"].data_ptr(),
                            bufs["em"].data_ptr(), binding._stream())
    assert rc == 0
    torch.cuda.synchronize()
    err = C.c_int32(-1)
    assert lib.dflash2_device_error(C.c_void_p(ws.data_ptr() + off), C.byref(err), binding._stream()) == 0
    assert err.value == 0
    _check(ws, off + dr.ws_bytes, "workspace")
    assert bool((ws[:off] == PATTERN).all()), "write before the workspace"
    for k, n in sizes.items():
        _check(bufs[k], n, k)
