"""Consecutive speculative rounds kept on the device.

The acceptance writes the next round's n_new and block tokens itself (dflash2_accept_chain), so
rounds follow one another with no host work in between (FastFlowLM card, "How it is used": the
target keeps the longest agreeing prefix plus one token of its own, and drafting continues from
there).  A serial chain is checked round by round against the oracle (each step through
parity.check_request, each acceptance bit-exact against oracle.accept_chain); the same rounds,
captured once as a CUDA graph of [target stand-in, dflash2_spec_round] and replayed, must
reproduce the serial chain bit for bit.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from block_diffusion_drafter_dflash2_b200 import inputs
from block_diffusion_drafter_dflash2_b200.binding import Drafter
from tests import parity

pytestmark = pytest.mark.gpu

ROUNDS = 5


def _clone(st):
    return {k: ([t.clone() for t in v] if isinstance(v, list) else (v.clone() if isinstance(v, torch.Tensor) else v))
            for k, v in st.items()}


def _target(path, m, V):
    """Stand-in for the target's verify pass (device ops, capturable): it agrees with the draft
    before position m[b] and disagrees from there on; position block-1 holds its bonus token."""
    B, D = path.shape
    ext = torch.cat([path, (path[:, :1] * 7 + 3) % V], dim=1)
    i = torch.arange(D + 1, device=path.device)[None, :]
    return torch.where(i < m[:, None], ext, (ext + 1) % V).to(torch.int32)


def test_device_chained_rounds_match_oracle_and_replay_as_one_graph():
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=4, ctx_lo=5, ctx_hi=300, shuffled_pages=True)
    d = wl.dims
    B, Bk, D, V = wl.batch, d.block, d.block - 1, d.vocab
    mask = V - 1
    torch.cuda.set_device(0)
    w = inputs.make_weights(d, wl.wseed, "cuda")
    hw_t, hw = parity.host_weights(w)
    st0 = inputs.make_state(wl, "cuda", extra_tokens=ROUNDS * Bk)
    m = torch.tensor([2, D, 0, 5], dtype=torch.int64, device="cuda")  # first disagreement per request

    # ---- serial chain, each round checked against the oracle ----
    st = _clone(st0)
    dr = Drafter(d, w, B)
    record = []
    run = parity.run_gpu(wl, w, range(B), state=st)
    for b in range(B):
        parity.check_request(run, hw_t, hw, b)
    path = run["path"]
    record.append((path.clone(), run["scores"].clone(), None))
    for r in range(1, ROUNDS):
        target = _target(path, m, V)
        acc = torch.full((B,), -5, dtype=torch.int32, device="cuda")
        em = torch.full((B, Bk), -5, dtype=torch.int32, device="cuda")
        dr.accept_chain(path, target, mask, acc, em, st["n_new"], st["block_tokens"])
        torch.cuda.synchronize()
        o_acc, o_em, o_nn, o_bt = oracle.accept_chain(path.cpu(), target.cpu(), mask)
        assert np.array_equal(acc.cpu().numpy(), o_acc) and np.array_equal(em.cpu().numpy(), o_em)
        assert np.array_equal(st["n_new"].cpu().numpy(), o_nn) and np.array_equal(st["block_tokens"].cpu().numpy(),
                                                                                    o_bt)
        assert np.array_equal(o_acc, np.minimum(m.cpu().numpy(), D))
        run = parity.run_gpu(wl, w, range(B), state=st)
        for b in range(B):
            parity.check_request(run, hw_t, hw, b)
        path = run["path"]
        record.append((path.clone(), run["scores"].clone(), (acc.clone(), st["n_new"].clone(),
                                                             st["block_tokens"].clone())))
    final_serial = st

    # ---- the same rounds from one captured graph ----
    st2 = _clone(st0)
    dr2 = Drafter(d, w, B)
    ins2 = {"taps": st2["taps"], "n_new": st2["n_new"], "block_tokens": st2["block_tokens"]}
    path2 = torch.empty((B, D), dtype=torch.int32, device="cuda")
    scores2 = torch.empty((B, D), dtype=torch.float32, device="cuda")
    acc2 = torch.empty((B,), dtype=torch.int32, device="cuda")
    em2 = torch.empty((B, Bk), dtype=torch.int32, device="cuda")
    tgt2 = torch.empty((B, Bk), dtype=torch.int32, device="cuda")
    dr2.draft_step(ins2, st2, path2, scores2)  # round 0 (also sets the kernels' attributes on the device)
    torch.cuda.synchronize()
    assert torch.equal(path2, record[0][0]) and torch.equal(scores2.view(torch.int32), record[0][1].view(torch.int32))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tgt2.copy_(_target(path2, m, V))
        dr2.spec_round(ins2, st2, path2, tgt2, mask, acc2, em2, path2, scores2, stream=s)
    torch.cuda.synchronize()
    for r in range(1, ROUNDS):
        g.replay()
        torch.cuda.synchronize()
        p_ref, s_ref, (a_ref, nn_ref, bt_ref) = record[r]
        assert torch.equal(acc2, a_ref) and torch.equal(st2["n_new"], nn_ref)
        assert torch.equal(st2["block_tokens"], bt_ref)
        assert torch.equal(path2, p_ref), (r, path2, p_ref)
        assert torch.equal(scores2.view(torch.int32), s_ref.view(torch.int32))
    assert dr2.device_error() == 0
    assert torch.equal(st2["seq_len"], final_serial["seq_len"])
    for l in range(d.layers):
        assert torch.equal(st2["k_cache"][l], final_serial["k_cache"][l])
        assert torch.equal(st2["v_cache"][l], final_serial["v_cache"][l])
    del g
