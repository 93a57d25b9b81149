"""Exact rejection-sampling acceptance on the GPU (dflash2_accept_sampled) against the oracle,
bit for bit: accepted lengths and emitted tokens are integers taken by exact rules, so any
difference is a bug.  Target distributions are softmaxes of random logits at several
temperatures (peaked and flat), drafted tokens are drawn from them (so acceptances of every length
occur), with and without a draft distribution, at a small vocabulary and at the full 248320."""
import numpy as np
import pytest
import torch

import oracle
from block_diffusion_drafter_dflash2_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _case(B, Bk, V, seed, with_q):
    g = np.random.default_rng(seed)
    D = Bk - 1
    temps = g.choice([0.3, 1.0, 3.0], size=(B, 1, 1))
    lg = g.standard_normal((B, Bk, V)) * 4.0 / temps
    p = np.exp(lg - lg.max(-1, keepdims=True))
    p = (p / p.sum(-1, keepdims=True)).astype(np.float32)
    draft = np.zeros((B, D), np.int32)
    for b in range(B):
        for i in range(D):  # mostly the target's likely tokens, so long acceptances happen
            draft[b, i] = np.argmax(p[b, i]) if g.random() < 0.7 else g.integers(0, V)
    q = None
    if with_q:
        lq = lg[:, :D] + g.standard_normal((B, D, V))
        q = np.exp(lq - lq.max(-1, keepdims=True))
        q = (q / q.sum(-1, keepdims=True)).astype(np.float32)
    ua = g.random((B, D)).astype(np.float32)
    us = g.integers(0, 2 ** 32, B, dtype=np.uint64).astype(np.uint32)
    us[0] = 0
    if B > 1:
        us[1] = 2 ** 32 - 1
    return draft, p, q, ua, us


@pytest.mark.parametrize("V,B,with_q", [(1000, 64, False), (1000, 64, True), (248320, 8, False), (248320, 4, True)])
def test_sampled_acceptance_matches_oracle(V, B, with_q):
    Bk = 8
    draft, p, q, ua, us = _case(B, Bk, V, 7 + V + B, with_q)
    dims = inputs.Dims(layers=1, hidden=256, ffn=256, n_q=1, n_kv=1, head_dim=128, window=16, vocab=V, n_taps=1,
                       block=Bk, topk=16, rank=16)
    draft[0, 3] = V + 5  # an id outside the vocabulary: rejected, never used as an index
    draft[-1, 1] = -2
    lib = binding.load()
    t = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a)).to("cuda", dt)
    acc = torch.full((B,), -5, dtype=torch.int32, device="cuda")
    em = torch.full((B, Bk), -5, dtype=torch.int32, device="cuda")
    # every device buffer stays referenced until the call has completed
    d_draft, d_p, d_ua = t(draft, torch.int32), t(p, torch.float32), t(ua, torch.float32)
    d_us = t(us.view(np.int32), torch.int32)
    d_q = t(q, torch.float32) if q is not None else None
    rc = lib.dflash2_accept_sampled(d_draft.data_ptr(), d_p.data_ptr(), d_q.data_ptr() if d_q is not None else None,
                                    d_ua.data_ptr(), d_us.data_ptr(), B, Bk, V, acc.data_ptr(), em.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    o_acc, o_em = oracle.accept_sampled(draft, p, ua, us, q=q)
    assert np.array_equal(acc.cpu().numpy(), o_acc), (acc.cpu().numpy(), o_acc)
    assert np.array_equal(em.cpu().numpy(), o_em)
    assert len(set(o_acc.tolist())) > 1  # the case exercises several acceptance lengths
