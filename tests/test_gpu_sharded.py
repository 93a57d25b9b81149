"""The vocabulary-sharded output head on one GPU: three shards' steps run one after another (as
three ranks would), their local candidates are stacked as the all-gather would stack them, and
dflash2_select picks the path.  Checked stage-wise against the oracle on the step's own final
rows: the merged top-16 against the oracle's top-16 of the whole vocabulary, the path against the
oracle's selector on the merged candidates; every shard's cache and sequence lengths equal the
unsharded step's bit for bit (the layers are the same kernels on the same inputs)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from block_diffusion_drafter_dflash2_b200 import inputs
from block_diffusion_drafter_dflash2_b200.sharded import ShardedDrafter, vocab_shards
from tests import parity

pytestmark = pytest.mark.gpu


def _clone(st):
    return {k: ([t.clone() for t in v] if isinstance(v, list) else (v.clone() if isinstance(v, torch.Tensor) else v))
            for k, v in st.items()}


@pytest.mark.parametrize("batch,G", [(1, 3), (2, 4)])
def test_sharded_head_matches_oracle_and_unsharded_step(batch, G):
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=batch, ctx_lo=10, ctx_hi=150)
    d = wl.dims
    B, D = batch, d.block - 1
    torch.cuda.set_device(0)
    w = inputs.make_weights(d, wl.wseed, "cuda")
    hw_t, _ = parity.host_weights(w)
    st0 = inputs.make_state(wl, "cuda")
    ref = parity.run_gpu(wl, w, list(range(B)), state=_clone(st0))  # the unsharded step, debug outputs
    g_fh = ref["dbg"]["final_h"]
    vals, ids, states, z = [], [], [], None
    shards = vocab_shards(d.vocab, G)
    drafters = []
    for r in range(G):
        st = _clone(st0)
        sd = ShardedDrafter(d, w, B, rank=r, world=G)
        sd.local_step({"taps": st["taps"], "n_new": st["n_new"], "block_tokens": st["block_tokens"]}, st)
        torch.cuda.synchronize()
        assert sd.base.device_error() == 0
        v0, rows = shards[r]
        cid = sd.cand_id.cpu().numpy()
        assert np.all((cid >= v0) & (cid < v0 + rows)), (r, v0, rows)  # vocabulary ids of this shard
        vals.append(sd.cand_val.clone())
        ids.append(sd.cand_id.clone())
        states.append(st)
        drafters.append(sd)
        z = sd.z if z is None else z
        assert torch.equal(st["seq_len"], ref["state"]["seq_len"])
        for l in range(d.layers):
            assert torch.equal(st["k_cache"][l], ref["state"]["k_cache"][l])
            assert torch.equal(st["v_cache"][l], ref["state"]["v_cache"][l])
    gv, gi = torch.stack(vals), torch.stack(ids)  # [G][rows][16], as the all-gather stacks them
    path = torch.full((B, D), -3, dtype=torch.int32, device="cuda")
    scores = torch.full((B, D), float("nan"), dtype=torch.float32, device="cuda")
    drafters[0].select(gv, gi, st0["block_tokens"], path, scores)
    torch.cuda.synchronize()
    assert drafters[0].base.device_error() == 0
    # merged candidates (what the selector merges), stage-wise against the oracle on the GPU's rows
    o_ids, o_vals = oracle.lmhead_topk(g_fh, hw_t["lm_head"], 16)
    gvn, gin = gv.cpu().double().numpy(), gi.cpu().numpy()
    m_ids = np.zeros((B * D, 16), np.int32)
    m_vals = np.zeros((B * D, 16))
    for row in range(B * D):
        v, i = gvn[:, row].reshape(-1), gin[:, row].reshape(-1)
        order = np.lexsort((i, -v))[:16]
        m_ids[row], m_vals[row] = i[order], v[order]
    o_at_g = oracle.logits_at(g_fh, hw_t["lm_head"], m_ids)
    for row in range(B * D):
        parity.check_topk_row(m_ids[row], m_vals[row], o_ids[row], o_vals[row], o_at_g[row])
    # the path: the oracle's selector on the merged candidates, with the shard's z
    zz = z.cpu().double().numpy()
    for b in range(B):
        rs = slice(b * D, (b + 1) * D)
        s_path, s_scores = oracle.selector(m_ids[rs], m_vals[rs], zz[rs], int(st0["block_tokens"][b, 0]),
                                           hw_t["cb_a"], hw_t["cb_b"])
        g_path = path[b].cpu().numpy()
        if not np.array_equal(s_path, g_path):
            tau = oracle.selector_trans(m_ids[rs], zz[rs], int(st0["block_tokens"][b, 0]), hw_t["cb_a"], hw_t["cb_b"])
            idx = [int(np.where(m_ids[rs][t] == g_path[t])[0][0]) for t in range(D)]
            sc = m_vals[rs][0, idx[0]] + tau[0, 0, idx[0]]
            for t in range(1, D):
                sc += m_vals[rs][t, idx[t]] + tau[t, idx[t - 1], idx[t]]
            assert abs(sc - s_scores[-1]) <= parity.STAGE_TOL * max(1.0, abs(s_scores[-1]))
