"""Vocabulary-sharded output head: partition and exchange on world-size-2 gloo ranks (CPU).

Each rank stands in for its GPU with the oracle: the LM head + top-16 over its own vocabulary
rows of the oracle's final rows.  The product's partition (vocab_shards) and exchange
(exchange_candidates) then bring both ranks' lists together, and the merged top-16 and the
selector's path must equal the oracle's single-rank results exactly.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from block_diffusion_drafter_dflash2_b200 import inputs
from block_diffusion_drafter_dflash2_b200.sharded import vocab_shards


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    from block_diffusion_drafter_dflash2_b200.sharded import exchange_candidates
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = inputs.WORKLOADS["tiny"]
        d = wl.dims
        w = inputs.make_weights(d, wl.seed)
        st = inputs.make_state(wl)
        hw = oracle.HostWeights(w)
        kc = [oracle._np(t).copy() for t in st["k_cache"]]
        vc = [oracle._np(t).copy() for t in st["v_cache"]]
        err, path, scores, sl, tr = oracle.draft_request(d, hw, st["taps"][0], int(st["n_new"][0]),
                                                         st["block_tokens"][0], kc, vc, st["page_table"][0],
                                                         int(st["seq_len"][0]), trace=True)
        assert err == 0
        v0, rows = vocab_shards(d.vocab, world)[rank]
        # this rank's local candidates: the oracle's head over rows [v0, v0 + rows) (fp64 rows in,
        # so the ranks' logits are the single-rank logits exactly)
        fh = tr["final_h"]
        lm = oracle.bf16_to_f64(oracle._np(w["lm_head"]))[v0:v0 + rows]
        logits = fh @ lm.T
        val = np.zeros((fh.shape[0], 16))
        ids = np.zeros((fh.shape[0], 16), np.int32)
        for t in range(fh.shape[0]):
            i, v = oracle.topk(logits[t], 16)
            ids[t], val[t] = i + v0, v
        gv, gi = exchange_candidates(torch.tensor(val, dtype=torch.float64).float(), torch.tensor(ids))
        if rank == 0:
            q.put((gv.numpy(), gi.numpy(), tr["cand"], tr["cand_logit"], tr["z"], path, wl.seed))
    finally:
        dist.destroy_process_group()


def test_vocab_shards_partition():
    for V, G in [(248320, 2), (248320, 8), (8192, 3), (8192, 8), (4096, 16)]:
        sh = vocab_shards(V, G)
        assert sh[0][0] == 0 and sum(r for _, r in sh) == V
        assert all(sh[i][0] + sh[i][1] == sh[i + 1][0] for i in range(G - 1))
        assert all(v0 % 256 == 0 for v0, _ in sh)
        assert max(r for _, r in sh) - min(r for _, r in sh) <= 256


def test_sharded_head_exchange_matches_single_rank_oracle():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    gv, gi, cand, cand_logit, z, path, seed = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert gv.shape == (world, cand.shape[0], 16)
    wl = inputs.WORKLOADS["tiny"]
    w = inputs.make_weights(wl.dims, seed)
    for t in range(cand.shape[0]):
        # merge of the gathered lists: logit descending, then smaller id
        v, i = gv[:, t].reshape(-1), gi[:, t].reshape(-1)
        order = np.lexsort((i, -v.astype(np.float64)))[:16]
        assert np.array_equal(i[order], cand[t]), (t, i[order], cand[t])
        assert np.allclose(v[order], cand_logit[t], rtol=1e-6)
    # the selector on the merged candidates gives the single-rank path
    p2, _ = oracle.selector(cand, cand_logit, z, int(inputs.make_state(wl)["block_tokens"][0, 0]), w["cb_a"], w["cb_b"])
    assert np.array_equal(p2, path)
