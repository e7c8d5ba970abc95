"""The multi-rank path of the replicas (bench.py --gpus N) on CPU: two gloo
ranks, each running the oracle forward on its own rows, meet in the same
host-side reductions the bench uses.  The global mean loss of the two
replicas must equal the mean over the union of their rows computed in one
process ([Math] §Cross-Entropy Loss: the mean over every valid target), and
the timing reductions must pick the slowest rank."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from decoder_only_transformer_fwd_b200 import replicas, synth
from oracle import nanochat_fwd as O

WORLD = 2
DEPTH, B, T = 1, 2, 24


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    ocfg = O.make_config(DEPTH, T, T, vocab=512)
    C, H = O.model_dims(DEPTH)
    p = synth.params(7, n_layer=DEPTH, n_embd=C, n_head=H, n_kv_head=H, head_dim=128, vocab=512,
                     vocab_padded=512, ve_layers=ocfg["ve_layers"], bf16=False)
    return ocfg, p


def _rank_rows(rank):
    seed = replicas.rank_seed(11, rank)
    tok = synth.tokens(seed, B, T, 512)
    tgt = synth.targets(seed, B, T, 512).copy()
    tgt[0, : 3 + rank] = -1   # ignored targets, a different count per rank
    return tok, tgt


def _worker(rank, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        ocfg, p = _case()
        tok, tgt = _rank_rows(rank)
        loss, _ = O.forward(ocfg, p, tok, tgt)
        valid = tgt >= 0
        mean = replicas.global_mean_loss(float(loss[valid].sum()), int(valid.sum()))
        slowest = replicas.max_over_ranks(1.0 + rank * 0.5)   # rank 1 "took" 1.5 s
        rate = replicas.aggregate_throughput(B * T, WORLD, 3, slowest)
        dist.barrier()
        out[rank] = (mean, slowest, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_reduce_like_one_process():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, port, out)) for r in range(WORLD)]
        for pr in procs:
            pr.start()
        for pr in procs:
            pr.join(timeout=300)
        assert all(pr.exitcode == 0 for pr in procs), [pr.exitcode for pr in procs]
        res = dict(out)
    # one process over the union of both ranks' rows
    ocfg, p = _case()
    rows = [_rank_rows(r) for r in range(WORLD)]
    tok = np.concatenate([r[0] for r in rows])
    tgt = np.concatenate([r[1] for r in rows])
    loss, _ = O.forward(ocfg, p, tok, tgt)
    ref = O.mean_loss(loss, tgt)
    for r in range(WORLD):
        mean, slowest, rate = res[r]
        assert abs(mean - ref) <= 1e-12 * abs(ref), (r, mean, ref)
        assert slowest == 1.5
        assert rate == pytest.approx(B * T * WORLD * 3 / 1.5)
    # the ranks drew different rows
    assert not np.array_equal(rows[0][0], rows[1][0])


def test_single_process_reductions_are_identities():
    assert replicas.max_over_ranks(2.5) == 2.5
    assert replicas.global_mean_loss(6.0, 4) == 1.5
    assert np.isnan(replicas.global_mean_loss(0.0, 0))
    assert replicas.aggregate_throughput(100, 1, 2, 0.5) == 400.0
