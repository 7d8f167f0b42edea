"""Context-sharded decode, host side: two gloo ranks (one process per rank, as
torchrun starts them) each hold one token range of a context and its split
partials (m, l, o); ``gather_partials`` brings every rank's partials side by
side.  The merge of the gathered slots (done here in NumPy float64; on GPUs by
``tq_merge_partials``) must equal softmax attention over the whole context,
whatever the ranks' split counts."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LOG2E = 1.4426950408889634


def _problem(seed=0, rows=6, T=50, d=16):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((rows, T)) * 3.0          # already scaled
    values = rng.standard_normal((T, d))
    return logits, values


def _partials(logits, values, token_splits):
    """(m, l, o) per split of a shard, as the decode leaves them: m in log2 units."""
    rows, d = logits.shape[0], values.shape[1]
    S = len(token_splits)
    ml = np.zeros((rows, S, 2))
    o = np.zeros((rows, S, d))
    for s, (a, b) in enumerate(token_splits):
        if b <= a:
            ml[:, s, 0] = -np.inf
            continue
        z = logits[:, a:b] * LOG2E
        m = z.max(axis=1)
        p = np.exp2(z - m[:, None])
        ml[:, s, 0] = m
        ml[:, s, 1] = p.sum(axis=1)
        o[:, s] = p @ values[a:b]
    return ml, o


def _merge(ml, o):
    M = ml[:, :, 0].max(axis=1)
    w = np.where(np.isneginf(ml[:, :, 0]), 0.0, np.exp2(ml[:, :, 0] - M[:, None]))
    return (w[:, :, None] * o).sum(axis=1) / (w * ml[:, :, 1]).sum(axis=1)[:, None]


def _dense(logits, values):
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)) @ values


# rank 0 holds tokens 0..29 in 3 splits (one of them empty), rank 1 tokens 30..49 in 2
SHARDS = {0: [(0, 12), (12, 30), (30, 30)], 1: [(30, 41), (41, 50)]}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from compressed_attention_turboquantprod_b200 import gather_partials
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        logits, values = _problem()
        ml, o = _partials(logits, values, SHARDS[rank])
        gml, go = gather_partials(torch.from_numpy(ml).float(), torch.from_numpy(o).float(), slots=3)
        out[rank] = (gml.double().numpy(), go.double().numpy())
    finally:
        dist.destroy_process_group()


def test_gathered_partials_merge_to_whole_context_attention():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    logits, values = _problem()
    want = _dense(logits, values)
    for r in range(world):
        gml, go = res[r]
        assert gml.shape == (6, 6, 2) and go.shape == (6, 6, 16)
        # rank-major slots; rank 1's third slot is padding
        assert np.all(np.isneginf(gml[:, 5, 0])) and np.all(gml[:, 5, 1] == 0) and np.all(go[:, 5] == 0)
        assert np.max(np.abs(_merge(gml, go) - want)) < 1e-5     # float32 partials


def test_stack_partials_pads_and_orders():
    from compressed_attention_turboquantprod_b200 import stack_partials
    logits, values = _problem(1)
    parts = [_partials(logits, values, sh) for sh in SHARDS.values()]
    tp = [(torch.from_numpy(a).float(), torch.from_numpy(b).float()) for a, b in parts]
    ml, o = stack_partials(tp, slots=4)
    assert ml.shape == (6, 8, 2) and o.shape == (6, 8, 16)
    assert torch.isneginf(ml[:, 3, 0]).all() and torch.isneginf(ml[:, 6:, 0]).all()
    assert np.max(np.abs(_merge(ml.double().numpy(), o.double().numpy()) - _dense(logits, values))) < 1e-5
    with pytest.raises(ValueError):
        stack_partials(tp, slots=2)
