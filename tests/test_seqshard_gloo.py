"""The sequence-shard exchange on CPU, world size 2 over gloo: each rank holds
a slice of the positions, produces its unnormalised partial, the partials are
all-gathered, and the merge gives the attention over the whole context.  The
CUDA entry points are replaced by the fp64 oracle's range attention and
log-sum-exp merge (so this checks the exchange and layout, on CPU)."""
import math
import os
import socket
import sys
import traceback

import numpy as np
import torch
import torch.multiprocessing as mp

LOG2E = 1.0 / math.log(2.0)
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:  # spawned ranks import this module afresh
    sys.path.insert(0, ROOT)


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_q):
    try:
        _run(rank, world, port, out_q)
    except Exception:
        out_q.put((rank, float("inf"), traceback.format_exc()))


def _run(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import oracle
    from decode_attention_yocopp_b200.seqshard import local_lengths, seq_shard_decode, shard_bounds
    dist.init_process_group("gloo", rank=rank, world_size=world)
    orc = oracle.default()
    rng = np.random.default_rng(0)  # identical full context on every rank
    B, hkv, G, d = 2, 2, 4, 16
    lens = [301, 5]
    K = rng.standard_normal((B, hkv, max(lens), d)) * 2
    V = rng.standard_normal((B, hkv, max(lens), d))
    q = rng.standard_normal((B, hkv * G, d))
    ll = local_lengths(lens, world, rank)

    def partial_fn(qt, cache, local_lens, partial):
        for b in range(B):
            s0, e0 = shard_bounds(lens[b], world, rank)
            for g in range(hkv):
                m, l, o = orc.attention_partial(q[b, g * G:(g + 1) * G], K[b, g, :lens[b]], V[b, g, :lens[b]], "f64",
                                                s0, e0, 0.25)
                partial[b, g * G:(g + 1) * G, :d] = torch.from_numpy(o)
                partial[b, g * G:(g + 1) * G, d] = torch.from_numpy(m * LOG2E)
                partial[b, g * G:(g + 1) * G, d + 1] = torch.from_numpy(l)

    def combine_fn(gathered, out):
        g = gathered.numpy().astype(np.float64)
        for b in range(B):
            for h in range(hkv * G):
                mm = g[:, b, h, d] / LOG2E
                out[b, h] = torch.from_numpy(orc.lse_combine(mm[:, None], g[:, b, h, d + 1][:, None], g[:, b, h, None, :d])[0])

    out = torch.empty((B, hkv * G, d), dtype=torch.float64)
    seq_shard_decode(torch.from_numpy(q), None, torch.tensor(ll), out, None, partial_fn=partial_fn, combine_fn=combine_fn)
    ref = np.stack([np.concatenate([orc.attention(q[b, g * G:(g + 1) * G], K[b, g, :lens[b]], V[b, g, :lens[b]], "f64", 0.25)
                                    for g in range(hkv)]) for b in range(B)])
    out_q.put((rank, float(np.max(np.abs(out.numpy() - ref))), ll))
    dist.destroy_process_group()


def test_two_rank_sequence_shard():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda r: r[0])
    for r in res:
        assert r[1] != float("inf"), r[2]
    assert res[0][2] == [151, 3] and res[1][2] == [150, 2]  # the two slices cover every position once
    for _, err, _ in res:
        assert err < 1e-6  # the partials travel as fp32, the layout the C ABI defines
