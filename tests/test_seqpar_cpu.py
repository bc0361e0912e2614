"""Host logic of the sequence-sharded attention cores (softmax_attention_video_gated_b200.seqpar)
on CPU ranks over gloo: the token shards, the all-reduce of the linear-attention
state and the all-gather of K and V. The kernel calls are replaced by the fp64
oracle's steps; what is checked is that sharding, collectives and read-out
give the unsharded result (GPU runs of the same phases are in the -m gpu tests)."""
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, N, H, d = 2, 37, 2, 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(5)
    D = H * d
    x = {n: rng.standard_normal((B, N, D)) for n in ("q", "k", "v", "g")}
    x["w"] = rng.standard_normal((B, N, H)) * 2.0
    return x


def _oracle_ops():
    import torch

    import oracle as O

    def state_bytes(b, h, dd):
        return b * h * (dd * dd + dd) * 4

    def state_fwd(k, v, state, h, flags=0, wgate=None):
        S, z = O.lin_state(k.numpy(), v.numpy(), h, None if wgate is None else wgate.numpy())
        flat = np.concatenate([S.reshape(B * h, -1), z.reshape(B * h, -1)], axis=1)
        state.copy_(torch.from_numpy(flat.reshape(-1)))

    def readout_fwd(q, gate, out, state, h, residual=None, eps=1e-6, flags=0):
        st = state.double().numpy().reshape(B * h, d * d + d)
        S = st[:, :d * d].reshape(B, h, d, d)
        z = st[:, d * d:].reshape(B, h, d)
        y = O.gate(O.lin_readout(q.numpy(), S, z, h, eps), gate.numpy())
        out.copy_(torch.from_numpy(y))

    def anchor_fwd(q, k, v, gate, out, h, residual=None, scale=0.0):
        y = O.softmax_anchor(q.numpy(), k.numpy(), v.numpy(), gate.numpy(), h)
        out.copy_(torch.from_numpy(y))

    return SimpleNamespace(state_bytes=state_bytes, state_fwd=state_fwd,
                           readout_fwd=readout_fwd, anchor_fwd=anchor_fwd)


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from softmax_attention_video_gated_b200 import seqpar

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    a, b = seqpar.shard_bounds(N, world, rank)
    x = {n: torch.from_numpy(np.ascontiguousarray(t[:, a:b])) for n, t in _inputs().items()}
    ops = _oracle_ops()
    y_lin = torch.empty_like(x["q"])
    seqpar.sharded_linear_attn(x["q"], x["k"], x["v"], x["g"], y_lin, H, wgate=x["w"], ops=ops)
    y_anc = torch.empty_like(x["q"])
    K, _ = seqpar.sharded_anchor(x["q"], x["k"], x["v"], x["g"], y_anc, H, N, ops=ops)
    out.put((rank, a, b, y_lin.numpy(), y_anc.numpy(), K.shape))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_cores_equal_the_unsharded_layer(world):
    import torch.multiprocessing as mp

    sys.path.insert(0, ROOT)
    import oracle as O

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    x = _inputs()
    lin = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, wgate=x["w"])
    anc = O.softmax_anchor(x["q"], x["k"], x["v"], x["g"], H)
    covered = []
    for rank, a, b, y_lin, y_anc, kshape in res:
        covered.append((a, b))
        assert tuple(kshape) == (B, N, H * d)          # every rank sees all keys
        # the state crosses ranks in fp32: relative error ~1e-7
        np.testing.assert_allclose(y_lin, lin[:, a:b], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(y_anc, anc[:, a:b], rtol=1e-12, atol=1e-12)
    assert covered[0][0] == 0 and covered[-1][1] == N
    assert all(covered[i][1] == covered[i + 1][0] for i in range(world - 1))


def test_shard_bounds_partition_the_tokens():
    sys.path.insert(0, ROOT)
    from softmax_attention_video_gated_b200 import seqpar

    for n, w in ((37, 2), (37, 3), (19320, 8), (8, 8)):
        lens = seqpar.shard_lengths(n, w)
        assert sum(lens) == n and max(lens) - min(lens) <= 1
        bounds = [seqpar.shard_bounds(n, w, r) for r in range(w)]
        assert bounds[0][0] == 0 and bounds[-1][1] == n
    with pytest.raises(ValueError):
        seqpar.shard_bounds(3, 4, 0)
