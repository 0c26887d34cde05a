"""The expert-parallel layer's exchange logic on CPU ranks (gloo).

int8_weight_moe_b200.ep.ep_forward splits the experts over the ranks, sends
every assignment's token row to the rank that owns its expert, runs the owned
experts there and sends the results back for the gate-weighted combine.  Here
world-size-2 and -4 process groups over gloo run ep_forward with a stand-in
for the per-rank compute written from the CPU oracle (its grouping, experts
and combine in fp64; the GPU kernels of the same steps are checked against
the oracle in the -m gpu tests).  Every rank's output must equal the oracle's
single-process MoE forward of its tokens bit for bit: the exchange moves fp64
rows untouched, and the expert outputs and their weighted sum are the same
fp64 operations in the same order.
"""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleEpOps:
    """Per-rank compute of the expert-parallel layer from the CPU oracle:
    rows are bf16 bit patterns (int16) going out and fp64 expert outputs
    coming back."""

    def __init__(self, experts, E, top_k):
        self.experts_w = experts  # {global expert id: (qg, sg, qd, sd)} of this rank
        self.E, self.top_k = E, top_k

    def dispatch(self, x, ids, G):
        import oracle

        ids_np = ids.numpy()
        offsets, perm, inv = oracle.permute(ids_np, self.E)
        el = self.E // G
        x_send = x[torch.from_numpy(perm.astype(np.int64) // self.top_k)]
        local = torch.from_numpy((ids_np.reshape(-1)[perm] % el).astype(np.int32))
        return offsets.tolist(), torch.from_numpy(inv), x_send, local

    def experts(self, x_recv, ids_recv):
        import oracle

        R = x_recv.shape[0]
        if R == 0:
            return torch.empty((0, x_recv.shape[1]), dtype=torch.float64)
        owned = sorted(self.experts_w)
        el = len(owned)
        tables = [[self.experts_w[e][i] for e in owned] for i in range(4)]
        y = oracle.moe_forward(x_recv.numpy().view(np.uint16), ids_recv.numpy().reshape(R, 1),
                               np.ones((R, 1)), *tables)
        assert ids_recv.numpy().max() < el
        return torch.from_numpy(y)

    def combine(self, y_back, inv, gates):
        T, k = gates.shape
        out = torch.zeros((T, y_back.shape[1]), dtype=torch.float64)
        for t in range(T):
            for j in range(k):
                out[t] += gates[t, j].item() * y_back[inv[t * k + j]]
        return out


def _layer(T, d, f, E, top_k, seed):
    import oracle
    import synth
    from synth.workloads import SIGMA_R, SIGMA_W, SIGMA_X

    x = synth.normal_bf16_bits(seed, synth.X, SIGMA_X, (T, d))
    wr = synth.normal_f32(seed, synth.WR, SIGMA_R, (E, d))
    _, ids, gates = oracle.route(x, wr, top_k)
    experts = {}
    for e in range(E):
        qg, sg = oracle.quantize(synth.normal_bf16_bits(seed, synth.WGU, SIGMA_W, (2 * f, d),
                                                        start=e * 2 * f * d))
        qd, sd = oracle.quantize(synth.normal_bf16_bits(seed, synth.WD, SIGMA_W, (d, f),
                                                        start=e * d * f))
        experts[e] = (qg, sg, qd, sd)
    return x, ids, gates, experts


def _worker(rank, world, port, shape, queue):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    for p in (ROOT, HERE):
        sys.path.insert(0, p)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from int8_weight_moe_b200.ep import ep_forward

        T, d, f, E, top_k = shape
        x, ids, gates, experts = _layer(T * world, d, f, E, top_k, seed=90)
        mine = slice(rank * T, (rank + 1) * T)  # this rank's tokens
        el = E // world
        owned = {e: experts[e] for e in range(rank * el, (rank + 1) * el)}
        ops = OracleEpOps(owned, E, top_k)
        out = ep_forward(ops, torch.from_numpy(x[mine].view(np.int16)),
                         torch.from_numpy(ids[mine]), torch.from_numpy(gates[mine]), E)
        queue.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


def _run(world, shape):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


@pytest.mark.parametrize("world,shape", [(2, (24, 64, 128, 16, 2)), (4, (9, 64, 64, 8, 3))],
                         ids=["G2_E16_top2", "G4_E8_top3"])
def test_expert_parallel_forward_equals_oracle(world, shape):
    import oracle

    for p in (ROOT, HERE):
        if p not in sys.path:
            sys.path.insert(0, p)
    T, d, f, E, top_k = shape
    outs = _run(world, shape)
    x, ids, gates, experts = _layer(T * world, d, f, E, top_k, seed=90)
    tables = [[experts[e][i] for e in range(E)] for i in range(4)]
    ref = oracle.moe_forward(x, ids, gates, *tables)
    for r in range(world):
        np.testing.assert_array_equal(outs[r], ref[r * T:(r + 1) * T])


def test_owner_splits():
    sys.path.insert(0, ROOT)
    from int8_weight_moe_b200.ep import owner_splits

    offsets = [0, 3, 3, 7, 10, 10, 12, 15, 20]  # 8 experts
    assert owner_splits(offsets, 8, 1) == [20]
    assert owner_splits(offsets, 8, 2) == [10, 10]
    assert owner_splits(offsets, 8, 4) == [3, 7, 2, 8]
    with pytest.raises(ValueError):
        owner_splits(offsets, 8, 3)
