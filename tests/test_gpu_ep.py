"""The expert-parallel layer's kernels on one GPU, against the CPU oracle.

G ranks are emulated in one process on one GPU: every virtual rank routes its
own tokens and builds its send buffer with jmoe_ep_dispatch; the all-to-all
is done by slicing and concatenating those buffers (what
torch.distributed.all_to_all_single does between GPUs); each rank runs
jmoe_forward on the rows it received with its own slice of the experts, the
results go back the same way, and jmoe_ep_combine finishes.  Nothing waits on
another rank.  The exchange code itself (int8_weight_moe_b200.ep.ep_forward)
is covered on CPU ranks by test_ep_gloo.py.
"""
import numpy as np
import pytest

from layers import DeviceLayer, OracleLayer, assert_close, bf16_to_f64
from synth.workloads import Workload

torch = pytest.importorskip("torch")

import int8_weight_moe_b200 as jm  # noqa: E402
from int8_weight_moe_b200.ep import JmoeEpOps, local_slices, owner_splits  # noqa: E402


def emulated_ep_forward(dev, ids, gates, G, path):
    E = dev.wl.E
    T = dev.x.shape[0] // G
    ranks = []
    for r in range(G):
        ops = JmoeEpOps(*local_slices(dev.w_gu, dev.s_gu, dev.w_d, dev.s_d, E, G, r), E=E,
                        path=path)
        mine = slice(r * T, (r + 1) * T)
        offsets, inv, x_send, local_ids = ops.dispatch(dev.x[mine].contiguous(),
                                                       ids[mine].contiguous(), G)
        send = owner_splits(offsets, E, G)
        starts = np.concatenate([[0], np.cumsum(send)])
        ranks.append(dict(ops=ops, inv=inv, x_send=x_send, ids=local_ids, send=send,
                          starts=starts, back=[None] * G))
    for q in range(G):  # rank q receives block q of every rank, in rank order
        xs = [ranks[r]["x_send"][ranks[r]["starts"][q]:ranks[r]["starts"][q + 1]] for r in range(G)]
        ls = [ranks[r]["ids"][ranks[r]["starts"][q]:ranks[r]["starts"][q + 1]] for r in range(G)]
        y = ranks[q]["ops"].experts(torch.cat(xs).contiguous(), torch.cat(ls).contiguous())
        at = 0
        for r in range(G):
            n = xs[r].shape[0]
            ranks[r]["back"][q] = y[at:at + n]
            at += n
    outs = []
    for r in range(G):
        mine = slice(r * T, (r + 1) * T)
        y_back = torch.cat(ranks[r]["back"]).contiguous()
        outs.append(ranks[r]["ops"].combine(y_back, ranks[r]["inv"], gates[mine].contiguous()))
    return torch.cat(outs)


@pytest.mark.gpu
@pytest.mark.parametrize("G,T,E,top_k,path", [
    (2, 40, 16, 2, jm.JMOE_PATH_DECODE),
    (4, 24, 16, 2, jm.JMOE_PATH_AUTO),
    (2, 600, 16, 2, jm.JMOE_PATH_PREFILL),
    (8, 16, 64, 4, jm.JMOE_PATH_AUTO),
], ids=["G2_decode", "G4_auto", "G2_prefill", "G8_E64_top4"])
def test_expert_parallel_kernels_match_oracle(G, T, E, top_k, path):
    wl = Workload(f"ep_G{G}", 21, G * T, 256, 512, E=E, top_k=top_k)
    dev, ora = DeviceLayer(wl), OracleLayer(wl)
    ids, gates = jm.jmoe_route(dev.x, dev.w_router, top_k)
    out = emulated_ep_forward(dev, ids, gates, G, path)
    torch.cuda.synchronize()
    assert jm.jmoe_last_error() == jm.JMOE_OK
    _, io, go = ora.route()
    assert np.array_equal(ids.cpu().numpy(), io)
    tokens = np.arange(wl.T) if wl.T <= 256 else np.r_[0:64, wl.T - 64:wl.T]
    assert_close(bf16_to_f64(out)[tokens], ora.forward_tokens(tokens, io, go), wl.name)


@pytest.mark.gpu
def test_dispatch_matches_grouping_and_combine_sums_in_order():
    wl = Workload("ep_parts", 22, 50, 256, 512, E=16, top_k=2)
    dev = DeviceLayer(wl)
    ids, gates = jm.jmoe_route(dev.x, dev.w_router, 2)
    offsets, perm, inv, x_send, local_ids = jm.jmoe_ep_dispatch(dev.x, ids, 16, 4)
    o2, p2, i2 = jm.jmoe_permute(ids, 16)
    assert torch.equal(offsets, o2) and torch.equal(perm, p2) and torch.equal(inv, i2)
    tok = (perm // 2).long()
    assert torch.equal(x_send, dev.x[tok])
    assert torch.equal(local_ids, ids.reshape(-1)[perm.long()] % 4)
    # combine with identity "experts": sum_j g_j x_t in fp32, rounded once to
    # bf16 (within one bf16 rounding of the fp64 sum; the kernel may fuse the
    # multiply-add)
    out = jm.jmoe_ep_combine(x_send.contiguous(), inv, gates)
    ref = (gates.double().sum(dim=1, keepdim=True) * dev.x.double())
    torch.cuda.synchronize()
    err = (out.double() - ref).abs()
    assert bool((err <= ref.abs() * 2.0 ** -7 + 1e-30).all())
