"""The expert-parallel layer's dispatch, exchange and combine on 2 CPU ranks
(gloo), with the library calls replaced by their oracle-built CPU stand-ins
(tests/_fake_abi.py): each rank holds the routed experts e with e % 2 == rank,
routes its own tokens, and must produce exactly the oracle's single-process
layer output for those tokens; the bias update from the all-gathered expert
loads must equal the oracle's update from the loads of all ranks' tokens."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, dedupe=False):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import datetime
        import torch
        import torch.distributed as dist
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        import oracle
        import synth
        from sparse_moe_layer_group_b200.ep import EPMoELayer
        from sparse_moe_layer_group_b200.layer import QuantWeights
        from tests import _fake_abi
        s = synth.TINY
        H, E, K, I = s.H, s.E, s.K, s.I
        T = 24

        def master(kind, e):
            tid = (synth.SH13 if kind == "w13" else synth.SH2) if e < 0 else (synth.W13 if kind == "w13" else synth.W2)
            rows, cols = (2 * I, H) if kind == "w13" else (H, I)
            return synth.expert_weight(rows, cols, s.w_std, synth.seed_of(s, tid, max(e, 0))).float().numpy()

        # this rank's routed experts and the shared one, quantised by the oracle: per-slot
        # dispatch places expert e on rank e % world, node-limited dispatch on rank e // (E/world)
        El = E // world
        mine = ([rank * El + l for l in range(El)] if dedupe else [l * world + rank for l in range(El)]) + [-1]
        q13 = [oracle.quant_128x128(master("w13", e)) for e in mine]
        q2 = [oracle.quant_128x128(master("w2", e)) for e in mine]
        qw = QuantWeights(torch.from_numpy(np.stack([a for a, _ in q13])), torch.from_numpy(np.stack([b for _, b in q13])),
                          torch.from_numpy(np.stack([a for a, _ in q2])), torch.from_numpy(np.stack([b for _, b in q2])))
        wr = synth.router_weights(E, H, s.wr_std, synth.seed_of(s, synth.WR))
        b = synth.expert_bias(E, s.bias_range, synth.seed_of(s, synth.BIAS))
        x_all = synth.activations(world * T, H, synth.seed_of(s, synth.X))
        x = x_all[rank * T:(rank + 1) * T].contiguous()
        layer = EPMoELayer(T, H, E, K, s.n_group, s.topk_group, I, s.rho, wr, b, qw, device="cpu", abi=_fake_abi,
                           dedupe=dedupe, placement="block" if dedupe else "cyclic")
        out = layer.forward(x).float().numpy()
        ref = oracle.moe_forward(x.float().numpy(), wr.numpy(), b.numpy(), oracle.LayerWeights(master), s.n_group,
                                 s.topk_group, K, s.rho)
        if dedupe:
            # each rank's gated partial sum crosses back in bf16
            ref["out"] = oracle.round_bf16(oracle.combine_by_rank(ref["yperm"], ref["row_of"], ref["w"],
                                                                  ref["idx"] // El, ref["ysh"]))
            # a token crosses to each rank at most once
            sent = int(layer.send_load.sum())
            assert sent == sum(len(set(int(e) // El for e in row)) for row in ref["idx"])
        recv = int(layer.recv_counts.sum())
        # bias update from the global loads: same on every rank, equal to the oracle's
        gamma = 0.001
        b0 = layer.e_bias.clone()
        layer.bias_update(gamma)
        s32 = oracle.router_scores(x_all.float().numpy(), wr.numpy(), None).astype(np.float32)
        idx_all, _ = oracle.select_experts(s32, b0.numpy(), s.n_group, s.topk_group, K, s.rho)
        load_all = np.bincount(idx_all.reshape(-1), minlength=E)
        ref_b = oracle.bias_update(b0.numpy(), load_all, world * T, K, gamma)
        same_b = bool(np.array_equal(layer.e_bias.numpy(), ref_b)) and bool(np.array_equal(
            layer.load_all.numpy(), load_all))
        moved = bool((layer.e_bias != b0).any())
        dist.destroy_process_group()
        q.put((rank, bool(np.array_equal(out, ref["out"])) and same_b and moved,
               f"out {float(np.abs(out - ref['out']).max())} bias {same_b} moved {moved}", recv))
    except Exception as exc:                     # report instead of hanging the parent
        q.put((rank, False, repr(exc), -1))


import pytest


@pytest.mark.parametrize("dedupe,world", [(False, 2), (True, 2), (True, 4)])
def test_expert_parallel_layer_matches_the_oracle_on_cpu_ranks(dedupe, world):
    """Per-slot dispatch: the oracle's layer bit for bit.  Node-limited dispatch
    (one row per token and rank, block placement): the oracle's layer with the
    per-rank partial sums of combine_by_rank, bit for bit, and exactly one row
    sent per (token, rank) pair."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, dedupe)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    res.sort()
    for rank, same, err, recv in res:
        assert same, f"rank {rank}: {err}"
        assert recv > 0                      # each rank computed rows for the other rank's tokens too
