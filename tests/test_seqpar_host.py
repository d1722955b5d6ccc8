"""Host logic of the sequence-parallel prefill (Chunk Parallelism), run as
three gloo ranks on the CPU.

Each rank holds a contiguous slice of the same sequences.  The exchange step
(all-gather of the slices' state increments and decays, then the fold into
each rank's initial state) is the product code in
``gated_retention_sequence_b200.seqpar``; its three computing steps are
replaced here by the fp64 oracle, so the test checks the exchange -- rank
order, gathered layout, fold -- against one oracle prefill of the whole
sequence.  (The GPU kernels of those steps have their own parity tests.)"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

CUTS = (0, 70, 150, 260)     # three ragged slices of 260 tokens


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The three computing steps in fp64 on the CPU (test stand-in)."""

    def state(self, K, V, z, tau, chunk):
        import oracle
        lg = oracle.log_gamma(z, tau)
        _, S = oracle.recurrent(K, K, V, lg)
        return torch.from_numpy(S), torch.from_numpy(np.asarray(lg).sum(axis=1))

    def fold(self, dS_all, decay_all, rank, S0):
        run = np.zeros(dS_all.shape[1:]) if S0 is None else S0.numpy().copy()
        for q in range(rank):
            run = np.exp(decay_all[q].numpy())[:, :, None, None] * run + dS_all[q].numpy()
        return torch.from_numpy(run)

    def prefill_from(self, Q, K, V, z, G, tau, chunk, eps, S_in):
        import oracle
        O, _, S = oracle.prefill(Q, K, V, z, G, tau, eps, S0=S_in.numpy())
        return torch.from_numpy(O), torch.from_numpy(S)


def _inputs():
    import gret_inputs as gi
    cfg = gi.C1.scaled(B=2, H=2, N=CUTS[-1], seed=55)
    inp = gi.prefill_inputs(cfg)
    S0 = gi.random_unit(55, 903, (cfg.B, cfg.H, cfg.dk, cfg.dv), var=0.04, io="f32").double()
    return cfg, inp, S0


def _rank_main(rank, world, port, out):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    from gated_retention_sequence_b200.seqpar import prefill_sequence_parallel
    from test_seqpar_host import OracleOps, _inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg, inp, S0 = _inputs()
        a, b = CUTS[rank], CUTS[rank + 1]
        sl = {k: v[:, a:b].contiguous() for k, v in inp.items()}
        O, S = prefill_sequence_parallel(sl["Q"], sl["K"], sl["V"], sl["z"], sl["G"], cfg.tau, cfg.chunk,
                                         eps=cfg.eps, S0=S0, ops=OracleOps())
        out[rank] = (O.numpy(), S.numpy())
    finally:
        dist.destroy_process_group()


def test_three_ranks_match_one_whole_prefill():
    import oracle
    world = len(CUTS) - 1
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    cfg, inp, S0 = _inputs()
    O_ref, _, S_ref = oracle.prefill(inp["Q"], inp["K"], inp["V"], inp["z"], inp["G"], cfg.tau, cfg.eps,
                                     S0=S0.numpy())
    O = np.concatenate([out[r][0] for r in range(world)], axis=1)
    np.testing.assert_allclose(O, O_ref, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(out[world - 1][1], S_ref, rtol=1e-9, atol=1e-12)
    # a middle rank's state is the state after its slice
    _, _, S_mid = oracle.prefill(inp["Q"][:, :CUTS[2]], inp["K"][:, :CUTS[2]], inp["V"][:, :CUTS[2]],
                                 inp["z"][:, :CUTS[2]], inp["G"][:, :CUTS[2]], cfg.tau, cfg.eps, S0=S0.numpy())
    np.testing.assert_allclose(out[1][1], S_mid, rtol=1e-9, atol=1e-12)
