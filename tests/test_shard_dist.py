"""The time-split protocol (selective_state_space_52_b200/shard.py) across
gloo ranks on CPU: world sizes 2 and 3, each rank holding one slice of a
sequence.  The per-slice operations are CPU stand-ins here (the oracle's scan,
numpy for the dt sum and the fold), so what is tested is the protocol: conv
halo from the previous rank, which state each slice starts from, the order of
the gathered summaries, the fold.  The concatenated outputs and the last
rank's caches must equal the oracle's scan over the whole sequence.  The CUDA
operations themselves are tested on the GPU in tests/test_shard_gpu.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def oracle_ops():
    import oracle
    from selective_state_space_52_b200.shard import SliceOps

    def scan(x, z, dt, Bm, Cm, params, cache):
        cc, ss = (None, None) if cache is None else cache
        y, cco, sso = oracle.scan_fwd(x, z, dt, Bm, Cm, params["conv_w"], params["conv_b"],
                                      params["dt_bias"], params["A_log"], params["D"], cc, ss)
        return torch.from_numpy(y), (torch.from_numpy(cco), torch.from_numpy(sso))

    def dt_sum(dt_raw, dt_bias):
        v = dt_raw.double().numpy() + dt_bias.double().numpy()
        return torch.from_numpy(np.clip(np.logaddexp(0.0, v), 1e-4, 100.0).sum(axis=1))

    def fold(r, A_log, h_all, dts_all):
        A = -np.exp(A_log.double().numpy())
        h = h_all[0].double().numpy()
        for j in range(1, r):
            h = np.exp(A * dts_all[j].double().numpy()[..., None]) * h + h_all[j].double().numpy()
        return torch.from_numpy(h)

    return SliceOps(scan=scan, dt_sum=dt_sum, fold=fold)


def _problem(with_state):
    from selective_state_space_52_b200 import workloads as W
    wl = W.custom(2, 30, 16, io="f32", seed=91)
    return W.make_inputs(wl, with_state=with_state)


def _worker(rank, world, port, with_state, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    from selective_state_space_52_b200.shard import sharded_scan_fwd
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    inp = _problem(with_state)
    L = inp["x"].shape[1]
    cut = [L * r // world for r in range(world + 1)]
    sl = {k: inp[k][:, cut[rank]:cut[rank + 1]].contiguous() for k in ("x", "z", "dt_raw", "B", "C")}
    params = {k: inp[k] for k in ("conv_w", "conv_b", "dt_bias", "A_log", "D")}
    cache = (inp["conv_cache"], inp["ssm_state"]) if with_state else None
    y, (cc, ss) = sharded_scan_fwd(sl, params, cache, ops=oracle_ops())
    q.put((rank, y.numpy(), cc.numpy(), ss.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("with_state", [False, True])
def test_time_split_protocol_on_gloo_ranks(world, with_state):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, with_state, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    finally:
        for p in procs:                      # never leave a rank behind
            if p.is_alive():
                p.terminate()
                p.join(timeout=10)
    inp = _problem(with_state)
    y_ref, cc_ref, ss_ref = oracle.scan_fwd(
        inp["x"], inp["z"], inp["dt_raw"], inp["B"], inp["C"], inp["conv_w"], inp["conv_b"],
        inp["dt_bias"], inp["A_log"], inp["D"],
        inp["conv_cache"] if with_state else None, inp["ssm_state"] if with_state else None)
    y = np.concatenate([r[1] for r in res], axis=1)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res[-1][3], ss_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(res[-1][2], cc_ref)
