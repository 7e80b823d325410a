"""Ring attention with real process groups on the GPU: each rank is a process of its own, the shards move
through ``ring_attention_forward`` / ``ring_attention_backward`` themselves (their send/recv sequencing
and buffer reuse), and every block runs the library's kernels.

Every run here has one GPU, so the ranks share it and the transport is gloo (host-staged copies, the
path ``ring._exchange`` takes for a backend that moves host memory); under NCCL the same functions hand
device tensors to the library.  No kernel waits on another rank's kernel: a rank's kernels only read
what its own stream copied in after the exchange completed.  Each rank checks its shard of O, LSE and
the gradients against the fp64 oracle of the whole sequence.
"""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, causal, layout, d, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        import workloads
        from _gpu import GRAD_TOL, LSE_TOL, O_TOL, f64, max_abs, rel_l2
        from exact_io_aware_90_b200.ring import ring_attention_backward, ring_attention_forward, zigzag_shard
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        C = 96  # chunk: a contiguous shard is 2 chunks, a zigzag shard chunks r and 2W − 1 − r
        L = 2 * world * C
        inp = workloads.random_inputs(2, d, "bf16", seed=880 + world + d + 2 * int(causal) + 4 * (layout == "zigzag"),
                                      B=1, N=L, causal=causal)
        if layout == "zigzag":
            shard = lambda x: zigzag_shard(x, rank, world)
        else:
            shard = lambda x: x[rank * 2 * C:(rank + 1) * 2 * C]
        q, k, v, do = (shard(t).contiguous().to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
        k0, v0 = k.clone(), v.clone()
        o, lse = ring_attention_forward(q, k, v, causal=causal, scale=inp.scale, layout=layout)
        dq, dk, dv = ring_attention_backward(q, k, v, o, lse, do, causal=causal, scale=inp.scale, layout=layout)
        torch.cuda.synchronize()
        O_ref, L_ref = oracle.attention_forward(inp.q, inp.k, inp.v, inp.scale, causal)
        G_ref = oracle.attention_backward(inp.q, inp.k, inp.v, inp.do, inp.scale, causal)
        sh = lambda a: shard(torch.from_numpy(np.ascontiguousarray(a))).numpy()
        res = {"o": max_abs(f64(o), sh(O_ref)) <= O_TOL, "lse": max_abs(f64(lse), sh(L_ref)) <= LSE_TOL,
               "untouched": bool(torch.equal(k, k0) and torch.equal(v, v0))}
        for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), G_ref):
            res[name] = rel_l2(f64(g), sh(r)) <= GRAD_TOL
        dist.barrier()
        out_q.put((rank, res))
    except Exception as exc:  # reported to the parent, which fails the test
        out_q.put((rank, {"error": f"{type(exc).__name__}: {exc}"}))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_processes_on_one_gpu(layout, causal):
    d = 128
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, causal, layout, d, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, p.exitcode
    for rank, res in got:
        assert "error" not in res, (rank, res)
        assert all(res.values()), (rank, res)
