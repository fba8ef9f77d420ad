"""The combine path of the tensor-parallel layer on the CPU: two gloo ranks, each
holding one half of the intermediate dimension, sum their partial outputs with the
all-reduce of TensorParallelMoE. The GPU layer is replaced by a stand-in that
returns the rank's partial output as the CPU oracle computes it for the rank's slice,
so the test checks the partition and the combine: the all-reduced result on every
rank must be the unsharded layer's output."""

import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _OracleShard:
    """Stand-in for MoELayer on a CPU rank: its forward is the oracle on the loaded slice."""

    def __init__(self, k, dtype):
        self.k, self.dtype = k, dtype

    def load_weights_shard(self, wg, wu, wd, shard, num_shards, stream=None):
        from oracle import moe_oracle as O
        self.w = O.shard_weights(wg.numpy(), wu.numpy(), wd.numpy(), shard, num_shards)

    def forward(self, x, logits, out=None, stream=None):
        from oracle import moe_oracle as O
        part = O.moe_forward(x.numpy(), logits.numpy(), self.k, *self.w)
        res = torch.from_numpy(part.astype(np.float32)).to(self.dtype)
        if out is not None:
            out.copy_(res)
            return out
        return res

    def close(self):
        pass


def _rank_main(rank, world, port, dtype, results):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mixture_experts_layer_sort_b200.parallel import TensorParallelMoE
        from tests.test_oracle_layer import rand_layer
        M, E, k, H, I = 6, 8, 2, 32, 256
        x, logits, wg, wu, wd = rand_layer(M, E, k, H, I, seed=5)
        tp = TensorParallelMoE(E, k, H, I, layer=_OracleShard(k, dtype))
        assert tp.rank == rank and tp.world == world
        tp.load_weights(torch.from_numpy(wg), torch.from_numpy(wu), torch.from_numpy(wd))
        out = tp.forward(torch.from_numpy(x), torch.from_numpy(logits))
        results[rank] = out.float().numpy().tolist()
        tp.close()
    finally:
        dist.destroy_process_group()


def _run(dtype):
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_rank_main, args=(2, _free_port(), dtype, results), nprocs=2, join=True)
    return np.array(results[0]), np.array(results[1])


def test_two_ranks_sum_to_the_unsharded_layer():
    sys.path.insert(0, ROOT)
    from oracle import moe_oracle as O
    from tests.test_oracle_layer import rand_layer
    r0, r1 = _run(torch.float32)
    assert np.array_equal(r0, r1)                     # every rank holds the combined output
    x, logits, wg, wu, wd = rand_layer(6, 8, 2, 32, 256, seed=5)
    full = O.moe_forward(x, logits, 2, wg, wu, wd)
    np.testing.assert_allclose(r0, full, rtol=1e-5, atol=1e-5)


def test_shard_sizes_must_be_multiples_of_128():
    sys.path.insert(0, ROOT)
    import pytest
    from mixture_experts_layer_sort_b200.parallel import TensorParallelMoE
    with pytest.raises(ValueError):
        TensorParallelMoE(8, 2, 256, 768, rank=0, world=8, layer=object())   # 96 per rank
    tp = TensorParallelMoE(8, 2, 256, 1024, rank=3, world=8, layer=object())
    assert tp.I_full == 1024 and tp.rank == 3


def test_all_reduce_runs_on_the_forward_stream(monkeypatch):
    """With an explicit stream the all-reduce is issued inside that stream's context, so
    it is ordered after the forward that wrote `out` (the CUDA stream objects are
    replaced by recorders: no GPU is needed)."""
    sys.path.insert(0, ROOT)
    import contextlib
    import torch
    from mixture_experts_layer_sort_b200 import parallel
    events = []

    class FakeStream:
        def __init__(self, handle):
            self.handle = handle

    @contextlib.contextmanager
    def fake_stream_ctx(s):
        events.append(("enter", s.handle))
        yield
        events.append(("exit", s.handle))

    class Layer:
        def forward(self, x, logits, out=None, stream=None):
            events.append(("forward", stream))
            return out

    monkeypatch.setattr(torch.cuda, "ExternalStream", FakeStream)
    monkeypatch.setattr(torch.cuda, "stream", fake_stream_ctx)
    monkeypatch.setattr(parallel.dist, "all_reduce", lambda t, op=None, group=None: events.append(("all_reduce",)))
    tp = parallel.TensorParallelMoE(8, 2, 256, 1024, rank=0, world=2, layer=Layer())
    out = torch.zeros(2, 4)
    tp.forward(None, None, out=out, stream=0x1234)
    assert events == [("forward", 0x1234), ("enter", 0x1234), ("all_reduce",), ("exit", 0x1234)]
    events.clear()
    tp.forward(None, None, out=out)                   # no stream: the current one, no context switch
    assert events == [("forward", None), ("all_reduce",)]
