"""World-size-2 data-parallel host logic on CPU (gloo): token sharding, the adapter-gradient
all-reduce and max-over-ranks timing.  The per-rank gradients come from the oracle, so the
check is that the sharded-and-reduced gradients equal the full-batch ones."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import oracle as O
    from qlora_parameter_efficient_b200 import dp
    from qlora_parameter_efficient_b200 import synthetic as S

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = S.make_layer(48, 64, 4, 8.0, 37, dtype="f32", seed=3)
        b, e = dp.token_shard(case.T, world, rank)
        dA, dB = O.lora_adapter_grads(case.X[b:e], case.dH[b:e], case.A, case.B, 8.0, 4)
        tA, tB = torch.from_numpy(dA.copy()), torch.from_numpy(dB.copy())
        dp.allreduce_adapter_grads(tA, tB)
        slow = dp.max_over_ranks(1.0 + rank)
        out[rank] = (tA.numpy(), tB.numpy(), slow, (b, e))
    finally:
        dist.destroy_process_group()


def test_token_shard_covers_all_tokens():
    from qlora_parameter_efficient_b200 import dp
    for T in (1, 7, 4096):
        for world in (1, 2, 3, 8):
            spans = [dp.token_shard(T, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1


def test_world2_allreduce_equals_full_batch():
    import oracle as O
    from qlora_parameter_efficient_b200 import synthetic as S

    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    case = S.make_layer(48, 64, 4, 8.0, 37, dtype="f32", seed=3)
    dA, dB = O.lora_adapter_grads(case.X, case.dH, case.A, case.B, 8.0, 4)
    for rank in range(2):
        gA, gB, slow, span = out[rank]
        assert np.allclose(gA, dA, rtol=1e-12, atol=1e-12)
        assert np.allclose(gB, dB, rtol=1e-12, atol=1e-12)
        assert slow == 2.0
    assert out[0][3] == (0, 19) and out[1][3] == (19, 37)


def _overlap_worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    from qlora_parameter_efficient_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        order = []
        grads = torch.zeros(6, dtype=torch.float64)
        dX = torch.zeros(3, dtype=torch.float64)

        def grads_fn():
            order.append("grads")
            grads.copy_(torch.arange(6, dtype=torch.float64) + 10 * rank)

        def dx_fn():
            order.append("dx")
            dX.fill_(rank + 1)

        dp.backward_overlapped(grads_fn, dx_fn, grads)
        out[rank] = (grads.numpy().copy(), dX.numpy().copy(), order)
    finally:
        dist.destroy_process_group()


def test_world2_overlapped_backward_sums_grads_and_keeps_dx_local():
    # dA and dB (one flat tensor) are summed over ranks; dX stays per rank; the gradient phase
    # is enqueued before the dX phase, which runs while the reduction is in flight
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_overlap_worker, args=(2, port, out), nprocs=2, join=True)
    want = 2 * np.arange(6, dtype=np.float64) + 10
    for rank in range(2):
        g, dx, order = out[rank]
        assert np.array_equal(g, want)
        assert np.array_equal(dx, np.full(3, rank + 1.0))
        assert list(order) == ["grads", "dx"]
