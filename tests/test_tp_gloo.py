"""Row-sharded (tensor-parallel) host logic on CPU: aligned row shards, the NF4 quantization of a
shard equal to the same rows of the unsharded quantization, and world-size-2 gloo exchanges
(H column gather; dX, dA all-reduce; dB local) reproducing the unsharded layer.  The per-rank
layer arithmetic comes from the oracle."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import oracle as O


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_row_shards_are_aligned_and_cover_d_out():
    from qlora_parameter_efficient_b200 import tp
    for d_in in (64, 128, 192, 4096, 8192, 11008):
        a = tp.row_align(d_in)
        assert a % 16 == 0 and (a * d_in // 64) % 256 == 0
        for d_out in (16, 200, 4096, 11008, 28672):
            for world in (1, 2, 3, 8):
                spans = [tp.row_shard(d_out, d_in, world, r) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == d_out
                assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
                assert all(b % a == 0 or b == d_out for b, _ in spans)


def test_shard_quantization_equals_rows_of_full_quantization():
    from qlora_parameter_efficient_b200 import tp
    rng = np.random.default_rng(4)
    d_in = 192                                 # 3 blocks per row
    a = tp.row_align(d_in)
    assert a == 256                            # 256 rows x 3 blocks = 3 whole groups
    d_out = 2 * a + 48                         # a ragged last shard
    W = (rng.standard_normal((d_out, d_in)) * 0.141).astype(np.float32)
    codes, q8, c2, _ = O.nf4_quantize(W)
    for world in (2, 3):
        for r in range(world):
            b, e = tp.row_shard(d_out, d_in, world, r)
            if b == e:
                continue
            sc, sq, s2, _ = O.nf4_quantize(W[b:e])
            bpr = d_in // 64
            assert np.array_equal(sc, codes[b:e])
            assert np.array_equal(sq, q8[b * bpr:e * bpr])
            g0 = b * bpr // 256
            assert np.array_equal(s2, c2[g0:g0 + len(s2)])


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    from qlora_parameter_efficient_b200 import synthetic as S
    from qlora_parameter_efficient_b200 import tp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = S.make_layer(40, 4096, 4, 8.0, 9, dtype="f32", seed=5)
        W = case.W0.astype(np.float64)
        b, e = tp.row_shard(case.d_out, case.d_in, world, rank)
        s = 8.0 / 4
        Wp, Bp, dHp = W[b:e], case.B[b:e].astype(np.float64), case.dH[:, b:e].astype(np.float64)
        X, A = case.X.astype(np.float64), case.A.astype(np.float64)
        Hp = O.lora_forward(Wp, X, A, Bp, 8.0, 4)                    # this rank's columns of H
        U = X @ A.T
        Gp = dHp @ Bp
        dXp = dHp @ Wp + s * (Gp @ A)                                 # partial sums over ranks
        dAp = s * (Gp.T @ X)
        dBp = s * (dHp.T @ U)                                         # local rows of dB
        H = tp.allgather_columns(torch.from_numpy(Hp), case.d_out, world)
        tdX, tdA = torch.from_numpy(dXp.copy()), torch.from_numpy(dAp.copy())
        tp.allreduce_partials(tdX, tdA)
        out[rank] = (H.numpy(), tdX.numpy(), tdA.numpy(), dBp, (b, e))
    finally:
        dist.destroy_process_group()


def test_world2_row_sharded_layer_equals_unsharded():
    from qlora_parameter_efficient_b200 import synthetic as S
    from qlora_parameter_efficient_b200 import tp

    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    case = S.make_layer(40, 4096, 4, 8.0, 9, dtype="f32", seed=5)
    W = case.W0.astype(np.float64)
    H = O.lora_forward(W, case.X, case.A, case.B, 8.0, 4)
    dX, dA, dB = O.lora_backward(W, case.X, case.dH, case.A, case.B, 8.0, 4)
    spans = [tp.row_shard(40, 4096, 2, r) for r in range(2)]      # 16-row alignment at d_in = 4096
    assert spans == [(0, 32), (32, 40)]
    for rank in range(2):
        gH, gdX, gdA, dBp, (b, e) = out[rank]
        assert (b, e) == spans[rank]
        assert np.allclose(gH, H, rtol=1e-12, atol=1e-12)
        assert np.allclose(gdX, dX, rtol=1e-12, atol=1e-12)
        assert np.allclose(gdA, dA, rtol=1e-12, atol=1e-12)
        assert np.allclose(dBp, dB[b:e], rtol=1e-12, atol=1e-12)
