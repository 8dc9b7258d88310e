"""Column-parallel (N-split) sharding of the quantized linear.

CPU: the shard boundaries, and two gloo ranks that each compute their
columns of a layer (with the oracle standing in for the GPU kernel, passed
to the shard explicitly), all-gather them and must reassemble exactly the
oracle's unsharded output.  GPU: the shards of a layer computed one after
the other on one GPU through the library give the unsharded layer's bits
column for column (a column depends on its own weight row only).
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from int4_weight_quantized_block_b200.column_parallel import ColumnParallelLinear, shard_bounds


@pytest.mark.parametrize("N,world", [(9216, 1), (9216, 2), (9216, 8), (3072, 8), (272, 3),
                                     (16, 4), (48, 5), (12288, 7), (0, 2)])
def test_shard_bounds_cover_disjoint_aligned(N, world):
    b = shard_bounds(N, world)
    assert len(b) == world
    assert b[0][0] == 0 and b[-1][1] == N
    for (lo, hi), (lo2, _) in zip(b, b[1:]):
        assert hi == lo2                                   # contiguous, disjoint
    for lo, hi in b:
        assert lo <= hi and lo % 16 == 0 and (hi % 16 == 0 or hi == N)
    widths = [hi - lo for lo, hi in b]
    assert max(widths) - min(widths) <= 16 or N < 16 * world   # as equal as 16-row blocks allow


def test_shard_bounds_rejects_bad_arguments():
    with pytest.raises(ValueError):
        shard_bounds(-1, 2)
    with pytest.raises(ValueError):
        shard_bounds(16, 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_linear(x_bits, wp, sr, g, bias, y, workspace):
    """The oracle in the kernel's place (CPU test of the host logic): bf16
    output bits as an int16 tensor."""
    import oracle
    out = oracle.convrot_linear(x_bits.numpy().view(np.uint16), wp.numpy(), sr.numpy(), g, 8)
    return torch.from_numpy(out.view(np.int16))


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import oracle
    from int4_weight_quantized_block_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        M, N, K, g = 5, 272, 256, 64          # 17 row blocks over 2 ranks: 144 + 128
        x = inputs.activations(M, K, seed=70)
        W = inputs.weights(N, K, seed=71)
        wp, sr, _ = oracle.pack_weights(W, g)
        wps, srs, _ = ColumnParallelLinear.shard(torch.from_numpy(wp), torch.from_numpy(sr),
                                                 rank, world)
        layer = ColumnParallelLinear(wps, srs, g, N, rank, world, gather=True,
                                     linear=_oracle_linear)
        y = layer(torch.from_numpy(x.view(np.int16)))
        ref = oracle.convrot_linear(x, wp, sr, g, 8)
        q.put((rank, (layer.lo, layer.hi), np.array_equal(y.numpy().view(np.uint16), ref)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_unsharded_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [(0, 144), (144, 272)]
    assert all(o[2] for o in out)


@pytest.mark.gpu
@pytest.mark.parametrize("world,act_bits", [(2, 8), (8, 8), (3, 4)])
def test_shards_on_one_gpu_give_the_unsharded_bits(world, act_bits):
    import int4_weight_quantized_block_b200 as t4
    from int4_weight_quantized_block_b200 import inputs
    dev = torch.device("cuda", 0)
    M, N, K, g = 200, 1040, 768, 256
    x = torch.from_numpy(inputs.activations(M, K, seed=72).view(np.int16)).view(torch.bfloat16).to(dev)
    W = torch.from_numpy(inputs.weights(N, K, seed=73)).to(dev)
    wp, sr = t4.tint4_pack_weights(W, g)
    fn = t4.convrot_w4a8_linear if act_bits == 8 else t4.convrot_w4a4_linear
    y_full = fn(x, wp, sr, g)
    parts = []
    for r in range(world):
        wps, srs, _ = ColumnParallelLinear.shard(wp, sr, r, world)
        layer = ColumnParallelLinear(wps, srs, g, N, r, world, act_bits=act_bits)
        # each shard packed on its own from its rows of W gives the same bytes
        lo, hi = layer.lo, layer.hi
        if hi > lo:
            wp_r, sr_r = t4.tint4_pack_weights(W[lo:hi].contiguous(), g)
            assert torch.equal(wp_r, wps) and torch.equal(sr_r, srs)
        parts.append(layer(x))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1).view(torch.int16), y_full.view(torch.int16))
