"""Data-parallel host logic on CPU: two gloo ranks, each holding a shard of the tokens, reduce their
adapter gradients (computed by the oracle) with the package's bucket; the result must equal the
oracle's full-batch gradient.  No GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import layer as OL
from oracle import quantize as Q
from quantized_base_lora_nf4_b200.dp import GradBucket, OverlappedBuckets, allreduce_adapter_grads, shard_rows
from synth import LinearSpec, linear_tensors


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_rows_cover_every_token_once():
    for total in (0, 1, 7, 12, 2048, 2049):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(total, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def test_bucket_rejects_mixed_dtypes():
    with pytest.raises(ValueError):
        GradBucket([torch.zeros(3), torch.zeros(3, dtype=torch.float64)])


def _spec(pooled: bool) -> LinearSpec:
    if pooled:
        return LinearSpec("w", 48, 128, "int4g", group=32, r=8, s=1.0, pooled=True)
    return LinearSpec("w", 48, 128, "nfk", 4, 64, 256, r=8, s=0.5)


def _dequant(spec, W):
    if spec.fmt == "int4g":
        return Q.dequant_int4_group(Q.quantize_int4_group(W, spec.group))
    return Q.dequant_nfk(Q.quantize_nfk(W, spec.bits, spec.block, spec.dq_block))


def _rank_main(rank: int, world: int, port: int, pooled: bool, M: int, q) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        spec = _spec(pooled)
        t = linear_tensors(spec, M, seed=5)
        Wdq = _dequant(spec, t["W"])
        L = spec.group if spec.pooled else None
        a, b = shard_rows(M, rank, world)
        g = OL.backward(t["dY"][a:b], t["X"][a:b], Wdq, t["A"], t["B"], spec.s, L)
        dA = torch.from_numpy(np.ascontiguousarray(g["dA"], dtype=np.float64))
        dB = torch.from_numpy(np.ascontiguousarray(g["dB"], dtype=np.float64))
        allreduce_adapter_grads([dA, dB])
        full = OL.backward(t["dY"], t["X"], Wdq, t["A"], t["B"], spec.s, L)
        ok = bool(np.allclose(dA.numpy(), full["dA"], rtol=1e-12, atol=1e-14)
                  and np.allclose(dB.numpy(), full["dB"], rtol=1e-12, atol=1e-14))
        q.put((rank, ok, None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, False, repr(e)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.parametrize("pooled", [False, True])
def test_two_rank_gradient_allreduce_matches_full_batch(pooled):
    world, M = 2, 13  # an odd token count: shards of 7 and 6
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, pooled, M, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert all(ok for _, ok, _ in results), results


def test_overlapped_buckets_follow_layer_order_and_cap():
    grads = [[torch.zeros(100), torch.zeros(28)], [torch.zeros(64)], [torch.zeros(200)], [torch.zeros(8)]]
    ob = OverlappedBuckets(grads, cap_bytes=4 * 150)  # 150 floats
    # layer 0 (128 floats) stays under the cap, layer 1 brings it to 192: first bucket after layer 1;
    # layer 2 alone exceeds it; layer 3 is the last layer and closes the final bucket
    assert ob.start_after == {1: 0, 2: 1, 3: 2}
    assert [len(b.grads) for b in ob.buckets] == [3, 1, 1]
    ob.layer_done(0)
    ob.layer_done(1)  # no process group: nothing to exchange, nothing pending to wait on
    ob.finish()


def _overlap_rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        g = torch.Generator().manual_seed(17)
        shapes = [[(16, 64), (96, 16)], [(16, 32)], [(8, 128), (40, 8)], [(4, 4)], [(16, 256), (64, 16)]]
        base = [[torch.randn(s, generator=g, dtype=torch.float64) for s in layer] for layer in shapes]
        mine = [[(rank + 1) * t for t in layer] for layer in base]
        ob = OverlappedBuckets(mine, cap_bytes=8 * 2000)
        for i in range(len(mine)):  # the backward: a layer's gradients are final when it is done
            ob.layer_done(i)
        ob.finish()
        total = sum(r + 1 for r in range(world))
        ok = all(torch.equal(t, total * b) for lm, lb in zip(mine, base) for t, b in zip(lm, lb))
        q.put((rank, ok and len(ob.buckets) > 1, None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, False, repr(e)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_overlapped_buckets_sum_every_gradient():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_overlap_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert all(ok for _, ok, _ in results), results
