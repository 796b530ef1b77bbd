"""Multi-rank host logic on CPU (gloo, world size 2): ahead-of-time placement of sequences on
ranks, the per-rank shard layouts, and detection of a rank that dies (on the host, through a
short process-group timeout; no GPU involved)."""
import os
import socket
import sys
import traceback

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _init(rank, world, port, timeout_s=30):
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=timeout_s))


def _shard_worker(rank, world, port, cfg, slow_bits, q):
    """One rank of `bench.py --gpus N`'s set-up, on the bench's own functions and full-size
    workloads: the global spec, this rank's sequences by ahead-of-time placement, its layout
    (checked against the oracle's) and plan, and the max / sum reduction over ranks."""
    try:
        sys.path.insert(0, ROOT)
        import torch
        import bench
        import non_uniform_paged_flash_b200 as tg
        from non_uniform_paged_flash_b200 import workload
        from oracle import workload as ow

        _init(rank, world, port)
        bench.SLOW_BITS = slow_bits
        sp = bench._global_spec(cfg, world)
        # the multi-layer workload places each layer's sequences by that layer's bytes; the
        # rest of the check runs on its last layer here
        for layer in ((0, 17) if sp.layers > 1 else (0,)):
            kv, fast = workload.retained(sp, layer)
            mine = bench._my_sequences(sp, rank, world, kv, fast)
            lay = workload.layout(sp, layer, mine)
            ow.assert_same_layout(lay, ow.layout(sp, layer, mine))
        shape = tg.make_shape(len(mine), sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages)
        plan = tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off,
                                 fast_len=lay.fast_len,
                                 slow_table_len=0 if lay.slow_table is None else lay.slow_table.size,
                                 host_only=True, num_workers=64, slow_bits=slow_bits if fast is not None else 0)
        items = tg.tg_plan_items(plan)
        pages_local = int((items[:, 2] - items[:, 1]).sum())
        # the bench's reduction: times / flags as the max over ranks, work as the sum
        vals = torch.tensor([float(rank + 1), 10.0 * (rank + 1), float(len(mine)), float(pages_local)],
                            dtype=torch.float64)
        reduced = bench._over_ranks(dist, vals, 2)
        seqs = torch.from_numpy(np.pad(mine, (0, sp.B - len(mine)), constant_values=-1))
        alls = [torch.zeros_like(seqs) for _ in range(world)]
        dist.all_gather(alls, seqs)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, reduced, [x.numpy() for x in alls], sp.B, None))
    except Exception:
        q.put((rank, None, None, None, traceback.format_exc()))


def _seq_bytes(sp, kv, fast, slow_bits):
    """Retained K/V bytes per sequence, written out from the tier layouts (bf16 K + V: 4 D per
    token-head; a slow token-head: codes of K and V plus two fp32 scales)."""
    if fast is None:
        return kv.astype(np.int64).sum(1) * 4 * sp.D
    f = np.minimum(fast, kv).astype(np.int64)
    code = sp.D if slow_bits == 8 else sp.D // 2
    return ((kv - f) * (2 * code + 8) + f * 4 * sp.D).sum(1)


@pytest.mark.parametrize("cfg,slow_bits", [(2, 8), (3, 8), (4, 8), (5, 8), (5, 4)])
def test_two_rank_shards_cover_batch_once_and_balance(cfg, slow_bits):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, cfg, slow_bits, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, reduced, alls, B, err in res:
        assert err is None, err
    import synth
    from dataclasses import replace
    from oracle import workload as ow
    _, reduced, alls, B, _ = res[0]
    seqs = np.concatenate([a[a >= 0] for a in alls])
    assert sorted(seqs.tolist()) == list(range(B))                     # each exactly once
    sp = replace(synth.preset(cfg), B=B)
    if sp.kind == "tiered":
        sp = replace(sp, slow_bits=slow_bits)
    kv, fast = ow.retained(sp, 17 if sp.layers > 1 else 0)     # the worker's last layer
    per_seq = _seq_bytes(sp, kv, fast, slow_bits)
    loads = [int(per_seq[a[a >= 0]].sum()) for a in alls]
    assert max(loads) <= per_seq.sum() / world + per_seq.max()        # LPT bound
    # every rank sees the same reduction: max of the times, sums of the work
    if fast is None:
        want_pages = int(((kv.astype(np.int64) + 15) // 16).sum())
    else:
        f = np.minimum(fast, kv).astype(np.int64)
        want_pages = int((((kv - f) + 15) // 16 + (f + 15) // 16).sum())
    for _, r, _, _, _ in res:
        assert r == [float(world), 10.0 * world, float(B), float(want_pages)]


def _dying_worker(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        _init(rank, world, port, timeout_s=3)
        dist.barrier()                       # both ranks reach the first step
        if rank == 1:
            os._exit(3)                      # leaves between steps, nothing in flight
        try:
            dist.barrier()                   # the next step's collective
            q.put((rank, "no error"))
        except Exception as e:               # the survivor learns of it on the host
            q.put((rank, "detected: " + type(e).__name__))
    except Exception:
        q.put((rank, "setup failed: " + traceback.format_exc()))


def test_dead_rank_is_detected_by_the_survivor():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dying_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    rank, msg = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert rank == 0 and msg.startswith("detected"), msg
    assert procs[1].exitcode == 3
