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


def _shard_worker(rank, world, port, cfg, q):
    try:
        sys.path.insert(0, ROOT)
        import torch
        import non_uniform_paged_flash_b200 as tg
        import synth
        from dataclasses import replace
        from non_uniform_paged_flash_b200 import workload
        from oracle import workload as ow

        _init(rank, world, port)
        sp = replace(synth.small(cfg), B=synth.small(cfg).B * world)
        kv, fast = workload.retained(sp, 0)
        per_seq = kv.astype(np.int64).sum(1) * 2 * sp.D * 2 if fast is None else \
            ((kv - fast) * 2 * (sp.D + 4) + fast * 2 * sp.D * 2).sum(1)
        gpu = tg.tg_place_sequences(per_seq, world)
        mine = np.nonzero(gpu == rank)[0]
        lay = workload.layout(sp, 0, mine)
        ow.assert_same_layout(lay, ow.layout(sp, 0, mine))
        shape = tg.make_shape(len(mine), sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages)
        plan = tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off,
                                 fast_len=lay.fast_len,
                                 slow_table_len=0 if lay.slow_table is None else lay.slow_table.size,
                                 host_only=True, num_workers=64)
        items = tg.tg_plan_items(plan)
        pages_local = int((items[:, 2] - items[:, 1]).sum())
        # gather: sequences and page counts of every rank
        t = torch.tensor([len(mine), pages_local, int(per_seq[mine].sum())], dtype=torch.int64)
        allt = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(allt, t)
        seqs = torch.from_numpy(np.pad(mine, (0, sp.B - len(mine)), constant_values=-1))
        alls = [torch.zeros_like(seqs) for _ in range(world)]
        dist.all_gather(alls, seqs)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, [x.tolist() for x in allt], [x.numpy() for x in alls], per_seq.tolist(),
               None))
    except Exception:
        q.put((rank, None, None, None, traceback.format_exc()))


@pytest.mark.parametrize("cfg", [2, 4, 5])
def test_two_rank_shards_cover_batch_once_and_balance(cfg):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, cfg, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, allt, alls, per_seq, err in res:
        assert err is None, err
    _, allt, alls, per_seq, _ = res[0]
    seqs = np.concatenate([a[a >= 0] for a in alls])
    assert sorted(seqs.tolist()) == list(range(len(per_seq)))           # each exactly once
    loads = [x[2] for x in allt]
    assert max(loads) <= sum(per_seq) / world + max(per_seq)            # LPT bound
    # pages of the shards add up to the pages of the whole batch
    import synth
    from dataclasses import replace
    from oracle import workload as ow
    sp = replace(synth.small(cfg), B=synth.small(cfg).B * world)
    kv, fast = ow.retained(sp, 0)
    if fast is None:
        want = int(((kv.astype(np.int64) + 15) // 16).sum())
    else:
        want = int((((kv - fast).astype(np.int64) + 15) // 16 + (fast.astype(np.int64) + 15) // 16).sum())
    assert sum(x[1] for x in allt) == want


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
