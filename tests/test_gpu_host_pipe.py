"""GPU: the host-buffer decode pipe. Several calls in flight with different queries give, per
call, exactly the device-buffer call's outputs (bit for bit), and the first call matches the
fp64 oracle; shape mismatches and unpinned host buffers are rejected.
"""
import numpy as np
import pytest
import torch

import non_uniform_paged_flash_b200 as tg
import synth
from non_uniform_paged_flash_b200 import workload
from tests import _oracle_side as ors

pytestmark = pytest.mark.gpu


def _queries(db, n, seed):
    g = torch.Generator().manual_seed(seed)
    qs = [db.q.cpu()] + [torch.randn(db.q.shape, generator=g).to(torch.bfloat16) for _ in range(n - 1)]
    return [q.pin_memory() for q in qs]


@pytest.mark.parametrize("cfg,kw", [(2, {}), (5, dict(min_splits=8, max_chunk_pages=16)),
                                    (4, dict(cascade=True))])
def test_pipelined_calls_equal_device_calls(cfg, kw):
    sp = synth.small(cfg)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, **kw)
    n = 5
    qs = _queries(db, n, 90 + cfg)
    outs = [torch.empty(db.out.shape, dtype=db.out.dtype).pin_memory() for _ in range(n)]
    lses = [torch.empty(db.lse.shape, dtype=db.lse.dtype).pin_memory() for _ in range(n)]
    pipe = tg.HostPipe(db.plan)
    for i in range(n):
        db.run_host(pipe, qs[i], outs[i], lses[i])
    pipe.wait()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    for i in range(n):   # the device-buffer call on the same query
        db.q.copy_(qs[i])
        db.run()
        torch.cuda.synchronize()
        assert torch.equal(outs[i], db.out.cpu()), i
        assert torch.equal(lses[i], db.lse.cpu()), i
    # the first query is the workload's own: against the oracle
    ol = ors.layout(sp, 0)
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    out = outs[0].float().numpy().reshape(-1, sp.D)
    lse = lses[0].numpy().reshape(-1)
    fin = np.isfinite(ref_lse)
    assert np.abs(out - ref_out).max() <= 2e-2
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= 1e-3
    pipe.destroy()


def test_pipe_bracketed_by_events_and_reused():
    """after / join put the pipe's copies inside a pair of events on the main stream; a pipe
    outlives many calls (set reuse every second call)."""
    sp = synth.small(2)
    db = workload.to_device(sp, workload.layout(sp, 0), 0)
    pipe = tg.HostPipe(db.plan)
    q = db.q.cpu().pin_memory()
    out = torch.empty(db.out.shape, dtype=db.out.dtype).pin_memory()
    lse = torch.empty(db.lse.shape, dtype=db.lse.dtype).pin_memory()
    db.run()
    torch.cuda.synchronize()
    ref_out, ref_lse = db.out.cpu(), db.lse.cpu()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    pipe.after()
    for _ in range(9):
        db.run_host(pipe, q, out, lse)
    pipe.join()
    e1.record()
    e1.synchronize()
    assert e0.elapsed_time(e1) > 0
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_pipe_rejects_mismatch_and_pageable():
    sp = synth.small(2)
    db = workload.to_device(sp, workload.layout(sp, 0), 0)
    other = workload.to_device(synth.small(1), workload.layout(synth.small(1), 0), 0)
    pipe = tg.HostPipe(db.plan)
    q = db.q.cpu().pin_memory()
    out = torch.empty(db.out.shape, dtype=db.out.dtype).pin_memory()
    lse = torch.empty(db.lse.shape, dtype=db.lse.dtype).pin_memory()
    with pytest.raises(tg.TGError) as ei:
        tg.tg_ragged_paged_decode_host(pipe, other.plan, q, other.k, other.v, other.table,
                                       other.head_off, other.kv_len, other.group_of_head,
                                       other.spec.scale, out, lse)
    assert ei.value.status == tg.TG_EINVAL
    B = db.lay.kv_len.shape[0]
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, db.lay.num_pages)
    p32 = tg.tg_plan_create(shape, db.lay.kv_len, db.lay.group_of_head, db.lay.group_off,
                            out_f32=True)
    with pytest.raises(tg.TGError) as e32:       # fp32 outputs do not fit the bf16 staging
        tg.tg_ragged_paged_decode_host(pipe, p32, q, db.k, db.v, db.table, db.head_off,
                                       db.kv_len, db.group_of_head, sp.scale, out, lse)
    assert e32.value.status == tg.TG_EINVAL
    with pytest.raises(tg.TGError):
        tg.HostPipe(p32)
    with pytest.raises(ValueError):
        db.run_host(pipe, db.q.cpu(), out, lse)   # pageable q
    with pytest.raises(ValueError):
        db.run_host(pipe, db.q, out, lse)         # device tensor where a host one belongs
    db.run_host(pipe, q, out, lse)
    pipe.wait()
    db.run()
    torch.cuda.synchronize()
    assert torch.equal(out, db.out.cpu())
