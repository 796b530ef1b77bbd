"""The bench line's parity sample, on CPU: the CPU-baseline leg hands back its first chunk of
oracle rows, and `_parity_sample` compares a step's outputs with them row by row (here the
"step" outputs are the oracle's own rows rounded to the device dtypes, so the differences are
rounding only, and a planted error shows up)."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import bench
import synth


@pytest.mark.parametrize("cfg,bits", [(2, 8), (4, 8), (5, 8), (5, 4)])
def test_parity_sample_against_oracle_rows(monkeypatch, cfg, bits):
    def small(c):
        sp = synth.small(c)
        return replace(sp, slow_bits=bits) if sp.kind == "tiered" else sp

    monkeypatch.setattr(bench, "_preset", small)
    sp = small(cfg)
    first = []
    base = bench.cpu_baseline(cfg, budget_s=5.0, min_s=1e-9, sample=first)
    assert base["kind"] == "oracle" and base["value"] > 0
    assert len(first) == 1
    sel, (o_ref, l_ref) = first[0]
    assert len(sel) == o_ref.shape[0] == l_ref.shape[0] > 0
    rows = sp.B * sp.Hq
    out = torch.zeros(rows, sp.D, dtype=torch.float64)
    lse = torch.full((rows,), float("-inf"), dtype=torch.float64)
    out[torch.from_numpy(sel)] = torch.from_numpy(o_ref)
    lse[torch.from_numpy(sel)] = torch.from_numpy(l_ref)
    out_d = out.to(torch.bfloat16).float().numpy()      # the step's outputs in device dtypes
    lse_d = lse.to(torch.float32).numpy()
    rep = bench._parity_sample(first, out_d, lse_d)
    assert "error" not in rep, rep
    assert rep["rows"] == len(sel)
    assert rep["max_abs_out"] <= 2 ** -8 * max(1.0, float(np.abs(o_ref).max()))   # bf16 rounding
    assert rep["max_abs_lse"] <= 1e-5 * max(1.0, float(np.abs(l_ref[np.isfinite(l_ref)]).max()))
    # a planted error in one sampled row is reported as it is
    r0 = int(sel[len(sel) // 2])
    out_d[r0, 3] += 0.5
    assert bench._parity_sample(first, out_d, lse_d)["max_abs_out"] >= 0.4


def test_parity_sample_records_a_failure_instead_of_raising():
    rep = bench._parity_sample([], None, None)
    assert set(rep) == {"error"}
