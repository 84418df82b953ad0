"""The workloads at full size on the GPU (the five of the method's benchmarks, workload 5's token split in the
no-padding layout, workload 3 with B in the NN orientation, workload 3's token counts as the K extents of a
K-grouped GEMM, and workload 3 with B in E2M1), in the launch configuration the bench times.

Outputs are checked against the oracle on sampled rows (every group's first and last valid row, the rows
on each side of every 128-row tile boundary of the sample's blocks, plus random rows), all N columns; the
rows the GEMM does not own are checked in full against the sentinel.
"""
import numpy as np
import pytest

import oracle
import synth
from _helpers import assert_close, bf16_to_f64, run_problem, untouched_rows_ok

pytestmark = pytest.mark.gpu


def sample_rows(p, n_random=192, seed=0):
    rng = np.random.default_rng(seed)
    valid = p.valid_rows()
    picks = set()
    if p.kind == "dense":
        picks.update([0, p.M - 1])
    else:
        groups = p.row_groups(valid)
        for g in np.unique(groups):
            rows = valid[groups == g]
            picks.update([int(rows[0]), int(rows[-1])])
    for r in valid[(valid % 128 == 0) | (valid % 128 == 127)][:64]:
        picks.add(int(r))
    picks.update(int(r) for r in rng.choice(valid, size=min(n_random, len(valid)), replace=False))
    return np.array(sorted(picks), np.int64)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5, 6, 7, 8, 9])
def test_full_config(cfg):
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_config(cfg)
    out = run_problem(p)
    dg.check_device_error()
    flat = out.reshape(-1, p.N)
    valid = np.zeros(p.rows, bool)
    valid[p.valid_rows()] = True
    assert untouched_rows_ok(out, valid)
    rows = sample_rows(p) if cfg != 1 else p.valid_rows()
    ref = oracle.problem_rows(p, rows)
    got = bf16_to_f64(flat[rows.tolist()])
    assert_close(got, ref, p.name)
