"""Parity of the whole layer on the five synthetic workloads, in the launch
configuration the benchmark times: every row's selection checked for its
invariants and compared bit for bit with the oracle's on every row (prefill
chunks: the oracle's per-row scoring and top-512 spread over the host's cores),
and the attention output compared with the oracle's on every row (decode) or on
a stratified sample of rows (prefill chunks)."""

import numpy as np
import pytest
import torch

from oracle import oracle as O
from qsa_synth import workloads as W

import gpu_util as gu
import oracle_parallel as OP

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gu.ensure_built()
    O.lib()


def sample_rows(n, k=24, seed=0):
    """First, last, tile edges and random rows of an n-row chunk."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, 2, 3, 127, 128, 129, n // 2, n - 129, n - 128, n - 4, n - 3, n - 2, n - 1}
    rest = rng.choice(n, size=k, replace=False)
    return sorted(r for r in fixed | set(rest.tolist()) if 0 <= r < n)


@pytest.mark.parametrize("cid", [0, 1, 2, 3, 4])
def test_workload_parity(cid, request):
    from qsa_synth import device as sdev
    wl = W.by_id(cid)
    dw = sdev.DeviceWorkload(wl)
    wo = O.WorkloadOracle(wl)
    gu.pool_history(dw, 0)
    for step in range(len(wl.steps)):
        out, sel_idx, sel_cnt, flags = gu.run_forward(dw, step)
        assert flags == 0
        gu.check_selection_properties(wl, step, sel_idx, sel_cnt)
        n = len(wl.steps[step].q_pos)
        rows = list(range(n)) if wl.mode == "decode" else sample_rows(n, seed=cid)
        sel = sel_idx.cpu().numpy()
        cnt = sel_cnt.cpu().numpy()
        if wl.mode == "prefill":
            # selection of every row of the chunk against the oracle, rows shared out over the cores
            want_all, secs, procs = OP.oracle_selections(wl, step)
            assert len(want_all) == n
            for r in range(n):
                np.testing.assert_array_equal(sel[r, : cnt[r]], want_all[r], err_msg=f"{wl.name} step {step} row {r}")
            request.config._qsa_notes.append(
                f"{wl.name}: selection of all {n} rows bit-exact vs the oracle "
                f"({secs:.1f} s wall on {procs} host cores)")
        got = gu.bf16_to_f64(out[rows])
        want = np.zeros_like(got)
        for j, r in enumerate(rows):
            s_want, o_want = wo.query(step, r)
            np.testing.assert_array_equal(sel[r, : cnt[r]], s_want, err_msg=f"{wl.name} step {step} row {r}")
            want[j] = o_want
        gu.compare_outputs(got, want)
        del out, sel_idx, sel_cnt
    del dw
    torch.cuda.empty_cache()
