"""Other micro-block sizes and selection budgets, through the C ABI against the oracle.

blog.cecily.jp/6295 (Raschka's explainer paragraph) contrasts QSA's 4-token blocks
with DSA's per-token selection; keieiax.jp glossary "Qwen Sparse Attention" gives
512 blocks as the published budget.  The library takes the block size (a power of
two up to 16; 1 is per-token selection) and the budget (1..512 blocks) at run
time; the oracle is written for any block size and budget.  Every step of the
layer (pooling, scoring, selection, attention) runs at the given sizes, in decode,
prefill, multi-token and paged calls.
"""

import numpy as np
import pytest
import torch

from oracle import oracle as O
from qsa_synth import workloads as W

import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gu.ensure_built()
    O.lib()


def _check_forward(wl, rows=None):
    """qsa_forward on every step; selection and output of the given rows (all by
    default) against the oracle."""
    from qsa_synth import device as sdev
    dw = sdev.DeviceWorkload(wl)
    wo = O.WorkloadOracle(wl)
    gu.pool_history(dw, 0)
    for step in range(len(wl.steps)):
        out, sel_idx, sel_cnt, flags = gu.run_forward(dw, step)
        assert flags == 0
        gu.check_selection_properties(wl, step, sel_idx, sel_cnt)
        n = len(wl.steps[step].q_pos)
        rr = list(range(n)) if rows is None else [r for r in rows if r < n]
        sel, cnt = sel_idx.cpu().numpy(), sel_cnt.cpu().numpy()
        got = gu.bf16_to_f64(out[rr])
        want = np.zeros_like(got)
        for j, r in enumerate(rr):
            s_want, o_want = wo.query(step, r)
            np.testing.assert_array_equal(sel[r, : cnt[r]], s_want, err_msg=f"{wl.name} step {step} row {r}")
            want[j] = o_want
        gu.compare_outputs(got, want)


# (block size, budget): per-token selection with the published 2,048-token budget capped at
# 512 tokens, 2-token blocks, coarse blocks with a small budget, a budget of one block
CASES = [(1, 512), (2, 300), (8, 128), (16, 64), (4, 1), (4, 200)]


@pytest.mark.parametrize("bs,k", CASES)
def test_decode_block_size_and_budget(bs, k):
    # ragged positions: below and above the budget, every offset within a block
    cap = 16384
    pos = [cap - 1, cap - 2, 9000 + bs // 2, 4 * 512 + 3, 700, 5, 0, 64 * bs - 1]
    n = len(pos)
    wl = W.Workload(f"dec_bs{bs}_k{k}", 120 + bs * 7 + k, "decode", n, 32, 4, cap,
                    [W.Step(list(pos), [p + 1 for p in pos], list(range(n)), pos, list(range(n)))],
                    block_size=bs, top_k=k)
    _check_forward(wl)


@pytest.mark.parametrize("bs,k", [(1, 512), (8, 128), (2, 300)])
def test_decode_long_rows_two_pass_select(bs, k):
    """Rows beyond 16,384 blocks take the two-pass select."""
    cap = 65536 * bs if bs <= 2 else 32768 * bs
    pos = [cap - 1, cap // 2 + 1]
    wl = W.Workload(f"dec_long_bs{bs}", 130 + bs, "decode", 2, 8, 1, cap,
                    [W.Step(list(pos), [p + 1 for p in pos], [0, 1], pos, [0, 1])], block_size=bs, top_k=k)
    _check_forward(wl)


@pytest.mark.parametrize("bs,k", [(1, 512), (16, 64), (2, 300)])
def test_prefill_block_size_and_budget(bs, k):
    cap = 8192 * max(bs, 2)
    t0 = cap - 300
    wl = W.Workload(f"pf_bs{bs}_k{k}", 140 + bs, "prefill", 1, 32, 4, cap, [W._prefill_step(t0, 260)],
                    block_size=bs, top_k=k)
    _check_forward(wl, rows=[0, 1, 2, 3, 4, 5, 126, 127, 128, 129, 200, 255, 256, 259])


def test_mtp_and_paged_with_two_token_blocks():
    """Draft groups sharing one selection, K/V in pages, at block size 2."""
    import test_gpu_mtp_paged as M
    k, bs = 2, 2
    t0s = [16380, 16381, 9001, 1501]
    q_seq, q_pos = [], []
    for s, t0 in enumerate(t0s):
        q_seq += [s] * k
        q_pos += [t0 + j for j in range(k)]
    n = len(q_pos)
    wl = W.Workload("mtp_bs2", 150, "decode", len(t0s), 32, 4, 16384 + 64,
                    [W.Step(list(t0s), [t0 + k for t0 in t0s], q_seq, q_pos, list(range(n)))], block_size=bs,
                    top_k=400)
    out, sel, cnt, flags = M._run_mtp(wl, k, page=M._paged(12, 32))
    assert flags == 0
    want_sel, want_out = M._oracle_mtp(wl, k)
    for g, ws_ in enumerate(want_sel):
        np.testing.assert_array_equal(sel[g, : cnt[g]], ws_, err_msg=f"group {g}")
    gu.compare_outputs(gu.bf16_to_f64(out), want_out)
