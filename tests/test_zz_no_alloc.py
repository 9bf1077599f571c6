"""The allocation-free attention entry point (qsa_sparse_attn_noalloc).

It serves callers that cannot allocate device memory (an engine whose allocator
already gave all of HBM to its KV cache, a frozen CUDA-graph memory plan, a C host
that only owns the tensors it passes) and so cannot hand qsa_sparse_attn a
workspace.  It must give the same results as qsa_sparse_attn on the same inputs,
call after call, since every call reuses the library's one built-in scratch array.
This file is collected last and builds its own inputs, so it passes alone in a
fresh process as well as after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

import gpu_util as gu
from qsa_synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    gu.ensure_built()
    import block_sparse_attention_key_b200 as qsa
    from qsa_synth import device as sdev
    # 16 sequences with 32 query / 4 KV heads at ragged positions near 16K tokens:
    # split-K attention, so the scratch holds partials and completion counters
    cap = 16384
    pos = [cap - 1 - 7 * i for i in range(16)]
    wl = W.Workload("noalloc", 77, "decode", 16, 32, 4, cap,
                    [W.Step([cap] * 16, [cap] * 16, list(range(16)), pos, list(range(16)))])
    dw = sdev.DeviceWorkload(wl)
    T = dw.step_tensors(0)
    rng = np.random.default_rng(1)
    sel = np.full((16, 512), -1, dtype=np.int32)
    cnt = np.zeros(16, dtype=np.int32)
    for r, t in enumerate(pos):
        n_c = (t + 1) // 4
        sel[r] = np.sort(rng.choice(n_c, size=512, replace=False))
        cnt[r] = 512
    return qsa, wl, dw, T, torch.tensor(sel, device="cuda"), torch.tensor(cnt, device="cuda")


def test_noalloc_matches_workspace_entry_point_twice(setup):
    qsa, wl, dw, T, sel, cnt = setup
    dims = gu.dims_of(wl)
    n = T["n_q"]
    ws = gu.new_workspace(qsa.qsa_workspace_bytes(dims, n, 0, qsa.QSA_MODE_DECODE))
    want = torch.empty((n, wl.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    qsa.qsa_sparse_attn(dims, T["q"], dw.k_cache, dw.v_cache, T["q_seq"], T["q_pos"], sel, cnt, n, want, ws)
    ref = gu.bf16_to_f64(want)
    for _ in range(2):  # the second call starts from the first call's leftover scratch
        got = torch.full_like(want, float("nan"))
        qsa.qsa_sparse_attn_noalloc(dims, T["q"], dw.k_cache, dw.v_cache, T["q_seq"], T["q_pos"], sel, cnt, n,
                                    got)
        torch.cuda.synchronize()
        gu.compare_outputs(gu.bf16_to_f64(got), ref)


def test_noalloc_rejects_calls_beyond_its_scratch(setup):
    qsa, wl, dw, T, sel, cnt = setup
    lib = qsa.load()
    # 65,535 queries x 128 KV heads need 32 MiB of completion counters (4 bytes per
    # query and KV head): over the 16 MiB limit, refused on the host before any launch
    dims = qsa.make_dims(batch=1, n_q_heads=128, n_kv_heads=128, kv_capacity=wl.kv_capacity)
    fake = 1 << 40
    rc = lib.qsa_sparse_attn_noalloc(ctypes.byref(dims), *([fake] * 7), 65535, fake, None)
    assert rc == qsa.QSA_ERR_WORKSPACE_TOO_SMALL
    assert lib.qsa_sparse_attn_noalloc(ctypes.byref(dims), *([None] * 7), 16, None, None) == qsa.QSA_ERR_INVALID_ARG
