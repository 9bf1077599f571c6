"""CPU-side checks of the C ABI: the library loads, exports what include/qsa.h
declares, and rejects bad arguments on the host before launching anything."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def qsa():
    from block_sparse_attention_key_b200 import build, qsa
    build.build()
    qsa.load()
    return qsa


def declared_functions():
    text = open(os.path.join(ROOT, "include", "qsa.h")).read()
    return sorted(set(re.findall(r"^(?:int|size_t|const char\*)\s+(qsa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_five_layer_calls():
    names = declared_functions()
    for n in ["qsa_pool_block_keys", "qsa_index_scores", "qsa_topk_blocks", "qsa_sparse_attn", "qsa_forward"]:
        assert n in names


def test_library_exports_every_declared_symbol(qsa):
    lib = qsa.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(qsa.EXPORTED) <= set(declared_functions())


def test_binding_names_match_abi(qsa):
    import block_sparse_attention_key_b200 as pkg
    for name in declared_functions():
        if name != "qsa_status_string":
            assert callable(getattr(pkg, name)), name


def test_status_strings(qsa):
    assert qsa.status_string(0) == "QSA_OK"
    assert qsa.status_string(-1) == "QSA_ERR_INVALID_ARG"
    assert qsa.status_string(-2) == "QSA_ERR_WORKSPACE_TOO_SMALL"
    assert qsa.status_string(-3) == "QSA_ERR_UNSUPPORTED"
    assert qsa.status_string(-4) == "QSA_ERR_CUDA"
    assert qsa.status_string(-99) == "QSA_ERR_UNKNOWN"


def _dims(qsa, **kw):
    base = dict(batch=16, n_q_heads=32, n_kv_heads=4, kv_capacity=65536)
    base.update(kw)
    return qsa.make_dims(**base)


def test_workspace_bytes_rejects_bad_dims(qsa):
    ok = qsa.qsa_workspace_bytes(_dims(qsa), 16, 16384, qsa.QSA_MODE_DECODE)
    assert ok > 0
    bad = [dict(block_size=3), dict(block_size=0), dict(block_size=32), dict(top_k=0), dict(top_k=513),
           dict(head_dim=64), dict(idx_dim=32), dict(n_idx_heads=2), dict(n_q_heads=30), dict(kv_capacity=65537),
           dict(batch=0), dict(batch=65536), dict(n_q_heads=128, n_kv_heads=2),
           dict(block_size=16, kv_capacity=65544)]
    for kw in bad:
        assert qsa.qsa_workspace_bytes(_dims(qsa, **kw), 16, 16384, 0) == 0, kw
    # other micro-block sizes and budgets: per-token selection (block 1), coarser blocks, smaller k
    for kw in [dict(block_size=1), dict(block_size=2), dict(block_size=8), dict(block_size=16), dict(top_k=1),
               dict(top_k=256), dict(block_size=1, top_k=512)]:
        assert qsa.qsa_workspace_bytes(_dims(qsa, **kw), 16, 4096, 0) > 0, kw
    assert qsa.qsa_workspace_bytes(_dims(qsa), 16, 16385 + 65536 // 4, 0) == 0   # max_blocks > capacity/4
    assert qsa.qsa_workspace_bytes(_dims(qsa), -1, 16384, 0) == 0
    assert qsa.qsa_workspace_bytes(_dims(qsa), 16, 16384, 7) == 0


def test_workspace_has_no_query_by_block_term_in_prefill(qsa):
    """Prefill workspace must not grow like n_q x n_blocks (no mask, no score matrix):
    per query it holds a fixed-capacity candidate list; only a fixed number of
    fallback score rows grows with the context."""
    d = _dims(qsa, batch=1, kv_capacity=1 << 20)
    nb = (1 << 20) // 4
    w_full = qsa.qsa_workspace_bytes(d, 8192, nb, qsa.QSA_MODE_PREFILL)
    w_half = qsa.qsa_workspace_bytes(d, 8192, nb // 2, qsa.QSA_MODE_PREFILL)
    assert 0 < w_half <= w_full
    assert w_full < 8192 * nb * 4 // 4          # well below the f32 score matrix (8 GiB)
    assert w_full - w_half <= 64 * (nb // 2) * 4 + (1 << 20)  # 64 fallback rows, not n_q rows


def test_decode_workspace_is_small(qsa):
    d = _dims(qsa, batch=4, kv_capacity=1 << 20)
    w = qsa.qsa_workspace_bytes(d, 4, (1 << 20) // 4, qsa.QSA_MODE_DECODE)
    assert 0 < w < 64 << 20


def _no_device():
    """Tests that hand the library fabricated addresses run only where no CUDA
    device is visible, so a regression in the host-side checks can never launch a
    kernel on them."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("uses fabricated addresses: host-only test")


def _call(fn, *args):
    return fn(*args)


def test_entry_points_reject_null_and_misaligned_pointers_on_host(qsa):
    _no_device()
    lib = qsa.load()
    d = ctypes.byref(_dims(qsa))
    P = None
    # every call below fails validation before touching CUDA
    assert lib.qsa_pool_block_keys(d, P, P, P, P, 4, P, P) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_pool_block_keys(d, 17, 32, 32, 32, 4, P, P) == qsa.QSA_ERR_INVALID_ARG  # misaligned
    assert lib.qsa_index_scores(d, P, P, P, P, P, 16, 16384, P, 16384, P, P) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_index_scores(d, 16, 16, 16, 16, 16, 16, 16384, 16, 100, P, P) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_topk_blocks(d, P, 16384, P, 16, 16384, P, P, P, 0, P) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_sparse_attn(d, P, P, P, P, P, P, P, 16, P, P, 0, P) == qsa.QSA_ERR_INVALID_ARG
    args = qsa.qsa_forward_args()
    args.n_q = 16
    args.max_blocks = 16384
    assert lib.qsa_forward(d, ctypes.byref(args), P, 0, P) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_forward(d, None, 16, 1 << 20, P) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_workspace_init(P, 0, P) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_read_device_status(P, None, P) == qsa.QSA_ERR_INVALID_ARG


def test_workspace_too_small_is_reported_before_launch(qsa):
    _no_device()
    lib = qsa.load()
    dims = _dims(qsa)
    d = ctypes.byref(dims)
    need = qsa.qsa_workspace_bytes(dims, 16, 16384, 0)
    fake = 1 << 40  # 16-byte aligned, never dereferenced: the size check fails first
    rc = lib.qsa_topk_blocks(d, fake, 16384, fake, 16, 16384, fake, fake, fake, need - 1, None)
    assert rc == qsa.QSA_ERR_WORKSPACE_TOO_SMALL
    args = qsa.qsa_forward_args(*([fake] * 11), 16, 1, 16384, 0, None, None, fake)
    assert lib.qsa_forward(d, ctypes.byref(args), fake, need - 1, None) == qsa.QSA_ERR_WORKSPACE_TOO_SMALL


def test_unsupported_group_size(qsa):
    _no_device()
    lib = qsa.load()
    d = ctypes.byref(_dims(qsa, n_q_heads=128, n_kv_heads=2))
    assert lib.qsa_sparse_attn(d, *([16] * 7), 1, 16, 16, 1 << 20, None) == qsa.QSA_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors(qsa):
    import torch
    with pytest.raises(ValueError):
        qsa._ptr(torch.zeros(4))


def test_binding_constants_match_the_header(qsa):
    """Every QSA_* value the header defines has the same value in the binding."""
    text = open(os.path.join(ROOT, "include", "qsa.h")).read()
    defs = dict(re.findall(r"^#define\s+(QSA_(?:OK|ERR_\w+|DEV_\w+|MODE_\w+))\s+(-?(?:0x)?[0-9A-Fa-f]+)u?\b", text, re.M))
    assert len(defs) == 16  # 5 return codes, 8 device status bits, 3 modes
    for name, val in defs.items():
        assert getattr(qsa, name) == int(val, 0), name
    cap = re.search(r"^#define\s+QSA_SEL_CAP\s+(\d+)", text, re.M)
    assert cap and int(cap.group(1)) == qsa.QSA_SEL_CAP


def test_workspace_grows_with_queries_and_blocks(qsa):
    """Workspace is monotone in the query count and the block bound, in both modes."""
    d = _dims(qsa, batch=4, kv_capacity=1 << 20)
    for mode in (qsa.QSA_MODE_DECODE, qsa.QSA_MODE_PREFILL):
        prev = 0
        for n_q in (1, 16, 256, 4096):
            w = qsa.qsa_workspace_bytes(d, n_q, 1 << 16, mode)
            assert w >= prev > 0 or prev == 0
            prev = w
        assert qsa.qsa_workspace_bytes(d, 256, 1 << 12, mode) <= qsa.qsa_workspace_bytes(d, 256, 1 << 16, mode)


def test_attention_plans_fit_the_hardware(qsa):
    """Every attention launch shape (host arithmetic of qsa_attn_plan, no device work):
    shared memory within the 227 KB a CTA may use (plus its 1 KB of static alignment),
    two CTAs per SM for the one-CTA-per-pair plan, split partials within the 148
    slots the workspace holds and split pairs within its 148 arrival counters, at
    most 6 stages, at most 32 rows per CTA."""
    import itertools
    max_block = 227 * 1024
    per_sm = 228 * 1024
    for (hq, hkv), gq, bs, n_groups in itertools.product(
            [(8, 1), (32, 4), (16, 16), (16, 1), (32, 1), (32, 2), (4, 2), (64, 8)], [1, 2, 3, 4, 8],
            [1, 2, 4, 8, 16], [1, 2, 3, 5, 16, 37, 64, 147, 148, 300, 4096]):
        G = hq // hkv
        d = qsa.make_dims(4, hq, hkv, 65536, block_size=bs)
        n_q = n_groups * gq
        if G * gq > 32:
            with pytest.raises(qsa.QsaError):
                qsa.qsa_attn_plan(d, n_q, gq)
            continue
        p = qsa.qsa_attn_plan(d, n_q, gq)
        pairs = n_groups * hkv
        assert p["rows"] == G * gq
        assert p["threads"] == (256 if p["rows"] <= 16 else 128)
        assert 1 <= p["n_stages"] <= 6
        assert p["smem_bytes"] + 1024 <= max_block, p
        assert p["ctas"] == pairs * p["n_split"]
        if p["n_split"] > 1:
            assert p["ctas"] <= 148, p
            # arrivals are counted per pair in a fixed region of 148 words
            assert pairs < 148, p
        elif pairs >= 148:
            assert 2 * (p["smem_bytes"] + 2048) <= per_sm, p
    empty = qsa.qsa_attn_plan(qsa.make_dims(4, 32, 4, 65536), 0)
    assert empty["ctas"] == 0


def _header_rules(d, n_q, group_q):
    """The argument rules include/qsa.h states, restated: None when qsa_attn_plan must
    accept (d, n_q, group_q), else the error class it must return."""
    import math
    invalid = (d["batch"] < 1 or d["n_q_heads"] < 1 or d["n_kv_heads"] < 1
               or d["n_q_heads"] % d["n_kv_heads"] != 0
               or d["block_size"] not in (1, 2, 4, 8, 16) or not 1 <= d["top_k"] <= 512
               or d["kv_capacity"] <= 0 or d["kv_capacity"] % d["block_size"] != 0 or d["kv_capacity"] >= 2 ** 31
               or not math.isfinite(d["softmax_scale"]))
    if invalid:
        return "invalid"
    G = d["n_q_heads"] // d["n_kv_heads"]
    if d["head_dim"] != 128 or d["n_idx_heads"] != 4 or d["idx_dim"] != 64 or G > 32 or d["batch"] > 65535:
        return "unsupported"
    if n_q < 0:
        return "invalid"
    if n_q > 65535:
        return "unsupported"
    if group_q < 1 or n_q % group_q != 0:
        return "invalid"
    if group_q * G > 32:
        return "unsupported"
    return None


def test_host_checks_follow_the_header_rules(qsa):
    """Random dims, query counts and draft-group sizes: qsa_attn_plan (host arithmetic
    only) and qsa_workspace_bytes accept exactly what the header's rules allow and
    return the error class they name.  Each example starts from valid dims and breaks
    up to two fields."""
    from hypothesis import given, settings, strategies as st
    lib = qsa.load()
    good = dict(batch=[1, 3, 16, 65535], heads=[(8, 1), (32, 4), (16, 16), (32, 1), (64, 2), (12, 4), (64, 8)],
                head_dim=[128], n_idx_heads=[4], idx_dim=[64], block_size=[1, 2, 4, 8, 16], top_k=[1, 200, 512],
                kv_capacity=[4096, 65536, 2 ** 31 - 16], softmax_scale=[0.0, 0.1])
    bad = dict(batch=[0, -1, 65536], heads=[(30, 4), (0, 1), (4, 0), (128, 2), (66, 2)], head_dim=[64],
               n_idx_heads=[2], idx_dim=[32], block_size=[0, 3, 32], top_k=[0, -1, 513],
               kv_capacity=[0, 65540, 2 ** 31], softmax_scale=[float("inf"), float("nan")])
    base_st = st.fixed_dictionaries({k: st.sampled_from(v) for k, v in good.items()})
    breaks_st = st.lists(st.sampled_from([(k, v) for k, vs in bad.items() for v in vs]), max_size=2)

    @settings(max_examples=600, deadline=None, derandomize=True)
    @given(base_st, breaks_st, st.sampled_from([-1, 0, 1, 6, 16, 96, 65535, 65536]),
           st.sampled_from([-1, 0, 1, 2, 3, 4, 8]))
    def check(base, breaks, n_q, group_q):
        d = dict(base)
        d.update(breaks)
        d["n_q_heads"], d["n_kv_heads"] = d.pop("heads")
        dims = qsa.make_dims(d["batch"], d["n_q_heads"], d["n_kv_heads"], d["kv_capacity"], d["head_dim"],
                             d["n_idx_heads"], d["idx_dim"], d["block_size"], d["top_k"], d["softmax_scale"])
        want = _header_rules(d, n_q, group_q)
        info = qsa.qsa_attn_plan_info()
        rc = lib.qsa_attn_plan(ctypes.byref(dims), n_q, group_q, ctypes.byref(info))
        expect = {None: qsa.QSA_OK, "invalid": qsa.QSA_ERR_INVALID_ARG, "unsupported": qsa.QSA_ERR_UNSUPPORTED}
        assert rc == expect[want], (d, n_q, group_q, rc)
        if want is None and n_q > 0:
            assert info.ctas >= 1 and info.rows == group_q * (d["n_q_heads"] // d["n_kv_heads"])
        # the workspace query accepts the same dims and query counts (no groups there)
        ws_ok = _header_rules(d, n_q, 1) is None
        assert (qsa.qsa_workspace_bytes(dims, n_q, 0, qsa.QSA_MODE_DECODE) > 0) == ws_ok, (d, n_q)

    check()
