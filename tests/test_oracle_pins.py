"""Pins of the CPU oracle against things other than itself.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
sign, an off-by-one block boundary, a transposed operand, the wrong GQA head
map, the wrong tie rule) fails at least one of them:

* a hand-worked example (tests/golden/hand_example.json);
* closed forms and special cases (one-hot tokens, ties to even, Q = 0, one token);
* library routines the method reduces to in special cases (torch's fp32 -> bf16
  conversion, einsum on exact integers, scaled_dot_product_attention in fp64 for
  dense causal GQA and for an explicit token mask);
* brute force on tiny inputs (Python sort, the count rule for top-k).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import qsa_synth as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    """bf16 bit patterns of exactly representable values (via torch, a library routine)."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def val(b):
    return syn.bf16_bits_to_f32(b).astype(np.float64)


# ------------------------------------------------------------------ bf16 helpers

def test_bf16_value_known_patterns(oracle_lib):
    o = oracle_lib
    assert o.bf16_value(0x3F80) == 1.0
    assert o.bf16_value(0xC000) == -2.0
    assert o.bf16_value(0x3E80) == 0.25
    assert math.isinf(o.bf16_value(0x7F80))
    assert o.bf16_value(0x0001) == 2.0 ** -133


def test_round_bf16_ties_to_even_by_hand(oracle_lib):
    o = oracle_lib
    # spacing at 1.0 is 2^-7: half way goes to the even neighbour
    assert o.round_bf16(1 + 2 ** -8) == 0x3F80
    assert o.round_bf16(1 + 3 * 2 ** -8) == 0x3F82
    assert o.round_bf16(1 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert o.round_bf16(-(1 + 2 ** -8)) == 0xBF80
    assert o.round_bf16(0.0) == 0
    assert o.round_bf16(3.5e38) == 0x7F80


def test_round_bf16_matches_torch_conversion(oracle_lib):
    rng = np.random.default_rng(7)
    mags = np.exp2(rng.uniform(-140, 127, 20000))
    x = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    want = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_lib.round_bf16(float(v)) for v in x], dtype=np.uint16)
    np.testing.assert_array_equal(got, want)


# ------------------------------------------------------------------ hand example

def test_hand_example_all_steps(oracle_lib):
    o = oracle_lib
    ex = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    idx_k = bits(ex["idx_k"])
    pooled = o.pool_blocks(idx_k, ex["block_size"])
    np.testing.assert_array_equal(val(pooled), np.array(ex["pooled"], dtype=np.float64))
    sc = o.block_scores(bits(ex["q_idx"]), np.array(ex["w"], np.float32), pooled)
    np.testing.assert_array_equal(sc, np.array(ex["scores"], dtype=np.float64))
    sel = o.select_top_blocks(sc, ex["top_k"])
    assert sel.tolist() == ex["selected"]
    toks = o.attended_tokens(sel, ex["t"], ex["block_size"])
    assert toks.tolist() == ex["attended_tokens"]


# ------------------------------------------------------------------ step 1: pooling

@pytest.mark.parametrize("j", [0, 3, 4, 7, 8, 30, 31])
def test_pool_one_hot_token_lands_in_its_block(oracle_lib, j):
    idx_k = np.zeros((32, 8), dtype=np.float32)
    idx_k[j, 5] = 4.0
    pooled = val(oracle_lib.pool_blocks(bits(idx_k)))
    want = np.zeros((8, 8))
    want[j // 4, 5] = 1.0
    np.testing.assert_array_equal(pooled, want)


def test_pool_mean_rounds_once_to_bf16(oracle_lib):
    u = 2.0 ** -7  # one bf16 step at 1.0
    cases = [
        ([1 + u, 1, 1, 1], 1.0),                  # mean 1 + u/4: rounds down
        ([1 + u, 1 + u, 1, 1], 1.0),              # mean 1 + u/2: tie -> even (1.0)
        ([1 + u, 1 + u, 1 + u, 1], 1 + u),        # mean 1 + 3u/4: rounds up
        ([3, 3, 3, 3], 3.0),
        ([-4, 4, -4, 3], -0.25),
    ]
    for toks, want in cases:
        x = np.array(toks, dtype=np.float32)[:, None]
        got = val(oracle_lib.pool_blocks(bits(x)))[0, 0]
        assert got == want, (toks, got, want)


def test_pool_integer_keys_equal_exact_quarter_means(oracle_lib):
    k = syn.gen_idx_k(5, 0, 0, 4096, 64)
    pooled = val(oracle_lib.pool_blocks(k))
    ints = syn.bf16_bits_to_f32(k).astype(np.int64).reshape(1024, 4, 64).sum(axis=1)
    np.testing.assert_array_equal(pooled * 4, ints.astype(np.float64))


# ------------------------------------------------------------------ step 2: scores

def test_scores_sign_relu_weights_by_hand(oracle_lib):
    q = bits([[1, 0, 0, 0], [0, -1, 0, 0]])
    w = np.array([2, 3], np.float32)
    pooled = bits([[3, 1, 0, 0], [-2, -5, 0, 0], [0, 0, 7, 7]])
    sc = oracle_lib.block_scores(q, w, pooled)
    # block0: 2*relu(3) + 3*relu(-1) = 6; block1: 2*relu(-2) + 3*relu(5) = 15; block2: 0
    np.testing.assert_array_equal(sc, [6.0, 15.0, 0.0])


def test_scores_match_einsum_on_integers(oracle_lib):
    rng = np.random.default_rng(3)
    q = rng.integers(-4, 5, (4, 64)).astype(np.float32)
    pooled = (rng.integers(-16, 17, (300, 64)) / 4).astype(np.float32)
    w = rng.integers(1, 4, 4).astype(np.float32)
    got = oracle_lib.block_scores(bits(q), w, bits(pooled))
    dots = torch.einsum("hd,bd->bh", torch.tensor(q, dtype=torch.float64),
                        torch.tensor(pooled, dtype=torch.float64))
    want = (torch.relu(dots) * torch.tensor(w, dtype=torch.float64)).sum(dim=1).numpy()
    np.testing.assert_array_equal(got, want)


def test_scores_weights_are_linear_and_nonnegative(oracle_lib):
    rng = np.random.default_rng(4)
    q = bits(rng.integers(-4, 5, (4, 64)))
    pooled = bits(rng.integers(-4, 5, (100, 64)))
    w = np.array([1, 2, 3, 1], np.float32)
    s1 = oracle_lib.block_scores(q, w, pooled)
    s2 = oracle_lib.block_scores(q, 2 * w, pooled)
    assert (s1 >= 0).all()
    np.testing.assert_array_equal(s2, 2 * s1)


# ------------------------------------------------------------------ step 3: top-k

def _brute_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda b: (-scores[b], b))
    return sorted(order[:k])


@pytest.mark.parametrize("n,k,seed", [(50, 7, 0), (300, 37, 1), (5, 9, 2), (1, 1, 3), (513, 512, 4)])
def test_select_matches_sort_and_count_rule(oracle_lib, n, k, seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, 6, n).astype(np.float64)  # heavy ties
    sel = oracle_lib.select_top_blocks(s, k).tolist()
    assert sel == _brute_topk(list(s), k)
    chosen = set(sel)
    for b in range(n):
        better = sum(1 for c in range(n) if s[c] > s[b] or (s[c] == s[b] and c < b))
        assert (b in chosen) == (better < k)


def test_select_tie_storm_takes_lowest_indices(oracle_lib):
    sel = oracle_lib.select_top_blocks(np.zeros(2048), 512)
    assert sel.tolist() == list(range(512))


def test_select_fewer_candidates_than_budget(oracle_lib):
    assert oracle_lib.select_top_blocks(np.array([3.0, 1.0, 2.0]), 512).tolist() == [0, 1, 2]
    assert oracle_lib.select_top_blocks(np.zeros(0), 512).tolist() == []


# ------------------------------------------------------------------ step 4: tokens

def test_attended_tokens_closed_forms(oracle_lib):
    o = oracle_lib
    assert o.attended_tokens(np.array([], np.int32), 0).tolist() == [0]
    assert o.attended_tokens(np.array([], np.int32), 2).tolist() == [0, 1, 2]
    assert o.attended_tokens(np.array([0], np.int32), 3).tolist() == [0, 1, 2, 3]
    assert o.attended_tokens(np.array([0], np.int32), 5).tolist() == [0, 1, 2, 3, 4, 5]
    assert o.attended_tokens(np.array([1], np.int32), 9).tolist() == [4, 5, 6, 7, 8, 9]
    assert o.attended_tokens(np.array([0, 2], np.int32), 11).tolist() == [0, 1, 2, 3, 8, 9, 10, 11]


# ------------------------------------------------------------------ step 5: attention

def _sdpa(q, k, v, mask=None):
    """torch SDPA in fp64 for one query: q [Hq][D], k/v [T][Hkv][D]."""
    qt = torch.tensor(val(q))[None, :, None, :]               # [1, Hq, 1, D]
    kt = torch.tensor(val(k)).permute(1, 0, 2)[None]          # [1, Hkv, T, D]
    vt = torch.tensor(val(v)).permute(1, 0, 2)[None]
    m = None if mask is None else torch.tensor(mask)[None, None, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, enable_gqa=True)
    return o[0, :, 0, :].numpy()


def test_attention_equals_dense_gqa_sdpa(oracle_lib):
    rng = np.random.default_rng(11)
    q = bits(rng.normal(size=(8, 32)))
    k = bits(rng.normal(size=(23, 2, 32)))
    v = bits(rng.normal(size=(23, 2, 32)))
    got = oracle_lib.gqa_attention(q, k, v)
    np.testing.assert_allclose(got, _sdpa(q, k, v), rtol=0, atol=1e-12)


def test_attention_closed_forms(oracle_lib):
    rng = np.random.default_rng(12)
    k = bits(rng.normal(size=(9, 1, 16)))
    v = bits(rng.normal(size=(9, 1, 16)))
    zero_q = bits(np.zeros((2, 16)))
    got = oracle_lib.gqa_attention(zero_q, k, v)
    np.testing.assert_allclose(got, np.tile(val(v)[:, 0, :].mean(axis=0), (2, 1)), atol=1e-12)
    one = oracle_lib.gqa_attention(bits(rng.normal(size=(2, 16))), k[:1], v[:1])
    np.testing.assert_allclose(one, np.tile(val(v)[0, 0], (2, 1)), atol=0)
    const_v = bits(np.full((9, 1, 16), 0.75))
    c = oracle_lib.gqa_attention(bits(rng.normal(size=(2, 16))), k, const_v)
    np.testing.assert_allclose(c, 0.75, atol=1e-12)


def test_attention_gqa_head_map_is_grouped(oracle_lib):
    # 4 query heads on 2 KV heads: heads 0,1 -> KV 0 and heads 2,3 -> KV 1.
    # V of KV head 0 is all 1, of KV head 1 all -1, so the map is visible directly.
    rng = np.random.default_rng(13)
    q = bits(rng.normal(size=(4, 8)))
    k = bits(rng.normal(size=(5, 2, 8)))
    v = np.ones((5, 2, 8), np.float32)
    v[:, 1, :] = -1
    out = oracle_lib.gqa_attention(q, k, bits(v))
    np.testing.assert_allclose(out[:2], 1.0, atol=1e-12)
    np.testing.assert_allclose(out[2:], -1.0, atol=1e-12)


# ------------------------------------------------------------------ whole query

def _dense_inputs(seed, T, Hq, Hkv, D, Di=64, Hi=4):
    rng = np.random.default_rng(seed)
    return dict(
        idx_k=bits(rng.integers(-4, 5, (T, Di))),
        q_idx=bits(rng.integers(-4, 5, (Hi, Di))),
        w=rng.integers(1, 4, Hi).astype(np.float32),
        q=bits(rng.normal(size=(Hq, D))),
        k=bits(rng.normal(size=(T, Hkv, D))),
        v=bits(rng.normal(size=(T, Hkv, D))),
    )


@pytest.mark.parametrize("t", [0, 1, 2, 3, 4, 6, 2047, 2050])
def test_query_with_at_most_512_blocks_is_dense_causal_gqa(oracle_lib, t):
    """<= 512 complete causal blocks: every token 0..t is attended, so QSA = dense causal GQA."""
    o = oracle_lib
    inp = _dense_inputs(21 + t, t + 1, 8, 2, 32)
    pooled = o.pool_blocks(inp["idx_k"])
    fetch = lambda toks: (inp["k"][toks], inp["v"][toks])
    sel, out = o.query_forward(pooled, inp["q_idx"], inp["w"], t, inp["q"], fetch)
    assert sel.tolist() == list(range((t + 1) // 4))
    np.testing.assert_allclose(out, _sdpa(inp["q"], inp["k"][: t + 1], inp["v"][: t + 1]),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("t,top_k", [(41, 3), (42, 5), (43, 2), (100, 7)])
def test_query_equals_explicit_mask_brute_force(oracle_lib, t, top_k):
    """The gathered form equals dense softmax attention under an explicit token mask
    built from the selection (a mask is used here only, on tiny inputs)."""
    o = oracle_lib
    inp = _dense_inputs(50 + t, t + 1, 4, 1, 16)
    pooled = o.pool_blocks(inp["idx_k"])
    fetch = lambda toks: (inp["k"][toks], inp["v"][toks])
    sel, out = o.query_forward(pooled, inp["q_idx"], inp["w"], t, inp["q"], fetch, top_k=top_k)
    # brute-force selection from exact integer scores
    pk = syn.bf16_bits_to_f32(inp["idx_k"]).astype(np.float64)[: 4 * ((t + 1) // 4)]
    mean = pk.reshape(-1, 4, pk.shape[1]).mean(axis=1)
    dots = val(inp["q_idx"]) @ mean.T
    scores = (np.maximum(dots, 0) * inp["w"][:, None]).sum(axis=0)
    assert sel.tolist() == _brute_topk(list(scores), top_k)
    mask = np.zeros(t + 1, dtype=bool)
    for b in sel:
        mask[4 * b: 4 * b + 4] = True
    mask[4 * ((t + 1) // 4):] = True
    np.testing.assert_allclose(out, _sdpa(inp["q"], inp["k"], inp["v"], mask), rtol=0, atol=1e-12)


def test_workload_query_selection_by_brute_force(oracle_lib):
    """decode_8k_b1's query (2,048 candidate blocks): selection equals a numpy brute force."""
    from oracle.oracle import WorkloadOracle
    from qsa_synth import workloads
    wl = workloads.decode_8k()
    wo = WorkloadOracle(wl)
    sel, out = wo.query(0, 0)
    st = wl.steps[0]
    idx_k = syn.bf16_bits_to_f32(syn.gen_idx_k(wl.seed, 0, 0, 8192, 64)).astype(np.float64)
    mean = idx_k.reshape(2048, 4, 64).mean(axis=1)
    q_idx = syn.bf16_bits_to_f32(syn.gen_q_idx(wl.seed, st.query_ids, 4, 64)[0]).astype(np.float64)
    w = syn.gen_w(wl.seed, st.query_ids, 4)[0].astype(np.float64)
    scores = (np.maximum(q_idx @ mean.T, 0) * w[:, None]).sum(axis=0)
    order = np.lexsort((np.arange(2048), -scores))[:512]
    assert sel.tolist() == sorted(order.tolist())
    assert out.shape == (8, 128) and np.isfinite(out).all()


# ------------------------------------------------------------------ multi-token decode (shared selection)

def test_shared_tokens_closed_forms(oracle_lib):
    """A draft query reusing the selection made at t_sel attends the selected blocks
    plus every token from the selection's first incomplete block up to itself."""
    o = oracle_lib
    # same position: the ordinary rule
    for sel, t in ([[0, 2], 11], [[1], 9], [[], 2], [[0], 3]):
        s = np.array(sel, np.int32)
        assert o.attended_tokens_shared(s, t, t).tolist() == o.attended_tokens(s, t).tolist()
    # selection at t_sel = 9 (2 complete blocks, partial block {8, 9}); drafts at 10, 11, 12, 13
    s = np.array([0], np.int32)
    assert o.attended_tokens_shared(s, 9, 10).tolist() == [0, 1, 2, 3, 8, 9, 10]
    assert o.attended_tokens_shared(s, 9, 11).tolist() == [0, 1, 2, 3, 8, 9, 10, 11]
    # draft 12 completes nothing new for the selection: block 2 (8..11) was not a candidate at t_sel
    assert o.attended_tokens_shared(s, 9, 12).tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 12]
    assert o.attended_tokens_shared(s, 9, 13).tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 12, 13]
    # t_sel = 11 completes block 2: the tail starts at 12
    s = np.array([2], np.int32)
    assert o.attended_tokens_shared(s, 11, 13).tolist() == [8, 9, 10, 11, 12, 13]


@pytest.mark.parametrize("t_sel,draft", [(40, 1), (41, 2), (43, 3), (102, 4)])
def test_shared_tokens_invariants(oracle_lib, t_sel, draft):
    """Counts, causality and coverage, for random selections below t_sel."""
    o = oracle_lib
    rng = np.random.default_rng(t_sel * 10 + draft)
    n_c = (t_sel + 1) // 4
    sel = np.sort(rng.choice(n_c, size=min(5, n_c), replace=False)).astype(np.int32)
    t = t_sel + draft
    toks = o.attended_tokens_shared(sel, t_sel, t)
    assert (np.diff(toks) > 0).all() and toks.max() == t and (toks <= t).all()
    assert len(toks) == 4 * len(sel) + (t + 1 - 4 * n_c)
    covered = set(toks.tolist())
    for b in range(n_c):  # a complete block below t_sel is attended whole or not at all
        inside = [p in covered for p in range(4 * b, 4 * b + 4)]
        assert all(inside) == (b in sel.tolist()) and (any(inside) == all(inside))
    assert all(p in covered for p in range(4 * n_c, t + 1))


@pytest.mark.parametrize("t_sel,draft", [(8, 1), (10, 3), (2047, 2), (2045, 4)])
def test_shared_selection_below_budget_is_dense_causal_gqa(oracle_lib, t_sel, draft):
    """With <= 512 complete blocks at t_sel every block is selected, so each draft
    query at t_sel + j attends tokens 0..t_sel+j: dense causal GQA (fp64 SDPA)."""
    o = oracle_lib
    t_last = t_sel + draft
    inp = _dense_inputs(70 + t_sel + draft, t_last + 1, 8, 2, 32)
    pooled = o.pool_blocks(inp["idx_k"])
    n_c = (t_sel + 1) // 4
    sel = o.select_top_blocks(o.block_scores(inp["q_idx"], inp["w"], pooled[:n_c]))
    assert sel.tolist() == list(range(n_c))
    for t in range(t_sel, t_last + 1):
        toks = o.attended_tokens_shared(sel, t_sel, t)
        out = o.gqa_attention(inp["q"], inp["k"][toks], inp["v"][toks])
        np.testing.assert_allclose(out, _sdpa(inp["q"], inp["k"][: t + 1], inp["v"][: t + 1]), rtol=0, atol=1e-12)
