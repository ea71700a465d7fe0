"""Pins for the CPU oracle: each test checks it against something other than
itself -- brute force, closed forms, hand-worked fixtures, invariants and
special cases that reduce to a library routine -- so that a dropped term, a
wrong index, a transposed operand or a swapped gate/up fails at least one."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import moe_inputs as mi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(v):
    if isinstance(v, str):
        return {"-0.0": np.float32(-0.0), "inf": np.float32(np.inf), "-inf": np.float32(-np.inf),
                "ln3": np.float32(math.log(3.0)), "-ln3": np.float32(-math.log(3.0))}[v]
    return np.float32(v)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- top-K

def brute_topk(row, K):
    """Subset whose (descending logit, ascending index) key list is the
    lexicographic maximum over all C(E,K) subsets."""
    E = len(row)
    best, best_key = None, None
    for sub in itertools.combinations(range(E), K):
        order = sorted(sub, key=lambda e: (-float(row[e]), e))
        key = [(float(row[e]), -e) for e in order]
        if best_key is None or key > best_key:
            best, best_key = order, key
    return best


@pytest.mark.parametrize("kind", ["gauss", "ties", "inf"])
def test_topk_matches_subset_bruteforce(kind):
    rng = np.random.default_rng(11)
    for E in range(1, 11):
        for K in range(1, min(E, 4) + 1):
            T = 12
            if kind == "gauss":
                lg = rng.standard_normal((T, E)).astype(np.float32)
            elif kind == "ties":
                lg = mi.tie_heavy_logits(T, E, seed=E * 10 + K, levels=1)
            else:
                lg = mi.tie_heavy_logits(T, E, seed=E * 7 + K, levels=2)
                lg[lg == 2] = np.inf
                lg[lg == -2] = -np.inf
            ids = oracle.topk(lg, K)
            for t in range(T):
                assert list(ids[t]) == brute_topk(lg[t], K), (E, K, lg[t], ids[t])


def test_topk_matches_stable_argsort():
    # A stable sort on the negated logit keeps the lower index first on ties;
    # numpy compares -0.0 equal to +0.0, as IEEE does.
    rng = np.random.default_rng(3)
    for E, K in [(8, 2), (64, 8), (256, 8), (37, 5)]:
        lg = np.concatenate([rng.standard_normal((20, E)).astype(np.float32),
                             mi.tie_heavy_logits(20, E, seed=E)], 0)
        ids = oracle.topk(lg, K)
        ref = np.argsort(-lg, axis=1, kind="stable")[:, :K]
        assert np.array_equal(ids, ref.astype(np.int32))


def test_topk_golden_ties():
    g = _load("topk_ties.json")
    lg = np.array([[_f32(v) for v in r["logits"]] for r in g["rows"]], np.float32)
    ids = oracle.topk(lg, g["K"])
    assert ids.tolist() == [r["ids"] for r in g["rows"]]


def test_topk_K_equals_E_is_a_permutation():
    lg = mi.tie_heavy_logits(30, 9, seed=5)
    ids = oracle.topk(lg, 9)
    for t in range(30):
        assert sorted(ids[t]) == list(range(9))
        vals = lg[t, ids[t]]
        assert np.all(vals[:-1] >= vals[1:])


def test_topk_rejects_nan():
    lg = np.zeros((2, 4), np.float32)
    lg[1, 2] = np.nan
    with pytest.raises(ValueError):
        oracle.topk(lg, 2)


# ---------------------------------------------------------------- weights

def test_gate_weights_golden():
    for c in _load("gate_weights.json")["cases"]:
        lg = np.array([[_f32(v) for v in c["logits"]]], np.float32)
        ids = oracle.topk(lg, c["K"])
        assert ids[0].tolist() == c["ids"]
        w = oracle.gate_weights(lg, ids, c["score_fn"], c["renorm"])
        assert np.allclose(w[0], c["w"], rtol=1e-6, atol=1e-7), (c, w)


def test_softmax_K_equals_E_is_full_softmax():
    rng = np.random.default_rng(4)
    lg = (3 * rng.standard_normal((16, 7))).astype(np.float32)
    ids = oracle.topk(lg, 7)
    for renorm in (0, 1):
        w = oracle.gate_weights(lg, ids, 0, renorm)
        ref = scipy.special.softmax(lg.astype(np.float64), axis=1)
        assert np.allclose(w, np.take_along_axis(ref, ids, 1), rtol=1e-12)


def test_softmax_renorm_is_topk_slice_renormalised():
    # renorm=0 gives the full softmax restricted to the selected experts; its
    # renormalisation over the K selected equals the renorm=1 weights.
    rng = np.random.default_rng(5)
    lg = (2 * rng.standard_normal((32, 16))).astype(np.float32)
    ids = oracle.topk(lg, 4)
    w0 = oracle.gate_weights(lg, ids, 0, 0)
    w1 = oracle.gate_weights(lg, ids, 0, 1)
    ref = scipy.special.softmax(lg.astype(np.float64), axis=1)
    assert np.allclose(w0, np.take_along_axis(ref, ids, 1), rtol=1e-12)
    assert np.allclose(w1, w0 / w0.sum(1, keepdims=True), rtol=1e-12)
    assert np.all(w1[:, :-1] >= w1[:, 1:])


def test_softmax_shift_invariance_and_sigmoid_values():
    lg = mi.tie_heavy_logits(16, 8, seed=9, levels=4).astype(np.float32)
    ids = oracle.topk(lg, 3)
    w = oracle.gate_weights(lg, ids, 0, 1)
    w_shift = oracle.gate_weights(lg + np.float32(5.0), ids, 0, 1)
    assert np.allclose(w, w_shift, rtol=1e-12)
    ws = oracle.gate_weights(lg, ids, 1, 0)
    ref = scipy.special.expit(np.take_along_axis(lg, ids, 1).astype(np.float64))
    assert np.allclose(ws, ref, rtol=1e-12)
    wsn = oracle.gate_weights(lg, ids, 1, 1)
    assert np.allclose(wsn.sum(1), 1.0, rtol=1e-12)


# ------------------------------------------------------------------ align

def _check_align_invariants(ids, E, B, r):
    T, K = ids.shape
    A = T * K
    counts, offsets, sid, be, pos = r["counts"], r["offsets"], r["sorted_ids"], r["block_expert"], r["pos"]
    assert counts.sum() == A
    assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
    padded = np.diff(offsets)
    assert offsets[0] == 0 and np.all(padded >= 0)
    assert np.all(padded % B == 0)
    assert np.all((padded - counts >= 0) & (padded - counts < B))
    assert np.all((padded == 0) == (counts == 0))
    assert offsets[E] == r["P"]
    # section 5.1 closed form of the padded rows
    assert r["P"] == int(sum(-(-int(n) // B) * B for n in counts))
    assert len(sid) == oracle.p_max(T, K, E, B)
    valid = sid[sid >= 0]
    assert np.array_equal(np.sort(valid), np.arange(A))          # bijection onto [0, A)
    assert np.all(sid[r["P"]:] == -1)
    for a in range(A):
        assert sid[pos[a]] == a
    for e in range(E):
        seg = sid[offsets[e]:offsets[e + 1]]
        real = seg[:counts[e]]
        assert np.all(seg[counts[e]:] == -1)
        assert np.all(np.diff(real) > 0)                         # ascending a
        assert np.all(ids.ravel()[real] == e)
        assert np.all(be[offsets[e] // B:offsets[e + 1] // B] == e)
    assert np.all(be[r["P"] // B:] == -1)
    assert r["E_active"] == int((counts > 0).sum())


def test_align_golden():
    g = _load("align_small.json")
    ids = np.array(g["ids"], np.int32)
    r = oracle.align(ids, g["E"], g["B"])
    assert oracle.p_max(g["T"], g["K"], g["E"], g["B"]) == g["P_max"]
    for key in ("counts", "offsets", "sorted_ids", "pos", "block_expert"):
        assert r[key].tolist() == g[key], key
    assert r["P"] == g["P"] and r["E_active"] == g["E_active"]
    _check_align_invariants(ids, g["E"], g["B"], r)


@pytest.mark.parametrize("B", [1, 4, 16, 128])
def test_align_invariants_random(B):
    rng = np.random.default_rng(B)
    for T, E, K in [(1, 8, 2), (37, 8, 2), (64, 64, 8), (50, 256, 8), (3, 5, 5), (0, 4, 2)]:
        lg = rng.standard_normal((T, E)).astype(np.float32)
        ids = oracle.topk(lg, K) if T else np.zeros((0, K), np.int32)
        r = oracle.align(ids, E, B)
        _check_align_invariants(ids, E, B, r)


def test_align_single_expert_closed_form():
    # every token on expert 0 (K=1): P = ceil(A/B)*B, one active expert
    for T, B in [(1, 16), (16, 16), (17, 16), (300, 128)]:
        ids = np.zeros((T, 1), np.int32)
        r = oracle.align(ids, 4, B)
        assert r["P"] == -(-T // B) * B
        assert r["E_active"] == 1
        assert r["sorted_ids"][:T].tolist() == list(range(T))


def _check_max_value_invariants(ids, E, B, r):
    # max-value padding (Section 5.1): every expert's segment has the padded
    # size of the most loaded expert, P = E * ceil(max N_i / B) * B
    T, K = ids.shape
    A = T * K
    counts, offsets, sid, be, pos = r["counts"], r["offsets"], r["sorted_ids"], r["block_expert"], r["pos"]
    assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
    M = -(-int(counts.max()) // B) * B if A else 0
    assert np.all(np.diff(offsets) == M)
    assert r["P"] == E * M == offsets[E]
    assert len(sid) == oracle.p_max(T, K, E, B, mode=1) >= r["P"]
    assert np.array_equal(np.sort(sid[sid >= 0]), np.arange(A))
    for a in range(A):
        assert sid[pos[a]] == a
    for e in range(E):
        seg = sid[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg[:counts[e]]) > 0) and np.all(ids.ravel()[seg[:counts[e]]] == e)
        assert np.all(seg[counts[e]:] == -1)
        assert np.all(be[offsets[e] // B:offsets[e + 1] // B] == e)
    assert np.all(be[r["P"] // B:] == -1)
    assert r["E_active"] == int((counts > 0).sum())


def test_align_max_value_worked_example():
    # T = 3, K = 2, E = 4, B = 4: counts (2, 1, 3, 0), the largest 3 pads to 4,
    # so every expert gets 4 rows and P = 16 (block-wise: 4 + 4 + 4 + 0 = 12)
    ids = np.array([[0, 2], [2, 1], [2, 0]], np.int32)
    r = oracle.align(ids, 4, 4, mode=1)
    assert r["counts"].tolist() == [2, 1, 3, 0]
    assert r["offsets"].tolist() == [0, 4, 8, 12, 16] and r["P"] == 16
    assert r["sorted_ids"][:16].tolist() == [0, 5, -1, -1, 3, -1, -1, -1, 1, 2, 4, -1, -1, -1, -1, -1]
    assert r["pos"].tolist() == [0, 8, 9, 4, 10, 1]
    assert r["block_expert"][:4].tolist() == [0, 1, 2, 3]
    assert r["E_active"] == 3
    assert oracle.align(ids, 4, 4)["P"] == 12


@pytest.mark.parametrize("B", [1, 4, 16, 128])
def test_align_max_value_invariants_random(B):
    rng = np.random.default_rng(100 + B)
    for T, E, K in [(1, 8, 2), (37, 8, 2), (64, 64, 8), (50, 256, 8), (3, 5, 5), (0, 4, 2)]:
        lg = rng.standard_normal((T, E)).astype(np.float32)
        ids = oracle.topk(lg, K) if T else np.zeros((0, K), np.int32)
        _check_max_value_invariants(ids, E, B, oracle.align(ids, E, B, mode=1))


def test_align_padding_schemes_extremes():
    # the two schemes' worst cases (Section 5.1): a concentrated distribution
    # (all tokens on one expert) costs max-value padding E times block-wise,
    # a dispersed one (each expert a single token) costs them the same
    E, B = 8, 16
    hot = np.zeros((40, 1), np.int32)
    assert oracle.align(hot, E, B)["P"] == 48
    assert oracle.align(hot, E, B, mode=1)["P"] == E * 48
    spread = np.arange(E, dtype=np.int32).reshape(E, 1)
    assert oracle.align(spread, E, B)["P"] == oracle.align(spread, E, B, mode=1)["P"] == E * B


def test_align_rejects_bad_ids():
    with pytest.raises(ValueError):
        oracle.align(np.array([[0, 5]], np.int32), 4, 4)


def test_align_max_value_rejects_rows_past_the_bound():
    # max-value padding's bound E * ceil(min(T, A) / B) * B holds when an
    # expert has at most one assignment per token (every top-K routing); ids
    # that repeat within a token can need more rows, and the oracle rejects
    # them.  Block-wise padding stays within A + min(E, A) (B - 1) for any ids.
    T, K, E, B = 4, 2, 4, 4
    ids = np.zeros((T, K), np.int32)         # expert 0 twice per token: N_0 = 8 > T
    assert oracle.p_max(T, K, E, B, 1) == 16
    with pytest.raises(ValueError):
        oracle.align(ids, E, B, mode=1)      # would need E * 8 = 32 rows
    r = oracle.align(ids, E, B)
    assert r["P"] == 8 and r["P"] <= oracle.p_max(T, K, E, B, 0)


# ----------------------------------------------------- permute / combine

def test_permute_then_combine_with_unit_weights_is_identity():
    # un-permuting the permuted rows by pos with w = 1 and K = 1 returns x;
    # padding rows of the permuted matrix are zero.
    rng = np.random.default_rng(7)
    T, E, B = 23, 5, 4
    x = rng.standard_normal((T, 6)).astype(np.float32)
    ids = rng.integers(0, E, size=(T, 1)).astype(np.int32)
    r = oracle.align(ids, E, B)
    xp = oracle.permute(x, r["sorted_ids"], 1, r["P"])
    pad = r["sorted_ids"][:r["P"]] < 0
    assert np.all(xp[pad] == 0.0)
    back = oracle.combine(xp.astype(np.float32), r["pos"], np.ones((T, 1)))
    assert np.array_equal(back, x.astype(np.float64))


def test_combine_closed_form_and_shared():
    # K = 2 rows with weights 3/4, 1/4 of constant rows c1, c2 give 3/4 c1 + 1/4 c2,
    # and the shared row is added once.
    y = np.array([[1.0, 1.0], [5.0, 5.0], [-2.0, 4.0]], np.float32)
    pos = np.array([[1, 0], [2, 1]], np.int32)
    w = np.array([[0.75, 0.25], [0.5, 0.5]])
    sh = np.array([[10.0, 0.0], [0.0, -1.0]], np.float32)
    out = oracle.combine(y, pos, w, sh)
    assert out.tolist() == [[0.75 * 5 + 0.25 * 1 + 10.0, 0.75 * 5 + 0.25 * 1], [0.5 * -2 + 0.5 * 5, 0.5 * 4 + 0.5 * 5 - 1.0]]


def test_permute_golden():
    g = _load("align_small.json")
    T, K = g["T"], g["K"]
    x = np.arange(T * 3, dtype=np.float32).reshape(T, 3)
    xp = oracle.permute(x, np.array(g["sorted_ids"], np.int32), K, g["P"])
    for p, a in enumerate(g["sorted_ids"][:g["P"]]):
        assert xp[p].tolist() == ([0.0] * 3 if a < 0 else x[a // K].tolist())


# -------------------------------------------------------------- FFN math

def _perm_matrix(perm):
    n = len(perm)
    m = np.zeros((n, n), np.float32)
    m[np.arange(n), perm] = 1.0     # (M v)[i] = v[perm[i]]
    return m


def test_swiglu_closed_form_on_permutation_weights():
    # W1, W3, W2 permutation matrices: g_i = x[s1(i)], u_i = x[s3(i)],
    # y_h = a[s2(h)] = silu(x[s1(s2(h))]) * x[s3(s2(h))], silu(v) = v/(1+e^-v).
    # A transposed W2 (s2^-1), a swapped gate/up or a dropped term fails.
    H = 7
    rng = np.random.default_rng(0)
    s1, s2, s3 = (rng.permutation(H) for _ in range(3))
    assert not np.array_equal(s2, np.argsort(s2))
    x = np.array([0.0, math.log(3.0), -1.5, 2.0, 0.25, -0.5, 3.0], np.float32)
    w13 = np.concatenate([_perm_matrix(s1), _perm_matrix(s3)], 0)
    w2 = _perm_matrix(s2)
    y = oracle.swiglu_ffn(x, w13, w2)
    xd = x.astype(np.float64)
    for h in range(H):
        v = xd[s1[s2[h]]]
        u = xd[s3[s2[h]]]
        assert y[h] == pytest.approx(v / (1.0 + math.exp(-v)) * u, rel=1e-14, abs=1e-15)


def test_swiglu_known_sigmoid_value():
    # sigmoid(ln 3) = 3/4: with H = I = 1 and unit weights, y = ln3 * 3/4 * ln3
    x = np.array([math.log(3.0)], np.float32)
    w13 = np.array([[1.0], [1.0]], np.float32)
    w2 = np.array([[1.0]], np.float32)
    l3 = float(np.float32(math.log(3.0)))
    assert oracle.swiglu_ffn(x, w13, w2)[0] == pytest.approx(l3 * l3 / (1 + math.exp(-l3)), rel=1e-14)
    assert oracle.swiglu_ffn(x, np.array([[0.0], [1.0]], np.float32), w2)[0] == 0.0


def test_swiglu_invariants():
    rng = np.random.default_rng(1)
    H, I = 24, 40
    x = rng.standard_normal(H).astype(np.float32)
    w13 = rng.standard_normal((2 * I, H)).astype(np.float32)
    w2 = rng.standard_normal((H, I)).astype(np.float32)
    y = oracle.swiglu_ffn(x, w13, w2)
    # linear in W2 and in W3 (exact power-of-two scaling)
    assert np.allclose(oracle.swiglu_ffn(x, w13, 2 * w2), 2 * y, rtol=1e-13)
    w13u = w13.copy()
    w13u[I:] *= 4
    assert np.allclose(oracle.swiglu_ffn(x, w13u, w2), 4 * y, rtol=1e-13)
    # permuting the intermediate dimension consistently changes nothing
    p = rng.permutation(I)
    w13p = np.concatenate([w13[:I][p], w13[I:][p]], 0)
    assert np.allclose(oracle.swiglu_ffn(x, w13p, np.ascontiguousarray(w2[:, p])), y, rtol=1e-12)
    # additive over a split of the intermediate dimension (shared-expert concatenation)
    J = 15
    ya = oracle.swiglu_ffn(x, np.concatenate([w13[:J], w13[I:I + J]]), np.ascontiguousarray(w2[:, :J]))
    yb = oracle.swiglu_ffn(x, np.concatenate([w13[J:I], w13[I + J:]]), np.ascontiguousarray(w2[:, J:]))
    assert np.allclose(ya + yb, y, rtol=1e-12, atol=1e-12)
    # gate/up are not interchangeable
    w13s = np.concatenate([w13[I:], w13[:I]])
    assert not np.allclose(oracle.swiglu_ffn(x, w13s, w2), y)


def test_dense_ffn_equals_per_token_expert_ffn():
    rng = np.random.default_rng(2)
    T, H, I = 9, 32, 48
    x = rng.standard_normal((T, H)).astype(np.float32)
    w13 = (rng.standard_normal((2 * I, H)) / np.sqrt(H)).astype(np.float32)
    w2 = (rng.standard_normal((H, I)) / np.sqrt(I)).astype(np.float32)
    out = oracle.dense_ffn(x, w13, w2, nthreads=2)
    for t in range(T):
        assert np.allclose(out[t], oracle.swiglu_ffn(x[t], w13, w2), rtol=1e-13, atol=1e-14)


def test_bf16_inputs_are_widened_exactly():
    rng = np.random.default_rng(3)
    x32 = rng.standard_normal((3, 16)).astype(np.float32)
    w32 = rng.standard_normal((5, 16)).astype(np.float32)
    xb = torch.from_numpy(x32).to(torch.bfloat16)
    wb = torch.from_numpy(w32).to(torch.bfloat16)
    lb = oracle.router_logits(mi.to_oracle(xb), mi.to_oracle(wb))
    lf = oracle.router_logits(xb.float().numpy(), wb.float().numpy())
    assert np.array_equal(lb, lf)


def test_router_logits_on_unit_vectors():
    rng = np.random.default_rng(6)
    E, H = 5, 11
    w = rng.standard_normal((E, H)).astype(np.float32)
    x = np.eye(H, dtype=np.float32)
    assert np.array_equal(oracle.router_logits(x, w), w.T.astype(np.float64))


# ------------------------------------------------------------- the layer

def _small_layer(seed, T=12, H=32, E=6, K=2, I=40, I_sh=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    w_r = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) / np.sqrt(H)).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) / np.sqrt(I)).astype(np.float32)
    sh = {}
    if I_sh:
        sh = dict(w13_sh=(rng.standard_normal((2 * I_sh, H)) / np.sqrt(H)).astype(np.float32),
                  w2_sh=(rng.standard_normal((H, I_sh)) / np.sqrt(I_sh)).astype(np.float32))
    return x, w_r, w13, w2, sh


@pytest.mark.parametrize("score_fn", [0, 1])
def test_layer_E1_K1_is_dense_ffn(score_fn):
    x, w_r, w13, w2, _ = _small_layer(0, E=1)
    out = oracle.moe_layer(x, w_r, w13, w2, K=1, score_fn=score_fn, renorm=1)
    assert np.allclose(out, oracle.dense_ffn(x, w13[0], w2[0]), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("score_fn", [0, 1])
def test_layer_identical_experts_is_dense_ffn(score_fn):
    x, w_r, w13, w2, _ = _small_layer(1, E=5, K=3)
    w13[:] = w13[0]
    w2[:] = w2[0]
    out = oracle.moe_layer(x, w_r, w13, w2, K=3, score_fn=score_fn, renorm=1)
    assert np.allclose(out, oracle.dense_ffn(x, w13[0], w2[0]), rtol=1e-12, atol=1e-13)


def test_layer_is_per_token_concatenated_dense_ffn():
    # out[t] = one dense FFN whose W1/W3 concatenate the selected experts (and
    # the shared FFN) along I and whose W2 columns are scaled by the gate
    # weights: DenseFA's shape with per-token weights.  The scaled W2 is
    # rounded to fp32, hence the 1e-6 tolerance.
    x, w_r, w13, w2, sh = _small_layer(2, E=6, K=3, I_sh=24)
    I = w2.shape[2]
    out, ids, w = oracle.moe_layer(x, w_r, w13, w2, K=3, score_fn=0, renorm=1, return_routing=True, **sh)
    for t in range(x.shape[0]):
        g = np.concatenate([w13[e][:I] for e in ids[t]] + [sh["w13_sh"][:24]])
        u = np.concatenate([w13[e][I:] for e in ids[t]] + [sh["w13_sh"][24:]])
        d = np.concatenate([(w2[e].astype(np.float64) * w[t, k]).astype(np.float32)
                            for k, e in enumerate(ids[t])] + [sh["w2_sh"]], 1)
        ref = oracle.dense_ffn(x[t:t + 1], np.concatenate([g, u]), np.ascontiguousarray(d))[0]
        assert np.allclose(out[t], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_layer_all_experts_then_mask():
    # brute force: evaluate every expert for every token, weight by a mask
    # that keeps only the brute-force top-K subset
    x, w_r, w13, w2, _ = _small_layer(3, T=8, E=6, K=2)
    logits = oracle.router_logits(x, w_r).astype(np.float32)
    out = oracle.moe_layer(x, w_r, w13, w2, K=2, score_fn=0, renorm=1)
    for t in range(8):
        sel = brute_topk(logits[t], 2)
        l = logits[t].astype(np.float64)
        den = sum(math.exp(l[e] - l[sel[0]]) for e in sel)
        ref = np.zeros(x.shape[1])
        for e in range(6):
            mask = math.exp(l[e] - l[sel[0]]) / den if e in sel else 0.0
            ref += mask * oracle.swiglu_ffn(x[t], w13[e], w2[e])
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-13)


def test_layer_linear_in_w2_and_token_permutation():
    x, w_r, w13, w2, sh = _small_layer(4, T=10, E=4, K=2, I_sh=16)
    out = oracle.moe_layer(x, w_r, w13, w2, K=2, **sh)
    routed_only = out - oracle.dense_ffn(x, sh["w13_sh"], sh["w2_sh"])
    out2 = oracle.moe_layer(x, w_r, w13, 2 * w2, K=2, **sh)
    assert np.allclose(out2 - oracle.dense_ffn(x, sh["w13_sh"], sh["w2_sh"]), 2 * routed_only,
                       rtol=1e-12, atol=1e-12)
    p = np.random.default_rng(0).permutation(10)
    outp = oracle.moe_layer(np.ascontiguousarray(x[p]), w_r, w13, w2, K=2, **sh)
    assert np.allclose(outp, out[p], rtol=1e-14, atol=1e-15)


def test_layer_token_subset_and_supplied_logits():
    x, w_r, w13, w2, _ = _small_layer(5, T=16, E=8, K=2)
    full = oracle.moe_layer(x, w_r, w13, w2, K=2)
    sub = np.array([15, 0, 7], np.int32)
    assert np.array_equal(oracle.moe_layer(x, w_r, w13, w2, K=2, tokens=sub), full[sub])
    lg = oracle.router_logits(x, w_r).astype(np.float32)
    assert np.array_equal(oracle.moe_layer(x, None, w13, w2, K=2, logits=lg), full)


# -------------------------------------------------------------- generator

def test_uniform_gumbel_routing_matches_expected_active():
    # s = 0: each token draws K distinct experts uniformly, so the number of
    # experts receiving at least one of m tokens has mean E(1-(1-K/E)^m).
    for E, K, m in [(8, 2, 1), (8, 2, 4), (64, 8, 8), (256, 8, 32)]:
        vals = []
        for seed in range(200):
            lg = mi.zipf_gumbel_logits(E, m, 0.0, seed=seed).numpy()
            vals.append(len(np.unique(oracle.topk(lg, K))))
        mean = float(np.mean(vals))
        sem = float(np.std(vals)) / math.sqrt(len(vals)) + 1e-9
        assert abs(mean - oracle.expected_active(E, K, m)) < 3 * sem + 1e-9, (E, K, m, mean)


def test_zipf_skew_reduces_active_experts():
    E, K, m = 256, 8, 32
    means = []
    for s in (0.0, 0.5, 1.0, 1.5):
        means.append(np.mean([len(np.unique(oracle.topk(mi.zipf_gumbel_logits(E, m, s, seed=q).numpy(), K)))
                              for q in range(20)]))
    assert all(a > b for a, b in zip(means, means[1:])), means


def test_router_generator_is_near_uniform():
    shape = mi.SHAPES["mixtral"]
    w = mi.make_weights(shape, seed=1, experts=False)
    x = mi.make_x(shape, 256, seed=2)
    lg = oracle.router_logits(mi.to_oracle(x), mi.to_oracle(w["w_r"])).astype(np.float32)
    counts = np.bincount(oracle.topk(lg, shape.K).ravel(), minlength=shape.E)
    expect = 256 * shape.K / shape.E
    assert np.all(np.abs(counts - expect) < 5 * math.sqrt(expect)), counts


# --------------------------------------------------- per-token dynamic K

def test_dynamic_k_topk_matches_bruteforce_prefix():
    # token t takes the first k_t experts of the (logit desc, index asc) order;
    # slots from k_t on are -1
    rng = np.random.default_rng(21)
    T, E, K = 40, 12, 5
    lg = mi.tie_heavy_logits(T, E, 3, levels=4)
    k = rng.integers(0, K + 1, size=T).astype(np.int32)
    ids = oracle.topk(lg, K, k)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))
        assert ids[t].tolist() == order[:k[t]] + [-1] * (K - k[t])


def test_dynamic_k_equal_to_K_is_static_topk():
    lg = np.random.default_rng(22).standard_normal((30, 16)).astype(np.float32)
    assert np.array_equal(oracle.topk(lg, 4, np.full(30, 4, np.int32)), oracle.topk(lg, 4))


@pytest.mark.parametrize("score_fn", [0, 1])
def test_dynamic_k_gate_weights_closed_forms(score_fn):
    # k_t = 1: the single weight is 1 (renormalised); k_t = 2 under softmax:
    # the pair's weights are sigma(l1 - l2) and sigma(l2 - l1); empty slots 0
    lg = np.array([[0.5, 2.0, -1.0, 1.0], [3.0, -2.0, 0.25, 1.5]], np.float32)
    k = np.array([1, 2], np.int32)
    ids = oracle.topk(lg, 3, k)
    assert ids.tolist() == [[1, -1, -1], [0, 3, -1]]
    w = oracle.gate_weights(lg, ids, score_fn=score_fn, renorm=1)
    assert w[0].tolist() == [1.0, 0.0, 0.0] and w[1, 2] == 0.0
    if score_fn == 0:
        assert math.isclose(w[1, 0], 1 / (1 + math.exp(-1.5)), rel_tol=1e-15)
        assert math.isclose(w[1, 1], 1 / (1 + math.exp(1.5)), rel_tol=1e-15)
    else:
        s0, s3 = 1 / (1 + math.exp(-3.0)), 1 / (1 + math.exp(-1.5))
        assert math.isclose(w[1, 0], s0 / (s0 + s3), rel_tol=1e-15)


@pytest.mark.parametrize("mode", [0, 1])
def test_dynamic_k_align_skips_empty_slots(mode):
    rng = np.random.default_rng(23)
    T, E, K, B = 33, 8, 4, 4
    k = rng.integers(0, K + 1, size=T).astype(np.int32)
    ids = oracle.topk(rng.standard_normal((T, E)).astype(np.float32), K, k)
    r = oracle.align(ids, E, B, mode=mode)
    real = ids.ravel() >= 0
    assert np.array_equal(r["counts"], np.bincount(ids.ravel()[real], minlength=E))
    assert np.all(r["pos"][~real] == -1)
    sid = r["sorted_ids"]
    assert np.array_equal(np.sort(sid[sid >= 0]), np.nonzero(real)[0])
    for a in np.nonzero(real)[0]:
        assert sid[r["pos"][a]] == a
    n = r["counts"]
    P = int(sum(-(-int(c) // B) * B for c in n)) if mode == 0 else E * (-(-int(n.max()) // B) * B)
    assert r["P"] == P


def test_dynamic_k_combine_skips_empty_slots():
    y = np.array([[1.0, 2.0], [10.0, 20.0]], np.float32)
    pos = np.array([[1, -1], [-1, -1]], np.int32)
    out = oracle.combine(y, pos, np.array([[0.5, 0.0], [0.0, 0.0]]))
    assert out.tolist() == [[5.0, 10.0], [0.0, 0.0]]


def test_dynamic_k_layer_is_static_layer_per_token():
    # each token with k_t equals the same token through the layer with K = k_t
    # (k_t = 0: the shared FFN alone)
    x, w_r, w13, w2, sh = _small_layer(24, T=9, E=6, K=3, I_sh=16)
    k = np.array([3, 0, 1, 2, 3, 1, 0, 2, 2], np.int32)
    out = oracle.moe_layer(x, w_r, w13, w2, K=3, k=k, **sh)
    shared = oracle.dense_ffn(x, sh["w13_sh"], sh["w2_sh"])
    for t in range(9):
        if k[t] == 0:
            assert np.allclose(out[t], shared[t], rtol=1e-14, atol=1e-15)
        else:
            ref = oracle.moe_layer(x, w_r, w13, w2, K=int(k[t]), tokens=np.array([t], np.int32), **sh)[0]
            assert np.allclose(out[t], ref, rtol=1e-13, atol=1e-14)


# -------------------------------------------------------- FP8 expert weights

def test_e4m3_value_table_from_the_format():
    # 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; subnormals at exponent 0
    v = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    assert v[0x38] == 1.0 and v[0x7E] == 448.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9
    assert v[0x30] == 0.5 and v[0x3C] == 1.5 and v[0x07] == 7 * 2.0 ** -9
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.array_equal(v[0x80:0xFF], -v[0x00:0x7F])
    assert np.all(np.diff(v[0x00:0x7F]) > 0)                   # codes order the values


def test_e4m3_encode_round_trip_ties_and_saturation():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_value(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)     # every finite code, -0 included
    # ties go to the even mantissa; magnitudes past 448 saturate
    cases = {1.0625: 0x38, 1.1875: 0x3A, 2.0 ** -10: 0x00, 3 * 2.0 ** -10: 0x02, 2.0 ** -6 - 2.0 ** -10: 0x08,
             464.0: 0x7E, 1000.0: 0x7E, -1e9: 0xFE, 0.3: 0x2A}
    for v, c in cases.items():
        assert int(oracle.e4m3_encode(np.float32(v))) == c, v


def test_e4m3_encode_matches_torch_inside_the_finite_range():
    # torch's float8_e4m3fn cast (round to nearest even) is an independent
    # implementation; it turns magnitudes >= 464 into NaN, so compare below that
    rng = np.random.default_rng(31)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 200.0)]).astype(np.float32)
    v = v[np.abs(v) < 464]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_quantize_fp8_rows():
    rng = np.random.default_rng(32)
    w = (rng.standard_normal((7, 300)) * np.array([1e-3, 0.1, 1, 3, 0, 50, 1e4])[:, None]).astype(np.float32)
    q, s = oracle.quantize_fp8(w)
    assert s[4] == 1.0 and np.all(oracle.e4m3_value(q[4]) == 0)       # an all-zero row (signed zeros kept)
    amax = np.abs(w).max(1)
    for r in (0, 1, 2, 3, 5, 6):
        assert s[r] == np.float32(amax[r]) / np.float32(448.0)
        assert abs(oracle.e4m3_value(q[r][np.abs(w[r]).argmax()])) == 448.0   # the largest maps to +-448
        deq = oracle.e4m3_value(q[r]) * s[r]
        # normal range: relative error at most half a mantissa step (2^-4); below it, half the subnormal step
        bound = np.maximum(np.abs(w[r]) * 2.0 ** -4, 2.0 ** -10 * s[r]) * (1 + 1e-6)
        assert np.all(np.abs(deq - w[r]) <= bound)


def test_fp8_layer_equals_float_layer_on_representable_weights():
    # with unit scales the dequantised weights are the codes' values, exactly
    # fp32; the FP8 layer must then equal the float layer (another code path)
    rng = np.random.default_rng(33)
    T, H, E, K, I, I_sh = 9, 32, 5, 2, 24, 16
    x = rng.standard_normal((T, H)).astype(np.float32)
    w_r = rng.standard_normal((E, H)).astype(np.float32)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    codes = lambda *sh: rng.choice(finite, size=sh).astype(np.uint8)
    q13, q2, q13s, q2s = codes(E, 2 * I, H), codes(E, H, I), codes(2 * I_sh, H), codes(H, I_sh)
    scale = lambda *sh: np.full(sh, 1.0 / 64, np.float32)            # a power of two: still exact
    s13, s2, s13s, s2s = scale(E, 2 * I), scale(E, H), scale(2 * I_sh), scale(H)
    out = oracle.moe_layer_fp8(x, w_r, q13, s13, q2, s2, K, q13_sh=q13s, s13_sh=s13s, q2_sh=q2s, s2_sh=s2s)
    f = lambda q, s: (oracle.e4m3_value(q) * s[..., None]).astype(np.float32)
    ref = oracle.moe_layer(x, w_r, f(q13, s13), f(q2, s2), K, w13_sh=f(q13s, s13s), w2_sh=f(q2s, s2s))
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


# ------------------------------------------- tensor parallelism over I (oracle)

def test_tp_shard_takes_the_reading_rows_and_columns():
    # weights whose entries encode their own indices: rank 1 of 3 over I = 6
    # holds gate rows 2, 3, up rows 6 + 2, 6 + 3 and W2 columns 2, 3
    E, I, H = 2, 6, 3
    w13 = np.array([[[1000 * e + 10 * j + h for h in range(H)] for j in range(2 * I)] for e in range(E)],
                   np.float32)
    w2 = np.array([[[1000 * e + 10 * h + i for i in range(I)] for h in range(H)] for e in range(E)], np.float32)
    s13, s2 = oracle.tp_shard(w13, w2, 1, 3)
    assert s13.shape == (E, 4, H) and s2.shape == (E, H, 2)
    for e in range(E):
        assert np.array_equal(s13[e], w13[e][[2, 3, 8, 9]])
        assert np.array_equal(s2[e], w2[e][:, [2, 3]])
    d13, d2 = oracle.tp_shard(w13[1], w2[1], 2, 3)  # one dense FFN: rows 4, 5, 10, 11
    assert np.array_equal(d13, w13[1][[4, 5, 10, 11]]) and np.array_equal(d2, w2[1][:, [4, 5]])
    one13, one2 = oracle.tp_shard(w13, w2, 0, 1)
    assert np.array_equal(one13, w13) and np.array_equal(one2, w2)
    with pytest.raises(ValueError):
        oracle.tp_shard(w13, w2, 0, 4)  # 6 does not split over 4 ranks
    with pytest.raises(ValueError):
        oracle.tp_shard(w13, w2, 3, 3)


@pytest.mark.parametrize("n_ranks", [1, 2, 4])
@pytest.mark.parametrize("score_fn", [0, 1])
def test_tp_layer_sums_to_the_whole_layer(n_ranks, score_fn):
    # linearity of the FFN output in the slices of I: the ranks' outputs add
    # up to the unsplit layer (routed and shared), up to float64 rounding
    x, w_r, w13, w2, sh = _small_layer(11, T=9, E=6, K=2, I=40, I_sh=24)
    full = oracle.moe_layer(x, w_r, w13, w2, K=2, score_fn=score_fn, **sh)
    tp = oracle.moe_layer_tp(x, w_r, w13, w2, 2, n_ranks, score_fn=score_fn, **sh)
    assert np.allclose(tp, full, rtol=1e-12, atol=1e-13 * np.abs(full).max())
    if n_ranks > 1:
        parts = oracle.moe_layer_tp(x, w_r, w13, w2, 2, n_ranks, score_fn=score_fn, partials=True, **sh)
        assert len(parts) == n_ranks
        assert all(np.abs(p - full).max() > 1e-3 * np.abs(full).max() for p in parts)


def test_tp_dense_slices_sum_and_routing_is_replicated():
    x, w_r, w13, w2, sh = _small_layer(12, T=7, E=5, K=3, I=32, I_sh=16)
    d = sum(oracle.dense_ffn(x, *oracle.tp_shard(sh["w13_sh"], sh["w2_sh"], r, 4)) for r in range(4))
    ref = oracle.dense_ffn(x, sh["w13_sh"], sh["w2_sh"])
    assert np.allclose(d, ref, rtol=1e-12, atol=1e-13 * np.abs(ref).max())
    routes = [oracle.moe_layer(x, w_r, *oracle.tp_shard(w13, w2, r, 2), K=3, return_routing=True)[1:]
              for r in range(2)]
    assert np.array_equal(routes[0][0], routes[1][0]) and np.array_equal(routes[0][1], routes[1][1])


def test_tp_pin_catches_a_misaligned_up_slice():
    # a plausible slicing mistake (up rows taken without the +I offset, i.e.
    # the next gate rows) must break the sum: the pin above would catch it
    x, w_r, w13, w2, _ = _small_layer(13, T=6, E=4, K=2, I=16)
    full = oracle.moe_layer(x, w_r, w13, w2, K=2)
    wrong = np.zeros_like(full)
    for r in range(2):
        lo, hi = 8 * r, 8 * r + 8
        bad13 = np.ascontiguousarray(np.concatenate([w13[:, lo:hi], w13[:, (lo + 8) % 16:(lo + 8) % 16 + 8]], 1))
        wrong += oracle.moe_layer(x, w_r, bad13, np.ascontiguousarray(w2[..., lo:hi]), K=2)
    assert np.abs(wrong - full).max() > 1e-2 * np.abs(full).max()


# -------------------------------------------- workload shapes (input recipe)

def test_layer_shapes_are_the_pages_models():
    with open(os.path.join(GOLDEN, "layer_shapes.json")) as f:
        g = json.load(f)
    for name in ("mixtral", "qwen2moe", "deepseekv3"):
        s, want = mi.SHAPES[name], g[name]
        assert (s.H, s.I, s.E, s.K) == (want["H"], want["I"], want["E"], want["K"]), name
        assert s.I_sh == want["shared"] * want["I"], name
        assert s.dtype == "bf16"
    assert mi.SHAPES["deepseekv3"].score_fn == 1 and mi.SHAPES["mixtral"].score_fn == 0
