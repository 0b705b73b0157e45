"""Pins of the CPU oracle against what the SAS paper and the mathematics fix.

None of these tests uses a GPU. Each pin is something other than the oracle
itself: hand-derived worked examples, closed forms, invariants, special cases
that reduce to torch's scaled_dot_product_attention / log_softmax / autograd,
brute force on tiny inputs, and central finite differences.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import sas_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _val(expr: str) -> float:
    expr = expr.strip()
    if expr.startswith("ln"):
        inner = expr[2:].strip().strip("()")
        return math.log(float(Fraction(inner)))
    return float(Fraction(expr))


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _selection_inputs(B=1, Hq=2, Hkv=1, T=256, d=16, block=64, K=3, seed=0, s_scale=1.0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, Hq, T, d))
    Kt = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d))
    dO = rng.standard_normal((B, Hq, T, d))
    NB = T // block
    s = s_scale * rng.standard_normal((B, Hkv, T, NB))
    logG = orc.gate_normalize(s, block)
    tau, tidx, sel = orc.select_threshold(logG, K, block)
    return Q, Kt, V, dO, s, logG, tau, tidx, sel


# ---------------------------------------------------------------- worked examples
@pytest.mark.parametrize("case_idx", [0, 1, 2])
def test_worked_example(case_idx):
    gold = json.load(open(GOLDEN))
    case = gold["cases"][case_idx]
    block, T = gold["block"], gold["T"]
    NB = T // block
    s = np.zeros((1, 1, T, NB))
    for r, vals in case["s_rows"].items():
        s[0, 0, int(r)] = vals
    logG = orc.gate_normalize(s, block)
    tau, tidx, _ = orc.select_threshold(logG, case["K"], block)
    Q = np.zeros((1, 1, T, 1))
    Kt = np.ones((1, 1, T, 1))
    V = np.asarray(gold["v"], float).reshape(1, 1, T, 1)
    dO = np.asarray(case["dO"], float).reshape(1, 1, T, 1)
    out = orc.forward_backward(Q, Kt, V, dO, logG, tau, tidx, block, 1.0)
    np.testing.assert_allclose(out["O"][0, 0, :, 0], [_val(x) for x in case["O"]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["LSE"][0, 0], [_val(x) for x in case["LSE"]], rtol=0, atol=1e-12)
    if "dLogG_row4" in case:
        np.testing.assert_allclose(out["dLogG"][0, 0, 4], [_val(x) for x in case["dLogG_row4"]], atol=1e-12)
        np.testing.assert_allclose(out["dV"][0, 0, :, 0], [_val(x) for x in case["dV"]], atol=1e-12)
        np.testing.assert_allclose(out["dQ"][0, 0, 4, 0], _val(case["dQ_row4"]), atol=1e-12)
        others = np.delete(out["dLogG"][0, 0], 4, axis=0)
        assert np.all(others == 0.0)


# ---------------------------------------------------------------- gate normalisation
def test_normalize_matches_log_softmax_prefix():
    block, T = 16, 160
    s = _rand((2, 3, T, T // block), 1)
    logG = orc.gate_normalize(s, block)
    st = torch.from_numpy(s)
    for t in range(T):
        c = t // block
        assert np.all(np.isneginf(logG[:, :, t, c:]))
        if c:
            ref = F.log_softmax(st[:, :, t, :c], dim=-1).numpy()
            np.testing.assert_allclose(logG[:, :, t, :c], ref, rtol=1e-13, atol=1e-13)


def test_gate_lse_matches_torch_logsumexp_prefix():
    """The compact gates' row normaliser is torch.logsumexp over the causal block prefix, -inf with no
    history; with it the raw scores give back gate_normalize's log gates (eq. 6)."""
    block, T = 16, 112
    s = 3.0 * _rand((2, 2, T, T // block), 21)
    lse = orc.gate_lse(s, block)
    st = torch.from_numpy(s)
    for t in range(T):
        c = t // block
        if c == 0:
            assert np.all(np.isneginf(lse[:, :, t]))
            continue
        ref = torch.logsumexp(st[:, :, t, :c], dim=-1).numpy()
        assert np.allclose(lse[:, :, t], ref, rtol=0, atol=1e-12)
    lg = orc.gate_normalize(s, block)
    c_t = np.arange(T) // block
    hist = np.arange(T // block)[None, :] < c_t[:, None]
    assert np.allclose(np.where(hist, s - lse[..., None], -np.inf)[..., hist], lg[..., hist], rtol=0, atol=1e-12)


def test_gate_lse_pin_catches_a_planted_mistake():
    """A normaliser over the wrong prefix (the current block included) fails the logsumexp pin."""
    block, T = 16, 80
    s = _rand((1, 1, T, T // block), 22)
    wrong = np.array([[[np.logaddexp.reduce(s[0, 0, t, :t // block + 1]) if t >= block else -np.inf
                        for t in range(T)]]])
    ref = torch.logsumexp(torch.from_numpy(s)[0, 0, 40, :40 // block], dim=-1).item()
    assert abs(orc.gate_lse(s, block)[0, 0, 40] - ref) < 1e-12
    assert abs(wrong[0, 0, 40] - ref) > 1e-3


def test_normalize_shift_invariance_and_unit_mass():
    block, T = 8, 96
    s = _rand((1, 2, T, T // block), 2) * 3
    a = orc.gate_normalize(s, block)
    b = orc.gate_normalize(s + 123.25, block)
    fin = np.isfinite(a)
    np.testing.assert_allclose(a[fin], b[fin], atol=1e-11)
    for t in range(block, T):
        c = t // block
        np.testing.assert_allclose(np.exp(a[:, :, t, :c]).sum(-1), 1.0, atol=1e-13)


# ---------------------------------------------------------------- top-k threshold
def _brute_force_topk(vals, c, H):
    """The unique H-subset whose every member beats every non-member under
    (value descending, index ascending); found by enumerating all subsets."""
    if min(c, H) == 0:
        return []
    if c <= H:
        return list(range(c))

    def beats(a, b):
        return vals[a] > vals[b] or (vals[a] == vals[b] and a < b)

    found = [sub for sub in itertools.combinations(range(c), H)
             if all(beats(a, b) for a in sub for b in range(c) if b not in sub)]
    assert len(found) == 1
    return list(found[0])


@pytest.mark.parametrize("H", [0, 1, 2, 3, 5])
def test_select_brute_force_with_ties(H):
    rng = np.random.default_rng(H)
    for trial in range(150):
        c = int(rng.integers(0, 9))
        vals = rng.integers(-2, 3, size=9).astype(np.float64)   # many ties
        if trial % 3 == 0:
            vals[rng.integers(0, 9)] = -0.0
            vals[rng.integers(0, 9)] = 0.0
        tau, tidx, chosen = orc.topk_threshold_row(vals, c, H)
        assert chosen == _brute_force_topk(vals, c, H)
        # The threshold pair reproduces the chosen set through the predicate.
        pred = [m for m in range(c) if vals[m] > tau or (vals[m] == tau and m <= tidx)]
        assert pred == chosen


def test_select_matches_lexsort_and_mask():
    block, T, K = 16, 256, 5
    s = _rand((2, 2, T, T // block), 3)
    logG = orc.gate_normalize(s, block).astype(np.float32).astype(np.float64)
    tau, tidx, sel = orc.select_threshold(logG, K, block)
    mask = orc.selection_mask(logG, tau, tidx, block)
    for b in range(2):
        for g in range(2):
            for t in range(T):
                c = t // block
                vals = logG[b, g, t, :c]
                ref = sorted(np.lexsort((np.arange(c), -vals))[: K - 1].tolist()) if c else []
                got = [m for m in sel[b, g, t] if m >= 0]
                assert got == ref
                assert np.flatnonzero(mask[b, g, t]).tolist() == ref


def test_select_signed_zero_ties():
    vals = np.array([0.0, -0.0, 0.0, -1.0, -0.0])
    tau, tidx, chosen = orc.topk_threshold_row(vals, 5, 2)
    assert chosen == [0, 1] and tau == 0.0 and tidx == 1


# ---------------------------------------------------------------- forward special cases
def _sdpa(Q, K, V, mask, sm_scale, G):
    q = torch.from_numpy(Q)
    k = torch.from_numpy(K).repeat_interleave(G, dim=1)
    v = torch.from_numpy(V).repeat_interleave(G, dim=1)
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=sm_scale).numpy()


def test_unit_gates_full_budget_is_dense_causal():
    B, Hq, Hkv, T, d, block = 1, 4, 2, 192, 16, 32
    rng = np.random.default_rng(4)
    Q, K, V = rng.standard_normal((B, Hq, T, d)), rng.standard_normal((B, Hkv, T, d)), rng.standard_normal((B, Hkv, T, d))
    logG = np.zeros((B, Hkv, T, T // block))        # unit gates
    tau, tidx, _ = orc.select_threshold(logG, T // block, block)
    O, LSE = orc.forward(Q, K, V, logG, tau, tidx, block, 0.25)
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    np.testing.assert_allclose(O, _sdpa(Q, K, V, causal, 0.25, Hq // Hkv), atol=1e-12)
    z = 0.25 * np.einsum("bhtd,bhsd->bhts", Q, np.repeat(K, 2, axis=1))
    z = np.where(causal.numpy(), z, -np.inf)
    np.testing.assert_allclose(LSE, torch.logsumexp(torch.from_numpy(z), -1).numpy(), atol=1e-12)


def test_budget_one_is_current_block_only():
    B, Hq, Hkv, T, d, block = 2, 2, 1, 128, 8, 16
    Q, K, V, _, s, logG, _, _, _ = _selection_inputs(B, Hq, Hkv, T, d, block, 1, seed=5)
    tau, tidx, _ = orc.select_threshold(logG, 1, block)
    O, _ = orc.forward(Q, K, V, logG, tau, tidx, block, 0.3)
    i = torch.arange(T)
    mask = (i[:, None] >= i[None, :]) & (i[:, None] // block == i[None, :] // block)
    np.testing.assert_allclose(O, _sdpa(Q, K, V, mask, 0.3, Hq), atol=1e-12)


def test_uniform_scores_full_budget_is_causal_with_log_count_bias():
    B, Hq, Hkv, T, d, block = 1, 2, 1, 160, 8, 32
    rng = np.random.default_rng(6)
    Q, K, V = rng.standard_normal((B, Hq, T, d)), rng.standard_normal((B, Hkv, T, d)), rng.standard_normal((B, Hkv, T, d))
    s = np.full((B, Hkv, T, T // block), 0.7)
    logG = orc.gate_normalize(s, block)
    tau, tidx, _ = orc.select_threshold(logG, T // block, block)
    O, _ = orc.forward(Q, K, V, logG, tau, tidx, block, 0.5)
    i = np.arange(T)
    c = i // block
    # Uniform softmax gates: each of the c_t historical blocks has g = 1/c_t.
    bias = np.where(i[None, :] // block < c[:, None], -np.log(np.maximum(c[:, None], 1)), 0.0)
    bias = np.where(i[None, :] <= i[:, None], bias, -np.inf)
    np.testing.assert_allclose(O, _sdpa(Q, K, V, torch.from_numpy(bias), 0.5, Hq), atol=1e-12)


def test_materialised_equals_gathered_rows():
    Q, K, V, dO, s, logG, tau, tidx, sel = _selection_inputs(1, 4, 2, 256, 16, 32, 3, seed=7)
    full = orc.forward_backward(Q, K, V, dO, logG, tau, tidx, 32, 0.25)
    for g in range(2):
        rows = np.arange(0, 256, 7)
        gat = orc.rows_gathered(Q, K, V, dO, logG, sel, 0, g, rows, 32, 0.25)
        for hh in range(2):
            h = g * 2 + hh
            np.testing.assert_allclose(gat["O"][hh], full["O"][0, h, rows], atol=1e-12)
            np.testing.assert_allclose(gat["LSE"][hh], full["LSE"][0, h, rows], atol=1e-12)
            np.testing.assert_allclose(gat["dQ"][hh], full["dQ"][0, h, rows], atol=1e-12)
        np.testing.assert_allclose(gat["dLogG"], full["dLogG"][0, g, rows], atol=1e-12)
        for j in range(256 // 32):
            dK, dV = orc.kv_block_gathered(Q, K, V, dO, logG, sel, 0, g, j, 32, 0.25)
            np.testing.assert_allclose(dK, full["dK"][0, g, j * 32:(j + 1) * 32], atol=1e-11)
            np.testing.assert_allclose(dV, full["dV"][0, g, j * 32:(j + 1) * 32], atol=1e-11)


def test_row_subset_matches_full():
    Q, K, V, dO, s, logG, tau, tidx, sel = _selection_inputs(1, 2, 1, 128, 8, 16, 3, seed=8)
    full = orc.forward_backward(Q, K, V, dO, logG, tau, tidx, 16, 0.4)
    rows = np.array([0, 15, 16, 17, 63, 100, 127])
    sub = orc.forward_backward(Q, K, V, dO, logG, tau, tidx, 16, 0.4, rows=rows)
    for k in ("O", "LSE", "dQ"):
        np.testing.assert_allclose(sub[k], full[k][:, :, rows], atol=1e-13)
    np.testing.assert_allclose(sub["dLogG"], full["dLogG"][:, :, rows], atol=1e-13)


def test_attention_weights_bounded_and_lse_finite():
    Q, K, V, dO, s, logG, tau, tidx, sel = _selection_inputs(1, 2, 1, 128, 8, 16, 2, seed=9, s_scale=4.0)
    _, LSE = orc.forward(Q, K, V, logG, tau, tidx, 16, 3.0)
    assert np.all(np.isfinite(LSE))
    # p_i = exp(z_i - LSE) <= 1 (eq. 7): every logit is at most the row LSE.
    mask = orc.selection_mask(logG, tau, tidx, 16)
    for h in range(2):
        z = 3.0 * Q[0, h] @ K[0, 0].T + orc.bias_rows(logG[0, 0], mask[0, 0], np.arange(128), 128, 16)
        assert np.all(z <= LSE[0, h][:, None] + 1e-12)


# ---------------------------------------------------------------- backward
def _loss(Q, K, V, dO, logG, tau, tidx, block, sm):
    O, _ = orc.forward(Q, K, V, logG, tau, tidx, block, sm)
    return float((O * dO).sum())


@pytest.mark.parametrize("Kbud", [2, 3])
def test_backward_central_finite_differences(Kbud):
    B, Hq, Hkv, T, d, block, sm = 1, 2, 1, 256, 16, 64, 0.25
    Q, K, V, dO, s, logG, tau, tidx, sel = _selection_inputs(B, Hq, Hkv, T, d, block, Kbud, seed=10 + Kbud)
    out = orc.forward_backward(Q, K, V, dO, logG, tau, tidx, block, sm)
    rng = np.random.default_rng(Kbud)
    eps = 1e-6

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + eps
        lp = _loss(Q, K, V, dO, logG, tau, tidx, block, sm)
        arr[idx] = old - eps
        lm = _loss(Q, K, V, dO, logG, tau, tidx, block, sm)
        arr[idx] = old
        return (lp - lm) / (2 * eps)

    for name, arr, grad in (("Q", Q, out["dQ"]), ("K", K, out["dK"]), ("V", V, out["dV"])):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            assert abs(fd(arr, idx) - grad[idx]) < 1e-6 * max(1.0, abs(grad[idx])), name
    # Selected log-gate entries, with the selected set held fixed: an entry that
    # is the threshold itself carries tau along with it.
    mask = orc.selection_mask(logG, tau, tidx, block)
    picks = np.argwhere(mask)
    assert len(picks) > 0

    def fd_gate(idx):
        row = idx[:3]
        at_tau = logG[idx] == tau[row]
        vals = []
        for sgn in (1.0, -1.0):
            old_g, old_t = logG[idx], tau[row]
            logG[idx] = old_g + sgn * eps
            if at_tau:
                tau[row] = logG[idx]
            assert np.array_equal(orc.selection_mask(logG, tau, tidx, block), mask)
            vals.append(_loss(Q, K, V, dO, logG, tau, tidx, block, sm))
            logG[idx], tau[row] = old_g, old_t
        return (vals[0] - vals[1]) / (2 * eps)

    for k in rng.choice(len(picks), size=min(10, len(picks)), replace=False):
        idx = tuple(int(x) for x in picks[k])
        assert abs(fd_gate(idx) - out["dLogG"][idx]) < 1e-6 * max(1.0, abs(out["dLogG"][idx]))
    assert np.all(out["dLogG"][~mask] == 0.0)


def test_backward_unit_gates_matches_autograd_causal_sdpa():
    B, Hq, Hkv, T, d, block, sm = 1, 4, 2, 128, 8, 32, 0.35
    rng = np.random.default_rng(11)
    Q, K, V, dO = (rng.standard_normal(s) for s in ((B, Hq, T, d), (B, Hkv, T, d), (B, Hkv, T, d), (B, Hq, T, d)))
    logG = np.zeros((B, Hkv, T, T // block))
    tau, tidx, _ = orc.select_threshold(logG, T // block, block)
    out = orc.forward_backward(Q, K, V, dO, logG, tau, tidx, block, sm)
    q, k, v = (torch.from_numpy(a).requires_grad_() for a in (Q, K, V))
    o = F.scaled_dot_product_attention(q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), is_causal=True, scale=sm)
    (o * torch.from_numpy(dO)).sum().backward()
    np.testing.assert_allclose(out["dQ"], q.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(out["dK"], k.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(out["dV"], v.grad.numpy(), atol=1e-12)


def test_gate_gradient_eq5_closed_form_and_zero_sum():
    B, Hq, Hkv, T, d, block, sm = 1, 2, 1, 128, 8, 16, 0.5
    Q, K, V, dO, s, logG, tau, tidx, sel = _selection_inputs(B, Hq, Hkv, T, d, block, 3, seed=12)
    out = orc.forward_backward(Q, K, V, dO, logG, tau, tidx, block, sm)
    mask = orc.selection_mask(logG, tau, tidx, block)
    own_total = np.zeros(T)
    for h in range(Hq):
        z = sm * Q[0, h] @ K[0, 0].T + orc.bias_rows(logG[0, 0], mask[0, 0], np.arange(T), T, block)
        p = np.exp(z - out["LSE"][0, h][:, None])
        o = out["O"][0, h]
        # eq. 5 (inner gate) times g_m: d log g_m = sum_{i in B_m} p_i do.(v_i - o)
        w = p * (dO[0, h] @ V[0, 0].T - (dO[0, h] * o).sum(1, keepdims=True))
        for t in range(T):
            c = t // block
            own_total[t] += w[t, c * block:t + 1].sum()
    eq5 = np.zeros((T, T // block))
    for h in range(Hq):
        z = sm * Q[0, h] @ K[0, 0].T + orc.bias_rows(logG[0, 0], mask[0, 0], np.arange(T), T, block)
        p = np.exp(z - out["LSE"][0, h][:, None])
        o = out["O"][0, h]
        for t in range(T):
            for m in range(t // block):
                if mask[0, 0, t, m]:
                    sl = slice(m * block, (m + 1) * block)
                    eq5[t, m] += (p[t, sl] * ((V[0, 0, sl] - o[t]) @ dO[0, h, t])).sum()
    np.testing.assert_allclose(out["dLogG"][0, 0], eq5, atol=1e-12)
    # sum_i dS_i = 0 per row: the selected blocks' gradients cancel the current block's.
    np.testing.assert_allclose(out["dLogG"][0, 0].sum(1), -own_total, atol=1e-12)


# ---------------------------------------------------------------- decode
def test_decode_full_budget_is_dense_attention_and_topk_bruteforce():
    B, Hq, Hkv, L, d, block = 3, 4, 2, 200, 16, 16
    rng = np.random.default_rng(13)
    q = rng.standard_normal((B, Hq, d))
    Kc, Vc = rng.standard_normal((B, Hkv, L, d)), rng.standard_normal((B, Hkv, L, d))
    s = np.round(rng.standard_normal((B, Hkv, (L + block - 1) // block)), 1)   # rounded: ties happen
    seqlen = np.array([200, 129, 17])
    o, sel = orc.decode(q, Kc, Vc, seqlen, s, 100, block, 0.25)
    for b in range(B):
        Lb = int(seqlen[b])
        ref = F.scaled_dot_product_attention(
            torch.from_numpy(q[b][:, None]), torch.from_numpy(Kc[b, :, :Lb]).repeat_interleave(2, 0),
            torch.from_numpy(Vc[b, :, :Lb]).repeat_interleave(2, 0), scale=0.25)[:, 0].numpy()
        np.testing.assert_allclose(o[b], ref, atol=1e-12)
    o, sel = orc.decode(q, Kc, Vc, seqlen, s, 4, block, 0.25)
    for b in range(B):
        c = (int(seqlen[b]) - 1) // block
        for g in range(Hkv):
            got = [m for m in sel[b, g] if m >= 0]
            assert got == _brute_force_topk(s[b, g], c, 3)
            keys = np.zeros(L, bool)
            for m in got:
                keys[m * block:(m + 1) * block] = True
            keys[c * block:int(seqlen[b])] = True
            ref = F.scaled_dot_product_attention(
                torch.from_numpy(q[b, 2 * g:2 * g + 2][:, None]), torch.from_numpy(Kc[b, g][None].repeat(2, 0)),
                torch.from_numpy(Vc[b, g][None].repeat(2, 0)), attn_mask=torch.from_numpy(keys)[None], scale=0.25)[:, 0].numpy()
            np.testing.assert_allclose(o[b, 2 * g:2 * g + 2], ref, atol=1e-12)


def test_decode_with_log_gate_equals_training_last_row():
    B, Hq, Hkv, T, d, block, Kb = 1, 2, 1, 192, 8, 32, 3
    rng = np.random.default_rng(14)
    Q, K, V = rng.standard_normal((B, Hq, T, d)), rng.standard_normal((B, Hkv, T, d)), rng.standard_normal((B, Hkv, T, d))
    s = rng.standard_normal((B, Hkv, T, T // block))
    logG = orc.gate_normalize(s, block)
    tau, tidx, _ = orc.select_threshold(logG, Kb, block)
    O, _ = orc.forward(Q, K, V, logG, tau, tidx, block, 0.3)
    o, _ = orc.decode(Q[:, :, T - 1], K, V, np.array([T]), s[:, :, T - 1], Kb, block, 0.3, apply_log_gate=True)
    np.testing.assert_allclose(o, O[:, :, T - 1], atol=1e-12)


# ---------------------------------------------------------------- the pins catch planted mistakes
def _bad_normalize(s, block):
    """Mistake: raw scores used as log-gates (the LSE is not subtracted)."""
    out = np.full(np.shape(s), -np.inf)
    for t in range(np.shape(s)[2]):
        c = t // block
        out[:, :, t, :c] = np.asarray(s, float)[:, :, t, :c]
    return out


def _bad_topk(vals, c, H):
    """Mistake: ties broken toward the higher block index."""
    if min(c, H) == 0:
        return math.inf, -1, []
    if c <= H:
        return -math.inf, c - 1, list(range(c))
    order = sorted(range(c), key=lambda m: (-float(vals[m]), -m))
    taken = order[:H]
    tau = float(vals[taken[-1]])
    return tau, max(m for m in taken if float(vals[m]) == tau), sorted(taken)


_good_bias = orc.bias_rows


def _bad_bias_causal(logG_g, mask_g, rows, T, block):
    """Mistake: the current block lets each query see one key past itself."""
    b = _good_bias(logG_g, mask_g, rows, T, block)
    rows = np.asarray(rows)
    nxt = np.minimum(rows + 1, T - 1)
    same = (nxt // block) == (rows // block)
    b[np.arange(len(rows))[same], nxt[same]] = 0.0
    return b


def _bad_bias_sign(logG_g, mask_g, rows, T, block):
    """Mistake: the log-gate enters the logits with the wrong sign."""
    b = _good_bias(logG_g, mask_g, rows, T, block)
    fin = np.isfinite(b) & (b != 0.0)
    b[fin] = -b[fin]
    return b


@pytest.mark.parametrize("mistake,target", [
    ("gate_normalize", lambda: test_worked_example(0)),
    ("topk_threshold_row", lambda: test_worked_example(2)),
    ("bias_causal", test_unit_gates_full_budget_is_dense_causal),
    ("bias_sign", test_uniform_scores_full_budget_is_causal_with_log_count_bias),
    ("bias_sign", lambda: test_worked_example(0)),
])
def test_pins_catch_planted_mistakes(monkeypatch, mistake, target):
    bad = {"gate_normalize": ("gate_normalize", _bad_normalize),
           "topk_threshold_row": ("topk_threshold_row", _bad_topk),
           "bias_causal": ("bias_rows", _bad_bias_causal),
           "bias_sign": ("bias_rows", _bad_bias_sign)}[mistake]
    monkeypatch.setattr(orc, bad[0], bad[1])
    with pytest.raises(AssertionError):
        target()


# ---------------------------------------------------------------- selector-score gradient
def _gate_loss(s, w, block):
    lg = orc.gate_normalize(s, block)
    return float(np.sum(np.where(np.isfinite(lg), lg * w, 0.0)))


def test_gate_grad_matches_central_differences():
    """ds from gate_grad against central differences of L(s) = sum_m w_m logG_m(s) on every entry."""
    rng = np.random.default_rng(11)
    block, T, NB = 4, 20, 5
    s = rng.standard_normal((1, 2, T, NB)) * 1.5
    w = rng.standard_normal((1, 2, T, NB))
    ds = orc.gate_grad(s, w, block)
    h = 1e-6
    fd = np.zeros_like(s)
    for idx in np.ndindex(s.shape):
        sp, sm = s.copy(), s.copy()
        sp[idx] += h
        sm[idx] -= h
        fd[idx] = (_gate_loss(sp, w, block) - _gate_loss(sm, w, block)) / (2 * h)
    np.testing.assert_allclose(ds, fd, atol=1e-8)


def test_gate_grad_rows_sum_to_zero_and_single_block_rows_vanish():
    """Shifting a row of s by a constant leaves logG unchanged, so each row of ds sums to zero; a row with a
    single historical block has logG = 0 whatever s is, so its ds is zero; future blocks get zero."""
    rng = np.random.default_rng(12)
    block, T, NB = 8, 64, 8
    s = rng.standard_normal((2, 1, T, NB))
    d = rng.standard_normal((2, 1, T, NB))
    ds = orc.gate_grad(s, d, block)
    np.testing.assert_allclose(ds.sum(axis=-1), 0.0, atol=1e-12)
    one = (np.arange(T) // block) == 1
    assert np.all(ds[:, :, one] == 0.0)
    c = (np.arange(T) // block)[None, None, :, None]
    assert np.all(ds[np.broadcast_to(np.arange(NB)[None, None, None, :] >= c, ds.shape)] == 0.0)


def _bad_gate_grad(s, dLogG, block):
    """Mistake: the softmax Jacobian applied without the gate weights (ds = dLogG - mean(dLogG))."""
    s = np.asarray(s, float)
    d = np.asarray(dLogG, float)
    ds = np.zeros(s.shape)
    for t in range(s.shape[2]):
        c = min(t // block, s.shape[3])
        if c:
            ds[:, :, t, :c] = d[:, :, t, :c] - d[:, :, t, :c].mean(axis=-1, keepdims=True)
    return ds


def test_gate_grad_pin_catches_planted_mistake(monkeypatch):
    monkeypatch.setattr(orc, "gate_grad", _bad_gate_grad)
    with pytest.raises(AssertionError):
        test_gate_grad_matches_central_differences()


# ---------------------------------------------------------------- paged decode
def _paged_layout(Kc, Vc, seqlen, block, rng, spare=5):
    """Scatter a contiguous cache into a shuffled pool of one-block pages (plus unused pages)."""
    B, Hkv, Lmax, d = Kc.shape
    max_pages = Lmax // block
    used = [(b, m) for b in range(B) for m in range((int(seqlen[b]) + block - 1) // block)]
    num_pages = len(used) + spare
    perm = rng.permutation(num_pages)
    Kp = rng.standard_normal((num_pages, Hkv, block, d))     # unused pages hold noise
    Vp = rng.standard_normal((num_pages, Hkv, block, d))
    pt = np.full((B, max_pages), -1, dtype=np.int32)
    for i, (b, m) in enumerate(used):
        pt[b, m] = perm[i]
        Kp[perm[i]] = Kc[b, :, m * block:(m + 1) * block]
        Vp[perm[i]] = Vc[b, :, m * block:(m + 1) * block]
    return Kp, Vp, pt


def test_paged_decode_equals_contiguous_decode_under_a_page_shuffle():
    B, Hq, Hkv, Lmax, d, block = 3, 4, 2, 256, 8, 16
    rng = np.random.default_rng(21)
    q = rng.standard_normal((B, Hq, d))
    Kc, Vc = rng.standard_normal((B, Hkv, Lmax, d)), rng.standard_normal((B, Hkv, Lmax, d))
    seqlen = np.array([256, 131, 16])
    s = rng.standard_normal((B, Hkv, Lmax // block))
    Kp, Vp, pt = _paged_layout(Kc, Vc, seqlen, block, rng)
    for Kb, gate in ((4, False), (3, True), (100, False)):
        o_ref, sel_ref = orc.decode(q, Kc, Vc, seqlen, s, Kb, block, 0.3, apply_log_gate=gate)
        o, sel = orc.decode_paged(q, Kp, Vp, pt, seqlen, s, Kb, block, 0.3, apply_log_gate=gate)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        assert np.array_equal(sel, sel_ref)
    # the logical cache itself, token by token
    Kl = orc.paged_cache(Kp, pt, block)
    for b in range(B):
        for p in range(int(seqlen[b])):
            np.testing.assert_array_equal(Kl[b, :, p], Kc[b, :, p])


def _bad_paged_cache(pool, page_table, block):
    """Mistake: the page table read with sequence and block swapped."""
    pool = np.asarray(pool, float)
    B, max_pages = page_table.shape
    out = np.zeros((B, pool.shape[1], max_pages * block, pool.shape[3]))
    for b in range(B):
        for m in range(max_pages):
            pg = int(page_table.T.reshape(B, max_pages)[b, m])
            if pg >= 0:
                out[b, :, m * block:(m + 1) * block] = pool[pg]
    return out


def test_paged_pin_catches_planted_mistake(monkeypatch):
    monkeypatch.setattr(orc, "paged_cache", _bad_paged_cache)
    with pytest.raises(AssertionError):
        test_paged_decode_equals_contiguous_decode_under_a_page_shuffle()


# ---------------------------------------------------------------- noisy (full*) selection
def test_select_noisy_without_noise_is_the_plain_selection():
    rng = np.random.default_rng(31)
    B, Hkv, T, NB, block, K = 1, 2, 320, 5, 64, 3
    logG32 = orc.gate_normalize(rng.standard_normal((B, Hkv, T, NB)), block).astype(np.float32)
    logG_sel, tau, tidx, sel = orc.select_noisy(logG32, np.zeros_like(logG32), K, block)
    t2, i2, s2 = orc.select_threshold(logG32.astype(np.float64), K, block)
    assert np.array_equal(tau, t2) and np.array_equal(tidx, i2) and np.array_equal(sel, s2)
    mask = orc.selection_mask(logG32, t2, i2, block)
    assert np.array_equal(logG_sel, np.where(mask, logG32.astype(np.float64), -np.inf))


def test_select_noisy_brute_force_and_predicate():
    """Tiny rows with integer-valued keys (many ties): the chosen set is the first H blocks under
    (key descending, block ascending) by brute force over all subsets, and the threshold of logG_sel
    picks exactly that set again."""
    rng = np.random.default_rng(32)
    B, Hkv, T, NB, block, K = 1, 1, 8 * 4, 7, 4, 4
    logG32 = rng.integers(-3, 3, size=(B, Hkv, T, NB)).astype(np.float32)
    noise32 = rng.integers(-2, 3, size=(B, Hkv, T, NB)).astype(np.float32)
    logG_sel, tau, tidx, sel = orc.select_noisy(logG32, noise32, K, block)
    keys = logG32 + noise32
    mask = orc.selection_mask(logG_sel, tau, tidx, block)
    for t in range(T):
        c = min(t // block, NB)
        want = _brute_force_topk(keys[0, 0, t].astype(np.float64), c, K - 1)
        assert [m for m in sel[0, 0, t] if m >= 0] == want
        assert sorted(np.nonzero(mask[0, 0, t])[0].tolist()) == want
        for m in range(NB):
            expect = float(logG32[0, 0, t, m]) if m in want else -np.inf
            assert logG_sel[0, 0, t, m] == expect


def test_select_noisy_planted_noise_wins_and_keys_are_fp32():
    B, Hkv, NB, block, K = 1, 1, 6, 2, 4
    T = block * (NB + 1)
    logG32 = np.tile(np.linspace(0.0, -5.0, NB, dtype=np.float32), (B, Hkv, T, 1))
    noise32 = np.zeros_like(logG32)
    noise32[..., [1, 3, 5]] = 100.0            # the three lowest gates but the largest keys
    _, _, _, sel = orc.select_noisy(logG32, noise32, K, block)
    assert sel[0, 0, T - 1].tolist() == [1, 3, 5]
    # keys formed in float32: 1 + 2^-24 rounds to 1, a tie that goes to the lower block
    lg = np.ones((1, 1, 3 * block, 2), np.float32)     # last row: c = 2 historical blocks, H = 1
    nz = np.zeros_like(lg)
    nz[..., 1] = 2.0 ** -24
    assert np.float64(1.0) + 2.0 ** -24 > 1.0          # in float64 block 1 would win
    _, _, _, sel = orc.select_noisy(lg, nz, 2, block)
    assert sel[0, 0, 3 * block - 1, 0] == 0


def _bad_select_noisy(logG32, noise32, K, block):
    """Mistake: the noise ignored (the clean Top-K)."""
    return _real_select_noisy(logG32, np.zeros_like(np.asarray(logG32, np.float32)), K, block)


_real_select_noisy = orc.select_noisy


def test_select_noisy_pin_catches_planted_mistake(monkeypatch):
    monkeypatch.setattr(orc, "select_noisy", _bad_select_noisy)
    with pytest.raises(AssertionError):
        test_select_noisy_planted_noise_wins_and_keys_are_fp32()


# ---------------------------------------------------------------- variable-length packing
def _packed_from_docs(docs, block, rng, NB_extra=0):
    """Pack per-document inputs (each its own problem) along T; score columns of other documents get noise."""
    B, Hq, Hkv, d = 1, 4, 2, 8
    cu = np.cumsum([0] + [L for L in docs])
    T = int(cu[-1])
    NB = T // block + NB_extra
    per = []
    Q = rng.standard_normal((B, Hq, T, d))
    Kt, Vt, dO = rng.standard_normal((B, Hkv, T, d)), rng.standard_normal((B, Hkv, T, d)), rng.standard_normal((B, Hq, T, d))
    s = rng.standard_normal((B, Hkv, T, NB)) * 5.0 + 50.0       # leaked columns would dominate
    for i, L in enumerate(docs):
        a = int(cu[i])
        sd = rng.standard_normal((B, Hkv, L, L // block))
        s[:, :, a:a + L, a // block:a // block + L // block] = sd
        per.append((slice(a, a + L), sd))
    return Q, Kt, Vt, dO, s, cu, per


def test_varlen_equals_each_document_alone():
    rng = np.random.default_rng(41)
    block, Kb, sm = 16, 3, 0.3
    docs = [48, 16, 80]
    Q, Kt, Vt, dO, s, cu, per = _packed_from_docs(docs, block, rng, NB_extra=2)
    logG = orc.gate_normalize_varlen(s, cu, block)
    out = orc.forward_backward_varlen(Q, Kt, Vt, dO, logG, Kb, cu, block, sm)
    mask = orc.selection_mask_varlen(logG, Kb, cu, block)
    for ts, sd in per:
        lg = orc.gate_normalize(sd, block)
        tau, tidx, _ = orc.select_threshold(lg, Kb, block)
        ref = orc.forward_backward(Q[:, :, ts], Kt[:, :, ts], Vt[:, :, ts], dO[:, :, ts], lg, tau, tidx, block, sm)
        b0 = ts.start // block
        nb = lg.shape[-1]
        np.testing.assert_array_equal(logG[:, :, ts, b0:b0 + nb], lg)
        assert np.all(np.isneginf(np.delete(logG[:, :, ts], np.s_[b0:b0 + nb], axis=-1)))
        np.testing.assert_array_equal(mask[:, :, ts, b0:b0 + nb], orc.selection_mask(lg, tau, tidx, block))
        for k in ("O", "LSE", "dQ", "dK", "dV"):
            np.testing.assert_allclose(out[k][:, :, ts], ref[k], atol=1e-12)
        np.testing.assert_allclose(out["dLogG"][:, :, ts, b0:b0 + nb], ref["dLogG"], atol=1e-12)
    assert not mask[..., sum(docs) // block:].any()


def test_varlen_uniform_scores_full_budget_is_block_diagonal_sdpa():
    """Uniform scores and a budget covering every block: each document is causal attention with a
    -log(historical blocks of its own) bias on its earlier blocks, and nothing across documents."""
    B, Hq, Hkv, d, block = 1, 2, 1, 8, 16
    docs = [32, 64, 48]
    T = sum(docs)
    rng = np.random.default_rng(42)
    Q, K, V = rng.standard_normal((B, Hq, T, d)), rng.standard_normal((B, Hkv, T, d)), rng.standard_normal((B, Hkv, T, d))
    dO = rng.standard_normal((B, Hq, T, d))
    cu = np.cumsum([0] + docs)
    s = np.full((B, Hkv, T, T // block), 0.4)
    logG = orc.gate_normalize_varlen(s, cu, block)
    out = orc.forward_backward_varlen(Q, K, V, dO, logG, T // block, cu, block, 0.5)
    i = np.arange(T)
    doc = np.searchsorted(cu, i, side="right") - 1
    start_blk = cu[doc] // block
    c = i // block
    same = doc[:, None] == doc[None, :]
    hist = (i[None, :] // block < c[:, None]) & same
    bias = np.where(hist, -np.log(np.maximum(c - start_blk, 1))[:, None], 0.0)
    bias = np.where((i[None, :] <= i[:, None]) & same, bias, -np.inf)
    np.testing.assert_allclose(out["O"], _sdpa(Q, K, V, torch.from_numpy(bias), 0.5, Hq), atol=1e-12)


def _bad_gate_normalize_varlen(s, cu_seqlens, block):
    """Mistake: each document's gates read from the first block columns instead of its own."""
    s = np.asarray(s, float)
    out = np.full(s.shape, -np.inf)
    for ts, bs in orc.doc_slices(cu_seqlens, block):
        nb = bs.stop - bs.start
        out[:, :, ts, bs] = orc.gate_normalize(s[:, :, ts, :nb], block)
    return out


def test_varlen_pin_catches_planted_mistake(monkeypatch):
    monkeypatch.setattr(orc, "gate_normalize_varlen", _bad_gate_normalize_varlen)
    with pytest.raises(AssertionError):
        test_varlen_equals_each_document_alone()


def test_select_noisy_on_packed_gates_stays_in_each_document():
    """Packed gates carry -inf on other documents' blocks: the noisy choice of every row is its own
    document's (the per-document choice shifted by the document's first block), and the threshold of
    logG_sel passes exactly the chosen blocks, also on rows whose document has fewer blocks than K-1."""
    rng = np.random.default_rng(43)
    block, K = 16, 4
    docs = [32, 96, 64]
    cu = np.cumsum([0] + docs)
    T = int(cu[-1])
    s = rng.standard_normal((1, 2, T, T // block))
    lg = orc.gate_normalize_varlen(s, cu, block).astype(np.float32)
    noise = rng.gumbel(size=lg.shape).astype(np.float32)
    logG_sel, tau, tidx, sel = orc.select_noisy(lg, noise, K, block)
    mask = orc.selection_mask(logG_sel, tau, tidx, block)
    for ts, bs in orc.doc_slices(cu, block):
        _, _, _, sd = orc.select_noisy(lg[:, :, ts, bs], noise[:, :, ts, bs], K, block)
        want = np.where(sd >= 0, sd + bs.start, -1)
        assert np.array_equal(sel[:, :, ts], want)
    for b, g, t in np.ndindex(*sel.shape[:3]):
        chosen = [m for m in sel[b, g, t] if m >= 0]
        assert sorted(np.nonzero(mask[b, g, t])[0].tolist()) == chosen
