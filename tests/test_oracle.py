"""Pins for the fp64 oracle, on the CPU.

The oracle is trusted only after it agrees with things that do not come from
itself: hand-derived worked examples (tests/golden), an independent
pure-Python brute force, PyTorch's scaled_dot_product_attention on fp64 CPU
for the cases it covers, closed forms, invariants and finite differences.
Each check is chosen so that a plausible slip in the oracle (a dropped scale,
a transposed operand, an off-by-one in the mask, a wrong GQA head map, a
missing softcap derivative) fails at least one of them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import attn_workloads as W
from oracle import (alibi_bias, attention_bwd, attention_fwd, head_bwd, head_fwd,
                    kvcache_decode, lse_combine, rotary, round_to, scores, visible_mask)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# independent brute force: pure Python loops, math.fsum, no numpy in the math
# ---------------------------------------------------------------------------
def brute_head(q, k, v, scale, causal, wl, wr, softcap, slope=0.0):
    sq, sk, d = len(q), len(k), len(q[0])
    outs, lses = [], []
    for i in range(sq):
        logits = []
        for j in range(sk):
            delta = sk - sq
            right = 0 if causal else wr
            if right >= 0 and j > i + delta + right:
                continue
            if wl >= 0 and j < i + delta - wl:
                continue
            s = scale * math.fsum(q[i][t] * k[j][t] for t in range(d))
            if softcap > 0:
                s = softcap * math.tanh(s / softcap)
            s -= slope * abs(i + delta - j)
            logits.append((j, s))
        if not logits:
            outs.append([0.0] * d)
            lses.append(-math.inf)
            continue
        m = max(s for _, s in logits)
        w = [(j, math.exp(s - m)) for j, s in logits]
        z = math.fsum(e for _, e in w)
        outs.append([math.fsum(e * v[j][t] for j, e in w) / z for t in range(d)])
        lses.append(m + math.log(z))
    return outs, lses


CASES = [
    # sq, sk, causal, wl, wr, softcap
    (5, 5, False, -1, -1, 0.0),
    (7, 7, True, -1, -1, 0.0),
    (6, 6, True, 2, 0, 0.0),
    (6, 6, False, 1, 2, 0.0),
    (6, 6, True, 0, 0, 0.0),
    (5, 5, False, -1, -1, 0.7),
    (7, 7, True, 3, 0, 1.5),
    (3, 9, True, -1, -1, 0.0),   # Sq < Sk: bottom-right alignment
    (4, 11, True, 2, 0, 0.9),
    (9, 4, True, -1, -1, 0.0),   # Sq > Sk: leading rows see nothing
    (12, 12, False, 4, 4, 0.0),
]


@pytest.mark.parametrize("sq,sk,causal,wl,wr,softcap", CASES)
def test_brute_force_forward(sq, sk, causal, wl, wr, softcap):
    r = rng(sq * 100 + sk)
    d = 5
    q = r.standard_normal((sq, d))
    k = r.standard_normal((sk, d))
    v = r.standard_normal((sk, d))
    scale = 0.61
    o, lse = head_fwd(q, k, v, scale, causal, wl, wr, softcap)
    bo, bl = brute_head(q.tolist(), k.tolist(), v.tolist(), scale, causal, wl, wr, softcap)
    np.testing.assert_allclose(o, np.array(bo), rtol=0, atol=1e-12)
    bl = np.array(bl)
    assert np.array_equal(np.isinf(lse), np.isinf(bl))
    fin = np.isfinite(bl)
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=0, atol=1e-12)


def test_brute_force_full_gqa_layout():
    """attention_fwd over (B, S, H, D) with GQA vs brute force per head."""
    r = rng(7)
    B, S, Hq, Hkv, D = 2, 6, 4, 2, 3
    q = r.standard_normal((B, S, Hq, D))
    k = r.standard_normal((B, S, Hkv, D))
    v = r.standard_normal((B, S, Hkv, D))
    o, lse = attention_fwd(q, k, v, 0.5, causal=True, window=(3, 0), softcap=2.0)
    assert o.shape == (B, S, Hq, D) and lse.shape == (B, Hq, S)
    for b in range(B):
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            bo, bl = brute_head(q[b, :, h].tolist(), k[b, :, kvh].tolist(), v[b, :, kvh].tolist(),
                                0.5, True, 3, 0, 2.0)
            np.testing.assert_allclose(o[b, :, h], np.array(bo), atol=1e-12)
            np.testing.assert_allclose(lse[b, h], np.array(bl), atol=1e-12)


# ---------------------------------------------------------------------------
# worked examples derived by hand (tests/golden)
# ---------------------------------------------------------------------------
def load_golden():
    with open(GOLDEN, encoding="utf-8") as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", load_golden(), ids=lambda c: c["name"])
def test_golden_worked_examples(case):
    kind = case["kind"]
    if kind in ("fwd", "fwd_bwd"):
        q = np.array(case["q"], dtype=np.float64)
        k = np.array(case["k"], dtype=np.float64)
        v = np.array(case["v"], dtype=np.float64)
        hq, hkv = q.shape[1], k.shape[1]
        g = hq // hkv
        wl, wr = case["window"]
        for h in range(hq):
            o, lse = head_fwd(q[:, h], k[:, h // g], v[:, h // g], case["scale"], case["causal"],
                              wl, wr, case["softcap"])
            np.testing.assert_allclose(o, np.array(case["expect_o"])[:, h], atol=1e-14)
            np.testing.assert_allclose(lse, np.array(case["expect_lse_value"])[h], atol=1e-14)
        if kind == "fwd_bwd":
            do = np.array(case["do"], dtype=np.float64)
            dq, dk, dv = head_bwd(q[:, 0], k[:, 0], v[:, 0], do[:, 0], case["scale"],
                                  case["causal"], wl, wr, case["softcap"])
            np.testing.assert_allclose(dq, np.array(case["expect_dq"])[:, 0], atol=1e-14)
            np.testing.assert_allclose(dk, np.array(case["expect_dk"])[:, 0], atol=1e-14)
            np.testing.assert_allclose(dv, np.array(case["expect_dv"])[:, 0], atol=1e-14)
    elif kind == "decode":
        q = np.array(case["q"])[None, None]            # (B=1, 1, Hq=1, D)
        kn = np.array(case["k_new"])[None, None]
        vn = np.array(case["v_new"])[None, None]
        o, lse, ks, vs = kvcache_decode(q, kn, vn, [np.array(case["k_cache"])],
                                        [np.array(case["v_cache"])], [case["cache_seqlen"]],
                                        case["scale"], case["causal"])
        np.testing.assert_allclose(o[0, 0], np.array(case["expect_o"]), atol=1e-14)
        np.testing.assert_allclose(lse[0, :, 0], np.array(case["expect_lse_value"]), atol=1e-14)
        np.testing.assert_array_equal(ks[0], np.array(case["expect_k_after"]))
        np.testing.assert_array_equal(vs[0], np.array(case["expect_v_after"]))
    elif kind == "alibi":
        o, lse = head_fwd(np.array(case["q"]), np.array(case["k"]), np.array(case["v"]),
                          case["scale"], True, alibi_slope=case["slope"])
        np.testing.assert_allclose(o, np.array(case["expect_o"]), atol=1e-12)
        np.testing.assert_allclose(lse, np.array(case["expect_lse"]), atol=1e-12)
    elif kind == "rotary":
        got = rotary(np.array(case["x"]), np.array(case["pos"]), np.array(case["cos"]),
                     np.array(case["sin"]))
        np.testing.assert_allclose(got, np.array(case["expect"]), atol=1e-15)
    elif kind == "combine":
        o, lse = lse_combine(np.array(case["o_parts"]), np.array(case["lse_parts"]))
        np.testing.assert_allclose(o, np.array(case["expect_o"]), atol=1e-14)
        assert abs(float(lse) - case["expect_lse_value"]) < 1e-14
    else:
        raise AssertionError(kind)


# ---------------------------------------------------------------------------
# library special case: PyTorch SDPA on fp64 CPU (no softcap, square)
# ---------------------------------------------------------------------------
def _sdpa(q, k, v, scale, causal):
    # (B, S, H, D) -> (B, H, S, D)
    qt = torch.tensor(q).permute(0, 2, 1, 3)
    kt = torch.tensor(k).permute(0, 2, 1, 3)
    vt = torch.tensor(v).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(3, 3), (4, 2), (6, 1)])
def test_sdpa_pin_forward(causal, hq, hkv):
    r = rng(11 + hq + 10 * causal)
    B, S, D = 2, 33, 16
    q = r.standard_normal((B, S, hq, D))
    k = r.standard_normal((B, S, hkv, D))
    v = r.standard_normal((B, S, hkv, D))
    o, _ = attention_fwd(q, k, v, 0.3, causal=causal)
    g = hq // hkv
    kr = np.repeat(k, g, axis=2)   # GQA == repeat_interleave of kv heads
    vr = np.repeat(v, g, axis=2)
    ref = _sdpa(q, kr, vr, 0.3, causal)
    np.testing.assert_allclose(o, ref, atol=1e-10)


@pytest.mark.parametrize("causal", [False, True])
def test_autograd_pin_backward(causal):
    r = rng(21 + causal)
    B, S, hq, hkv, D = 1, 17, 4, 2, 8
    q = r.standard_normal((B, S, hq, D))
    k = r.standard_normal((B, S, hkv, D))
    v = r.standard_normal((B, S, hkv, D))
    do = r.standard_normal((B, S, hq, D))
    dq, dk, dv = attention_bwd(q, k, v, do, 0.4, causal=causal)
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    g = hq // hkv
    o = torch.nn.functional.scaled_dot_product_attention(
        qt.permute(0, 2, 1, 3), kt.repeat_interleave(g, dim=2).permute(0, 2, 1, 3),
        vt.repeat_interleave(g, dim=2).permute(0, 2, 1, 3), is_causal=causal, scale=0.4)
    (o.permute(0, 2, 1, 3) * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-10)


# ---------------------------------------------------------------------------
# finite differences (covers softcap, window and GQA, which SDPA does not)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal,window,softcap", [(False, (-1, -1), 0.0), (True, (2, 0), 0.0),
                                                   (True, (-1, -1), 1.3), (False, (1, 2), 0.8)])
def test_finite_difference_backward(causal, window, softcap):
    r = rng(31)
    B, S, hq, hkv, D = 1, 6, 4, 2, 3
    q = r.standard_normal((B, S, hq, D))
    k = r.standard_normal((B, S, hkv, D))
    v = r.standard_normal((B, S, hkv, D))
    do = r.standard_normal((B, S, hq, D))
    scale = 0.7
    dq, dk, dv = attention_bwd(q, k, v, do, scale, causal, window, softcap)

    def f(q_, k_, v_):
        o, _ = attention_fwd(q_, k_, v_, scale, causal, window, softcap)
        return float(np.sum(o * do))

    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in itertools.product(*map(range, x.shape)):
            xp = x.copy()
            xm = x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name] = xp
            args_m[name] = xm
            num[idx] = (f(args_p["q"], args_p["k"], args_p["v"]) -
                        f(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
        err = np.linalg.norm(num - grad) / max(np.linalg.norm(num), 1e-30)
        assert err < 1e-6, (name, err)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal,window,softcap", [(False, (-1, -1), 0.0), (True, (3, 0), 0.0),
                                                   (True, (-1, -1), 2.0)])
def test_softmax_rows_sum_to_one(causal, window, softcap):
    """With V = identity (D = Sk) the output row *is* the probability row."""
    r = rng(41)
    S = 10
    q = r.standard_normal((S, 4))
    k = r.standard_normal((S, 4))
    p, _ = head_fwd(q, k, np.eye(S), 0.9, causal, window[0], window[1], softcap)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(p >= 0)
    vis = visible_mask(S, S, causal, window[0], window[1])
    assert np.all(p[~vis] == 0.0)


def test_shift_invariance():
    """Adding a constant c_i to every logit of row i leaves O unchanged and
    shifts LSE by c_i."""
    r = rng(43)
    S = 9
    q, k, v = (r.standard_normal((S, 4)) for _ in range(3))
    c = r.standard_normal(S) * 5.0
    o0, l0 = head_fwd(q, k, v, 0.8, True)
    o1, l1 = head_fwd(q, k, v, 0.8, True, _score_hook=lambda x: x + c[:, None])
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    np.testing.assert_allclose(l1, l0 + c, atol=1e-12)


def test_key_permutation_equivariance():
    r = rng(47)
    q, k, v = (r.standard_normal((8, 5)) for _ in range(3))
    perm = r.permutation(8)
    o0, l0 = head_fwd(q, k, v, 0.5)
    o1, l1 = head_fwd(q, k[perm], v[perm], 0.5)
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    np.testing.assert_allclose(l1, l0, atol=1e-12)


def test_softcap_bounds_logits():
    r = rng(53)
    q = r.standard_normal((6, 4)) * 2.5
    k = r.standard_normal((6, 4)) * 2.5
    x, y = scores(q, k, 1.0, 3.0)
    assert np.all(np.abs(x) < 3.0)
    np.testing.assert_allclose(x, 3.0 * np.tanh(y / 3.0), atol=0)
    assert np.max(np.abs(y)) > 3.0  # the cap actually engaged


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------
def test_zero_keys_give_mean_of_values():
    r = rng(59)
    S, D = 11, 4
    q = r.standard_normal((S, D))
    k = np.zeros((S, D))
    v = r.standard_normal((S, D))
    o, lse = head_fwd(q, k, v, 0.7)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-13)
    np.testing.assert_allclose(lse, np.log(S), atol=1e-13)
    o, lse = head_fwd(q, k, v, 0.7, causal=True)
    prefix = np.cumsum(v, axis=0) / np.arange(1, S + 1)[:, None]
    np.testing.assert_allclose(o, prefix, atol=1e-13)
    np.testing.assert_allclose(lse, np.log(np.arange(1, S + 1)), atol=1e-13)


def test_one_hot_scores_select_a_value_row():
    r = rng(61)
    S, D = 7, 7
    target = r.permutation(S)
    q = np.eye(D)[target] * 40.0  # row i points at key target[i]
    k = np.eye(D) * 40.0
    v = r.standard_normal((S, 3))
    o, _ = head_fwd(q, k, v, 1.0)  # logit gap 1600 -> weight e^-1600 == 0
    np.testing.assert_allclose(o, v[target], atol=1e-13)


def test_window_zero_zero_copies_values():
    r = rng(67)
    S = 8
    q, k, v = (r.standard_normal((S, 4)) for _ in range(3))
    o, lse = head_fwd(q, k, v, 0.6, True, 0, 0)
    np.testing.assert_allclose(o, v, atol=1e-14)
    np.testing.assert_allclose(lse, 0.6 * np.sum(q * k, axis=1), atol=1e-13)


def test_wide_window_equals_causal_and_huge_softcap_equals_none():
    r = rng(71)
    S = 9
    q, k, v = (r.standard_normal((S, 4)) for _ in range(3))
    a = head_fwd(q, k, v, 0.6, True)
    b = head_fwd(q, k, v, 0.6, True, S + 5, 0)
    np.testing.assert_allclose(a[0], b[0], atol=1e-14)
    c = head_fwd(q, k, v, 0.6, True, softcap=1e9)
    np.testing.assert_allclose(a[0], c[0], atol=1e-10)
    np.testing.assert_allclose(a[1], c[1], atol=1e-10)


def test_varlen_equals_separate_sequences():
    r = rng(73)
    lens = [5, 1, 9, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    t = int(cu[-1])
    q = r.standard_normal((t, 4, 3))
    k = r.standard_normal((t, 2, 3))
    v = r.standard_normal((t, 2, 3))
    o, lse = attention_fwd(q, k, v, 0.5, True, (2, 0), 1.1, cu_seqlens=cu)
    assert lse.shape == (4, t)
    for b in range(len(lens)):
        sl = slice(cu[b], cu[b + 1])
        ob, lb = attention_fwd(q[sl][None], k[sl][None], v[sl][None], 0.5, True, (2, 0), 1.1)
        np.testing.assert_allclose(o[sl], ob[0], atol=1e-14)
        np.testing.assert_allclose(lse[:, sl], lb[0], atol=1e-14)
    dq, dk, dv = attention_bwd(q, k, v, q * 0.5, 0.5, True, (2, 0), 1.1, cu_seqlens=cu)
    for b in range(len(lens)):
        sl = slice(cu[b], cu[b + 1])
        a, bb, c = attention_bwd(q[sl][None], k[sl][None], v[sl][None], q[sl][None] * 0.5, 0.5,
                                 True, (2, 0), 1.1)
        np.testing.assert_allclose(dq[sl], a[0], atol=1e-14)
        np.testing.assert_allclose(dk[sl], bb[0], atol=1e-14)
        np.testing.assert_allclose(dv[sl], c[0], atol=1e-14)


def test_decode_equals_last_row_of_causal_prefill():
    r = rng(79)
    B, hq, hkv, D = 3, 4, 2, 5
    lens = [6, 1, 12]
    kc = [r.standard_normal((n, hkv, D)) for n in lens]
    vc = [r.standard_normal((n, hkv, D)) for n in lens]
    q = r.standard_normal((B, 1, hq, D))
    kn = r.standard_normal((B, 1, hkv, D))
    vn = r.standard_normal((B, 1, hkv, D))
    for window, softcap in (((-1, -1), 0.0), ((3, 0), 2.5)):
        o, lse, ks, vs = kvcache_decode(q, kn, vn, kc, vc, lens, 0.45, True, window, softcap)
        for b in range(B):
            n = lens[b] + 1
            qq = np.concatenate([r.standard_normal((n - 1, hq, D)), q[b]], axis=0)
            of, lf = attention_fwd(qq[None], ks[b][None], vs[b][None], 0.45, True, window, softcap)
            np.testing.assert_allclose(o[b, 0], of[0, -1], atol=1e-13)
            np.testing.assert_allclose(lse[b, :, 0], lf[0, :, -1], atol=1e-13)
            np.testing.assert_array_equal(ks[b][-1], kn[b, 0])
            np.testing.assert_array_equal(ks[b][:-1], kc[b])


def test_combine_of_splits_reproduces_whole():
    r = rng(83)
    S, D = 23, 6
    q = r.standard_normal((4, D))
    k = r.standard_normal((S, D))
    v = r.standard_normal((S, D))
    o_full, l_full = head_fwd(q, k, v, 0.5)
    for cuts in ([0, 7, 23], [0, 1, 2, 20, 23], [0, 11, 12, 23]):
        parts = [head_fwd(q, k[a:b], v[a:b], 0.5) for a, b in zip(cuts[:-1], cuts[1:])]
        o, lse = lse_combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        np.testing.assert_allclose(o, o_full, atol=1e-12)
        np.testing.assert_allclose(lse, l_full, atol=1e-12)
    # an empty part (LSE = -inf) carries no weight
    o, lse = lse_combine(np.stack([o_full, np.zeros_like(o_full)]),
                         np.stack([l_full, np.full_like(l_full, -np.inf)]))
    np.testing.assert_allclose(o, o_full, atol=1e-14)


def test_backward_identities():
    """Without softcap every softmax-gradient row sums to zero, so
    sum_j dK_j = scale * sum_i (sum_j dX_ij) q_i = 0; and
    rowsum(P * dP) = rowsum(dO * O) (the quantity a tiled backward
    precomputes)."""
    r = rng(89)
    S, D = 12, 5
    q, k, v, do = (r.standard_normal((S, D)) for _ in range(4))
    dq, dk, dv = head_bwd(q, k, v, do, 0.7, True, 4, 0)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    o, _ = head_fwd(q, k, v, 0.7, True, 4, 0)
    p, _ = head_fwd(q, k, np.eye(S), 0.7, True, 4, 0)
    dp = do @ v.T
    np.testing.assert_allclose(np.sum(p * dp, axis=1), np.sum(do * o, axis=1), atol=1e-12)
    # dV columns: sum over keys of dV equals sum over queries of dO (rows of P sum to 1)
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)


def test_empty_rows_are_zero():
    q = np.ones((4, 2))
    k = np.ones((2, 2))
    v = np.ones((2, 2))
    o, lse = head_fwd(q, k, v, 1.0, True)  # Sq > Sk: rows 0,1 see nothing
    assert np.all(o[:2] == 0) and np.all(np.isneginf(lse[:2]))
    dq, dk, dv = head_bwd(q, k, v, np.ones((4, 2)), 1.0, True)
    assert np.all(dq[:2] == 0)


# ---------------------------------------------------------------------------
# accounting helpers used for FLOP/s must match the mask the oracle applies
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("sq,sk,causal,wl,wr", [(17, 17, True, -1, -1), (17, 17, True, 5, 0),
                                                (9, 30, True, -1, -1), (20, 20, False, 3, 6),
                                                (30, 9, True, 2, 0)])
def test_visible_pairs_matches_mask(sq, sk, causal, wl, wr):
    assert W.visible_pairs(sq, sk, causal, wl, wr) == int(visible_mask(sq, sk, causal, wl, wr).sum())


def test_oracle_is_independent_of_cuda_package():
    here = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for fn in os.listdir(os.path.join(here, "oracle")):
        if fn.endswith(".py"):
            src = open(os.path.join(here, "oracle", fn), encoding="utf-8").read()
            assert "exact_attention_149_b200" not in src.replace(
                "imports nothing from\nthe CUDA library", "")


# ---------------------------------------------------------------------------
# rotary embedding and multi-token decode
# ---------------------------------------------------------------------------
def rope_tables(positions, rdim, base=10000.0):
    """Standard angle tables: theta(p, i) = p * base^(-2i / rdim)."""
    inv = base ** (-np.arange(0, rdim, 2) / rdim)
    ang = np.arange(positions)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


@pytest.mark.parametrize("interleaved", [False, True])
def test_rotary_preserves_pair_norms_and_tail(interleaved):
    r = rng(97)
    x = r.standard_normal((5, 3, 8))
    cos, sin = rope_tables(40, 6)
    pos = np.array([0, 3, 7, 20, 39])
    y = rotary(x, pos, cos, sin, interleaved)
    if interleaved:
        px, py = (x[..., 0:6:2], x[..., 1:6:2]), (y[..., 0:6:2], y[..., 1:6:2])
    else:
        px, py = (x[..., :3], x[..., 3:6]), (y[..., :3], y[..., 3:6])
    np.testing.assert_allclose(px[0] ** 2 + px[1] ** 2, py[0] ** 2 + py[1] ** 2, atol=1e-12)
    np.testing.assert_array_equal(y[..., 6:], x[..., 6:])
    np.testing.assert_array_equal(y[0], x[0])  # position 0: identity rotation


@pytest.mark.parametrize("interleaved", [False, True])
def test_rotary_scores_depend_on_relative_position(interleaved):
    """<R(m) q, R(n) k> depends on m - n only: the property that makes the
    rotation a relative position encoding (fails for a sign or pairing slip
    between the cos and sin terms)."""
    r = rng(101)
    q = r.standard_normal((1, 1, 16))
    k = r.standard_normal((1, 1, 16))
    cos, sin = rope_tables(100, 16)
    s1 = np.sum(rotary(q, [10], cos, sin, interleaved) * rotary(k, [3], cos, sin, interleaved))
    s2 = np.sum(rotary(q, [57], cos, sin, interleaved) * rotary(k, [50], cos, sin, interleaved))
    s3 = np.sum(rotary(q, [10], cos, sin, interleaved) * rotary(k, [4], cos, sin, interleaved))
    assert abs(s1 - s2) < 1e-10 and abs(s1 - s3) > 1e-3


def test_rotary_interleaved_is_a_permutation_of_half_split():
    r = rng(103)
    x = r.standard_normal((4, 2, 8))
    cos, sin = rope_tables(10, 8)
    pos = np.array([1, 2, 5, 9])
    perm = np.array([0, 2, 4, 6, 1, 3, 5, 7])  # interleaved slot -> half-split slot
    half = rotary(x[..., perm], pos, cos, sin, interleaved=False)
    inter = rotary(x, pos, cos, sin, interleaved=True)
    np.testing.assert_allclose(half, inter[..., perm], atol=1e-14)


def test_round_to_matches_torch_casts():
    r = rng(107)
    x = r.standard_normal(10000) * np.exp(r.uniform(-20, 20, 10000))
    bf = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(round_to(x.astype(np.float32).astype(np.float64), "bf16"), bf)
    hf = torch.tensor(x, dtype=torch.float32).to(torch.float16).to(torch.float64).numpy()
    np.testing.assert_array_equal(round_to(x.astype(np.float32).astype(np.float64), "fp16"), hf)


@pytest.mark.parametrize("window,softcap,causal", [((-1, -1), 0.0, True), ((4, 0), 1.7, True),
                                                   ((-1, -1), 0.0, False)])
def test_multi_token_decode_equals_prefill_rows(window, softcap, causal):
    """Sq new tokens appended after L cached ones: the outputs are the last Sq
    rows of an ordinary (bottom-right aligned) attention over all L + Sq
    tokens; with rotary, q and the new keys are rotated at their positions."""
    r = rng(109)
    B, Sq, hq, hkv, D = 2, 3, 4, 2, 8
    lens = [5, 9]
    kc = [r.standard_normal((n, hkv, D)) for n in lens]
    vc = [r.standard_normal((n, hkv, D)) for n in lens]
    q = r.standard_normal((B, Sq, hq, D))
    kn = r.standard_normal((B, Sq, hkv, D))
    vn = r.standard_normal((B, Sq, hkv, D))
    cos, sin = rope_tables(32, 6)
    for rot in (False, True):
        kw = dict(rotary_cos=cos, rotary_sin=sin) if rot else {}
        o, lse, ks, vs = kvcache_decode(q, kn, vn, kc, vc, lens, 0.37, causal, window, softcap, **kw)
        for b in range(B):
            n = lens[b] + Sq
            pos = np.arange(lens[b], n)
            kfull = np.concatenate([kc[b], rotary(kn[b], pos, cos, sin) if rot else kn[b]])
            np.testing.assert_allclose(ks[b], kfull, atol=1e-14)
            qb = rotary(q[b], pos, cos, sin) if rot else q[b]
            for h in range(hq):
                of, lf = head_fwd(qb[:, h], kfull[:, h // 2], vs[b][:, h // 2], 0.37, causal,
                                  window[0], window[1], softcap)
                # the same rows through a full-length prefill (bottom-right = top-left here)
                qq = np.concatenate([r.standard_normal((lens[b], D)), qb[:, h]])
                op, lp = head_fwd(qq, kfull[:, h // 2], vs[b][:, h // 2], 0.37, causal,
                                  window[0], window[1], softcap)
                np.testing.assert_allclose(o[b, :, h], of, atol=1e-13)
                np.testing.assert_allclose(o[b, :, h], op[-Sq:], atol=1e-13)
                np.testing.assert_allclose(lse[b, h], lp[-Sq:], atol=1e-13)


def test_rotary_rejects_positions_outside_the_table():
    cos, sin = rope_tables(8, 4)
    x = np.ones((1, 1, 4))
    with pytest.raises(ValueError):
        rotary(x, [-1], cos, sin)  # numpy would silently wrap to the last row
    with pytest.raises(ValueError):
        rotary(x, [8], cos, sin)


# ---------------------------------------------------------------------------
# ALiBi (guide §进阶参数 alibi_slopes; the linear-distance form is a reading)
# ---------------------------------------------------------------------------
ALIBI_CASES = [
    # sq, sk, causal, wl, wr, softcap, slope
    (6, 6, True, -1, -1, 0.0, 0.5),
    (5, 5, False, -1, -1, 0.0, 0.25),
    (7, 7, True, 2, 0, 1.2, 0.7),
    (3, 8, True, -1, -1, 0.0, 1.5),   # Sq < Sk: distances from the bottom-right diagonal
    (6, 6, False, 1, 2, 0.0, 0.3),
]


@pytest.mark.parametrize("sq,sk,causal,wl,wr,softcap,slope", ALIBI_CASES)
def test_alibi_brute_force(sq, sk, causal, wl, wr, softcap, slope):
    r = rng(sq * 7 + sk)
    q, k, v = r.standard_normal((sq, 4)), r.standard_normal((sk, 4)), r.standard_normal((sk, 4))
    o, lse = head_fwd(q, k, v, 0.6, causal, wl, wr, softcap, alibi_slope=slope)
    bo, bl = brute_head(q.tolist(), k.tolist(), v.tolist(), 0.6, causal, wl, wr, softcap, slope)
    np.testing.assert_allclose(o, np.array(bo), atol=1e-12)
    np.testing.assert_allclose(lse, np.array(bl), atol=1e-12)


def _alibi_mask(sq, sk, slopes, causal):
    """(H, sq, sk) additive float mask for SDPA: the bias, -inf where hidden."""
    m = np.stack([alibi_bias(sq, sk, sl) for sl in slopes])
    if causal:
        vis = visible_mask(sq, sk, True, -1, -1)
        m = np.where(vis[None], m, -np.inf)
    return torch.tensor(m)


@pytest.mark.parametrize("causal", [False, True])
def test_alibi_sdpa_pin(causal):
    """SDPA with the bias as an additive float mask (a library routine that
    knows nothing of ALiBi), per-head slopes and GQA."""
    r = rng(71 + causal)
    B, S, hq, hkv, D = 2, 19, 4, 2, 8
    q = r.standard_normal((B, S, hq, D))
    k = r.standard_normal((B, S, hkv, D))
    v = r.standard_normal((B, S, hkv, D))
    slopes = np.array([0.5, 0.25, 0.125, 0.0625])
    o, _ = attention_fwd(q, k, v, 0.35, causal=causal, alibi_slopes=slopes)
    g = hq // hkv
    qt = torch.tensor(q).permute(0, 2, 1, 3)
    kt = torch.tensor(np.repeat(k, g, axis=2)).permute(0, 2, 1, 3)
    vt = torch.tensor(np.repeat(v, g, axis=2)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=_alibi_mask(S, S, slopes, causal), scale=0.35)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-10)


def test_alibi_autograd_pin_backward():
    r = rng(73)
    B, S, hq, hkv, D = 1, 13, 4, 2, 8
    q = r.standard_normal((B, S, hq, D))
    k = r.standard_normal((B, S, hkv, D))
    v = r.standard_normal((B, S, hkv, D))
    do = r.standard_normal((B, S, hq, D))
    slopes = np.array([0.9, 0.3, 0.1, 0.05])
    dq, dk, dv = attention_bwd(q, k, v, do, 0.45, causal=True, alibi_slopes=slopes)
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    g = hq // hkv
    o = torch.nn.functional.scaled_dot_product_attention(
        qt.permute(0, 2, 1, 3), kt.repeat_interleave(g, dim=2).permute(0, 2, 1, 3),
        vt.repeat_interleave(g, dim=2).permute(0, 2, 1, 3), attn_mask=_alibi_mask(S, S, slopes, True),
        scale=0.45)
    (o.permute(0, 2, 1, 3) * torch.tensor(do)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-10)


def test_alibi_finite_difference_with_softcap_and_window():
    r = rng(79)
    B, S, hq, hkv, D = 1, 6, 2, 1, 3
    q = r.standard_normal((B, S, hq, D))
    k = r.standard_normal((B, S, hkv, D))
    v = r.standard_normal((B, S, hkv, D))
    do = r.standard_normal((B, S, hq, D))
    slopes = np.array([[0.8, 0.2]])  # (B, Hq) layout
    args = (0.7, True, (3, 0), 1.1)
    dq, dk, dv = attention_bwd(q, k, v, do, *args, alibi_slopes=slopes)

    def f(q_, k_, v_):
        return float(np.sum(attention_fwd(q_, k_, v_, *args, alibi_slopes=slopes)[0] * do))

    h = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        x = {"q": q, "k": k, "v": v}[name]
        num = np.zeros_like(x)
        for idx in itertools.product(*map(range, x.shape)):
            pl = {"q": q, "k": k, "v": v}
            mi = {"q": q, "k": k, "v": v}
            pl[name] = x.copy()
            mi[name] = x.copy()
            pl[name][idx] += h
            mi[name][idx] -= h
            num[idx] = (f(pl["q"], pl["k"], pl["v"]) - f(mi["q"], mi["k"], mi["v"])) / (2 * h)
        assert np.linalg.norm(num - grad) / np.linalg.norm(num) < 1e-6, name


def test_alibi_per_batch_slopes_and_zero_slope():
    r = rng(83)
    B, S, H, D = 2, 9, 2, 4
    q, k, v = (r.standard_normal((B, S, H, D)) for _ in range(3))
    o2, l2 = attention_fwd(q, k, v, 0.5, True, alibi_slopes=np.array([[0.3, 0.6], [1.2, 0.1]]))
    for b, sl in ((0, [0.3, 0.6]), (1, [1.2, 0.1])):
        o1, l1 = attention_fwd(q[b:b + 1], k[b:b + 1], v[b:b + 1], 0.5, True, alibi_slopes=np.array(sl))
        np.testing.assert_allclose(o2[b:b + 1], o1, atol=1e-14)
        np.testing.assert_allclose(l2[b:b + 1], l1, atol=1e-14)
    o0, l0 = attention_fwd(q, k, v, 0.5, True, alibi_slopes=np.zeros(H))
    on, ln = attention_fwd(q, k, v, 0.5, True)
    np.testing.assert_array_equal(o0, on)
    np.testing.assert_array_equal(l0, ln)
