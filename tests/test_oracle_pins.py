"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources of truth used here:
  * the worked example's printed values (tests/golden/worked_example.txt),
  * textbook constants (tests/golden/textbook_values.txt),
  * library routines (torch CPU matmul / activations / softmax, numpy bincount),
  * brute force with pure-Python loops on tiny inputs,
  * invariants that any correct dispatch satisfies.

Every ``check_*`` takes the oracle module ``O`` so that test_oracle_mutations.py
can plant mistakes in a patched copy and show that some check fails.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as tF
from scipy.special import softmax as sp_softmax

import oracle.moe_oracle as ORACLE
from conftest import read_golden

GOLD = read_golden("worked_example.txt")
TEXT = read_golden("textbook_values.txt")


# ---------------------------------------------------------------------------
# helpers that use only library routines (never the oracle)
# ---------------------------------------------------------------------------

def torch_mlp(x, w_up, w_down, act):
    """Dense two-layer MLP with torch CPU float64 ops (library reference)."""
    x = torch.as_tensor(np.asarray(x, dtype=np.float64))
    wu = torch.as_tensor(np.asarray(w_up, dtype=np.float64))
    wd = torch.as_tensor(np.asarray(w_down, dtype=np.float64))
    h = x @ wu
    if act == "swiglu":
        F = wu.shape[1] // 2
        a = tF.silu(h[:, :F]) * h[:, F:]
    else:
        a = tF.gelu(h, approximate="none")
    return (a @ wd).numpy()


def bf16_vals(shape, std, rng):
    """Random bf16-representable values (as float64) via torch's bf16 cast."""
    t = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * std)
    return t.to(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------------------
# worked example
# ---------------------------------------------------------------------------

def _worked_example_inputs(O):
    E, k = GOLD["num_experts"][0], GOLD["top_k"][0]
    D, F = 64, 128
    e_a, e_b = GOLD["chosen_experts"]
    wa, wb = GOLD["routing_weights"]
    x = np.zeros((1, D), dtype=np.float32)
    x[0, 0] = 1.0
    # Router column 0 (the only feature the token has): exp(l_a - l_b) = wa / wb.
    w_r = np.full((E, D), 0.0, dtype=np.float32)
    w_r[:, 0] = -10.0
    w_r[e_a, 0] = np.float32(math.log(wa / wb))
    w_r[e_b, 0] = 0.0
    # GELU experts: hidden unit e sees +x0, unit 64+e sees -x0; output feature 1
    # collects c_e * gelu(+1), feature 2 collects c_e * gelu(-1); c_e = (e+1)/16.
    w1 = np.zeros((E, D, F))
    w2 = np.zeros((E, F, D))
    for e in range(E):
        w1[e, 0, e] = 1.0
        w1[e, 0, 64 + e] = -1.0
        w2[e, e, 1] = (e + 1) / 16.0
        w2[e, 64 + e, 2] = (e + 1) / 16.0
    return x, w_r, w1, w2, E, k


def check_worked_example_placement(O):
    E = GOLD["num_experts"][0]
    ep = GOLD["num_devices"][0]
    assert E // ep == GOLD["experts_per_device"][0]
    for e, dev in zip(GOLD["chosen_experts"], GOLD["device_of_chosen"]):
        r, _ = O.expert_placement(e, E, ep)
        assert int(r) == dev
    # Step 2 prints the remote entry's tag: expert 11 is local expert 11 mod 4 = 3
    _, l = O.expert_placement(GOLD["chosen_experts"][1], E, ep)
    assert int(l) == GOLD["local_index_of_remote"][0]
    ranks, _ = O.expert_placement(np.arange(E), E, ep)
    assert list(np.nonzero(ranks == 0)[0]) == GOLD["experts_on_device_0"]
    assert list(np.nonzero(ranks == 2)[0]) == GOLD["experts_on_device_2"]


def check_worked_example_routing(O):
    x, w_r, w1, w2, E, k = _worked_example_inputs(O)
    logits = O.router_logits(x, w_r)
    idx, w = O.topk_select(logits, k, renormalize=True)
    assert list(idx[0]) == GOLD["chosen_experts"]
    assert np.allclose(w[0], GOLD["routing_weights"], rtol=0, atol=1e-7)
    # Step 2: the two dispatch entries land in device 0's and device 2's segments.
    pre = O.preprocess(idx, E, GOLD["num_devices"][0])
    ro = pre["rank_offsets"]
    rows = pre["pos"]
    for j, dev in enumerate(GOLD["device_of_chosen"]):
        assert ro[dev] <= rows[j] < ro[dev + 1]
    assert list(pre["rank_splits"]) == [1, 0, 1, 0]


def check_worked_example_output(O):
    x, w_r, w1, w2, E, k = _worked_example_inputs(O)
    res = O.moe_layer(x, w_r, None, w1, w2, None, None, E=E, ep_size=GOLD["num_devices"][0],
                      top_k=k, act="gelu", renormalize=True, x_is_f32=True)
    e_a, e_b = GOLD["chosen_experts"]
    ca, cb = GOLD["combine_coefficients"]
    w = res["topk_w"][0]
    g_pos = 1.0 * TEXT["phi_1"][0]             # gelu(+1) = Phi(1)
    g_neg = -1.0 * TEXT["phi_minus_1"][0]      # gelu(-1) = -Phi(-1)
    sa, sb = (e_a + 1) / 16.0, (e_b + 1) / 16.0
    expect = np.zeros(64)
    expect[0] = GOLD["residual_coefficient"][0] * 1.0
    expect[1] = w[0] * sa * g_pos + w[1] * sb * g_pos
    expect[2] = w[0] * sa * g_neg + w[1] * sb * g_neg
    assert np.allclose(res["out"][0], expect, rtol=0, atol=1e-12)
    # and with the page's rounded weights (the routing is exact to 1e-7)
    expect_page = expect.copy()
    expect_page[1] = ca * sa * g_pos + cb * sb * g_pos
    expect_page[2] = ca * sa * g_neg + cb * sb * g_neg
    assert np.allclose(res["out"][0], expect_page, rtol=0, atol=1e-7)


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------

def check_logits_exact(O):
    rng = np.random.default_rng(1)
    T, E, D = 6, 5, 37
    x = rng.standard_normal((T, D)).astype(np.float32)
    w = (rng.standard_normal((E, D)) * 0.02).astype(np.float32)
    b = (rng.standard_normal(E)).astype(np.float32)
    got = O.router_logits(x, w, b)
    for t in range(T):
        for e in range(E):
            exact = math.fsum(float(x[t, d]) * float(w[e, d]) for d in range(D))
            ref = np.float32(np.float32(exact) + b[e])
            assert got[t, e] == ref, (t, e)
    assert got.dtype == np.float32


def _brute_topk(row, k, renorm):
    E = len(row)
    order = sorted(range(E), key=lambda e: (-float(row[e]), e))
    ch = order[:k]
    m = float(row[ch[0]])
    num = [math.exp(float(row[e]) - m) for e in ch]
    den = math.fsum(num) if renorm else math.fsum(math.exp(float(v) - m) for v in row)
    return ch, [v / den for v in num]


def check_topk_bruteforce(O):
    rng = np.random.default_rng(2)
    T, E = 40, 7
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[0] = 0.5                          # all tied
    logits[1, [1, 4]] = 3.0                  # tie at the top
    logits[2, [2, 5, 6]] = -0.25             # ties in the middle
    logits[3] = np.array([1, 2, 2, 1, 0, 2, 1], dtype=np.float32)
    for k in (1, 3, E):
        for renorm in (True, False):
            idx, w = O.topk_select(logits, k, renorm)
            for t in range(T):
                ch, ww = _brute_topk(logits[t], k, renorm)
                assert list(idx[t]) == ch, (k, renorm, t)
                assert np.allclose(w[t], ww, rtol=1e-14, atol=0)


def check_ties_lower_index(O):
    logits = np.zeros((3, 8), dtype=np.float32)
    logits[1, [3, 6]] = 1.0
    logits[2, [7, 2, 5]] = 2.0
    idx, w = O.topk_select(logits, 2)
    assert idx.tolist() == [[0, 1], [3, 6], [2, 5]]
    assert np.allclose(w, 0.5)


def check_route_gaps(O):
    """The margins that decide which tokens the parity tests exempt, on logits whose
    sorted values are built from powers of two, so every gap is an exact fp32
    number known in advance.  Each row lists its logits out of order; the k-th/(k+1)-th
    gap, the gaps around it and the gaps inside the top-k all differ, so taking the
    wrong neighbour, forgetting to sort, or letting the (k+1)-th into the inner gap
    each gives a different number."""
    h = 2.0 ** -17                          # ~7.6e-6: below the 1e-5 exemption threshold
    H = 2.0 ** -16                          # ~1.5e-5: above it
    # sorted descending: 4, 3.5, 3.25, 3.25 - h, 3 ... ; gaps 0.5, 0.25, h, 0.25 - h ...
    desc = np.array([4.0, 3.5, 3.25, 3.25 - h, 3.0, 1.0], dtype=np.float32)
    perm = [3, 0, 5, 1, 4, 2]
    rows = np.stack([desc[perm], desc[perm[::-1]]])
    # k = 3: gap_k = 3.25 - (3.25 - h) = h; inner = min(0.5, 0.25) = 0.25
    g, inner = O.route_gaps(rows, 3)
    assert g.tolist() == [h, h] and inner.tolist() == [0.25, 0.25]
    # k = 2: gap_k = 3.5 - 3.25 = 0.25; inner = 0.5
    g, inner = O.route_gaps(rows, 2)
    assert g.tolist() == [0.25, 0.25] and inner.tolist() == [0.5, 0.5]
    # k = 4: gap_k = (3.25 - h) - 3 = 0.25 - h; inner = h (the 3rd/4th pair)
    g, inner = O.route_gaps(rows, 4)
    assert g.tolist() == [0.25 - h, 0.25 - h] and inner.tolist() == [h, h]
    # k = 1: the set margin is the top two's gap; no order inside a single pick
    g, inner = O.route_gaps(rows, 1)
    assert g.tolist() == [0.5, 0.5] and np.all(np.isinf(inner))
    # k = E: every expert is chosen, the set has no margin to lose
    g, inner = O.route_gaps(rows, 6)
    assert np.all(np.isinf(g)) and inner.tolist() == [h, h]
    # exact ties give a zero gap, and one of 2^-16 stays above the threshold
    ties = np.array([[1.0, 2.0, 2.0, 0.0], [2.0, 2.0 - H, 0.0, 2.0 - H - 0.5]], dtype=np.float32)
    g, inner = O.route_gaps(ties, 1)
    assert g.tolist() == [0.0, H]
    g, inner = O.route_gaps(ties, 2)
    assert g.tolist() == [1.0, 0.5] and inner.tolist() == [0.0, H]
    # the rows' margins against the 1e-5 threshold the tests apply
    assert h < 1e-5 < H


def check_softmax_library(O):
    rng = np.random.default_rng(3)
    logits = (rng.standard_normal((20, 9)) * 3).astype(np.float32)
    full = sp_softmax(logits.astype(np.float64), axis=1)
    # k = E with renormalisation: the complete softmax, in descending order
    idx, w = O.topk_select(logits, 9, True)
    assert np.allclose(w, np.take_along_axis(full, idx.astype(np.int64), 1), rtol=1e-13)
    # no renormalisation: the complete softmax restricted to the chosen experts
    idx, w = O.topk_select(logits, 3, False)
    assert np.allclose(w, np.take_along_axis(full, idx.astype(np.int64), 1), rtol=1e-13)
    # renormalised weights sum to one
    idx, w = O.topk_select(logits, 3, True)
    assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# preprocess / permute
# ---------------------------------------------------------------------------

def _random_topk_idx(rng, T, E, k, p=None):
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def check_preprocess_invariants(O):
    rng = np.random.default_rng(4)
    T, E, k = 300, 12, 3
    p = np.array([0.4, 0.2, 0.1, 0.1, 0.05, 0.05, 0.05, 0.05, 0, 0, 0, 0])
    idx = _random_topk_idx(rng, T, E, k, p=p)      # experts 8..11 are empty
    for ep in (1, 2, 3, 4, 6, 12):
        pre = O.preprocess(idx, E, ep)
        El = E // ep
        counts, off = pre["counts"], pre["expert_offsets"]
        # brute-force recount
        rc = [0] * E
        for t in range(T):
            for j in range(k):
                rc[idx[t, j]] += 1
        assert counts.tolist() == rc
        assert counts.tolist() == np.bincount(idx.ravel(), minlength=E).tolist()
        assert counts.sum() == pre["rank_splits"].sum() == T * k
        assert off[0] == 0 and off[-1] == T * k and np.all(np.diff(off) == counts)
        for r in range(ep):
            assert pre["rank_splits"][r] == sum(rc[r * El:(r + 1) * El])
            assert pre["rank_offsets"][r] == off[r * El]
        # pos/src inverse bijections on [0, T*k)
        pos, src = pre["pos"].astype(np.int64), pre["src"].astype(np.int64)
        assert sorted(pos.tolist()) == list(range(T * k))
        assert np.all(src[pos] == np.arange(T * k)) and np.all(pos[src] == np.arange(T * k))
        # definition: pos[t,j] = off[e] + #{t' < t : e in topk(t')}
        seen = [0] * E
        for t in range(T):
            for j in range(k):
                e = idx[t, j]
                assert pos[t * k + j] == off[e] + seen[e]
            for j in range(k):
                seen[idx[t, j]] += 1
        # each expert segment holds only that expert's pairs, tokens strictly increasing
        for e in range(E):
            seg = src[off[e]:off[e + 1]]
            assert np.all(idx.ravel()[seg] == e)
            assert np.all(np.diff(seg // k) > 0)
    with pytest.raises(ValueError):
        O.preprocess(idx, E, 5)
    with pytest.raises(ValueError):
        O.expert_placement(3, 10, 4)


def check_permute_roundtrip(O):
    rng = np.random.default_rng(5)
    T, E, k, D = 57, 10, 4, 6
    idx = _random_topk_idx(rng, T, E, k)
    x = rng.standard_normal((T, D))
    pre = O.preprocess(idx, E, 5)
    xp = O.permute(x, pre["src"], k)
    back = O.unpermute(xp, pre["pos"], T, k)
    for j in range(k):
        assert np.array_equal(back[:, j], x)
    # and row r of the buffer is a copy of its source token
    for r in range(T * k):
        assert np.array_equal(xp[r], x[pre["src"][r] // k])


# ---------------------------------------------------------------------------
# expert FFN closed forms and library cross-checks
# ---------------------------------------------------------------------------

def check_activation_closed_forms(O):
    assert O.gelu(0.0) == 0.0
    assert abs(O.gelu(1.0) - TEXT["phi_1"][0]) < 1e-15
    assert abs(O.gelu(-1.0) + TEXT["phi_minus_1"][0]) < 1e-15
    assert abs(O.gelu(2.0) - 2 * TEXT["phi_2"][0]) < 1e-15
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(1.0) - TEXT["logistic_1"][0]) < 1e-15
    assert abs(O.silu(-1.0) + TEXT["logistic_minus_1"][0]) < 1e-15
    assert abs(O.silu(2.0) - 2 * TEXT["logistic_2"][0]) < 1e-15


def check_swiglu_gate_up_order(O):
    # x = e_0; gate column 0 sees 1, up column 0 sees 2 -> a0 = silu(1) * 2.
    x = np.array([[1.0, 0, 0, 0]])
    wgu = np.zeros((4, 4))            # F = 2: columns [g0, g1, u0, u1]
    wgu[0, 0], wgu[0, 2] = 1.0, 2.0
    wd = np.zeros((2, 4))
    wd[0, 3] = 1.0
    y = O.expert_ffn(x, wgu, wd, "swiglu")
    assert abs(y[0, 3] - 2.0 * TEXT["logistic_1"][0]) < 1e-15
    assert np.count_nonzero(y) == 1


def check_ffn_library(O):
    rng = np.random.default_rng(6)
    x = bf16_vals((13, 32), 1.0, rng)
    for act, up in (("swiglu", 2 * 24), ("gelu", 24)):
        wu = bf16_vals((32, up), 0.2, rng)
        wd = bf16_vals((24, 32), 0.2, rng)
        assert np.allclose(O.expert_ffn(x, wu, wd, act), torch_mlp(x, wu, wd, act), rtol=1e-12, atol=1e-13)


def check_bf16_round_library(O):
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(5000).astype(np.float32) * 10,
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0,
                                  3.0e38, 1e-40, 2 ** -126], dtype=np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(v)
    assert np.array_equal(got, ref)
    assert got[-8 + 0] == 1.0 and got[-8 + 1] == 1 + 2 ** -6      # ties to even
    bits = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_bits_to_f64(bits), ref)


# ---------------------------------------------------------------------------
# whole-layer reductions and brute force
# ---------------------------------------------------------------------------

def _layer(O, x, w_r, b, wu, wd, swu, swd, E, ep, k, act, renorm=True):
    return O.moe_layer(x, w_r, b, wu, wd, swu, swd, E=E, ep_size=ep, top_k=k, act=act,
                       renormalize=renorm)


def check_identical_experts_is_dense(O):
    rng = np.random.default_rng(8)
    T, D, E, F, k = 33, 16, 6, 24, 2
    x = bf16_vals((T, D), 1.0, rng)
    w_r = (rng.standard_normal((E, D)) * 0.5).astype(np.float32)
    wu1 = bf16_vals((D, 2 * F), 0.3, rng)
    wd1 = bf16_vals((F, D), 0.3, rng)
    res = _layer(O, x, w_r, None, np.stack([wu1] * E), np.stack([wd1] * E), None, None, E, 3, k, "swiglu")
    assert np.allclose(res["out"], x + torch_mlp(x, wu1, wd1, "swiglu"), rtol=1e-12, atol=1e-12)


def check_single_expert_is_dense(O):
    rng = np.random.default_rng(9)
    T, D, F = 21, 16, 32
    x = bf16_vals((T, D), 1.0, rng)
    w_r = rng.standard_normal((1, D)).astype(np.float32)
    wu = bf16_vals((1, D, F), 0.3, rng)
    wd = bf16_vals((1, F, D), 0.3, rng)
    res = _layer(O, x, w_r, None, wu, wd, None, None, 1, 1, 1, "gelu")
    assert np.allclose(res["out"], x + torch_mlp(x, wu[0], wd[0], "gelu"), rtol=1e-12, atol=1e-12)
    assert np.all(res["topk_w"] == 1.0)


def check_zero_experts_is_shared(O):
    rng = np.random.default_rng(10)
    T, D, E, F, k, S, Fs = 17, 16, 4, 8, 2, 2, 12
    x = bf16_vals((T, D), 1.0, rng)
    w_r = rng.standard_normal((E, D)).astype(np.float32)
    swu = bf16_vals((S, D, 2 * Fs), 0.3, rng)
    swd = bf16_vals((S, Fs, D), 0.3, rng)
    res = _layer(O, x, w_r, None, np.zeros((E, D, 2 * F)), np.zeros((E, F, D)), swu, swd, E, 2, k, "swiglu")
    shared = sum(torch_mlp(x, swu[i], swd[i], "swiglu") for i in range(S))
    assert np.allclose(res["out"], x + shared, rtol=1e-12, atol=1e-12)


def check_k_equals_e_mixture(O):
    rng = np.random.default_rng(11)
    T, D, E, F = 19, 8, 4, 8
    x = bf16_vals((T, D), 1.0, rng)
    w_r = rng.standard_normal((E, D)).astype(np.float32)
    wu = bf16_vals((E, D, 2 * F), 0.3, rng)
    wd = bf16_vals((E, F, D), 0.3, rng)
    res = _layer(O, x, w_r, None, wu, wd, None, None, E, 2, E, "swiglu")
    logits = torch.as_tensor(x) @ torch.as_tensor(w_r.astype(np.float64)).T
    p = torch.softmax(logits.to(torch.float32).to(torch.float64), dim=1).numpy()
    ref = x + sum(p[:, e:e + 1] * torch_mlp(x, wu[e], wd[e], "swiglu") for e in range(E))
    assert np.allclose(res["out"], ref, rtol=1e-9, atol=1e-9)


def check_bruteforce_layer(O):
    """Dense formulation on tiny inputs: every expert on every token, gate matrix
    from a per-token Python sort, out = x + s + G @ Y."""
    rng = np.random.default_rng(12)
    for (T, D, E, ep, k, F, act, S, renorm, bias) in [
        (24, 8, 8, 4, 2, 8, "swiglu", 1, True, False),
        (16, 8, 16, 4, 2, 16, "gelu", 0, True, False),
        (20, 8, 6, 3, 3, 8, "swiglu", 2, False, True),
    ]:
        x = bf16_vals((T, D), 1.0, rng)
        w_r = (rng.standard_normal((E, D)) * 0.5).astype(np.float32)
        b = np.array([2 * math.log(1 / (e + 1)) for e in range(E)], dtype=np.float32) if bias else None
        up = 2 * F if act == "swiglu" else F
        wu = bf16_vals((E, D, up), 0.3, rng)
        wd = bf16_vals((E, F, D), 0.3, rng)
        swu = bf16_vals((S, D, 2 * 8), 0.3, rng) if S else None
        swd = bf16_vals((S, 8, D), 0.3, rng) if S else None
        res = _layer(O, x, w_r, b, wu, wd, swu, swd, E, ep, k, act, renorm)
        # brute force
        G = np.zeros((T, E))
        for t in range(T):
            row = [np.float32(np.float32(math.fsum(x[t, d] * float(w_r[e, d]) for d in range(D)))
                              + (b[e] if b is not None else np.float32(0))) for e in range(E)]
            ch, ww = _brute_topk(np.array(row, dtype=np.float32), k, renorm)
            for e, v in zip(ch, ww):
                G[t, e] = v
        Y = np.stack([torch_mlp(x, wu[e], wd[e], act) for e in range(E)])     # [E, T, D]
        s = sum(torch_mlp(x, swu[i], swd[i], "swiglu") for i in range(S)) if S else 0.0
        ref = x + s + np.einsum("te,etd->td", G, Y)
        assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


ALL_CHECKS = [
    check_worked_example_placement, check_worked_example_routing, check_worked_example_output,
    check_logits_exact, check_topk_bruteforce, check_ties_lower_index, check_route_gaps,
    check_softmax_library,
    check_preprocess_invariants, check_permute_roundtrip, check_activation_closed_forms,
    check_swiglu_gate_up_order, check_ffn_library, check_bf16_round_library,
    check_identical_experts_is_dense, check_single_expert_is_dense, check_zero_experts_is_shared,
    check_k_equals_e_mixture, check_bruteforce_layer,
]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(ORACLE)


def test_textbook_constants_consistent():
    # the table values agree with the closed forms computed by the C library
    assert abs(TEXT["phi_1"][0] - 0.5 * (1 + math.erf(1 / math.sqrt(2)))) < 1e-16
    assert abs(TEXT["phi_minus_1"][0] - 0.5 * (1 + math.erf(-1 / math.sqrt(2)))) < 1e-16
    assert abs(TEXT["logistic_1"][0] - 1 / (1 + math.exp(-1))) < 1e-16
