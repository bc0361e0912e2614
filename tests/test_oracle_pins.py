"""Pins of the fp64 oracle against things other than itself: hand-worked
closed forms (tests/golden), brute force, library routines (torch's fp64 CPU
attention, scipy's expit), and invariants the definitions imply. Each pin is
chosen so a plausible slip in the oracle (a dropped term, a wrong sign, a
transposed operand, a wrong axis) fails at least one of them."""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_cases.json")


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def rel(a, b):
    return np.linalg.norm(np.ravel(a - b)) / max(np.linalg.norm(np.ravel(b)), 1e-300)


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ------------------------------------------------------------ golden cases

def test_golden_linear(golden):
    c = golden["linear_core"]
    a = O.lin_core(np.array([c["q"]]), np.array([c["k"]]), np.array([c["v"]]), H=1, eps=c["eps"])
    np.testing.assert_allclose(a[0], c["expect"], rtol=0, atol=1e-14)


def test_golden_softmax(golden):
    c = golden["softmax_core"]
    a = O.softmax_core(np.array([c["q"]]), np.array([c["k"]]), np.array([c["v"]]), H=1)
    np.testing.assert_allclose(a[0], c["expect"], rtol=0, atol=1e-14)


def test_golden_gate(golden):
    c = golden["gate"]
    np.testing.assert_allclose(O.gate(c["a"], c["g"]), c["expect"], rtol=0, atol=1e-14)


def test_golden_write_gated_linear(golden):
    c = golden["write_gated_linear_core"]
    a = O.lin_core(np.array([c["q"]]), np.array([c["k"]]), np.array([c["v"]]), H=1,
                   eps=c["eps"], wgate=np.array([c["wgate"]]))
    np.testing.assert_allclose(a[0], c["expect"], rtol=0, atol=1e-14)


def test_golden_linear_layer_residual_is_added_after_the_gate(golden):
    c = golden["linear_layer_residual"]
    y = O.linear_attn(np.array([c["q"]]), np.array([c["k"]]), np.array([c["v"]]),
                      np.array([c["g"]]), H=1, eps=c["eps"], residual=np.array([c["residual"]]))
    np.testing.assert_allclose(y[0], c["expect"], rtol=0, atol=1e-14)


def test_golden_softmax_layer_residual_is_added_after_the_gate(golden):
    c = golden["softmax_layer_residual"]
    y = O.softmax_anchor(np.array([c["q"]]), np.array([c["k"]]), np.array([c["v"]]),
                         np.array([c["g"]]), H=1, residual=np.array([c["residual"]]))
    np.testing.assert_allclose(y[0], c["expect"], rtol=0, atol=1e-14)


def test_golden_route(golden):
    c = golden["route"]
    h = np.array([c["h"]])
    s = [np.array([x]) for x in c["s"]]
    u, alpha = O.route(h, s, np.array(c["w_r"]))
    np.testing.assert_allclose(alpha[0], c["expect_alpha"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(u[0], c["expect_u"], rtol=0, atol=1e-14)


# ------------------------------------------------------------ linear core

@pytest.mark.parametrize("N,H,d", [(1, 1, 4), (37, 2, 8), (64, 3, 16)])
def test_linear_equals_bruteforce(N, H, d):
    q, k, v = (rand((2, N, H * d), s) for s in (1, 2, 3))
    a = O.lin_core(q, k, v, H, eps=1e-6)
    b = O.lin_core_bruteforce(q, k, v, H, eps=1e-6)
    assert rel(a, b) < 1e-12


def test_linear_constant_values_normalise_to_the_constant():
    # With V_t = c for every token and eps = 0, the normalised read-out is c
    # exactly wherever phi(Q_t) . z > 0 (the normaliser divides the state out).
    N, H, d = 50, 2, 8
    q, k = np.abs(rand((1, N, H * d), 4)), rand((1, N, H * d), 5)
    c = rand((H * d,), 6)
    v = np.broadcast_to(c, (1, N, H * d)).copy()
    a = O.lin_core(q, k, v, H, eps=0.0)
    np.testing.assert_allclose(a[0], np.broadcast_to(c, (N, H * d)), rtol=1e-12, atol=1e-12)


def test_linear_single_key_token():
    # One key token s: A_t = V_s * w / (w + eps), w = phi(Q_t).phi(K_s).
    H, d, eps = 1, 6, 0.25
    q, k, v = rand((1, 5, d), 7), np.abs(rand((1, 1, d), 8)), rand((1, 1, d), 9)
    a = O.lin_core(q, k, v, H, eps)
    for t in range(5):
        w = sum(max(q[0, t, i], 0.0) * k[0, 0, i] for i in range(d))
        np.testing.assert_allclose(a[0, t], v[0, 0] * w / (w + eps), rtol=1e-13, atol=1e-15)


def test_linear_scale_invariance_and_zero_query():
    N, H, d = 40, 2, 8
    q, k, v = (rand((1, N, H * d), s) for s in (10, 11, 12))
    qp = np.abs(q)        # every row has phi(Q_t) . z > 0, so eps = 0 is defined
    a = O.lin_core(qp, k, v, H, eps=0.0)
    assert rel(O.lin_core(qp, 3.5 * k, v, H, eps=0.0), a) < 1e-13
    assert rel(O.lin_core(0.25 * qp, k, v, H, eps=0.0), a) < 1e-13
    # a query row with no positive entry gives exactly zero (never NaN)
    q2 = q.copy()
    q2[0, 3, :] = -np.abs(q2[0, 3, :])
    a2 = O.lin_core(q2, k, v, H, eps=1e-6)
    assert np.all(a2[0, 3] == 0.0) and np.all(np.isfinite(a2))


def test_linear_is_noncausal_and_heads_are_independent():
    N, H, d = 30, 3, 4
    q, k, v = (rand((1, N, H * d), s) for s in (13, 14, 15))
    a = O.lin_core(q, k, v, H)
    v2 = v.copy()
    v2[0, -1, :d] += 1.0                     # last token, head 0 only
    a2 = O.lin_core(q, k, v2, H)
    assert np.abs(a2[0, 0, :d] - a[0, 0, :d]).max() > 0   # first token sees the last
    np.testing.assert_array_equal(a2[0, :, d:], a[0, :, d:])   # other heads untouched


def test_linear_state_rows_subset():
    # reading out a subset of rows gives the same rows as the full read-out
    N, H, d = 33, 2, 8
    q, k, v = (rand((1, N, H * d), s) for s in (16, 17, 18))
    S, z = O.lin_state(k, v, H)
    rows = [0, 5, 32]
    np.testing.assert_allclose(O.lin_readout(q[:, rows], S, z, H, 1e-6),
                               O.lin_core(q, k, v, H)[:, rows], rtol=1e-14, atol=0)


# ------------------------------------------------------------ write-gated linear core

@pytest.mark.parametrize("N,H,d", [(1, 1, 4), (29, 2, 8), (64, 3, 16)])
def test_write_gated_linear_equals_bruteforce(N, H, d):
    q, k, v = (rand((2, N, H * d), s) for s in (70, 71, 72))
    w = rand((2, N, H), 73, 3.0)
    a = O.lin_core(q, k, v, H, eps=1e-6, wgate=w)
    b = O.lin_core_bruteforce(q, k, v, H, eps=1e-6, wgate=w)
    assert rel(a, b) < 1e-12
    if N > 1:   # (one token: the gate cancels in the normalisation)
        assert rel(a, O.lin_core(q, k, v, H, eps=1e-6)) > 1e-3


def test_write_gate_open_is_ungated():
    # sigmoid(40) = 1 - 4e-18: a wide-open write gate is the ungated layer
    N, H, d = 45, 2, 8
    q, k, v = (rand((1, N, H * d), s) for s in (74, 75, 76))
    a = O.lin_core(q, k, v, H, wgate=np.full((1, N, H), 40.0))
    assert rel(a, O.lin_core(q, k, v, H)) < 1e-15


def test_write_gate_closed_token_is_removed():
    # a token whose gate is shut (sigmoid(-80) ~ 2e-35) writes nothing into S
    # or z: the result equals the layer run on the other tokens only, for the
    # gated head; other heads still see the token
    N, H, d = 20, 2, 8
    q, k, v = (np.abs(rand((1, N, H * d), s)) for s in (77, 78, 79))
    w = rand((1, N, H), 80)
    w[0, 7, 1] = -80.0
    a = O.lin_core(q, k, v, H, wgate=w)
    keep = [t for t in range(N) if t != 7]
    ref = O.lin_core(q, k[:, keep], v[:, keep], H, wgate=w[:, keep])
    np.testing.assert_allclose(a[0, :, d:], ref[0, :, d:], rtol=1e-13, atol=0)
    assert np.abs(a[0, :, :d] - ref[0, :, :d]).max() > 1e-3


def test_write_gate_constant_cancels_up_to_eps():
    # a constant gate omega scales S and z alike, so it only rescales eps:
    # A = phi(Q) S / (phi(Q) z + eps / omega). This fails if only S is gated.
    N, H, d, c, eps = 40, 2, 8, -1.5, 0.5
    q, k, v = (rand((1, N, H * d), s) for s in (81, 82, 83))
    om = 1.0 / (1.0 + math.exp(-c))
    a = O.lin_core(q, k, v, H, eps=eps, wgate=np.full((1, N, H), c))
    assert rel(a, O.lin_core(q, k, v, H, eps=eps / om)) < 1e-13
    assert rel(a, O.lin_core(q, k, v, H, eps=eps)) > 1e-3


def test_write_gate_heads_and_tokens_are_indexed_right():
    # changing the logit of (token 3, head 1) changes head 1 only
    N, H, d = 16, 3, 4
    q, k, v = (np.abs(rand((1, N, H * d), s)) for s in (84, 85, 86))
    w = rand((1, N, H), 87)
    a = O.lin_core(q, k, v, H, wgate=w)
    w2 = w.copy()
    w2[0, 3, 1] += 2.0
    a2 = O.lin_core(q, k, v, H, wgate=w2)
    np.testing.assert_array_equal(a2[0, :, :d], a[0, :, :d])
    np.testing.assert_array_equal(a2[0, :, 2 * d:], a[0, :, 2 * d:])
    assert np.abs(a2[0, :, d:2 * d] - a[0, :, d:2 * d]).max() > 1e-4


def test_write_weights_layout_and_values():
    w = rand((2, 5, 3), 88, 4.0)
    om = O.write_weights(w, 3)
    assert om.shape == (2, 3, 5, 1)
    from scipy.special import expit
    np.testing.assert_allclose(om[1, 2, 4, 0], expit(w[1, 4, 2]), rtol=1e-15)


# ------------------------------------------------------------ softmax core

def test_softmax_matches_torch_fp64_attention():
    torch = pytest.importorskip("torch")
    B, N, H, d = 2, 300, 2, 16
    q, k, v = (rand((B, N, H * d), s) for s in (20, 21, 22))
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(O.split_heads(t, H).copy()) for t in (q, k, v)))
    ref = O.merge_heads(ref.numpy())
    assert rel(O.softmax_core(q, k, v, H), ref) < 1e-12


def test_softmax_row_blocking_does_not_change_the_result():
    q, k, v = (rand((1, 70, 16), s) for s in (23, 24, 25))
    a = O.softmax_core(q, k, v, 2, row_block=256)
    b = O.softmax_core(q, k, v, 2, row_block=7)
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-15)


def test_softmax_special_cases():
    H, d = 1, 8
    q, v = rand((1, 9, d), 26), rand((1, 12, d), 27)
    k_same = np.broadcast_to(rand((d,), 28), (1, 12, d))
    # identical keys: uniform weights, the mean of V
    np.testing.assert_allclose(O.softmax_core(q, k_same, v, H)[0],
                               np.broadcast_to(v[0].mean(0), (9, d)), rtol=1e-13, atol=1e-14)
    # one dominant logit selects its value row
    k = rand((1, 12, d), 29) * 0.01
    k[0, 5] = 200.0 * np.sign(q[0, 0]) * (np.abs(q[0, 0]) > 0)
    a = O.softmax_core(q[:, :1], k, v, H)
    np.testing.assert_allclose(a[0, 0], v[0, 5], rtol=1e-10, atol=1e-10)
    # a single key returns its value
    np.testing.assert_allclose(O.softmax_core(q, k[:, :1], v[:, :1], H)[0],
                               np.broadcast_to(v[0, 0], (9, d)), rtol=1e-14, atol=0)


def test_softmax_key_shift_invariance_and_convexity():
    H, d = 2, 8
    q, k, v = (rand((1, 40, H * d), s) for s in (30, 31, 32))
    a = O.softmax_core(q, k, v, H)
    shifted = k + rand((H * d,), 33)                 # same vector added to every key
    assert rel(O.softmax_core(q, shifted, v, H), a) < 1e-12
    lo = v.min(axis=1, keepdims=True)
    hi = v.max(axis=1, keepdims=True)
    assert np.all(a >= lo - 1e-12) and np.all(a <= hi + 1e-12)


def test_softmax_default_scale_is_inverse_sqrt_d():
    q, k, v = (rand((1, 20, 32), s) for s in (34, 35, 36))
    np.testing.assert_allclose(O.softmax_core(q, k, v, 2),
                               O.softmax_core(q, k, v, 2, scale=1 / 4.0), rtol=1e-15, atol=0)
    assert rel(O.softmax_core(q, k, v, 2), O.softmax_core(q, k, v, 2, scale=1.0)) > 1e-3


# ------------------------------------------------------------ gate

def test_sigmoid_matches_scipy_and_limits():
    special = pytest.importorskip("scipy.special")
    g = np.concatenate([rand((1000,), 37, 8.0), [-800.0, 800.0, 0.0]])
    np.testing.assert_allclose(O.sigmoid(g), special.expit(g), rtol=1e-15, atol=0)
    a = rand((4, 8), 38)
    np.testing.assert_allclose(O.gate(a, np.full_like(a, 30.0)), a, rtol=1e-12, atol=0)
    np.testing.assert_allclose(O.gate(a, np.zeros_like(a)), 0.5 * a, rtol=0, atol=0)
    assert np.abs(O.gate(a, np.full_like(a, -60.0))).max() < 1e-25


# ------------------------------------------------------------ router

def test_router_weights_are_a_distribution():
    B, N, D = 2, 17, 24
    h, w_r = rand((B, N, D), 40), rand((D, D), 41, 1 / math.sqrt(D))
    s = [rand((B, N, D), 42 + i) for i in range(3)]
    u, alpha = O.route(h, s, w_r)
    assert alpha.shape == (B, N, 3)
    assert np.all(alpha >= 0)
    np.testing.assert_allclose(alpha.sum(-1), 1.0, rtol=0, atol=1e-15)


def test_router_single_block_identity_and_equal_summaries():
    B, N, D = 1, 9, 16
    h, w_r, s1 = rand((B, N, D), 45), rand((D, D), 46), rand((B, N, D), 47)
    u, alpha = O.route(h, [s1], w_r)
    np.testing.assert_array_equal(alpha, np.ones((B, N, 1)))
    np.testing.assert_allclose(u, h + s1, rtol=0, atol=1e-15)
    u2, _ = O.route(h, [s1, s1.copy()], w_r)
    np.testing.assert_allclose(u2, h + s1, rtol=1e-15, atol=1e-15)


def test_router_reassociated_key_form():
    # (h W_r^T) . s == h . (s W_r): the per-block key tensor form the GPU uses.
    B, N, D = 1, 11, 20
    h, w_r = rand((B, N, D), 48), rand((D, D), 49)
    s = [rand((B, N, D), 50), rand((B, N, D), 51)]
    _, alpha = O.route(h, s, w_r)
    logits = np.stack([np.einsum("bnd,bnd->bn", h, x @ w_r) for x in s], -1) / math.sqrt(D)
    ref = np.exp(logits - logits.max(-1, keepdims=True))
    ref /= ref.sum(-1, keepdims=True)
    np.testing.assert_allclose(alpha, ref, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------ projections

def test_projection_uses_out_in_layout():
    # W[i, j] = 1 iff j == i + 1: y_i = u_{i+1} under y = u W^T
    D = 6
    w = np.eye(D, k=1)
    u = rand((1, 3, D), 52)
    y = O.project(u, w)
    np.testing.assert_array_equal(y[..., :-1], u[..., 1:])
    np.testing.assert_array_equal(y[..., -1], 0.0)


# ------------------------------------------------------------ stack

def small_stack(L=8, B=1, N=24, H=2, d=4, seed=60, wo_zero=False):
    D = H * d
    x = rand((B, N, D), seed)
    wq = [rand((4 * D, D), seed + 1 + l, 1 / math.sqrt(D)) for l in range(L)]
    wo = [np.zeros((D, D)) if wo_zero else rand((D, D), seed + 100 + l, 1 / math.sqrt(D))
          for l in range(L)]
    wr = rand((D, D), seed + 200, 1 / math.sqrt(D))
    return x, wq, wo, wr, H


def test_stack_layer_kinds_follow_the_three_to_one_pattern():
    x, wq, wo, wr, H = small_stack(L=12)
    _, tr = O.stack(x, wq, wo, wr, H, keep_trace=True)
    assert tr["kind"] == ["linear"] * 3 + ["softmax"] + ["linear"] * 3 + ["softmax"] + \
        ["linear"] * 3 + ["softmax"]
    _, tr = O.stack(x, wq, wo, wr, H, all_softmax=True, keep_trace=True)
    assert tr["kind"] == ["softmax"] * 12


def test_stack_routes_only_later_block_linear_layers():
    x, wq, wo, wr, H = small_stack(L=24)
    _, tr = O.stack(x, wq, wo, wr, H, keep_trace=True)
    for l in range(1, 25):
        a = tr["alpha"][l - 1]
        if l <= 8 or l % 4 == 0:
            assert a is None, l
        else:
            assert a.shape[-1] == (l - 1) // 8, l


def test_stack_summary_is_block_end_stream():
    # layer 9 (first of block 2, linear) reads u = h_8 + s_1 = 2 h_8 (alpha = 1);
    # layer 12 (an anchor) is not routed and reads h_11.
    x, wq, wo, wr, H = small_stack(L=16)
    h8 = O.stack(x, wq[:8], wo[:8], wr, H)
    _, tr = O.stack(x, wq, wo, wr, H, keep_trace=True)
    np.testing.assert_allclose(tr["u"][8], 2.0 * h8, rtol=1e-14, atol=1e-14)
    h11 = O.stack(x, wq[:11], wo[:11], wr, H)
    np.testing.assert_allclose(tr["u"][11], h11, rtol=1e-14, atol=1e-14)


def test_stack_token_permutation_equivariance():
    x, wq, wo, wr, H = small_stack(L=24)
    perm = np.random.default_rng(61).permutation(x.shape[1])
    y = O.stack(x, wq, wo, wr, H)
    yp = O.stack(x[:, perm], wq, wo, wr, H)
    np.testing.assert_allclose(yp, y[:, perm], rtol=1e-11, atol=1e-12)


def test_stack_batch_entries_are_independent():
    x, wq, wo, wr, H = small_stack(L=12, B=2)
    y = O.stack(x, wq, wo, wr, H)
    for b in range(2):
        np.testing.assert_allclose(O.stack(x[b:b + 1], wq, wo, wr, H)[0], y[b],
                                   rtol=1e-13, atol=1e-14)


def test_stack_layer_observer_sees_the_traced_layers_and_changes_nothing():
    # on_layer is an observer: the result is unchanged, and it sees exactly the
    # per-layer values keep_trace records
    x, wq, wo, wr, H = small_stack(L=12)
    y, tr = O.stack(x, wq, wo, wr, H, keep_trace=True)
    seen = []
    y2 = O.stack(x, wq, wo, wr, H, on_layer=lambda *a: seen.append(a))
    np.testing.assert_array_equal(y2, y)
    assert [a[0] for a in seen] == list(range(1, 13))
    for l, kind, u, Y, o, alpha in seen:
        assert kind == tr["kind"][l - 1]
        np.testing.assert_array_equal(u, tr["u"][l - 1])
        np.testing.assert_array_equal(Y, tr["Y"][l - 1])
        np.testing.assert_array_equal(o, tr["o"][l - 1])
        if alpha is None:
            assert tr["alpha"][l - 1] is None
        else:
            np.testing.assert_array_equal(alpha, tr["alpha"][l - 1])


def test_stack_zero_output_projection_is_identity():
    x, wq, wo, wr, H = small_stack(L=12, wo_zero=True)
    np.testing.assert_array_equal(O.stack(x, wq, wo, wr, H), x)


def test_stack_single_block_attnres_on_equals_off():
    x, wq, wo, wr, H = small_stack(L=8)
    np.testing.assert_array_equal(O.stack(x, wq, wo, wr, H, attnres_block=8),
                                  O.stack(x, wq, wo, wr, H, attnres_block=0))


def test_stack_zero_write_gate_weights_double_eps():
    # W_wg = 0 gives every token the logit 0, a constant gate of 1/2, so the
    # write-gated stack is the ungated one with eps doubled; anchors ignore
    # their entry, so garbage there changes nothing
    x, wq, wo, wr, H = small_stack(L=12)
    D = x.shape[-1]
    w0 = [np.zeros((H, D)) for _ in range(12)]
    for l in (3, 7, 11):
        w0[l] = rand((H, D), 90 + l)
    y = O.stack(x, wq, wo, wr, H, eps=0.3, w_wg=w0)
    np.testing.assert_allclose(y, O.stack(x, wq, wo, wr, H, eps=0.6), rtol=1e-12, atol=1e-13)
    assert rel(y, O.stack(x, wq, wo, wr, H, eps=0.3)) > 1e-6


def test_stack_write_gate_logits_come_from_the_layer_input():
    # the logits of a routed linear layer are u W_wg^T with u the router output
    x, wq, wo, wr, H = small_stack(L=12)
    D = x.shape[-1]
    wwg = [rand((H, D), 95 + l, 1 / math.sqrt(D)) for l in range(12)]
    _, tr = O.stack(x, wq, wo, wr, H, w_wg=wwg, keep_trace=True)
    l = 10                                   # layer 10 of block 2: routed, linear
    u = tr["u"][l - 1]
    qkvg = u @ wq[l - 1].T
    q, k, v, g = (qkvg[..., i * D:(i + 1) * D] for i in range(4))
    Y = O.gate(O.lin_core_bruteforce(q, k, v, H, wgate=u @ wwg[l - 1].T), g)
    np.testing.assert_allclose(tr["Y"][l - 1], Y, rtol=1e-11, atol=1e-14)


def test_stack_qkvg_column_order():
    # Zeroing the V block of W_qkvg ([Q | K | V | G] along the output rows) makes
    # every core output zero, so y = x; zeroing the Q block of an anchor makes its
    # attention uniform, so Y = mean(V) * sigmoid(G).
    x, wq, wo, wr, H = small_stack(L=4)
    D = x.shape[-1]
    wq_v0 = [w.copy() for w in wq]
    for w in wq_v0:
        w[2 * D:3 * D] = 0.0
    np.testing.assert_allclose(O.stack(x, wq_v0, wo, wr, H), x, rtol=0, atol=0)
    wq_q0 = [w.copy() for w in wq]
    wq_q0[3][0:D] = 0.0
    _, tr = O.stack(x, wq_q0, wo, wr, H, keep_trace=True)
    u = tr["u"][3]
    v = u @ wq[3][2 * D:3 * D].T
    g = u @ wq[3][3 * D:4 * D].T
    expect = v.mean(axis=1, keepdims=True) * (1 / (1 + np.exp(-g)))
    np.testing.assert_allclose(tr["Y"][3], expect, rtol=1e-12, atol=1e-14)
