"""GPU parity: every entry point of the C ABI against the fp64 oracle on the same
seeded inputs, element by element, at sizes the oracle finishes in seconds
that still span several tiles and a ragged tail. bf16: rel-L2 <= 1e-2 and
max-abs <= 3e-2 max|ref|; fp32: rel-L2 <= 1e-5."""
import math

import numpy as np
import pytest

import oracle as O
import workloads as W
from tests._util import assert_close, rel_l2, to_dev, to_host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import softmax_attention_video_gated_b200 as sva  # noqa: E402

TDT = {"bf16": torch.bfloat16, "f32": torch.float32}


def core_case(B, N, H, d, dtype, seed, q_scale=1.0):
    x = W.core_inputs(B, N, H, d, dtype, seed, q_scale=q_scale)
    return x, {k: to_dev(v, dtype) for k, v in x.items()}


# ------------------------------------------------------------------ device status

def test_bounded_wait_times_out_and_context_survives():
    ws = sva.workspace(256)
    sva.sva_selftest_bounded_wait(ws, 2000)
    assert sva.sva_check_device_status(ws) == sva.SVA_ERR_DEVICE_TIMEOUT
    # the context is still usable: a real call succeeds and reports OK
    x = torch.randn(64, 128, device="cuda").to(torch.bfloat16)
    w = torch.randn(128, 128, device="cuda").to(torch.bfloat16)
    y = torch.empty(64, 128, device="cuda", dtype=torch.bfloat16)
    ws2 = sva.sva_projection_fwd(x, w, y)
    assert sva.sva_check_device_status(ws2) == sva.SVA_OK


# ------------------------------------------------------------------ projections

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,N", [(1, 64, 64), (300, 256, 512), (1000, 512, 320), (517, 192, 1024),
                                   (301, 136, 72), (64, 64, 40)])
def test_projection(dtype, M, K, N):
    rng = np.random.default_rng(M * 7 + N)
    x = W.round_to(rng.standard_normal((M, K)).astype(np.float32), dtype)
    w = W.round_to((rng.standard_normal((N, K)) / math.sqrt(K)).astype(np.float32), dtype)
    y = torch.empty(M, N, device="cuda", dtype=TDT[dtype])
    ws = sva.sva_projection_fwd(to_dev(x, dtype), to_dev(w, dtype), y)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    assert_close(to_host(y), O.project(x, w), dtype, "projection")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_projection_relu_columns(dtype):
    rng = np.random.default_rng(3)
    M, K, N = 260, 256, 768
    x = W.round_to(rng.standard_normal((M, K)).astype(np.float32), dtype)
    w = W.round_to((rng.standard_normal((N, K)) / 16).astype(np.float32), dtype)
    y = torch.empty(M, N, device="cuda", dtype=TDT[dtype])
    sva.sva_projection_fwd(to_dev(x, dtype), to_dev(w, dtype), y, relu_cols=512)
    ref = O.project(x, w)
    ref[:, :512] = O.phi(ref[:, :512])
    assert_close(to_host(y), ref, dtype, "projection+relu")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,N", [(333, 256, 512), (77, 136, 200)])
def test_projection_residual(dtype, M, K, N):
    # (77, 136, 200): the last N tile ends inside a 16-column chunk of h
    rng = np.random.default_rng(4 + N)
    x = W.round_to(rng.standard_normal((M, K)).astype(np.float32), dtype)
    w = W.round_to((rng.standard_normal((N, K)) / 16).astype(np.float32), dtype)
    h0 = rng.standard_normal((M, N)).astype(np.float32)
    h = torch.from_numpy(h0).cuda()
    hc = torch.empty(M, N, device="cuda", dtype=TDT[dtype])
    sva.sva_projection_residual_fwd(to_dev(x, dtype), to_dev(w, dtype), h, hc)
    o = O.project(x, w)
    # the fp32 stream update must carry the projection's accuracy
    assert_close(to_host(h) - h0, o, dtype, "residual update")
    assert_close(to_host(hc), h0 + o, dtype, "stream copy")


# ------------------------------------------------------------------ gated linear attention

@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64), ("f32", 128)])
@pytest.mark.parametrize("B,N,H", [(1, 1, 1), (2, 100, 2), (1, 128, 3), (2, 1000, 2), (1, 3001, 2)])
def test_linear_attn(dtype, d, B, N, H):
    x, t = core_case(B, N, H, d, dtype, seed=11 + N)
    out = torch.empty_like(t["q"])
    ws = sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], out, H, eps=1e-6)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    ref = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6)
    assert_close(to_host(out), ref, dtype, f"linear B={B} N={N}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_linear_attn_strided_features(dtype):
    # q, k, v, g as column slices of one fused [B, N, 4D] buffer, with phi
    # already applied to q and k (the flag)
    B, N, H, d = 2, 777, 2, 128
    D = H * d
    x, _ = core_case(B, N, H, d, dtype, seed=21)
    fq, fk = O.phi(x["q"]).astype(np.float32), O.phi(x["k"]).astype(np.float32)
    buf = to_dev(np.concatenate([fq, fk, x["v"], x["g"]], axis=-1), dtype)
    out = torch.empty(B, N, D, device="cuda", dtype=TDT[dtype])
    sva.sva_linear_attn_fwd(buf[..., :D], buf[..., D:2 * D], buf[..., 2 * D:3 * D],
                            buf[..., 3 * D:], out, H, eps=1e-6, flags=sva.SVA_FLAG_QK_FEATURES)
    ref = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6)
    assert_close(to_host(out), ref, dtype, "linear strided")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_linear_attn_residual_in_place(dtype):
    # out = residual + Y, written over the residual; the residual is scaled to
    # the size of Y so the check still sees Y through the output rounding
    B, N, H, d = 1, 1000, 2, 128
    D = H * d
    x, t = core_case(B, N, H, d, dtype, seed=22)
    res = W.round_to(0.03 * np.random.default_rng(5).standard_normal((B, N, D)).astype(np.float32),
                     dtype)
    out = to_dev(res, dtype)
    sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], out, H, residual=out, eps=1e-6)
    ref = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6, residual=res)
    assert_close(to_host(out), ref, dtype, "linear residual")


def test_linear_attn_zero_query_rows_are_zero_not_nan():
    B, N, H, d = 1, 300, 2, 128
    x, t = core_case(B, N, H, d, "bf16", seed=31)
    q = t["q"].clone()
    q[0, 17] = -q[0, 17].abs() - 0.5
    out = torch.empty_like(q)
    sva.sva_linear_attn_fwd(q, t["k"], t["v"], t["g"], out, H)
    o = to_host(out)
    assert np.isfinite(o).all()
    assert np.all(o[0, 17] == 0.0)


# ------------------------------------------------------------------ write-gated linear attention

def wgate_case(B, N, H, dtype, seed, width, std=2.0):
    """Write-gate logits [B, N, H] ~ N(0, std^2), handed to the library as the
    first H columns of a [B, N, width] buffer (row stride width)."""
    w = W.normal((B, N, width), std, seed, W.TAG_WGATE, dtype)
    return w[..., :H], to_dev(w, dtype)[..., :H]


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64), ("f32", 128)])
@pytest.mark.parametrize("B,N,H,width", [(1, 1, 1, 8), (2, 1000, 2, 2), (1, 3001, 3, 8), (2, 129, 2, 5)])
def test_write_gated_linear_attn(dtype, d, B, N, H, width):
    x, t = core_case(B, N, H, d, dtype, seed=41 + N)
    wg, twg = wgate_case(B, N, H, dtype, 42 + N, width)
    out = torch.empty_like(t["q"])
    ws = sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], out, H, eps=1e-6, wgate=twg)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    ref = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6, wgate=wg)
    assert_close(to_host(out), ref, dtype, f"write-gated linear B={B} N={N}")
    if N > 1:   # the gate changes the result by far more than the tolerance
        assert rel_l2(ref, O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6)) > 0.05


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_write_gated_linear_attn_saturated_gates_and_features(dtype):
    # logits ~ N(0, 30^2): most gates are shut or wide open; q and k given as
    # features (flag) in a fused buffer, as the stack calls it
    B, N, H, d = 1, 1500, 2, 128
    D = H * d
    x, _ = core_case(B, N, H, d, dtype, seed=43)
    wg, twg = wgate_case(B, N, H, dtype, 44, 8, std=30.0)
    fq, fk = O.phi(x["q"]).astype(np.float32), O.phi(x["k"]).astype(np.float32)
    buf = to_dev(np.concatenate([fq, fk, x["v"], x["g"]], axis=-1), dtype)
    out = torch.empty(B, N, D, device="cuda", dtype=TDT[dtype])
    ws = sva.sva_linear_attn_fwd(buf[..., :D], buf[..., D:2 * D], buf[..., 2 * D:3 * D],
                                 buf[..., 3 * D:], out, H, eps=1e-6,
                                 flags=sva.SVA_FLAG_QK_FEATURES, wgate=twg)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    ref = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6, wgate=wg)
    assert_close(to_host(out), ref, dtype, "write-gated linear, saturated gates")


def test_write_gated_linear_attn_noalloc_matches_workspace_call():
    B, N, H, d = 2, 700, 2, 128
    x, t = core_case(B, N, H, d, "bf16", seed=45)
    _, twg = wgate_case(B, N, H, "bf16", 46, 4)
    out1, out2 = torch.empty_like(t["q"]), torch.empty_like(t["q"])
    sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], out1, H, wgate=twg)
    sva.sva_linear_attn_fwd_noalloc(t["q"], t["k"], t["v"], t["g"], out2, H, wgate=twg)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


# ------------------------------------------------------------------ sequence-sharded cores

@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
@pytest.mark.parametrize("gated", [False, True])
def test_linear_state_and_readout_phases_over_two_shards(dtype, d, gated):
    # the states of two token shards, summed (what an all-reduce over two ranks
    # gives), read out by each shard's queries: the unsharded layer
    B, N, H = 2, 1000, 2
    x, t = core_case(B, N, H, d, dtype, seed=51 + d)
    wg, twg = wgate_case(B, N, H, dtype, 52, 8) if gated else (None, None)
    cut = 433
    st = [torch.empty(sva.sva_linear_attn_state_bytes(B, H, d) // 4, device="cuda") for _ in range(2)]
    outs = []
    for i, (a, b) in enumerate(((0, cut), (cut, N))):
        sl = lambda z: z[:, a:b].contiguous()  # noqa: E731
        sva.sva_linear_attn_state_fwd(sl(t["k"]), sl(t["v"]), st[i], H,
                                      wgate=None if twg is None else sl(twg))
    total = st[0] + st[1]
    for a, b in ((0, cut), (cut, N)):
        sl = lambda z: z[:, a:b].contiguous()  # noqa: E731
        o = torch.empty_like(sl(t["q"]))
        ws = sva.sva_linear_attn_readout_fwd(sl(t["q"]), sl(t["g"]), o, total, H, eps=1e-6)
        assert sva.sva_check_device_status(ws) == sva.SVA_OK
        outs.append(o)
    got = to_host(torch.cat(outs, dim=1))
    ref = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6, wgate=wg)
    assert_close(got, ref, dtype, "linear phases over two shards")
    # and the fp32 state itself against the oracle's S and z
    S, z = O.lin_state(x["k"], x["v"], H, wg)
    flat = np.concatenate([S.reshape(B * H, -1), z.reshape(B * H, -1)], axis=1).reshape(-1)
    assert rel_l2(to_host(total), flat) < (1e-2 if dtype == "bf16" else 1e-5)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64), ("f32", 128)])
@pytest.mark.parametrize("rows,keys", [((300, 777), 1000), ((0, 1000), 300), ((999, 1000), 1000)])
def test_softmax_anchor_query_shard_against_all_keys(dtype, d, rows, keys):
    # a shard's queries against the keys and values of the whole sequence
    # (n_keys != N), including more queries than keys and a one-row shard
    B, H = 2, 2
    a, b = rows
    nq = max(b, keys)
    x, t = core_case(B, nq, H, d, dtype, seed=61 + a + keys)
    q, g = t["q"][:, a:b].contiguous(), t["g"][:, a:b].contiguous()
    k, v = t["k"][:, :keys].contiguous(), t["v"][:, :keys].contiguous()
    out = torch.empty_like(q)
    ws = sva.sva_softmax_anchor_fwd(q, k, v, g, out, H)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    ref = O.softmax_anchor(x["q"][:, a:b], x["k"][:, :keys], x["v"][:, :keys], x["g"][:, a:b], H)
    assert_close(to_host(out), ref, dtype, f"anchor rows {a}:{b} keys {keys}")


# ------------------------------------------------------------------ gated softmax anchor

@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64), ("f32", 128)])
@pytest.mark.parametrize("B,N,H", [(1, 1, 1), (2, 100, 2), (1, 129, 2), (1, 700, 2), (2, 1111, 1)])
def test_softmax_anchor(dtype, d, B, N, H):
    x, t = core_case(B, N, H, d, dtype, seed=41 + N)
    out = torch.empty_like(t["q"])
    ws = sva.sva_softmax_anchor_fwd(t["q"], t["k"], t["v"], t["g"], out, H)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    ref = O.softmax_anchor(x["q"], x["k"], x["v"], x["g"], H)
    assert_close(to_host(out), ref, dtype, f"anchor B={B} N={N}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_softmax_anchor_peaky_rescale_path(dtype):
    # Q scaled by 8: logits spread over tens of units, so the running max moves
    # by more than the rescale threshold between key blocks
    B, N, H, d = 1, 1500, 2, 128
    x, t = core_case(B, N, H, d, dtype, seed=51, q_scale=8.0)
    out = torch.empty_like(t["q"])
    sva.sva_softmax_anchor_fwd(t["q"], t["k"], t["v"], t["g"], out, H)
    ref = O.softmax_anchor(x["q"], x["k"], x["v"], x["g"], H)
    assert_close(to_host(out), ref, dtype, "anchor peaky")


def test_softmax_anchor_strided_and_scale():
    B, N, H, d = 1, 555, 2, 128
    D = H * d
    x, _ = core_case(B, N, H, d, "bf16", seed=61)
    buf = to_dev(np.concatenate([x["q"], x["k"], x["v"], x["g"]], -1), "bf16")
    out = torch.empty(B, N, D, device="cuda", dtype=torch.bfloat16)
    sva.sva_softmax_anchor_fwd(buf[..., :D], buf[..., D:2 * D], buf[..., 2 * D:3 * D],
                               buf[..., 3 * D:], out, H, scale=0.05)
    ref = O.softmax_anchor(x["q"], x["k"], x["v"], x["g"], H, scale=0.05)
    assert_close(to_host(out), ref, "bf16", "anchor strided")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_softmax_anchor_residual_in_place(dtype):
    B, N, H, d = 1, 640, 2, 128
    D = H * d
    x, t = core_case(B, N, H, d, dtype, seed=62)
    res = W.round_to(0.03 * np.random.default_rng(6).standard_normal((B, N, D)).astype(np.float32),
                     dtype)
    out = to_dev(res, dtype)            # in place: out aliases residual
    sva.sva_softmax_anchor_fwd(t["q"], t["k"], t["v"], t["g"], out, H, residual=out)
    ref = O.softmax_anchor(x["q"], x["k"], x["v"], x["g"], H, residual=res)
    assert_close(to_host(out), ref, dtype, "anchor residual")


# ------------------------------------------------------------------ AttnRes

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("nb", [1, 2, 3, 5])
@pytest.mark.parametrize("D", [384, 512, 3072])
def test_attnres_route(dtype, nb, D):
    # D = 512 and 3072 take the bf16 row-group kernel (up to 4 blocks; 8 and 1
    # rows per CTA, 1234 rows leaves a ragged last CTA); D = 384, 5 blocks and
    # fp32 take the warp-per-row kernel
    rng = np.random.default_rng(70 + nb + D)
    rows = 1234
    h = rng.standard_normal((rows, D)).astype(np.float32)
    s = [W.round_to(rng.standard_normal((rows, D)).astype(np.float32), dtype) for _ in range(nb)]
    wr = W.round_to((rng.standard_normal((D, D)) / math.sqrt(D)).astype(np.float32), dtype)
    # keys from the oracle's own arithmetic, rounded to the run dtype like the GPU's
    keys = [W.round_to((si.astype(np.float64) @ wr.astype(np.float64)).astype(np.float32), dtype)
            for si in s]
    u = torch.empty(rows, D, device="cuda", dtype=TDT[dtype])
    alpha = torch.empty(rows, nb, device="cuda", dtype=torch.float32)
    sva.sva_attnres_route(torch.from_numpy(h).cuda(), [to_dev(k, dtype) for k in keys],
                          [to_dev(x, dtype) for x in s], u, alpha)
    uref, aref = O.route(h[None], [x[None] for x in s], wr)
    assert_close(to_host(alpha), aref[0], "bf16" if dtype == "bf16" else "f32", "alpha")
    np.testing.assert_allclose(to_host(alpha).sum(-1), 1.0, atol=1e-6)
    assert_close(to_host(u), uref[0], dtype, "routed input")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_attnres_keys(dtype):
    rng = np.random.default_rng(80)
    rows, D = 700, 256
    s = W.round_to(rng.standard_normal((rows, D)).astype(np.float32), dtype)
    wr = W.round_to((rng.standard_normal((D, D)) / 16).astype(np.float32), dtype)
    k = torch.empty(rows, D, device="cuda", dtype=TDT[dtype])
    ws = sva.sva_attnres_keys(to_dev(s, dtype), to_dev(wr, dtype), k)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    assert_close(to_host(k), s.astype(np.float64) @ wr.astype(np.float64), dtype, "keys")


# ------------------------------------------------------------------ the stack

def run_stack(x, wq, wo, wr, H, dtype, **kw):
    B, N, D = x.shape
    L = len(wq)
    tq = [to_dev(w, dtype) for w in wq]
    to = [to_dev(w, dtype) for w in wo]
    tr = to_dev(wr, dtype)
    trace_o = [torch.empty(B * N, D, device="cuda", dtype=torch.float32) for _ in range(L)]
    # router weights of a routed layer in block c: [B*N, c-1], contiguous
    trace_a = [torch.zeros(B * N * 8, device="cuda", dtype=torch.float32) for _ in range(L)]
    st = sva.Stack(tq, to, tr, B, N, H, trace_o=trace_o, trace_alpha=trace_a, **kw)
    xt = to_dev(x, dtype)
    y = torch.empty_like(xt)
    ws = sva.sva_hybrid_stack_fwd(st, xt, y)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    return to_host(y), [to_host(t).reshape(B, N, D) for t in trace_o], [to_host(t) for t in trace_a]


def alpha_rows(flat, rows, nb):
    return flat[:rows * nb].reshape(rows, nb)


def test_stack_fp32_hybrid_group_config():
    """The 4-layer fp32 hybrid group (3 linear + 1 anchor, no AttnRes), N = 1024."""
    w = W.HYBRID4_F32
    x = W.stack_x(w)
    p = W.stack_weights(w)
    y, tro, _ = run_stack(x, p["w_qkvg"], p["w_o"], p["w_r"], w.H, "f32", attnres_block=0)
    yref, tr = O.stack(x, p["w_qkvg"], p["w_o"], p["w_r"], w.H, attnres_block=0, keep_trace=True)
    for l in range(w.L):
        assert_close(tro[l], tr["o"][l], "f32", f"o_{l + 1}")
    assert_close(y - x, yref - x, "f32", "y - x")
    assert_close(y, yref, "f32", "y")


def small_bf16_stack(L, N=333, H=2, seed=90):
    D = H * 128
    rng = np.random.default_rng(seed)
    x = W.round_to(rng.standard_normal((1, N, D)).astype(np.float32), "bf16")
    wq = [W.round_to((rng.standard_normal((4 * D, D)) / math.sqrt(D)).astype(np.float32), "bf16")
          for _ in range(L)]
    wo = [W.round_to((rng.standard_normal((D, D)) / math.sqrt(D)).astype(np.float32), "bf16")
          for _ in range(L)]
    wr = W.round_to((rng.standard_normal((D, D)) / math.sqrt(D)).astype(np.float32), "bf16")
    return x, wq, wo, wr, H


def test_stack_bf16_three_blocks_with_router():
    x, wq, wo, wr, H = small_bf16_stack(24)
    y, tro, tra = run_stack(x, wq, wo, wr, H, "bf16")
    yref, tr = O.stack(x, wq, wo, wr, H, keep_trace=True)
    for l in range(24):
        assert_close(tro[l], tr["o"][l], "bf16", f"o_{l + 1}")
        if tr["alpha"][l] is not None:
            nb = tr["alpha"][l].shape[-1]
            assert_close(alpha_rows(tra[l], x.shape[1], nb), tr["alpha"][l][0], "bf16",
                         f"alpha_{l + 1}")
    assert_close(y - x, yref - x, "bf16", "y - x")


def wwg_weights(L, H, D, dtype, seed):
    return [W.normal((H, D), 1.0 / math.sqrt(D), seed, W.TAG_WWG + l, dtype) for l in range(1, L + 1)]


def run_wg_stack(x, wq, wo, wr, wwg, H, dtype, **kw):
    return run_stack(x, wq, wo, wr, H, dtype,
                     w_wg=[None if l % 4 == 0 else to_dev(w, dtype)
                           for l, w in enumerate(wwg, start=1)], **kw)


def test_stack_bf16_write_gated_two_blocks():
    x, wq, wo, wr, H = small_bf16_stack(12, N=333, seed=93)
    wwg = wwg_weights(12, H, x.shape[-1], "bf16", 93)
    y, tro, tra = run_wg_stack(x, wq, wo, wr, wwg, H, "bf16")
    yref, tr = O.stack(x, wq, wo, wr, H, keep_trace=True, w_wg=wwg)
    for l in range(12):
        assert_close(tro[l], tr["o"][l], "bf16", f"o_{l + 1}")
    assert_close(y - x, yref - x, "bf16", "y - x")
    assert rel_l2(yref - x, O.stack(x, wq, wo, wr, H) - x) > 0.05   # the gate matters


def test_stack_fp32_write_gated_hybrid_group():
    w = W.HYBRID4_F32
    x = W.stack_x(w)
    p = W.stack_weights(w)
    wwg = wwg_weights(w.L, w.H, w.D, "f32", w.seed)
    y, tro, _ = run_wg_stack(x, p["w_qkvg"], p["w_o"], p["w_r"], wwg, w.H, "f32", attnres_block=0)
    yref, tr = O.stack(x, p["w_qkvg"], p["w_o"], p["w_r"], w.H, attnres_block=0, keep_trace=True,
                       w_wg=wwg)
    for l in range(w.L):
        assert_close(tro[l], tr["o"][l], "f32", f"o_{l + 1}")
    assert_close(y - x, yref - x, "f32", "y - x")


def test_stack_bf16_zero_write_gate_weights_double_eps():
    # W_wg = 0: every gate is sigmoid(0) = 1/2, which only doubles eps. eps is
    # set near the denominators phi(Q).z (about 300 keys x 20) so it matters.
    x, wq, wo, wr, H = small_bf16_stack(8, N=300, seed=94)
    zeros = [np.zeros((H, x.shape[-1]), np.float32) for _ in range(8)]
    y_wg, _, _ = run_wg_stack(x, wq, wo, wr, zeros, H, "bf16", eps=3000.0)
    y_2e, _, _ = run_stack(x, wq, wo, wr, H, "bf16", eps=6000.0)
    y_1e, _, _ = run_stack(x, wq, wo, wr, H, "bf16", eps=3000.0)
    assert rel_l2(y_wg - x, y_2e - x) < 2e-3
    assert rel_l2(y_1e - x, y_2e - x) > 2e-2


@pytest.mark.parametrize("n", [0, 1, 3])
def test_stack_host_batches_match_device_passes(n):
    # the pipelined host-batch call gives, bit for bit, what one device-resident
    # pass per batch gives (the same kernels on the same inputs)
    x, wq, wo, wr, H = small_bf16_stack(12, N=300, seed=97)
    st = sva.Stack([to_dev(w, "bf16") for w in wq], [to_dev(w, "bf16") for w in wo],
                   to_dev(wr, "bf16"), 1, 300, H)
    xs = [to_dev(W.round_to(np.random.default_rng(98 + i).standard_normal(x.shape)
                            .astype(np.float32), "bf16"), "bf16") for i in range(n)]
    xh = [t.cpu().pin_memory() for t in xs]
    yh = [torch.empty_like(t).pin_memory() for t in xh]
    ws, _ = sva.sva_hybrid_stack_fwd_host(st, xh, yh)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    for i in range(n):
        y = torch.empty_like(xs[i])
        sva.sva_hybrid_stack_fwd(st, xs[i], y)
        torch.cuda.synchronize()
        assert torch.equal(yh[i], y.cpu()), i


def test_stack_bf16_single_block_attnres_on_equals_off():
    x, wq, wo, wr, H = small_bf16_stack(8, N=257, seed=91)
    y_on, _, _ = run_stack(x, wq, wo, wr, H, "bf16", attnres_block=8)
    y_off, _, _ = run_stack(x, wq, wo, wr, H, "bf16", attnres_block=0)
    np.testing.assert_array_equal(y_on, y_off)
    yref = O.stack(x, wq, wo, wr, H)
    assert_close(y_on - x, yref - x, "bf16", "y - x")


def test_stack_bf16_all_softmax():
    x, wq, wo, wr, H = small_bf16_stack(8, N=300, seed=92)
    y, tro, _ = run_stack(x, wq, wo, wr, H, "bf16", all_softmax=True)
    yref, tr = O.stack(x, wq, wo, wr, H, all_softmax=True, keep_trace=True)
    for l in range(8):
        assert_close(tro[l], tr["o"][l], "bf16", f"o_{l + 1}")
    assert_close(y - x, yref - x, "bf16", "y - x")
