"""Parity at the workloads' full sizes, in the launch configurations bench.py
times (one call per layer over all heads): attention outputs are checked on
sampled query rows the oracle computes one by one against all keys (tile
edges, the pair boundary of the anchor's two-tile CTAs and the ragged tail
included); the 8-layer 480p stack is checked whole; the 24-layer 720p stack
is also checked through properties that hold at any
size (token-permutation equivariance, run-to-run determinism); the oracle's
whole-stack comparison of the 720p stack is in test_gpu_stacks_whole.py. The
anchor is also checked at the duration sweep's longest lengths (N = 148,120
and 221,720).

Inputs up to 720p come from the chunked numpy generator; the linear sweep's
largest lengths (1.9 GB per tensor) are drawn by torch's seeded generator on
the device and copied to the host in chunks for the oracle. The linear sweep
(B = 2, up to N = 150,880) is compared on every row: the oracle's linear layer
is O(N)."""
import math

import numpy as np
import pytest

import oracle as O
import workloads as W
from tests._util import BF16_MAX_ABS, BF16_REL_L2, assert_close, to_dev, to_host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import softmax_attention_video_gated_b200 as sva  # noqa: E402


def sample_rows(N, extra=40, seed=0):
    rows = {0, 1, 127, 128, 255, 256, 257, N - 1, N - 2, (N // 128) * 128, (N // 256) * 256,
            (N // 256) * 256 - 1}
    rows |= set(np.random.default_rng(seed).integers(0, N, extra).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N))


def run_core(kind, t, H):
    out = torch.empty_like(t["q"])
    if kind == "anchor":
        ws = sva.sva_softmax_anchor_fwd(t["q"], t["k"], t["v"], t["g"], out, H)
    else:
        ws = sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], out, H, eps=1e-6)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    return out


def check_rows(kind, x, out, H, rows):
    got = to_host(out[:, torch.as_tensor(rows, device="cuda")])
    if kind == "anchor":
        ref = O.softmax_anchor(x["q"][:, rows], x["k"], x["v"], x["g"][:, rows], H)
    else:
        ref = O.linear_attn(x["q"][:, rows], x["k"], x["v"], x["g"][:, rows], H, eps=1e-6)
    assert_close(got, ref, "bf16", f"{kind} sampled rows")


# ------------------------------------------------------------------ 720p layer shapes

@pytest.fixture(scope="module")
def core720():
    w = W.STACK720P
    x = W.core_inputs_par(w.B, w.N, w.H, w.d, "bf16", w.seed)
    return x, {k: to_dev(v, "bf16") for k, v in x.items()}


@pytest.mark.parametrize("kind", ["anchor", "linear"])
def test_720p_layer_sampled_rows(core720, kind):
    x, t = core720
    out = run_core(kind, t, W.STACK720P.H)
    check_rows(kind, x, out, W.STACK720P.H, sample_rows(W.STACK720P.N))


def test_720p_write_gated_linear_layer_sampled_rows(core720):
    # write-gate logits [B, N, H] ~ N(0, 1), the spread of u W_wg^T at the
    # stack's weight scale
    x, t = core720
    w = W.STACK720P
    wg = W.normal((w.B, w.N, w.H), 1.0, w.seed, W.TAG_WGATE, "bf16")
    out = torch.empty_like(t["q"])
    ws = sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], out, w.H, eps=1e-6,
                                 wgate=to_dev(wg, "bf16"))
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    rows = sample_rows(w.N, seed=2)
    ref = O.linear_attn(x["q"][:, rows], x["k"], x["v"], x["g"][:, rows], w.H, eps=1e-6, wgate=wg)
    assert_close(to_host(out[:, torch.as_tensor(rows, device="cuda")]), ref, "bf16",
                 "720p write-gated linear sampled rows")


# ------------------------------------------------------------------ long video (N = 37,720)

def test_long_video_layers_sampled_rows():
    w = W.LONG4
    x = W.core_inputs_par(w.B, w.N, w.H, w.d, "bf16", w.seed)
    t = {k: to_dev(v, "bf16") for k, v in x.items()}
    rows = sample_rows(w.N, seed=1)
    for kind in ("anchor", "linear"):
        check_rows(kind, x, run_core(kind, t, w.H), w.H, rows)


# ------------------------------------------------------------------ anchor at long-video lengths

@pytest.mark.parametrize("N", [148120, 221720])
def test_anchor_long_duration_sampled_rows(N):
    # the softmax anchor at 161 and 241 latent frames of 23 x 40 patches (the
    # 40 s and 60 s rows of the duration sweep), one call over all 24 heads, as
    # the sweep times it; inputs drawn on the device, K and V copied to the host
    # in bf16 and handed to the oracle one head at a time (heads are independent)
    H, d, seed = 24, 128, 1234 + 5
    D = H * d
    t = {name: W.normal_torch((1, N, D), 1.0, seed, tag, "bf16")
         for name, tag in (("q", W.TAG_Q), ("k", W.TAG_K), ("v", W.TAG_V), ("g", W.TAG_G))}
    out = run_core("anchor", t, H)
    rows = sample_rows(N, seed=N)
    ri = torch.as_tensor(rows, device="cuda")
    q, g = to_host(t["q"][:, ri]), to_host(t["g"][:, ri])
    got = to_host(out[:, ri])
    k_h, v_h = t["k"].cpu(), t["v"].cpu()
    del t, out
    ref = np.empty_like(got)
    for h in range(H):
        c = slice(h * d, (h + 1) * d)
        ref[..., c] = O.softmax_anchor(q[..., c], k_h[..., c].to(torch.float64).numpy(),
                                       v_h[..., c].to(torch.float64).numpy(), g[..., c], 1)
    assert_close(got, ref, "bf16", f"anchor sampled rows N={N}")


# ------------------------------------------------------------------ linear sweep (B = 2)

@pytest.mark.parametrize("N", list(W.LINSWEEP.Ns))
def test_linear_sweep_all_rows(N):
    # the isolated linear layer at B = 2 (a CFG pair): every output row against
    # the oracle, which is O(N): its state over all N tokens, summed chunk by
    # chunk (S = sum_t ...), then the read-out of every row, chunk by chunk
    c = W.LINSWEEP
    D = c.H * c.d
    t = {name: W.normal_torch((c.B, N, D), 1.0, c.seed, tag, "bf16")
         for name, tag in (("q", W.TAG_Q), ("k", W.TAG_K), ("v", W.TAG_V), ("g", W.TAG_G))}
    out = run_core("linear", t, c.H)
    S = np.zeros((c.B, c.H, c.d, c.d))
    z = np.zeros((c.B, c.H, c.d))
    for t0 in range(0, N, 4096):
        Sc, zc = O.lin_state(to_host(t["k"][:, t0:t0 + 4096]), to_host(t["v"][:, t0:t0 + 4096]), c.H)
        S += Sc
        z += zc
    num = den = 0.0
    worst_abs, ref_max = 0.0, 0.0
    for t0 in range(0, N, 4096):
        q, g = to_host(t["q"][:, t0:t0 + 4096]), to_host(t["g"][:, t0:t0 + 4096])
        ref = O.gate(O.lin_readout(q, S, z, c.H, 1e-6), g)
        got = to_host(out[:, t0:t0 + 4096])
        assert np.all(np.isfinite(got))
        num += float(np.sum((got - ref) ** 2))
        den += float(np.sum(ref ** 2))
        worst_abs = max(worst_abs, float(np.abs(got - ref).max()))
        ref_max = max(ref_max, float(np.abs(ref).max()))
    # the bf16 bounds of tests/_util.py over all B * N rows
    assert math.sqrt(num / den) <= BF16_REL_L2, f"linear sweep N={N}: rel-L2 {math.sqrt(num / den):.3e}"
    assert worst_abs <= BF16_MAX_ABS * ref_max, f"linear sweep N={N}: max-abs {worst_abs:.3e}"


# ------------------------------------------------------------------ 480p stack, whole

def test_480p_stack_whole():
    w = W.STACK480P
    D, std = w.D, w.weight_std
    x = W.normal_par((w.B, w.N, D), 1.0, w.seed, W.TAG_X, "bf16")
    wq = [W.normal_par((4 * D, D), std, w.seed, W.TAG_WQKVG + l, "bf16") for l in range(1, w.L + 1)]
    wo = [W.normal_par((D, D), std, w.seed, W.TAG_WO + l, "bf16") for l in range(1, w.L + 1)]
    wr = W.normal_par((D, D), std, w.seed, W.TAG_WR, "bf16")
    trace_o = [torch.empty(w.B * w.N, D, device="cuda", dtype=torch.float32) for _ in range(w.L)]
    st = sva.Stack([to_dev(a, "bf16") for a in wq], [to_dev(a, "bf16") for a in wo],
                   to_dev(wr, "bf16"), w.B, w.N, w.H, attnres_block=w.attnres_block,
                   trace_o=trace_o)
    xt = to_dev(x, "bf16")
    y = torch.empty_like(xt)
    ws = sva.sva_hybrid_stack_fwd(st, xt, y)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    yref, tr = O.stack(x, wq, wo, wr, w.H, attnres_block=w.attnres_block, keep_trace=True)
    for l in range(w.L):
        assert_close(to_host(trace_o[l]).reshape(x.shape), tr["o"][l], "bf16", f"480p o_{l + 1}")
    # the fp32 residual update h_L - x (the bf16 rounding of y alone is ~2^-9 |x|,
    # not small next to the mixer's signal), then y itself
    update = to_host(torch.stack(trace_o).sum(0)).reshape(x.shape)
    assert_close(update, yref - x, "bf16", "480p h_L - x")
    assert_close(to_host(y), yref, "bf16", "480p y")


# ------------------------------------------------------------------ 720p stack, properties

@pytest.fixture(scope="module")
def stack720():
    w = W.STACK720P
    D, std = w.D, w.weight_std
    wq = [W.normal_torch((4 * D, D), std, w.seed, W.TAG_WQKVG + l, "bf16") for l in range(1, w.L + 1)]
    wo = [W.normal_torch((D, D), std, w.seed, W.TAG_WO + l, "bf16") for l in range(1, w.L + 1)]
    wr = W.normal_torch((D, D), std, w.seed, W.TAG_WR, "bf16")
    trace_o = [torch.empty(w.B * w.N, D, device="cuda", dtype=torch.float32) for _ in range(w.L)]
    st = sva.Stack(wq, wo, wr, w.B, w.N, w.H, trace_o=trace_o)
    x = W.normal_torch((w.B, w.N, D), 1.0, w.seed, W.TAG_X, "bf16")
    ws = sva.workspace(st.workspace_bytes())

    def run(inp):
        # returns y and the fp32 residual update h_L - x = sum_l o_l
        y = torch.empty_like(inp)
        sva.sva_hybrid_stack_fwd(st, inp, y, ws=ws)
        assert sva.sva_check_device_status(ws) == sva.SVA_OK
        return y, torch.stack(trace_o).sum(0).view(inp.shape)

    return x, run


def test_720p_stack_is_deterministic(stack720):
    x, run = stack720
    (y1, u1), (y2, u2) = run(x), run(x)
    assert torch.equal(y1, y2) and torch.equal(u1, u2)


def test_720p_stack_token_permutation_equivariance(stack720):
    # every layer is non-causal and the router works per token, so permuting
    # the tokens of x permutes the output
    x, run = stack720
    perm = torch.as_tensor(np.random.default_rng(3).permutation(x.shape[1]), device="cuda")
    _, u = run(x)
    u = u[:, perm].clone()
    _, up = run(x[:, perm].contiguous())
    assert_close(to_host(up), to_host(u), "bf16", "720p permuted h_L - x")
