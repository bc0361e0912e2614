"""The allocation-free linear-attention entry point, for callers that cannot
allocate device memory (an engine with a fixed memory plan, a plugin handed a
stream but no allocator): it must give the same results as the workspace entry
point and match the fp64 oracle, call after call, while its scratch lives in
the library's fixed device array. Collected last so a failure here leaves every
other test already run."""
import ctypes

import numpy as np
import pytest

import oracle as O
import workloads as W
from tests._util import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import softmax_attention_video_gated_b200 as sva  # noqa: E402


def noalloc_call(q, k, v, g, out, H, eps=1e-6, residual=None, wgate=None):
    a = sva._attn_args(q, k, v, g, out, H, residual, eps, 0.0, 0, wgate)
    return sva._lib().sva_linear_attn_fwd_noalloc(ctypes.byref(a), sva._stream())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(dtype):
    # two calls with different shapes and values: the second must not see the
    # first one's scratch
    for B, N, H, seed in ((2, 1000, 2, 101), (1, 3001, 3, 102)):
        x = W.core_inputs(B, N, H, 128, dtype, seed)
        t = {k: to_dev(v, dtype) for k, v in x.items()}
        ref = torch.empty_like(t["q"])
        sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], ref, H, eps=1e-6)
        out = torch.full_like(t["q"], float("nan"))
        assert noalloc_call(t["q"], t["k"], t["v"], t["g"], out, H) == sva.SVA_OK
        torch.cuda.synchronize()
        assert_close(to_host(out), to_host(ref), dtype, f"noalloc B={B} N={N}")
        want = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6)
        assert_close(to_host(out), want, dtype, f"noalloc B={B} N={N} vs oracle")


def test_noalloc_with_residual_and_write_gate_matches_workspace_entry_point():
    # the residual and write-gate operands go through the same validation and
    # kernels as in the workspace entry point; out aliases the residual
    B, N, H = 1, 2333, 2
    x = W.core_inputs(B, N, H, 128, "bf16", 103)
    t = {k: to_dev(v, "bf16") for k, v in x.items()}
    wg_h = W.normal((B, N, H), 1.0, 103, W.TAG_WGATE, "bf16")
    wg = to_dev(wg_h, "bf16")
    # a residual of the layer output's own scale (~0.05), so neither term hides the other
    r_h = W.normal((B, N, H * 128), 0.05, 104, W.TAG_X, "bf16")
    r = to_dev(r_h, "bf16")
    want = O.linear_attn(x["q"], x["k"], x["v"], x["g"], H, eps=1e-6, residual=r_h, wgate=wg_h)
    for _ in range(2):
        ref = r.clone()
        sva.sva_linear_attn_fwd(t["q"], t["k"], t["v"], t["g"], ref, H, residual=ref, eps=1e-6,
                                wgate=wg)
        out = r.clone()
        assert noalloc_call(t["q"], t["k"], t["v"], t["g"], out, H, residual=out,
                            wgate=wg) == sva.SVA_OK
        torch.cuda.synchronize()
        assert_close(to_host(out), to_host(ref), "bf16", "noalloc residual + write gate")
        assert_close(to_host(out), want, "bf16", "noalloc residual + write gate vs oracle")


def test_noalloc_refuses_calls_beyond_its_scratch():
    # fp32, 128 heads of d = 128 over 100k tokens needs far more than 16 MiB
    a = sva.AttnArgs()
    a.B, a.N, a.H, a.d, a.dtype = 1, 100000, 128, 128, sva.SVA_F32
    for f in ("q", "k", "v", "gate", "out"):
        setattr(a, f, 0x10000)
    a.ldq = a.ldk = a.ldv = a.ldg = a.ldo = 128 * 128
    a.eps = 1e-6
    assert sva._lib().sva_linear_attn_fwd_noalloc(ctypes.byref(a), None) == sva.SVA_ERR_WORKSPACE
