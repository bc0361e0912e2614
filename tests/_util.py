"""Helpers shared by the GPU tests: moving the seeded inputs to the device and
comparing against the oracle with the tolerances the library commits to."""
import numpy as np

import workloads as W

# bf16 path: relative L2 <= 1e-2 and max-abs <= 3e-2 * max|ref|; fp32 path: 1e-5 relative L2
BF16_REL_L2, BF16_MAX_ABS = 1e-2, 3e-2
F32_REL_L2 = 1e-5


def to_dev(a: np.ndarray, dtype: str):
    """Exact values of `a` (already representable in dtype) as a CUDA tensor."""
    import torch
    if dtype == "bf16":
        bits = W.bf16_bits(a)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_host(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def rel_l2(x, ref) -> float:
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    return float(np.linalg.norm((x - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def assert_close(x, ref, dtype: str, what: str = ""):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), f"{what}: non-finite output"
    r = rel_l2(x, ref)
    if dtype == "bf16":
        m = float(np.abs(x - ref).max()) if x.size else 0.0
        bound = BF16_MAX_ABS * float(np.abs(ref).max()) if ref.size else 0.0
        assert r <= BF16_REL_L2, f"{what}: rel-L2 {r:.3e} > {BF16_REL_L2}"
        assert m <= bound, f"{what}: max-abs {m:.3e} > {bound:.3e}"
    else:
        assert r <= F32_REL_L2, f"{what}: rel-L2 {r:.3e} > {F32_REL_L2}"
    return r
