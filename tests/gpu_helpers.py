"""Shared pieces of the GPU parity tests: tolerances, comparisons, and runners that
call the library through its C ABI (hybrid_head_ssm_b200.runtime)."""
import numpy as np
import pytest

# Tolerances of the contract: bf16 layers max abs <= 2e-2 and relative L2 <= 5e-3;
# fp32 layers max abs <= 1e-4; indexing bit-exact.
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_MAX_ABS = 1e-4


def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def assert_close(got, ref, cfg, what="", max_abs=None, rel_l2=None):
    mx, rl = errors(got, ref)
    if cfg.dtype == 1:
        ma = BF16_MAX_ABS if max_abs is None else max_abs
        rt = BF16_REL_L2 if rel_l2 is None else rel_l2
        assert mx <= ma and rl <= rt, f"{what}: max abs {mx:.3e} (<= {ma}), rel L2 {rl:.3e} (<= {rt})"
    else:
        ma = F32_MAX_ABS if max_abs is None else max_abs
        assert mx <= ma, f"{what}: max abs {mx:.3e} (<= {ma}), rel L2 {rl:.3e}"
    return mx, rl


def to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


def merge_split_partials(part):
    """Softmax over the union of the key splits from per-split partials [..., dv + 2]:
    dv unnormalised sums of p v, then the split's max logit (base-2 domain) and its sum
    of p. Each split is rescaled by 2^(m_s - max m) before the sums are divided."""
    num, m, l = part[..., :-2], part[..., -2], part[..., -1]
    M = m.max(axis=-1, keepdims=True)
    w = np.where(np.isfinite(m), np.exp2(m - M), 0.0)
    return (w[..., None] * num).sum(axis=-2) / (w * l).sum(axis=-1)[..., None]
