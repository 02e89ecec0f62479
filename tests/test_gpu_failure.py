"""The failure path of the library's bounded device waits, exercised on the GPU without a
fault: a wait that runs out records HYMBA_ERR_DEVICE_TIMEOUT and where it gave up, its
block drains what it issued and exits, and the context stays usable.

1. hymba_debug_stalled_wait: one block waits on an mbarrier that nothing arrives on (a
   flag that nothing sets), with a short limit; the status word must read
   HYMBA_ERR_DEVICE_TIMEOUT with a diagnosis record of role 4.
2. A bf16 layer (tcgen05 GEMMs and attention, bulk-copy decode attention) run with a
   limit of a few hundred cycles: every wait that is not already satisfied gives up.
   The call must end without a CUDA error, report either success or the timeout, and
   a normal call afterwards must match the oracle.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import assert_close, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _small_bf16():
    return synth.hymba15_layer_cfg(window=40).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                    dt_rank=24, n_meta=8)


def _prefill_and_decode(cfg, w, x, T, cap):
    """Prefill T tokens, then one decode step; returns (status, y_prefill, y_decode)."""
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    B = x.shape[0]
    layer = rt.DeviceLayer(cfg, w)
    kv = rt.KV(cfg, B, seq_cap=cfg.n_meta + T, cache_cap=cap)
    st = rt.State(cfg, B)
    y = torch.empty((B, cfg.n_meta + T, cfg.d_model), dtype=rt.act_dtype(cfg), device="cuda")
    rt.prefill(layer, rt.to_device(x[:, :T], cfg), T, kv, y, rt.workspace(cfg, B, T, hy.HYMBA_MODE_PREFILL), st)
    xt = rt.to_device(x[:, T], cfg)
    yt = torch.empty_like(xt)
    rt.decode(layer, xt, kv.s, st, yt, rt.workspace(cfg, B, cap, hy.HYMBA_MODE_DECODE))
    torch.cuda.synchronize()
    return hy.hymba_get_device_status(None), y, yt


def test_stalled_wait_reports_the_timeout_and_where():
    torch_cuda()
    import hybrid_head_ssm_b200 as hy
    assert hy.hymba_get_device_status(None) == hy.HYMBA_OK
    hy.check(hy.hymba_debug_set_wait_limit(1_000_000))  # about 0.5 ms
    try:
        hy.check(hy.hymba_debug_stalled_wait(hy.current_stream_ptr()))
        assert hy.hymba_get_device_status(None) == hy.HYMBA_ERR_DEVICE_TIMEOUT
        diag = hy.device_diag()
        assert diag[0] == 1 and diag[4] == 4, diag
        # both are cleared once read
        assert hy.hymba_get_device_status(None) == hy.HYMBA_OK
        assert hy.device_diag()[0] == 0
    finally:
        hy.check(hy.hymba_debug_set_wait_limit(0))


def test_layer_with_a_tiny_wait_limit_fails_cleanly_then_runs_normally():
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    cfg = _small_bf16()
    w = synth.layer_weights(cfg, 131)
    B, T, cap = 2, 70, cfg.n_meta + 40
    x = synth.layer_input(cfg, B, T + 1, 131)
    hy.check(hy.hymba_debug_set_wait_limit(256))
    try:
        status, _, _ = _prefill_and_decode(cfg, w, x, T, cap)
        assert status in (hy.HYMBA_OK, hy.HYMBA_ERR_DEVICE_TIMEOUT), status
        diag = hy.device_diag()
        if status == hy.HYMBA_ERR_DEVICE_TIMEOUT:
            assert diag[0] == 1 and diag[4] in (0, 1, 2, 3), diag
        print(f"tiny wait limit: status {status}, diagnosis {diag}")
    finally:
        hy.check(hy.hymba_debug_set_wait_limit(0))
    # the context is intact: the same calls with the default limit match the oracle
    status, y, yt = _prefill_and_decode(cfg, w, x, T, cap)
    assert status == hy.HYMBA_OK
    ref = oracle.mixer_prefill(cfg, w, x[:, :T])
    assert_close(to_np(y), ref["y"], cfg, "prefill after the timeouts")
    cache = oracle.cache_from_prefill(cfg, ref["k"], ref["v"], cap)
    yd = oracle.mixer_decode(cfg, w, x[:, T], cache, ref["h"].copy(), ref["conv"].copy())
    assert_close(to_np(yt), yd, cfg, "decode after the timeouts")
    assert torch.isfinite(yt.float()).all()
