"""GPU parity of the Hymba block around the mixer (pre-norm residual mixer, then the
pre-norm SiLU-gated MLP; the 51cto Hymba-1.5B article, section 2, gives the MLP
intermediate size 5504) against the fp64 oracle, through the C ABI: a KV-sharing pair
of blocks in prefill and then in decode, on the fp32 residual stream."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import assert_close, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _block_pair(base, d_ff, seed):
    ca, cb = base, base.with_(is_kv_producer=0)
    wa = synth.with_pre_norm(synth.perturbed_weights(synth.layer_weights(ca, seed), ca, seed), ca, seed, 0.3)
    wb = synth.with_pre_norm(synth.perturbed_weights(synth.layer_weights(cb, seed + 1), cb, seed + 1), cb, seed + 1,
                             0.3)
    fa = synth.mlp_weights(ca.d_model, d_ff, ca.dtype, seed + 2)
    fb = synth.mlp_weights(cb.d_model, d_ff, cb.dtype, seed + 3)
    return ca, cb, wa, wb, fa, fb


@pytest.mark.parametrize("case", ["f32_tiny", "bf16_small", "bf16_hymba15"])
def test_block_pair_prefill_then_decode(case):
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    if case == "f32_tiny":
        base, d_ff, B, T0, steps = synth.tiny_layer_cfg().with_(window=12), 512, 2, 40, 6
    elif case == "bf16_small":
        base = synth.hymba15_layer_cfg(window=24).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                        dt_rank=24, n_meta=8)
        d_ff, B, T0, steps = 704, 3, 60, 6
    else:
        base, d_ff, B, T0, steps = synth.hymba15_layer_cfg(1024), synth.HYMBA15_D_FF, 1, 1200, 2
    ca, cb, wa, wb, fa, fb = _block_pair(base, d_ff, 151)
    m = ca.n_meta
    Tp = m + T0
    g = np.random.default_rng(152)
    h_np = g.standard_normal((B, Tp + steps, ca.d_model)).astype(np.float32)
    h_np[:, :m] = wa["meta"].astype(np.float32)  # the stream starts with the meta rows
    # oracle: the pair of blocks on the prompt, then decode steps
    ra = oracle.block_prefill(ca, wa, fa, h_np[:, :Tp])
    rb = oracle.block_prefill(cb, wb, fb, ra["y"], kv_shared=(ra["k"], ra["v"]))
    cap = m + ca.window
    cache = oracle.cache_from_prefill(ca, ra["k"], ra["v"], cap)
    sa = [ra["h"].copy(), ra["conv"].copy()]
    sb = [rb["h"].copy(), rb["conv"].copy()]
    # GPU
    la, lb = rt.DeviceLayer(ca, wa), rt.DeviceLayer(cb, wb)
    ma, mb = rt.DeviceMLP(ca, fa), rt.DeviceMLP(cb, fb)
    kv = rt.KV(ca, B, seq_cap=Tp, cache_cap=cap)
    kvb = hy.hymba_kv()
    hy.check(hy.hymba_kv_share(ctypes.byref(kv.s), ctypes.byref(lb.c), ctypes.byref(kvb)))
    gsa, gsb = rt.State(ca, B), rt.State(cb, B)
    fl = hy.HYMBA_X_HAS_META | hy.HYMBA_ADD_RESIDUAL | hy.HYMBA_PRE_NORM | (
        hy.HYMBA_IO_F32 if ca.dtype == synth.BF16 else 0)
    h = torch.from_numpy(h_np[:, :Tp].copy()).cuda()
    ws = rt.workspace(ca, B, T0, hy.HYMBA_MODE_PREFILL)
    wm = rt.mlp_workspace(ma, B * Tp)
    rt.prefill(la, h, T0, kv, h, ws, gsa, fl)
    rt.mlp(ma, h, wm)
    rt.prefill(lb, h, T0, kv, h, ws, gsb, fl, kv_struct_override=kvb)
    rt.mlp(mb, h, wm)
    torch.cuda.synchronize()
    assert hy.hymba_get_device_status(None) == 0
    mx, rl = assert_close(to_np(h), rb["y"], cb, "block pair prefill")
    print(f"block pair {case}: prefill max abs {mx:.3e}, rel L2 {rl:.3e}")
    fld = fl & ~hy.HYMBA_X_HAS_META
    wda = rt.workspace(ca, B, cap, hy.HYMBA_MODE_DECODE)
    wdm = rt.mlp_workspace(ma, B)
    for s in range(steps):
        xt = h_np[:, Tp + s]
        ya = oracle.block_decode(ca, wa, fa, xt, cache, sa[0], sa[1])
        yb = oracle.block_decode(cb, wb, fb, ya, cache, sb[0], sb[1])
        t = torch.from_numpy(xt.copy()).cuda()
        rt.decode(la, t, kv.s, gsa, t, wda, fld)
        rt.mlp(ma, t, wdm)
        rt.decode(lb, t, kvb, gsb, t, wda, fld)
        rt.mlp(mb, t, wdm)
        torch.cuda.synchronize()
        assert_close(to_np(t), yb, cb, f"block pair decode step {s}")
    assert hy.hymba_get_device_status(None) == 0
