"""GPU parity of the 32-layer mixer stack (B=8, T=4096 + 128 meta, layers 0/15/31
global, consecutive pairs sharing KV, fp32 residual stream between the bf16 layers),
run at full size through the C ABI. The oracle recomputes sequence 0 from the same
seeded inputs on its own, over a prefix of the positions: outputs at a position
depend only on earlier positions, so the GPU's full-size outputs there are exact
samples of the full computation."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import assert_close, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def run_stack_gpu(wl, x):
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    cfgs = synth.stack_layer_cfgs(wl["cfg"], wl["n_layers"], wl["global_layers"])
    B, T = x.shape[0], x.shape[1]
    Tp = cfgs[0].n_meta + T
    h = rt.to_device(x, cfgs[0], io_f32=True)
    out = torch.empty((B, Tp, cfgs[0].d_model), dtype=torch.float32, device="cuda")
    ws = rt.workspace(cfgs[0], B, T, hy.HYMBA_MODE_PREFILL)
    kv = None
    for l, cfg in enumerate(cfgs):
        layer = rt.DeviceLayer(cfg, synth.layer_weights(cfg, 1000 * wl["seed"] + l))
        fl = rt.stream_flags(cfg) | (hy.HYMBA_X_HAS_META if l > 0 else 0)
        if cfg.is_kv_producer:
            kv = rt.KV(cfg, B, seq_cap=Tp)
            kvs = kv.s
        else:
            kvs = hy.hymba_kv()
            hy.check(hy.hymba_kv_share(ctypes.byref(kv.s), ctypes.byref(layer.c), ctypes.byref(kvs)))
        if l == 0:
            rt.prefill(layer, h, T, kv, out, ws, None, fl, kv_struct_override=kvs)
        else:
            rt.prefill(layer, out, T, kv, out, ws, None, fl, kv_struct_override=kvs)  # in place
        del layer
    torch.cuda.synchronize()
    assert hy.hymba_get_device_status(None) == 0
    return out


def run_stack_oracle(wl, x_row, T_prefix):
    cfgs = synth.stack_layer_cfgs(wl["cfg"], wl["n_layers"], wl["global_layers"])
    h = x_row[None, :T_prefix]
    kv = None
    for l, cfg in enumerate(cfgs):
        w = synth.layer_weights(cfg, 1000 * wl["seed"] + l)
        r = oracle.mixer_prefill(cfg, w, h, kv_shared=None if cfg.is_kv_producer else kv, residual=True,
                                 x_has_meta=l > 0)
        if cfg.is_kv_producer:
            kv = (r["k"], r["v"])
        h = r["y"]
    return h[0]


def test_stack32_full_size_prefix_of_sequence0():
    wl = synth.workload("hymba15_stack32_b8_t4096")
    x = synth.layer_input(wl["cfg"], wl["B"], wl["T"], wl["seed"])
    y = to_np(run_stack_gpu(wl, x))
    T_prefix = 1536  # 1664 rows: past the 1024 window, so the sliding window is exercised
    ref = run_stack_oracle(wl, x[0], T_prefix)
    m = wl["cfg"].n_meta
    mx, rl = assert_close(y[0, :m + T_prefix], ref, wl["cfg"], "stack output, sequence 0")
    print(f"32-layer stack, sequence 0, {m + T_prefix} rows: max abs {mx:.3e}, rel L2 {rl:.3e}")
