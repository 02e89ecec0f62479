"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/hymba.h declares, its host-only helpers agree with the oracle and
the pages' printed cache sizes, and argument errors are caught before any launch."""
import ctypes
import json
import os
import re

import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hy():
    import hybrid_head_ssm_b200 as hy
    return hy


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(hymba_\w+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_function(hy):
    declared = _declared()
    assert "hymba_mixer_prefill" in declared and "hymba_kv_share" in declared
    lib = ctypes.CDLL(hy.LIB_PATH)
    for n in declared:
        assert hasattr(lib, n), n
        assert n in hy.EXPORTS, n


def test_kv_bytes_matches_pages(hy):
    gold = json.load(open(os.path.join(ROOT, "tests", "golden", "cache_sizes.json")))
    ex = gold["jamba_worked_example"]
    assert hy.hymba_kv_bytes(32, 8, 128, 128, 64000, 4, 2) == ex["dense_32_layers_bytes"]
    assert hy.hymba_kv_bytes(4, 8, 128, 128, 64000, 4, 2) == ex["hybrid_4_layers_bytes"]
    assert hy.hymba_kv_bytes(1, 8, 128, 128, 1, 1, 2) == ex["bytes_per_token_layer"]
    assert hy.hymba_ssm_state_bytes(64, 64 * 64, 128, 1, 2) == oracle.ssm_state_bytes(64, 4096, 128, 1, 2)
    assert hy.hymba_kv_bytes(80, 8, 128, 128, 128000, 1, 2) == oracle.kv_cache_bytes(80, 8, 128, 128000, 1, 2)


@pytest.mark.parametrize("window,producer", [(1024, 1), (0, 1), (1024, 0)])
def test_cache_bytes_matches_oracle(hy, window, producer):
    cfg = synth.hymba15_layer_cfg(window, producer)
    c = hy.cfg_struct(cfg)
    for B, T in [(1, 100), (64, 4224)]:
        assert hy.hymba_cache_bytes(ctypes.byref(c), B, T) == oracle.layer_cache_bytes(cfg, B, T)


def test_workspace_layout_is_consistent(hy):
    cfg = synth.hymba15_layer_cfg(1024)
    c = hy.cfg_struct(cfg)
    lay = hy.workspace_layout(c, 1, 2048, hy.HYMBA_MODE_PREFILL)
    assert lay["total"] == hy.hymba_workspace_bytes(ctypes.byref(c), 1, 2048, hy.HYMBA_MODE_PREFILL)
    assert lay["ldP"] % 64 == 0 and lay["ldP"] >= cfg.n_in
    offs = sorted(lay[k] for k in ("P", "delta", "O", "ypre", "U"))
    assert all(o % 256 == 0 for o in offs)
    assert len(set(offs)) == 5
    dec = hy.workspace_layout(c, 64, 1152, hy.HYMBA_MODE_DECODE)
    assert dec["n_split"] >= 1 and dec["part"] > 0
    # every split holds at most 256 keys (the decode attention's score buffer), and the
    # partials [B, H, splits, v_head_dim + 4] fp32 fit the last segment
    assert -(-1152 // dec["n_split"]) <= 256
    assert dec["total"] - dec["part"] >= 64 * cfg.n_q_heads * dec["n_split"] * (cfg.v_head_dim + 4) * 4


def test_invalid_configs_rejected(hy):
    base = synth.tiny_layer_cfg()
    for bad in (base.with_(head_dim=32), base.with_(d_state=8), base.with_(n_kv_heads=3),
                base.with_(v_head_dim=64), base.with_(dtype=7), base.with_(d_model=0), base.with_(fusion=2),
                base.with_(fusion=1, v_head_dim=96), base.with_(ssm_heads=-1), base.with_(ssm_heads=3),
                base.with_(ssm_heads=128), synth.hymba15_layer_cfg(1024).with_(ssm_heads=25)):
        c = hy.cfg_struct(bad)
        assert hy.hymba_workspace_bytes(ctypes.byref(c), 1, 10, 0) == 0
        assert hy.hymba_cache_bytes(ctypes.byref(c), 1, 10) == 0


def test_ssd_form_configs_accepted(hy):
    """The SSD form: any head width that is a multiple of 8 for fp32, 64 for bf16 (the
    tensor-core chunk kernel's width)."""
    for ok in (synth.tiny_layer_cfg().with_(ssm_heads=4), synth.tiny_layer_cfg().with_(ssm_heads=64),
               synth.hymba15_layer_cfg(1024).with_(ssm_heads=50)):
        c = hy.cfg_struct(ok)
        assert hy.hymba_workspace_bytes(ctypes.byref(c), 1, 10, 0) > 0


def test_concat_fusion_workspace_holds_the_wider_u(hy):
    """The concat fusion's U is d_inner + H * dv wide (the input of W_o); its 64-wide V
    heads need not add up to d_inner."""
    cat = synth.hymba15_layer_cfg(1024).with_(fusion=1, v_head_dim=64)
    lc = hy.workspace_layout(hy.cfg_struct(cat), 2, 100, hy.HYMBA_MODE_PREFILL)
    rows = 2 * (cat.n_meta + 100)
    assert cat.u_width == 3200 + 25 * 64
    order = sorted((lc[k], k) for k in ("P", "delta", "O", "ypre", "U", "rope"))
    nxt = {k: order[i + 1][0] for i, (_, k) in enumerate(order[:-1])}
    assert lc["total"] - lc["U"] >= rows * cat.u_width * 2  # U is the last of the exposed blocks
    assert nxt["O"] - lc["O"] >= rows * 25 * 64 * 2


def test_prefill_argument_errors_before_any_launch(hy):
    cfg = synth.tiny_layer_cfg()
    c = hy.cfg_struct(cfg)
    w = hy.hymba_layer_weights()
    kv = hy.hymba_kv()
    rc = hy.hymba_mixer_prefill(ctypes.byref(c), ctypes.byref(w), None, 1, 10, 0, None, ctypes.byref(kv),
                                None, None, 0, None)
    assert rc == hy.HYMBA_ERR_INVALID_ARG
    bad = hy.cfg_struct(cfg.with_(head_dim=48))
    rc = hy.hymba_mixer_prefill(ctypes.byref(bad), ctypes.byref(w), None, 1, 10, 0, None, ctypes.byref(kv),
                                None, None, 0, None)
    assert rc == hy.HYMBA_ERR_UNSUPPORTED
    # all pointers "present" (fake host addresses, never dereferenced) but workspace too small
    fake = 1 << 20
    wf = hy.hymba_layer_weights(*([fake] * 13))  # no affine shared-KV vectors
    kvf = hy.kv_struct(cfg, 1)
    kvf.k_seq = kvf.v_seq = fake
    kvf.seq_cap = cfg.n_meta + 10
    rc = hy.hymba_mixer_prefill(ctypes.byref(c), ctypes.byref(wf), 1 << 24, 1, 10, 0, 1 << 28, ctypes.byref(kvf),
                                None, 1 << 30, 256, None)
    assert rc == hy.HYMBA_ERR_WORKSPACE_TOO_SMALL
    kvf.seq_cap = 5
    rc = hy.hymba_mixer_prefill(ctypes.byref(c), ctypes.byref(wf), 1 << 24, 1, 10, 0, 1 << 28, ctypes.byref(kvf),
                                None, 1 << 30, 1 << 40, None)
    assert rc == hy.HYMBA_ERR_KV_INCOMPATIBLE
    # x and y overlap without the in-place form
    kvf.seq_cap = cfg.n_meta + 10
    rc = hy.hymba_mixer_prefill(ctypes.byref(c), ctypes.byref(wf), 1 << 24, 1, 10, 0, (1 << 24) + 64,
                                ctypes.byref(kvf), None, 1 << 30, 1 << 40, None)
    assert rc == hy.HYMBA_ERR_INVALID_ARG


def test_decode_argument_errors_before_any_launch(hy):
    """Every argument check of hymba_mixer_decode runs before the device is touched
    (fake host addresses, never dereferenced)."""
    cfg = synth.tiny_layer_cfg().with_(window=8)
    c = hy.cfg_struct(cfg)
    fake = 1 << 20
    wf = hy.hymba_layer_weights(*([fake] * 13))
    B = 2
    kv = hy.kv_struct(cfg, B)
    kv.k_cache = kv.v_cache = kv.len = fake
    kv.cache_cap = cfg.n_meta + 8
    st = hy.hymba_ssm_state(fake, fake)
    need = hy.hymba_workspace_bytes(ctypes.byref(c), B, kv.cache_cap, hy.HYMBA_MODE_DECODE)
    assert need > 0

    def call(cfg_s=c, x=1 << 24, flags=0, kv_s=kv, st_s=st, ws=1 << 30, ws_bytes=need, b=B):
        return hy.hymba_mixer_decode(ctypes.byref(cfg_s), ctypes.byref(wf), x, b, flags, 1 << 26,
                                     ctypes.byref(kv_s), ctypes.byref(st_s), ws, ws_bytes, None)

    assert call(ws_bytes=need - 256) == hy.HYMBA_ERR_WORKSPACE_TOO_SMALL
    assert call(x=None) == hy.HYMBA_ERR_INVALID_ARG
    assert call(b=0) == hy.HYMBA_ERR_INVALID_ARG
    assert call(st_s=hy.hymba_ssm_state(None, fake)) == hy.HYMBA_ERR_INVALID_ARG
    assert call(ws=(1 << 30) + 64) == hy.HYMBA_ERR_INVALID_ARG           # not 256-byte aligned
    assert call(flags=hy.HYMBA_IO_F32) == hy.HYMBA_ERR_INVALID_ARG       # fp32 layer
    assert call(flags=1 << 12) == hy.HYMBA_ERR_INVALID_ARG               # unknown flag
    short = hy.kv_struct(cfg, B)
    short.k_cache = short.v_cache = short.len = fake
    short.cache_cap = cfg.n_meta                                          # no ring slot
    assert call(kv_s=short) == hy.HYMBA_ERR_INVALID_ARG
    assert call(cfg_s=hy.cfg_struct(cfg.with_(head_dim=48))) == hy.HYMBA_ERR_UNSUPPORTED


def test_kv_share_rules(hy):
    prod_cfg = synth.tiny_layer_cfg().with_(window=8)
    kv = hy.kv_struct(prod_cfg, 2)
    kv.k_seq = kv.v_seq = 4096
    kv.seq_cap = 100
    out = hy.hymba_kv()
    # consumer with the same span: fine, pointers copied
    cons = hy.cfg_struct(prod_cfg.with_(is_kv_producer=0))
    assert hy.hymba_kv_share(ctypes.byref(kv), ctypes.byref(cons), ctypes.byref(out)) == 0
    assert out.k_seq == kv.k_seq and out.seq_cap == 100
    # a producer config cannot be a consumer
    assert hy.hymba_kv_share(ctypes.byref(kv), ctypes.byref(hy.cfg_struct(prod_cfg)), ctypes.byref(out)) == hy.HYMBA_ERR_INVALID_ARG
    # decode ring of 8 slots: a window-16 consumer does not fit, a global one neither
    kv.k_cache = kv.v_cache = kv.len = 8192
    kv.cache_cap = prod_cfg.n_meta + 8
    for w in (16, 0):
        c2 = hy.cfg_struct(prod_cfg.with_(is_kv_producer=0, window=w))
        assert hy.hymba_kv_share(ctypes.byref(kv), ctypes.byref(c2), ctypes.byref(out)) == hy.HYMBA_ERR_KV_INCOMPATIBLE
    # a different KV head count is incompatible
    c3 = hy.cfg_struct(prod_cfg.with_(is_kv_producer=0, n_kv_heads=4))
    assert hy.hymba_kv_share(ctypes.byref(kv), ctypes.byref(c3), ctypes.byref(out)) == hy.HYMBA_ERR_KV_INCOMPATIBLE


def test_strerror_covers_codes(hy):
    for code in range(0, -9, -1):
        assert hy.hymba_strerror(code).decode() != "unknown status"
    assert hy.hymba_strerror(-99).decode() == "unknown status"
