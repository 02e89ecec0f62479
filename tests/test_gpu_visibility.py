"""Bit-exact visible sets of the attention kernels on the GPU, through the C ABI.

Key j is visible to query i iff j <= i and (j < n_meta or i - j < window) ("Hymba
Guide", Learnable Meta-Tokens: every query attends to the meta prefix; 51cto
Hymba-1.5B article, section 2: sliding-window attention, global in a few layers).
The oracle's `visibility_mask` states that rule; here the GPU kernels must reproduce
it exactly, key by key.

Method: a consumer layer (it reads caller-owned K/V) is given K = 0, so every score
is 0 and the softmax weight of every visible key is exactly 1 / |S_i| (P = 2^0 = 1 in
the kernels, the row sum the count of visible keys). V carries one-hot codes: in run
r, the V row of position (or cache slot) j of KV head g is (b + 1) times the unit
vector e_c when j = r * G * dv + g * dv + c, else 0. Query head h of group g then
returns (b + 1) / |S_i| in column c exactly when key r*G*dv + g*dv + c is visible to
it, and 0 otherwise. The nonzero pattern is compared with the mask bit for bit; the
values check the count |S_i|, the sequence (factor b + 1) and the KV head (the
column offset) that was read.

Prefill: the bf16 path runs the tcgen05 flash kernel (query tiles of 128, key blocks
of 128 that skip invisible blocks), the fp32 path the CUDA-core kernel. Decode: the
split-KV partials a decode step leaves in its workspace (per split: sum of p v, max,
sum of p) reveal the visible slots directly, since p = 1; the allocation-free entry
point is checked on its normalised output.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import torch_cuda

pytestmark = pytest.mark.gpu


def _runs(n_keys, G, dv):
    return -(-n_keys // (G * dv))


def _onehot_v(B, G, n_keys, dv, r, torch, dtype):
    """[B, G, n_keys, dv]: (b + 1) * e_c at key j = r*G*dv + g*dv + c."""
    v = torch.zeros((B, G, n_keys, dv), dtype=dtype, device="cuda")
    base = r * G * dv
    scale = torch.arange(1, B + 1, dtype=torch.float32, device="cuda").to(dtype).view(B, 1)
    for g in range(G):
        lo = base + g * dv
        hi = min(lo + dv, n_keys)
        if lo >= hi:
            continue
        idx = torch.arange(lo, hi, device="cuda")
        v[:, g, idx, idx - lo] = scale
    return v


def _expected_cols(mask_row_block, G, H, dv, r):
    """[Lq, H*dv] bool: column h*dv + c is on iff key r*G*dv + g(h)*dv + c is visible."""
    Lq, Lk = mask_row_block.shape
    out = np.zeros((Lq, H * dv), dtype=bool)
    base = r * G * dv
    for h in range(H):
        g = oracle.gqa_group(h, H, G)
        lo = base + g * dv
        hi = min(lo + dv, Lk)
        if lo < hi:
            out[:, h * dv:h * dv + (hi - lo)] = mask_row_block[:, lo:hi]
    return out


def _check_run(got, mask, B, G, H, dv, r, what):
    """got [B, Lq, H*dv] (fp32 view of the kernel's output for run r)."""
    n_vis = mask.sum(axis=1).astype(np.float64)
    exp_on = _expected_cols(mask, G, H, dv, r)
    for b in range(B):
        on = got[b] != 0
        bad = np.argwhere(on != exp_on)
        assert bad.size == 0, (f"{what}: run {r}, sequence {b}: {len(bad)} visibility mismatches, first "
                               f"(query, column) {bad[:5].tolist()}")
        want = (b + 1) / n_vis[:, None] * np.ones((1, H * dv))
        rel = np.abs(got[b][exp_on] - want[exp_on]) / want[exp_on]
        assert rel.size == 0 or rel.max() <= 1e-3, f"{what}: run {r}, sequence {b}: value rel err {rel.max():.2e}"


def _prefill_visibility(cfg, B, T, seed):
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    cfg = cfg.with_(is_kv_producer=0)
    m, Tp = cfg.n_meta, cfg.n_meta + T
    H, G, dh, dv = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim
    mdt = rt.mid_dtype(cfg)
    layer = rt.DeviceLayer(cfg, synth.layer_weights(cfg, seed))
    x = rt.to_device(synth.layer_input(cfg, B, T, seed), cfg)
    y = torch.empty((B, Tp, cfg.d_model), dtype=rt.act_dtype(cfg), device="cuda")
    ws = rt.workspace(cfg, B, T, hy.HYMBA_MODE_PREFILL)
    lay = hy.workspace_layout(layer.c, B, T, hy.HYMBA_MODE_PREFILL)
    esz = torch.tensor([], dtype=mdt).element_size()
    k_seq = torch.zeros((B, G, Tp, dh), dtype=mdt, device="cuda")
    pos = np.arange(Tp)
    mask = oracle.visibility_mask(pos, pos, m, cfg.window)
    for r in range(_runs(Tp, G, dv)):
        v_seq = _onehot_v(B, G, Tp, dv, r, torch, mdt)
        kvs = hy.kv_struct(cfg, B, k_seq, v_seq)
        ws.fill_(0xFF)
        rt.prefill(layer, x, T, None, y, ws, None, 0, kv_struct_override=kvs)
        torch.cuda.synchronize()
        assert hy.hymba_get_device_status(None) == 0
        n = B * Tp * H * dv
        o = ws[lay["O"]:lay["O"] + n * esz].view(mdt).view(B, Tp, H * dv).float().cpu().numpy()
        _check_run(o, mask, B, G, H, dv, r, f"prefill {cfg.window=} {m=} {T=}")


@pytest.mark.parametrize("case", ["swa1024_meta128_t2048", "global_meta128_b2_t700", "swa200_nometa_t500",
                                  "swa5_meta16_b3_t333"])
def test_bf16_prefill_attention_visible_set_bit_exact(case):
    """The tcgen05 prefill attention of a bf16 layer visits exactly the visible keys:
    the 1.5B SWA layer (meta 128, window 1024, T 2048), a global layer with a ragged
    last query tile, no meta tokens, and a window far smaller than a key block."""
    base = synth.hymba15_layer_cfg(1024)
    if case == "swa1024_meta128_t2048":
        _prefill_visibility(base, 1, 2048, 11)
    elif case == "global_meta128_b2_t700":
        _prefill_visibility(base.with_(window=0), 2, 700, 12)
    elif case == "swa200_nometa_t500":
        _prefill_visibility(base.with_(window=200, n_meta=0), 1, 500, 13)
    else:
        small = base.with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640, dt_rank=24, n_meta=16, window=5)
        _prefill_visibility(small, 3, 333, 14)


def test_f32_prefill_attention_visible_set_bit_exact():
    """The CUDA-core attention of the fp32 layer: meta 16, window 64, two sequences."""
    _prefill_visibility(synth.tiny_layer_cfg(), 2, 300, 15)


def _slot_positions(L, m, cap):
    """Position held by each cache slot after positions 0..L-1 were written (-1: empty)."""
    ring = cap - m
    held = np.full(cap, -1)
    for p in range(L):
        held[oracle.ring_slot(p, m, ring)] = p
    return held


def _decode_visibility(cfg, B, cap, lens, seed, static=False):
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    cfg = cfg.with_(is_kv_producer=0)
    m = cfg.n_meta
    H, G, dh, dv = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim
    mdt = rt.mid_dtype(cfg)
    esz = torch.tensor([], dtype=mdt).element_size()
    layer = rt.DeviceLayer(cfg, synth.layer_weights(cfg, seed))
    st = rt.State(cfg, B)
    ws = rt.workspace(cfg, B, cap, hy.HYMBA_MODE_DECODE)
    lay = hy.workspace_layout(layer.c, B, cap, hy.HYMBA_MODE_DECODE)
    ns = lay["n_split"]
    k_cache = torch.zeros((B, G, cap, dh), dtype=mdt, device="cuda")
    x = rt.to_device(synth.layer_input(cfg, B, 1, seed)[:, 0], cfg)
    y = torch.empty_like(x)
    for L in lens:
        length = torch.full((B,), L, dtype=torch.int32, device="cuda")
        held = _slot_positions(L, m, cap)
        p = L - 1
        # the slot mask of the query at position p: slots whose held position is visible
        vis_slot = np.array([held[s] >= 0 and oracle.key_visible(p, int(held[s]), m, cfg.window)
                             for s in range(cap)])[None, :]
        n_vis = sum(oracle.key_visible(p, j, m, cfg.window) for j in range(p + 1))
        assert vis_slot.sum() == n_vis, "the cache must hold every visible position"
        for r in range(_runs(cap, G, dv)):
            v_cache = _onehot_v(B, G, cap, dv, r, torch, mdt)
            kvs = hy.kv_struct(cfg, B, None, None, k_cache, v_cache, length)
            if static:
                q = torch.zeros((B, H * dh), dtype=mdt, device="cuda")
                o = torch.full((B, H * dv), float("nan"), dtype=mdt, device="cuda")
                hy.check(hy.hymba_attn_decode_static(ctypes.byref(layer.c), q.data_ptr(), H * dh, ctypes.byref(kvs),
                                                     o.data_ptr(), B, hy.current_stream_ptr()))
                torch.cuda.synchronize()
                assert hy.hymba_get_device_status(None) == 0
                got = o.float().cpu().numpy()[:, None, :]
            else:
                ws.fill_(0xFF)
                rt.decode(layer, x, kvs, st, y, ws, 0)
                torch.cuda.synchronize()
                assert hy.hymba_get_device_status(None) == 0
                n = B * H * ns * (dv + 4)  # records: dv sums, max logit, sum of p, two pad words
                part = ws[lay["part"]:lay["part"] + n * 4].view(torch.float32).view(B, H, ns, dv + 4)
                part = part.double().cpu().numpy()
                # p = 1 for every visible key: the split sums of p v are 0/(b+1) one-hot
                # counts, the split sums of p count the keys; normalise by the total
                cnt = part[..., dv + 1].sum(axis=-1)
                assert np.all(cnt == n_vis), (L, np.unique(cnt))
                got = (part[..., :dv].sum(axis=2) / cnt[..., None]).reshape(B, 1, H * dv)
            _check_run(got, vis_slot, B, G, H, dv, r, f"decode {'static ' if static else ''}L={L}")


DECODE_LENS = (1, 100, 128 + 1024, 128 + 1024 + 1, 128 + 4096 + 1, 128 + 4096 + 700)


def test_bf16_decode_attention_visible_set_bit_exact():
    """The bulk-copy decode attention (128-key splits) of the 1.5B pair shape, B=64,
    ring 1024 + 128 meta: a query inside the meta block, before the ring fills, at the
    exact fill, one past it (first wrap) and deep into wrapped rings."""
    cfg = synth.hymba15_layer_cfg(1024)
    _decode_visibility(cfg, 64, 128 + 1024, DECODE_LENS, 21)


def test_bf16_decode_attention_small_window_and_global():
    """A window shorter than one split and a global layer whose cache holds every
    position."""
    small = synth.hymba15_layer_cfg(7).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640, dt_rank=24,
                                             n_meta=16)
    _decode_visibility(small, 3, 16 + 7, (3, 16, 23, 24, 61), 22)
    glob = small.with_(window=0)
    _decode_visibility(glob, 2, 400, (1, 17, 255, 256, 257, 400), 23)


def test_f32_decode_attention_visible_set_bit_exact():
    cfg = synth.tiny_layer_cfg().with_(window=40)
    _decode_visibility(cfg, 3, 16 + 40, (5, 16, 56, 57, 200), 24)
