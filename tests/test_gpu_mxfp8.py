"""MXFP8 quantisation on the GPU (moe_mxfp8_quantize) against the oracle's definition
(oracle/mxfp8.py, after the OCP Microscaling v1.0 MXFP8 (E4M3) format): the E4M3 bytes and
the E8M0 scale bytes must be the oracle's, bit for bit."""
import numpy as np
import pytest
import torch

import expert_dispatch_fp32_b200 as M
from oracle import mxfp8

pytestmark = pytest.mark.gpu


def _rows(rows, K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((rows, K), generator=g)
    # blocks over many binades, exact zeros, ties between E4M3 values, the clamp range
    x[0, :32] = 0.0
    x[1, :32] = torch.linspace(-3, 3, 32)
    x[2] *= 1e-30
    x[3] *= 1e30
    x[4, :32] = torch.tensor([448.0, 464.0, 480.0, 496.0] * 8)         # [448, 512): clamp and ties
    x[5, :32] = torch.tensor([1.0, 1.0625, 1.125, 1.1875] * 8) * 256   # halfway cases after scaling
    x[6] = torch.exp2(torch.randint(-40, 40, (K,), generator=g).float()) * torch.sign(x[6])
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,K", [(7, 64), (300, 2048), (129, 7168)])
def test_quantize_matches_the_oracle_bit_for_bit(rows, K):
    x = _rows(rows, K, seed=rows + K)
    xd = x.cuda()
    q = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows, K // 32), dtype=torch.uint8, device="cuda")
    M.moe_mxfp8_quantize(xd, rows, K, q, s)
    torch.cuda.synchronize()
    qv_ref, s_ref = mxfp8.quantize_mxfp8(x.to(torch.float64).numpy(), axis=-1)
    assert np.array_equal(s.cpu().numpy().astype(np.int64) - 127, s_ref)
    qv = q.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(qv, qv_ref)


def _mx_oracle_expert(x_rows, w_up, w_down, act):
    """The expert FFN on MXFP8 operands: x and both weight matrices quantised along their
    K axis (oracle/mxfp8.py), the activation quantised along F, from full precision,
    before the down projection."""
    import oracle
    dq = lambda a: mxfp8.dequantize_mxfp8(*mxfp8.quantize_mxfp8(a, axis=-1), axis=-1)
    xq = dq(x_rows)
    wu = dq(np.asarray(w_up).T).T            # [D, Nup], blocks of 32 along D
    wd = dq(np.asarray(w_down).T).T          # [F, D], blocks of 32 along F
    h = xq @ wu
    if act == "swiglu":
        F = wu.shape[1] // 2
        a = oracle.silu(h[:, :F]) * h[:, F:]
    else:
        a = oracle.gelu(h)
    return dq(a) @ wd


@pytest.mark.parametrize("case,half", [("swiglu_shared", "1"), ("gelu", "1"), ("deepseek_like", "1"),
                                       ("swiglu_shared", "0"), ("deepseek_like", "0")])
def test_mxfp8_expert_ffn_matches_the_oracle(case, half, monkeypatch):
    # half "1": a group's last <= 128 rows run as an M = 128 tile (the default); "0": M = 256
    monkeypatch.setenv("MOE_MX_HALF", half)
    import moe_workloads as W
    from parity_helpers import assert_layer_close, f64, make_layer, up_weights
    wl = {"swiglu_shared": W.Workload(name="mx1", T=300, D=512, E=8, ep_size=2, top_k=2, F=256,
                                      n_shared=1, F_shared=256, seed=31),
          "gelu": W.Workload(name="mx2", T=200, D=256, E=4, ep_size=2, top_k=2, F=256, act="gelu",
                             seed=32),
          "deepseek_like": W.Workload(name="mx3", T=512, D=1024, E=16, ep_size=4, top_k=8, F=512,
                                      n_shared=1, F_shared=512, seed=33)}[case]
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    T = wl.T
    b = layer.allocate(T)
    cfg = layer.config(T)
    layer.forward(inp["x"])                 # route, preprocess, dispatch (x_perm) and the bf16 FFN
    torch.cuda.synchronize()
    layer.check_status()
    y_bf16 = b["y_perm"].clone()
    packed_mx = torch.empty(M.moe_packed_weights_mxfp8_size(cfg), dtype=torch.uint8, device="cuda")
    M.moe_prepare_weights_mxfp8(cfg, layer.packed, packed_mx)
    ws = torch.zeros(M.moe_workspace_mxfp8_size(cfg), dtype=torch.uint8, device="cuda")
    y = torch.full_like(b["y_perm"], float("nan"))
    sh = None if b["shared_out"] is None else torch.empty_like(b["shared_out"])
    for it in range(2):                     # twice: the scratch and counters are reused
        M.moe_expert_ffn_mxfp8(cfg, b["x_perm"], inp["x"] if wl.x_dtype == "bf16" else None,
                               b["expert_offsets"], layer.packed, packed_mx, y, sh, ws, b["status"])
        torch.cuda.synchronize()
        layer.check_status()
    off = b["expert_offsets"].cpu().numpy()
    xp = f64(b["x_perm"])
    wup = up_weights(wl, inp)
    got, ref = [], []
    for e in range(wl.E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        r = _mx_oracle_expert(xp[lo:hi], f64(wup[e]), f64(inp["w_down"][e]), wl.act)
        g = f64(y[lo:hi])
        assert_layer_close(g, r, np.zeros_like(r), f"mxfp8 y_perm expert {e}")
        got.append(g); ref.append(r)
    err = np.linalg.norm(np.concatenate(got) - np.concatenate(ref)) / np.linalg.norm(np.concatenate(ref))
    vs_bf16 = (torch.linalg.norm(y.float() - y_bf16.float()) / torch.linalg.norm(y_bf16.float())).item()
    print(f"\n{case}: MXFP8 y_perm vs oracle rel-L2 {err:.2e}; vs the bf16 path {vs_bf16:.2e}")
    if sh is not None:
        assert torch.equal(sh, b["shared_out"])     # the shared experts stay bf16


@pytest.mark.parametrize("E", [16, 64])
def test_mxfp8_layer_forward_is_its_stages(E):
    """MoELayer(mxfp8=True): the forward is route+dispatch, the MXFP8 FFN and the combine
    (same bits as the calls one by one; with more than 32 experts the dispatch writes the
    quantised rows itself), and its MoE part stays within the format's error of the bf16
    layer's."""
    import moe_workloads as W
    from parity_helpers import f64
    wl = W.Workload(name="mxl", T=640, D=512, E=E, ep_size=4, top_k=4, F=256, n_shared=1,
                    F_shared=256, seed=41)
    inp = W.make_inputs(wl, device="cuda")
    kw = dict(D=wl.D, E=wl.E, ep_size=wl.ep_size, top_k=wl.top_k, F=wl.F, w_router=inp["w_router"],
              w_gate_up=inp["w_gate_up"], w_down=inp["w_down"], expert_bias=inp["bias"],
              ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"])
    ref = M.MoELayer(**kw)
    mx = M.MoELayer(**kw, mxfp8=True)
    x = inp["x"]
    out_ref = ref.forward(x).clone()
    out = mx.forward(x).clone()
    torch.cuda.synchronize()
    mx.check_status()
    b, cfg = mx.buf, mx.config(wl.T)
    y = torch.empty_like(b["y_perm"])
    sh = torch.empty_like(b["shared_out"])
    o = torch.empty_like(out)
    M.moe_route_dispatch(cfg, x, mx.w_router, mx.expert_bias, None, b["topk_idx"], b["topk_w"],
                         b["counts"], b["expert_offsets"], b["rank_splits"], b["rank_offsets"], b["pos"],
                         b["src"], b["x_perm"], b["workspace"], b["status"])
    x_perm = b["x_perm"]
    if not M.moe_route_dispatch_is_fused(cfg):
        M.moe_dispatch_mxfp8(cfg, x, b["src"], b["expert_offsets"], b["workspace"])
        x_perm = None
    M.moe_expert_ffn_mxfp8(cfg, x_perm, x, b["expert_offsets"], mx.packed, mx.packed_mx, y, sh,
                           b["workspace"], b["status"])
    M.moe_combine_unpermute(cfg, y, b["pos"], b["topk_w"], x, sh, o)
    torch.cuda.synchronize()
    mx.check_status()
    assert torch.equal(o, out)
    moe_mx, moe_ref = f64(out) - f64(x), f64(out_ref) - f64(x)
    rel = np.linalg.norm(moe_mx - moe_ref) / np.linalg.norm(moe_ref)
    print(f"\nMoE part, MXFP8 layer vs bf16 layer: rel-L2 {rel:.3e}")
    assert rel < 0.15


@pytest.mark.parametrize("half", ["1", "0"])
def test_mxfp8_dispatch_equals_quantised_x_perm(half, monkeypatch):
    """moe_dispatch_mxfp8 (each row quantised straight from x[src / k]) followed by the
    MXFP8 FFN with x_perm = NULL gives the bits of the bf16 dispatch followed by the FFN's
    own quantisation of x_perm, with M = 128 remainder tiles on and off."""
    import moe_workloads as W
    from parity_helpers import make_layer
    monkeypatch.setenv("MOE_MX_HALF", half)
    wl = W.Workload(name="mxd", T=700, D=512, E=64, ep_size=8, top_k=4, F=256, seed=43)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    x = inp["x"]
    layer.forward(x)
    torch.cuda.synchronize()
    layer.check_status()
    b, cfg = layer.buf, layer.config(wl.T)
    pmx = torch.empty(M.moe_packed_weights_mxfp8_size(cfg), dtype=torch.uint8, device="cuda")
    M.moe_prepare_weights_mxfp8(cfg, layer.packed, pmx)
    n = M.moe_workspace_mxfp8_size(cfg)
    ws_a = torch.zeros(n, dtype=torch.uint8, device="cuda")
    ws_b = torch.full((n,), 0x7F, dtype=torch.uint8, device="cuda")   # stale bytes everywhere
    y_a = torch.empty_like(b["y_perm"])
    y_b = torch.full_like(b["y_perm"], float("nan"))
    M.moe_expert_ffn_mxfp8(cfg, b["x_perm"], None, b["expert_offsets"], layer.packed, pmx, y_a, None,
                           ws_a, b["status"])
    M.moe_dispatch_mxfp8(cfg, x, b["src"], b["expert_offsets"], ws_b)
    M.moe_expert_ffn_mxfp8(cfg, None, None, b["expert_offsets"], layer.packed, pmx, y_b, None, ws_b,
                           b["status"])
    torch.cuda.synchronize()
    layer.check_status()
    assert torch.equal(y_a, y_b)


MX_UNEVEN = [0, 1, 64, 65, 128, 129, 200, 256, 257, 270, 288, 289, 300, 320, 321, 384, 385, 513, 3, 0,
             700, 260]


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
@pytest.mark.parametrize("fold", ["1", "0"])
def test_mxfp8_uneven_expert_tiles(act, fold, monkeypatch):
    """Every routed row of the MXFP8 expert FFN against the oracle on quantised operands,
    with hand-set expert sizes that put each expert's last tile in every case: folded
    remainders of 1..32 and 33..64 rows (257..320-row experts), M = 128 tiles, full tiles,
    several bands, a single row and empty experts; folding on and off."""
    import moe_workloads as W
    from parity_helpers import f64, make_layer, up_weights
    monkeypatch.setenv("MOE_MX_FOLD", fold)
    counts = np.array(MX_UNEVEN)
    E, T = counts.size, int(counts.sum())                # top-1: one row per token
    wl = W.Workload(name="mxu", T=T, D=256, E=E, ep_size=2, top_k=1, F=256, act=act, seed=44)
    inp = W.make_inputs(wl, device="cuda")
    layer = make_layer(wl, inp)
    b = layer.allocate(T)
    cfg = layer.config(T)
    rng = np.random.default_rng(12)
    assign = rng.permutation(np.repeat(np.arange(E), counts)).astype(np.int32)
    idx = torch.from_numpy(assign.reshape(T, 1)).cuda()
    b["status"].zero_()
    M.moe_preprocess(cfg, idx, b["counts"], b["expert_offsets"], b["rank_splits"], b["rank_offsets"],
                     b["pos"], b["src"], b["workspace"], b["status"])
    g = torch.Generator(device="cuda")
    g.manual_seed(6)
    x_perm = torch.randn((T, wl.D), generator=g, device="cuda").to(torch.bfloat16)
    pmx = torch.empty(M.moe_packed_weights_mxfp8_size(cfg), dtype=torch.uint8, device="cuda")
    M.moe_prepare_weights_mxfp8(cfg, layer.packed, pmx)
    ws = torch.full((M.moe_workspace_mxfp8_size(cfg),), 0x7F, dtype=torch.uint8, device="cuda")
    y = torch.full_like(b["y_perm"], float("nan"))
    M.moe_expert_ffn_mxfp8(cfg, x_perm, None, b["expert_offsets"], layer.packed, pmx, y, None, ws, b["status"])
    torch.cuda.synchronize()
    assert int(b["status"].item()) == 0
    off = b["expert_offsets"].cpu().numpy()
    assert np.array_equal(np.diff(off), counts)
    xp, yp = f64(x_perm), f64(y)
    wup = up_weights(wl, inp)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        ref = _mx_oracle_expert(xp[lo:hi], f64(wup[e]), f64(inp["w_down"][e]), act)
        assert np.isfinite(yp[lo:hi]).all(), f"expert {e}: unwritten rows"
        from parity_helpers import assert_layer_close
        assert_layer_close(yp[lo:hi], ref, np.zeros_like(ref), f"mxfp8 y_perm expert {e} ({hi - lo} rows)")
