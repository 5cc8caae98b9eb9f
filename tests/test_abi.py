"""C-ABI library checks that need no GPU: it loads, exports every symbol
include/moe.h declares, and rejects bad arguments on the host before touching
CUDA.  No call here enqueues device work."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from expert_dispatch_fp32_b200 import build
    build.build()
    import expert_dispatch_fp32_b200._binding as binding
    binding.lib()
    return binding


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_stage_calls():
    names = declared_symbols()
    for stage in ("moe_route", "moe_preprocess", "moe_dispatch_permute", "moe_expert_ffn",
                  "moe_combine_unpermute", "moe_forward"):
        assert stage in names


def test_library_exports_every_declared_symbol(B):
    L = ctypes.CDLL(B.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(L, n)]
    assert not missing, missing


def test_binding_names_match_header(B):
    import expert_dispatch_fp32_b200 as pkg
    for n in declared_symbols():
        assert callable(getattr(pkg, n, None)), n


def good_cfg(B, **kw):
    c = dict(T=64, D=64, E=16, ep_size=4, top_k=2, F=128, act=B.MOE_ACT_GELU, renormalize=1,
             x_dtype=B.MOE_DT_F32, router_dtype=B.MOE_DT_F32, n_shared=0, F_shared=0)
    c.update(kw)
    return B.MoeConfig(**c)


def test_version_and_strings(B):
    assert B.moe_abi_version() == B.ABI_VERSION == 3
    assert B.moe_status_string(B.MOE_OK) == "ok"
    assert "range" in B.moe_status_string(B.MOE_ERR_INDEX_OOB)
    assert B.moe_status_string(99) == "unknown status"


@pytest.mark.parametrize("kw,expect", [
    ({}, 0),
    ({"E": 10, "ep_size": 4}, 1),          # num_experts must be divisible by ep_size
    ({"top_k": 17}, 1),                     # k > E
    ({"top_k": 0}, 1),
    ({"T": -1}, 1),
    ({"router_dtype": 1}, 2),               # only the fp32 router
    ({"D": 96}, 2),                         # rows of 64-element K steps
    ({"act": 1, "F": 192}, 2),              # SwiGLU tiles need F % 128
    ({"act": 7}, 1),
    ({"renormalize": 2}, 1),
    ({"n_shared": 1, "F_shared": 0}, 1),
    ({"n_shared": 1, "F_shared": 128}, 2),  # shared experts read bf16 x
    ({"n_shared": 1, "F_shared": 128, "x_dtype": 1}, 0),
    ({"E": 2048, "ep_size": 8}, 2),
    ({"top_k": 33, "E": 64}, 2),
    ({"T": 0}, 0),
])
def test_validate_config(B, kw, expect):
    assert B.moe_validate_config(good_cfg(B, **kw)) == expect


def test_sizes_host_only(B):
    c = good_cfg(B)
    ws = B.moe_workspace_size(c)
    pk = B.moe_packed_weights_size(c)
    assert ws > 0 and ws % 256 == 0
    # packed = W1 [16,128,64] + W2 [16,64,128], bf16
    assert pk == 2 * (16 * 128 * 64) * 2
    assert B.moe_workspace_size(good_cfg(B, E=10)) == 0


def test_null_and_misaligned_pointers_rejected_on_host(B):
    c = good_cfg(B)
    lib = B.lib()
    by = ctypes.byref(c)
    # a real, 256-byte-aligned host buffer stands in for every non-null argument: the
    # calls must reject before they enqueue anything, and if one ever did not, it would
    # hand the runtime an address it can reject, never an arbitrary one
    import numpy as np
    buf = np.zeros(1 << 16, dtype=np.uint8)
    fake = (buf.ctypes.data + 255) // 256 * 256
    assert lib.moe_route(by, None, fake, None, None, fake, fake, fake, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_route(by, fake + 4, fake, None, None, fake, fake, fake, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_preprocess(by, fake, fake, fake, fake, fake, fake, fake, fake, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_dispatch_permute(by, fake, None, fake, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_check_wait_timeout(None, fake, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_check_wait_timeout(fake, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_ffn(by, fake, None, fake, None, fake, fake, None, fake, fake, None) == B.MOE_ERR_INVALID_ARG
    # out may not alias the residual
    assert lib.moe_combine_unpermute(by, fake, fake, fake, fake, None, fake, None) == B.MOE_ERR_INVALID_ARG
    bad = good_cfg(B, E=10)
    assert lib.moe_forward(ctypes.byref(bad), *([fake] * 20), None) == B.MOE_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op(B):
    c = good_cfg(B, T=0)
    lib = B.lib()
    assert lib.moe_route(ctypes.byref(c), None, None, None, None, None, None, None, None) == 0
    assert lib.moe_dispatch_permute(ctypes.byref(c), None, None, None, None) == 0
    assert lib.moe_combine_unpermute(ctypes.byref(c), None, None, None, None, None, None, None) == 0


def test_router_filter_view_says_which_router_runs(B):
    # the tensor-core filter: bf16 x, 256 experts, enough tokens, renormalised
    ds = good_cfg(B, T=8192, D=7168, E=256, ep_size=8, top_k=8, F=2048, act=B.MOE_ACT_SWIGLU,
                  x_dtype=B.MOE_DT_BF16)
    ao, ld, wo, coef = B.moe_router_filter_view(ds)
    assert ld == 256 and ao % 256 == 0 and wo % 256 == 0
    assert ao + 8192 * ld * 4 <= B.moe_workspace_size(ds) and wo + 7168 * 4 <= ao
    assert abs(coef - (4 * (7168 // 16 + 2) * 2.0 ** -23 + 2.0 ** -17)) < 1e-9
    # other paths: fp32 x, few experts, few tokens, no renormalisation
    assert B.moe_router_filter_view(good_cfg(B)) is None
    for kw in ({"E": 16, "ep_size": 4, "D": 2048}, {"T": 32}, {"renormalize": 0}):
        c = dict(T=8192, D=7168, E=256, ep_size=8, top_k=8, F=2048, act=B.MOE_ACT_SWIGLU,
                 x_dtype=B.MOE_DT_BF16)
        c.update(kw)
        assert B.moe_router_filter_view(good_cfg(B, **c)) is None, kw


def test_peer_exchange_calls_reject_bad_tables_on_host(B):
    c = good_cfg(B)                       # ep_size 4
    lib = B.lib()
    import numpy as np
    buf = np.zeros(1 << 12, dtype=np.uint8)
    h = (buf.ctypes.data + 255) // 256 * 256       # real host memory, never enqueued on
    peers = B.MoeEpPeers(4, 16, h, h, h, h, h, h)
    by, pa = ctypes.byref(c), ctypes.addressof(peers)
    assert lib.moe_ep_send_counts(by, None, 0, 4, h, 1, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_send_counts(by, pa, 3, 2, h, 1, None) == B.MOE_ERR_INVALID_ARG   # ranks 3..4 of 4
    assert lib.moe_ep_send_counts(by, pa, 0, 0, h, 1, None) == B.MOE_ERR_INVALID_ARG
    bad = B.MoeEpPeers(2, 16, h, h, h, h, h, h)   # P differs from ep_size
    assert lib.moe_ep_wait_returned(by, ctypes.addressof(bad), 0, 1, 1, h, None) == B.MOE_ERR_INVALID_ARG
    nul = B.MoeEpPeers(4, 16, h, None, h, h, h, h)
    assert lib.moe_ep_recv_layout(by, ctypes.addressof(nul), 0, 1, h, 1, h, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_send_rows(by, pa, 0, 1, h, h, h, None, 1, h, h, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_return_rows(by, pa, 0, 1, h, h, 1, None, h, None) == B.MOE_ERR_INVALID_ARG


def test_cycle_counters_exist_only_in_an_instrumented_build(B):
    """moe_instr_read answers MOE_ERR_UNSUPPORTED from the ordinary library (the counters
    are compiled out) and checks its arguments on the host first."""
    import numpy as np
    lib = B.lib()
    buf = np.zeros(B.INSTR_CTAS * B.INSTR_SLOTS, dtype=np.uint64)
    p = buf.ctypes.data
    assert lib.moe_instr_read(0, p, buf.size) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_instr_read(1, p, buf.size) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_instr_read(2, p, buf.size) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_instr_read(0, None, buf.size) == B.MOE_ERR_INVALID_ARG
    assert not buf.any()


def test_fused_return_call_checks_its_configs_on_host(B):
    """moe_ep_expert_ffn_return rejects, before enqueuing anything, a local config that is
    not the tokens config's local-expert view (E/P experts, top-1, T = cap, same D/F/act),
    a rank outside the exchange, a null or misaligned `done`, and a null table."""
    c = good_cfg(B, act=B.MOE_ACT_SWIGLU, F=128, x_dtype=B.MOE_DT_BF16)    # E 16, ep 4, D 64
    lib = B.lib()
    import numpy as np
    buf = np.zeros(1 << 12, dtype=np.uint8)
    h = (buf.ctypes.data + 255) // 256 * 256
    peers = B.MoeEpPeers(4, 16, h, h, h, h, h, h)
    pa = ctypes.addressof(peers)
    mk = lambda **kw: B.MoeConfig(**{**dict(T=16, D=64, E=4, ep_size=1, top_k=1, F=128,
                                            act=B.MOE_ACT_SWIGLU, renormalize=1, x_dtype=B.MOE_DT_BF16,
                                            router_dtype=B.MOE_DT_F32, n_shared=0, F_shared=0), **kw})
    call = lambda loc, rank=0, done=h, p=pa: lib.moe_ep_expert_ffn_return(
        ctypes.byref(c), ctypes.byref(loc), p, rank, h, h, h, h, h, h, None, h, 1, done, h, None)
    # both configs are valid on their own, so each rejection below is the one field changed
    # (a fully valid call would enqueue, which this host-memory test never does)
    assert lib.moe_validate_config(ctypes.byref(c)) == 0 and lib.moe_validate_config(ctypes.byref(mk())) == 0
    assert call(mk(E=8)) == B.MOE_ERR_INVALID_ARG          # not E / P experts
    assert call(mk(T=32)) == B.MOE_ERR_INVALID_ARG         # T is not the receive capacity
    assert call(mk(top_k=2)) == B.MOE_ERR_INVALID_ARG
    assert call(mk(F=256)) == B.MOE_ERR_INVALID_ARG
    assert call(mk(), rank=4) == B.MOE_ERR_INVALID_ARG
    assert call(mk(), done=None) == B.MOE_ERR_INVALID_ARG
    assert call(mk(), done=h + 2) == B.MOE_ERR_INVALID_ARG
    assert call(mk(), p=None) == B.MOE_ERR_INVALID_ARG
