"""User-facing MoE layer: owns packed weights and the per-batch buffers.

PyTorch only allocates device memory and provides the stream; every stage runs
in libmoe.so's kernels through the C ABI (``_binding``).  Buffers are allocated
once per batch size and reused, so a forward call only enqueues kernels.
"""
from __future__ import annotations

import torch

from . import _binding as B


def make_config(T, D, E, ep_size, top_k, F, act="swiglu", renormalize=True, x_dtype="bf16",
                n_shared=0, F_shared=0) -> B.MoeConfig:
    """Build and validate a ``moe_config``."""
    cfg = B.MoeConfig(T=T, D=D, E=E, ep_size=ep_size, top_k=top_k, F=F,
                      act=B.MOE_ACT_SWIGLU if act == "swiglu" else B.MOE_ACT_GELU,
                      renormalize=int(bool(renormalize)),
                      x_dtype=B.MOE_DT_F32 if x_dtype in ("f32", torch.float32) else B.MOE_DT_BF16,
                      router_dtype=B.MOE_DT_F32, n_shared=n_shared, F_shared=F_shared)
    st = B.moe_validate_config(cfg)
    if st != B.MOE_OK:
        raise B.MoeError("moe_validate_config", st)
    return cfg


def _empty(n, dtype, device):
    return torch.empty(n, dtype=dtype, device=device)


class MoELayer:
    """Forward of an expert-parallel MoE layer on one GPU.

    Weights (device tensors): w_router fp32 [E, D]; expert_bias fp32 [E] or None;
    w_gate_up bf16 [E, D, 2F] (SwiGLU) or W1 [E, D, F] (GELU); w_down bf16
    [E, F, D]; ws_gate_up bf16 [S, D, 2Fs] and ws_down bf16 [S, Fs, D] or None.
    The expert weights are repacked once at construction (moe_prepare_weights);
    the caller may drop its copies afterwards.

    mxfp8=True runs the routed experts in MXFP8 (moe_expert_ffn_mxfp8: E4M3 operands with
    one E8M0 scale per 32, quantised once for the weights at construction and per batch
    for the rows); routing, the shared experts and the combine stay as in the bf16 path.
    """

    def __init__(self, *, D, E, ep_size, top_k, F, w_router, w_gate_up, w_down, expert_bias=None,
                 ws_gate_up=None, ws_down=None, act="swiglu", renormalize=True, x_dtype="bf16",
                 keep_router_logits=False, mxfp8=False, stream=None):
        self.D, self.E, self.ep_size, self.top_k, self.F = D, E, ep_size, top_k, F
        self.act, self.renormalize, self.x_dtype = act, renormalize, x_dtype
        self.n_shared = 0 if ws_gate_up is None else ws_gate_up.shape[0]
        self.F_shared = 0 if ws_gate_up is None else ws_down.shape[1]
        self.keep_router_logits = keep_router_logits
        self.device = w_router.device
        self.w_router = w_router.contiguous()
        self.expert_bias = None if expert_bias is None else expert_bias.contiguous()
        cfg = self.config(1)
        self.packed = _empty(B.moe_packed_weights_size(cfg), torch.uint8, self.device)
        B.moe_prepare_weights(cfg, w_gate_up.contiguous(), w_down.contiguous(),
                              None if ws_gate_up is None else ws_gate_up.contiguous(),
                              None if ws_down is None else ws_down.contiguous(), self.packed, stream)
        self.mxfp8 = bool(mxfp8)
        self.packed_mx = None
        if self.mxfp8:
            n = B.moe_packed_weights_mxfp8_size(cfg)
            if n == 0:
                raise B.MoeError("moe_packed_weights_mxfp8_size", B.MOE_ERR_UNSUPPORTED)
            self.packed_mx = _empty(n, torch.uint8, self.device)
            B.moe_prepare_weights_mxfp8(cfg, self.packed, self.packed_mx, stream)
        self._bufT = None
        self.buf = {}

    def config(self, T) -> B.MoeConfig:
        return make_config(T, self.D, self.E, self.ep_size, self.top_k, self.F, self.act,
                           self.renormalize, self.x_dtype, self.n_shared, self.F_shared)

    def allocate(self, T):
        """(Re)allocate the per-batch buffers for T tokens."""
        if self._bufT == T:
            return self.buf
        dev, k, D, E = self.device, self.top_k, self.D, self.E
        R = T * k
        xdt = torch.float32 if self.x_dtype in ("f32", torch.float32) else torch.bfloat16
        cfg = self.config(T)
        self.buf = dict(
            logits=_empty((T, E), torch.float32, dev) if self.keep_router_logits else None,
            topk_idx=_empty((T, k), torch.int32, dev), topk_w=_empty((T, k), torch.float32, dev),
            counts=_empty(E, torch.int32, dev), expert_offsets=_empty(E + 1, torch.int32, dev),
            rank_splits=_empty(self.ep_size, torch.int32, dev),
            rank_offsets=_empty(self.ep_size + 1, torch.int32, dev),
            pos=_empty(R, torch.int32, dev), src=_empty(R, torch.int32, dev),
            x_perm=_empty((R, D), torch.bfloat16, dev), act=_empty((R, self.F), torch.bfloat16, dev),
            y_perm=_empty((R, D), torch.bfloat16, dev),
            shared_out=_empty((T, D), torch.bfloat16, dev) if self.n_shared else None,
            out=_empty((T, D), xdt, dev),
            workspace=_empty(max(B.moe_workspace_mxfp8_size(cfg) if self.mxfp8 else
                                 B.moe_workspace_size(cfg), 256), torch.uint8, dev),
            status=torch.zeros(1, dtype=torch.int32, device=dev),
        )
        self._bufT = T
        self._cfg = cfg
        return self.buf

    def forward(self, x, stream=None):
        """Enqueue the whole layer on ``stream``; returns the output buffer."""
        b = self.allocate(x.shape[0])
        self.forward_into(x, b["out"], stream)
        return b["out"]

    def forward_into(self, x, out, stream=None):
        """Enqueue the whole layer on ``stream`` with its output written to ``out``
        (a device tensor shaped like x)."""
        T = x.shape[0]
        b = self.allocate(T)
        if not self.mxfp8:
            B.moe_forward(self._cfg, x, self.w_router, self.expert_bias, self.packed, b["logits"],
                          b["topk_idx"], b["topk_w"], b["counts"], b["expert_offsets"], b["rank_splits"],
                          b["rank_offsets"], b["pos"], b["src"], b["x_perm"], b["act"], b["y_perm"],
                          b["shared_out"], out, b["workspace"], b["status"], stream)
            return
        if self.x_dtype != "bf16" or B.moe_route_dispatch_is_fused(self._cfg):
            # the one-launch router + preprocess + dispatch writes the bf16 x_perm; the
            # FFN call quantises it
            B.moe_route_dispatch(self._cfg, x, self.w_router, self.expert_bias, b["logits"],
                                 b["topk_idx"], b["topk_w"], b["counts"], b["expert_offsets"],
                                 b["rank_splits"], b["rank_offsets"], b["pos"], b["src"], b["x_perm"],
                                 b["workspace"], b["status"], stream)
            x_perm = b["x_perm"]
        else:
            # route and preprocess, then the dispatch quantises the rows as it copies them
            B.moe_route(self._cfg, x, self.w_router, self.expert_bias, b["logits"], b["topk_idx"],
                        b["topk_w"], b["workspace"], stream)
            B.moe_preprocess(self._cfg, b["topk_idx"], b["counts"], b["expert_offsets"], b["rank_splits"],
                             b["rank_offsets"], b["pos"], b["src"], b["workspace"], b["status"], stream)
            B.moe_dispatch_mxfp8(self._cfg, x, b["src"], b["expert_offsets"], b["workspace"], stream)
            x_perm = None
        B.moe_expert_ffn_mxfp8(self._cfg, x_perm, x if self.x_dtype == "bf16" else None,
                               b["expert_offsets"], self.packed, self.packed_mx, b["y_perm"],
                               b["shared_out"], b["workspace"], b["status"], stream)
        B.moe_combine_unpermute(self._cfg, b["y_perm"], b["pos"], b["topk_w"], x, b["shared_out"], out,
                                stream)

    __call__ = forward

    def check_status(self):
        """Read the device status word (synchronises); raise if a kernel reported an error."""
        st = int(self.buf["status"].item())
        if st != B.MOE_OK:
            raise B.MoeError("device status", st)
