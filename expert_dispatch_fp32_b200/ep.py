"""Expert parallelism over the ranks of a torch.distributed process group.

"Expert Parallel (EP)", Communication Pattern: each rank owns E / ep contiguous
experts (rank r: experts [r*El, (r+1)*El), the placement of the worked example's
Step 3) and its own batch of tokens.  A forward pass on every rank:

  1. router + top-k and preprocess of its tokens (split sizes per destination rank);
  2. dispatch into the rank-major buffer; the row counts per (destination rank,
     local expert) are exchanged first, then the token pre-all-to-all sends rows
     [rank_offsets[r], rank_offsets[r+1]) to rank r, with each row's local expert;
  3. the local experts run on the received rows (grouped by local expert with a
     one-slot preprocess, dispatched, FFN, put back in received order);
  4. the token post-all-to-all returns the output rows to their source ranks;
  5. the shared experts of the rank's own tokens, then combine (weighted sum of the
     k returned rows + residual) exactly as on one GPU.

The exchanges are torch.distributed all_to_all_single calls (NCCL over NVLink /
NVSwitch on GPUs); every computation is a call into libmoe.so through the C ABI.
The layer is written against a small set of stage operations (`GpuOps`) so the
exchange bookkeeping can be exercised on CPU ranks with another implementation.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding as B
from .layer import make_config


class GpuOps:
    """Stage operations of one rank on its CUDA device, through libmoe.so."""

    def __init__(self, *, D, E, ep_size, top_k, F, w_router, w_gate_up_local, w_down_local,
                 expert_bias=None, ws_gate_up=None, ws_down=None, act="swiglu", renormalize=True,
                 x_dtype="bf16"):
        self.D, self.E, self.ep, self.k, self.F = D, E, ep_size, top_k, F
        self.El = E // ep_size
        self.act, self.renorm, self.x_dtype = act, renormalize, x_dtype
        self.S = 0 if ws_gate_up is None else ws_gate_up.shape[0]
        self.Fs = 0 if ws_gate_up is None else ws_down.shape[1]
        self.dev = w_router.device
        self.w_router = w_router.contiguous()
        self.bias = None if expert_bias is None else expert_bias.contiguous()
        # one packed buffer: the El local routed experts, then the shared experts
        cfg = self._local_cfg(1)
        self.packed = torch.empty(B.moe_packed_weights_size(cfg), dtype=torch.uint8, device=self.dev)
        B.moe_prepare_weights(cfg, w_gate_up_local.contiguous(), w_down_local.contiguous(),
                              None if ws_gate_up is None else ws_gate_up.contiguous(),
                              None if ws_down is None else ws_down.contiguous(), self.packed)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.dev)

    # configurations: the rank's tokens over all E experts and ep ranks; the
    # received rows (one slot each) over the El local experts
    def _tok_cfg(self, T):
        return make_config(T, self.D, self.E, self.ep, self.k, self.F, self.act, self.renorm,
                           self.x_dtype, self.S, self.Fs)

    def _local_cfg(self, n):
        return make_config(n, self.D, self.El, 1, 1, self.F, self.act, True, "bf16", self.S, self.Fs)

    def _i32(self, n):
        return torch.empty(n, dtype=torch.int32, device=self.dev)

    def _ws(self, cfg):
        return torch.empty(max(B.moe_workspace_size(cfg), 256), dtype=torch.uint8, device=self.dev)

    def route_and_preprocess(self, x):
        T = x.shape[0]
        cfg = self._tok_cfg(T)
        st = dict(cfg=cfg, ws=self._ws(cfg), topk_idx=torch.empty((T, self.k), dtype=torch.int32, device=self.dev),
                  topk_w=torch.empty((T, self.k), dtype=torch.float32, device=self.dev),
                  counts=self._i32(self.E), offsets=self._i32(self.E + 1), splits=self._i32(self.ep),
                  rank_offsets=self._i32(self.ep + 1), pos=self._i32(T * self.k), src=self._i32(T * self.k))
        B.moe_route(cfg, x, self.w_router, self.bias, None, st["topk_idx"], st["topk_w"], st["ws"])
        B.moe_preprocess(cfg, st["topk_idx"], st["counts"], st["offsets"], st["splits"],
                         st["rank_offsets"], st["pos"], st["src"], st["ws"], self.status)
        return st

    def dispatch(self, x, st):
        x_perm = torch.empty((x.shape[0] * self.k, self.D), dtype=torch.bfloat16, device=self.dev)
        B.moe_dispatch_permute(st["cfg"], x, st["pos"], x_perm)
        ids = self._i32(x.shape[0] * self.k)
        B.moe_ep_local_ids(st["cfg"], st["topk_idx"], st["src"], ids)
        return x_perm, ids

    def local_experts(self, x_recv, ids_recv):
        """The rank's experts on the rows it received (any order), output rows in
        the same order."""
        n = x_recv.shape[0]
        y = torch.empty((n, self.D), dtype=torch.bfloat16, device=self.dev)
        if n == 0:
            return y
        cfg = self._local_cfg(n)
        ws = self._ws(cfg)
        counts, offs = self._i32(self.El), self._i32(self.El + 1)
        sp, ro, pos, src = self._i32(1), self._i32(2), self._i32(n), self._i32(n)
        B.moe_preprocess(cfg, ids_recv.view(n, 1), counts, offs, sp, ro, pos, src, ws, self.status)
        x_local = torch.empty((n, self.D), dtype=torch.bfloat16, device=self.dev)
        B.moe_dispatch_permute(cfg, x_recv, pos, x_local)
        act = torch.empty((n, self.F), dtype=torch.bfloat16, device=self.dev)
        y_local = torch.empty((n, self.D), dtype=torch.bfloat16, device=self.dev)
        B.moe_expert_ffn(cfg, x_local, None, offs, self.packed, act, y_local, None, ws, self.status)
        B.moe_gather_rows(y_local, pos, y, n, n, self.D)
        return y

    def shared_and_combine(self, x, st, y_back):
        T = x.shape[0]
        shared = None
        if self.S:
            shared = torch.empty((T, self.D), dtype=torch.bfloat16, device=self.dev)
            cfg_s = self._local_cfg(T)
            B.moe_shared_ffn(cfg_s, x, self.packed, shared, self._ws(cfg_s), self.status)
        out = torch.empty_like(x)
        B.moe_combine_unpermute(st["cfg"], y_back, st["pos"], st["topk_w"], x, shared, out)
        return out

    def check(self):
        v = int(self.status.item())
        if v != B.MOE_OK:
            raise B.MoeError("device status", v)


class EPMoELayer:
    """MoE layer whose experts are split over the ranks of `group` (ep = its size).

    `ops` holds this rank's weights (its El local experts, the replicated router and
    shared experts) and runs the stages; `forward(x)` takes this rank's tokens and
    returns their outputs, exchanging rows with the other ranks in between.
    """

    def __init__(self, ops, group=None):
        self.ops = ops
        self.group = group
        self.ws = dist.get_world_size(group) if dist.is_initialized() else 1
        if self.ws != ops.ep:
            raise ValueError(f"ep_size {ops.ep} differs from the group size {self.ws}")

    def _a2a(self, out, inp, out_splits, in_splits):
        if dist.is_initialized():
            dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
        else:                          # one rank without a process group
            out.copy_(inp)

    def forward(self, x):
        o = self.ops
        st = o.route_and_preprocess(x)
        x_perm, ids = o.dispatch(x, st)
        # rows per (destination rank, local expert), then the split sizes on the host
        send_counts = st["counts"].view(self.ws, o.El)
        recv_counts = torch.empty_like(send_counts)
        self._a2a(recv_counts, send_counts, None, None)
        send = st["splits"].tolist()
        recv = recv_counts.sum(dim=1).tolist()
        x_recv = x_perm.new_empty((sum(recv), x_perm.shape[1]))
        ids_recv = ids.new_empty(sum(recv))
        self._a2a(x_recv, x_perm, recv, send)           # token pre-all-to-all
        self._a2a(ids_recv, ids, recv, send)
        y_recv = o.local_experts(x_recv, ids_recv)
        y_back = y_recv.new_empty((x_perm.shape[0], y_recv.shape[1]))
        self._a2a(y_back, y_recv, send, recv)           # token post-all-to-all
        return o.shared_and_combine(x, st, y_back)

    __call__ = forward


class PeerEPGroup:
    """The expert-parallel forward of P ranks whose data is all on one device, the two
    exchanges done by libmoe.so's peer-memory calls (moe_ep_*): stores straight into
    the owning rank's receive buffer, flags with the forward's epoch, no host round
    trip and no collective library.

    Rank r owns experts [r*El, (r+1)*El) and its own T tokens; the shared experts and
    the router are replicated.  The same calls take peer-mapped buffers of other GPUs
    in their pointer tables; here every table entry is a slice of one device's tensors,
    and each call covers all P ranks in one launch (kernels of different ranks never
    wait on one another across launches).  forward(x) takes x [P, T, D] and returns
    out [P, T, D]: rank r's rows equal moe_forward of its tokens with all E experts.
    """

    def __init__(self, *, D, E, P, top_k, F, T, w_router, w_gate_up, w_down, expert_bias=None,
                 ws_gate_up=None, ws_down=None, act="swiglu", renormalize=True, x_dtype="bf16"):
        if E % P:
            raise ValueError("num_experts must be divisible by the number of ranks")
        dev = w_router.device
        self.D, self.E, self.P, self.k, self.F, self.T = D, E, P, top_k, F, T
        self.El = El = E // P
        self.S = 0 if ws_gate_up is None else ws_gate_up.shape[0]
        self.Fs = 0 if ws_gate_up is None else ws_down.shape[1]
        self.cap = cap = P * T * min(top_k, El)
        self.w_router = w_router.contiguous()
        self.bias = None if expert_bias is None else expert_bias.contiguous()
        self.tok_cfg = make_config(T, D, E, P, top_k, F, act, renormalize, x_dtype, self.S, self.Fs)
        self.loc_cfg = make_config(cap, D, El, 1, 1, F, act, True, "bf16", self.S, self.Fs)
        self.sh_cfg = make_config(T, D, El, 1, 1, F, act, True, "bf16", self.S, self.Fs)
        i32 = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)
        bf = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device=dev)
        # stacked per-rank int32 rows padded to 16 bytes (the calls' row stride); [:, :n]
        # views keep every rank's row aligned for the single-rank calls
        pad = lambda n: (n + 3) // 4 * 4
        rows = lambda n: torch.zeros((P, pad(n)), dtype=torch.int32, device=dev)[:, :n]
        R = T * top_k
        psize = B.moe_packed_weights_size(self.loc_cfg)
        self.packed = torch.empty((P, psize), dtype=torch.uint8, device=dev)
        for r in range(P):
            B.moe_prepare_weights(self.loc_cfg, w_gate_up[r * El:(r + 1) * El].contiguous(),
                                  w_down[r * El:(r + 1) * El].contiguous(),
                                  None if ws_gate_up is None else ws_gate_up.contiguous(),
                                  None if ws_down is None else ws_down.contiguous(), self.packed[r])
        # each rank's own stage outputs (stacked: rank r at index r)
        self.topk_idx, self.topk_w = rows(R), torch.zeros((P, T, top_k), device=dev)
        self.counts, self.offsets = rows(E), rows(E + 1)
        self.splits, self.rank_offsets = rows(P), rows(P + 1)
        self.pos, self.src = rows(R), rows(R)
        self.ws_tok = torch.empty((P, max(B.moe_workspace_size(self.tok_cfg), 256)), dtype=torch.uint8,
                                  device=dev)
        # exchange buffers, reached through the pointer tables
        self.cnt = i32(P, P, E)
        self.flags = i32(P, 3, P)
        self.recv_x, self.recv_src, self.recv_rank = bf(P, cap, D), i32(P, cap), i32(P, cap)
        self.y_back = bf(P, R, D)
        # the local experts' inputs and outputs
        self.local_off = rows(El + 1)
        self.act, self.y_recv = bf(P, cap, F), bf(P, cap, D)
        self.ws_loc = torch.empty((P, max(B.moe_workspace_size(self.loc_cfg), 256)), dtype=torch.uint8,
                                  device=dev)
        self.ws_sh = torch.empty((P, max(B.moe_workspace_size(self.sh_cfg), 256)), dtype=torch.uint8,
                                 device=dev)
        xdt = torch.float32 if x_dtype in ("f32", torch.float32) else torch.bfloat16
        self.shared_out = bf(P, T, D) if self.S else None
        self.out = torch.empty((P, T, D), dtype=xdt, device=dev)
        self.done, self.status = i32(P), i32(1)
        table = lambda t: torch.tensor([t[r].data_ptr() for r in range(P)], dtype=torch.int64, device=dev)
        self._tables = [table(t) for t in (self.cnt, self.flags, self.recv_x, self.recv_src,
                                          self.recv_rank, self.y_back)]
        self.peers = B.MoeEpPeers(P, cap, *[t.data_ptr() for t in self._tables])
        self.epoch = 0

    def forward(self, x, stream=None):
        P, c = self.P, self.tok_cfg
        self.epoch = self.epoch % 0xFFFFFFFF + 1          # never 0, the flags' initial value
        e = self.epoch
        for r in range(P):                                 # 1. each rank routes its tokens
            B.moe_route(c, x[r], self.w_router, self.bias, None, self.topk_idx[r], self.topk_w[r],
                        self.ws_tok[r], stream)
        for r in range(P):
            B.moe_preprocess(c, self.topk_idx[r], self.counts[r], self.offsets[r], self.splits[r],
                             self.rank_offsets[r], self.pos[r], self.src[r], self.ws_tok[r],
                             self.status, stream)
        # 2. counts, then the token pre-all-to-all into the owners' buffers
        B.moe_ep_send_counts(c, self.peers, 0, P, self.counts, e, stream)
        B.moe_ep_send_rows(c, self.peers, 0, P, x, self.topk_idx, self.pos, self.offsets, e, self.done,
                           self.status, stream)
        B.moe_ep_recv_layout(c, self.peers, 0, P, self.local_off, e, self.status, stream)
        for d in range(P):                                 # 3. each rank's local experts
            B.moe_expert_ffn(self.loc_cfg, self.recv_x[d], None, self.local_off[d], self.packed[d],
                             self.act[d], self.y_recv[d], None, self.ws_loc[d], self.status, stream)
        # 4. the token post-all-to-all back to the senders' dispatch rows
        B.moe_ep_return_rows(c, self.peers, 0, P, self.y_recv, self.local_off, e, self.done,
                             self.status, stream)
        B.moe_ep_wait_returned(c, self.peers, 0, P, e, self.status, stream)
        for r in range(P):                                 # 5. shared experts and combine
            sh = None
            if self.S:
                sh = self.shared_out[r]
                B.moe_shared_ffn(self.sh_cfg, x[r], self.packed[r], sh, self.ws_sh[r], self.status, stream)
            B.moe_combine_unpermute(c, self.y_back[r], self.pos[r], self.topk_w[r], x[r], sh, self.out[r],
                                    stream)
        return self.out

    __call__ = forward

    def check_status(self):
        v = int(self.status.item())
        if v != B.MOE_OK:
            raise B.MoeError("device status", v)
