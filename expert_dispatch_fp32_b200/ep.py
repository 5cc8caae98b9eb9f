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
    and each exchange call covers all P ranks in one launch (kernels of different ranks
    never wait on one another across launches); each rank's local experts run as their
    own launch whose down-projection epilogue stores the output rows straight into the
    senders' y_back (moe_ep_expert_ffn_return).  forward(x) takes x [P, T, D] and
    returns out [P, T, D]: rank r's rows equal moe_forward of its tokens with all E
    experts.
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
        # 3.-4. each rank's local experts, their output rows stored by the down GEMM's
        # epilogue straight back into the senders' y_back at their dispatch rows
        for d in range(P):
            B.moe_ep_expert_ffn_return(c, self.loc_cfg, self.peers, d, self.recv_x[d], self.recv_src[d],
                                       self.recv_rank[d], self.local_off[d], self.packed[d], self.act[d],
                                       self.y_recv[d], self.ws_loc[d], e, self.done[d:d + 1], self.status,
                                       stream)
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


# --------------------------------------------------------------------------------------
# One process per GPU: the same peer-memory exchange, each rank's buffers mapped into
# the other ranks' processes
# --------------------------------------------------------------------------------------

EXCHANGE_BUFFERS = ("cnt", "flags", "recv_x", "recv_src", "recv_rank", "y_back")


def exchange_layout(P, E, D, T, top_k, cap):
    """Byte offsets and sizes of one rank's exchange buffers inside its single exchange
    allocation (the same on every rank, so a peer's buffer is its mapped base plus the
    offset): count matrix int32 [P, E], flags uint32 [3, P], received rows bf16 [cap, D]
    with their sender rows and ranks int32 [cap], returned rows bf16 [T*k, D]."""
    sizes = {"cnt": 4 * P * E, "flags": 4 * 3 * P, "recv_x": 2 * cap * D, "recv_src": 4 * cap,
             "recv_rank": 4 * cap, "y_back": 2 * T * top_k * D}
    off, o = {}, 0
    for name in EXCHANGE_BUFFERS:
        off[name] = o
        o += (sizes[name] + 255) // 256 * 256
    return off, sizes, o


class CudaIpc:
    """Maps exchange allocations between the processes of one node (libmoe.so's
    moe_ipc_* calls: a CUDA IPC handle of the allocation plus the buffer's offset)."""

    def export(self, t):
        return B.moe_ipc_export(t)

    def import_(self, handle, offset):
        return B.moe_ipc_import(handle, offset)

    def close(self, ptr, offset):
        B.moe_ipc_close(ptr, offset)


def peer_tables(rank, own_base, offsets, infos, ipc):
    """Pointer tables of one rank: for each exchange buffer, entry p is rank p's buffer,
    i.e. rank p's exchange allocation (this rank's own, or rank p's export mapped into
    this process) plus the buffer's offset.  infos[p] is what rank p shared: its
    exported (handle, offset).  Returns the tables (name -> P addresses) and the
    mappings opened, (address, offset) pairs for ipc.close."""
    P = len(infos)
    bases, opened = [0] * P, []
    for p in range(P):
        if p == rank:
            bases[p] = own_base
            continue
        handle, off = infos[p]["export"]
        ptr = ipc.import_(handle, off)
        opened.append((ptr, off))
        bases[p] = ptr
    return {name: [bases[p] + offsets[name] for p in range(P)] for name in EXCHANGE_BUFFERS}, opened


def gather_infos(info, group=None):
    """Every rank's `info` (host-side: host name, device id, exported handle), in rank
    order, over the process group (any backend; one rank without a group)."""
    if not dist.is_initialized():
        return [info]
    infos = [None] * dist.get_world_size(group)
    dist.all_gather_object(infos, info, group=group)
    return infos


def check_peer_devices(infos):
    """Every rank on its own GPU of one node: kernels of two ranks on one device would
    wait on each other across launches (PeerEPGroup runs such ranks in one launch), and
    the handles map only within a node."""
    hosts = {inf["host"] for inf in infos}
    if len(hosts) > 1:
        raise RuntimeError(f"peer-memory exchange needs one node; ranks are on {sorted(hosts)}")
    seen = {}
    for p, inf in enumerate(infos):
        if inf["device"] in seen:
            raise RuntimeError(f"ranks {seen[inf['device']]} and {p} share device {inf['device']}: "
                               "run ranks that share a GPU as one PeerEPGroup")
        seen[inf["device"]] = p


class PeerEPRank:
    """One rank of the expert-parallel forward over peer memory, one process per GPU.

    "Expert Parallel (EP)", Communication Pattern: rank r (its rank in `group`, P = the
    group's size = ep) owns experts [r*El, (r+1)*El) and its own T tokens; the router
    and the shared experts are replicated.  The exchanges are the moe_ep_* calls of
    PeerEPGroup, each covering this rank alone (rank0 = r, nlocal = 1), with pointer
    tables whose other entries are the other ranks' exchange buffers mapped into this
    process once, at construction (moe_ipc_*: each rank exports its exchange
    allocation, the handles go round the group with all_gather_object, each rank maps
    the others').  Rows are stored straight into the owners' memory over NVLink /
    NVSwitch and every wait is a flag in peer memory: no collective library and no host
    round trip per forward.  Every rank calls forward the same number of times, with T
    tokens each; close() (after the last forward, on every rank) unmaps the peers.  Each
    process selects its own GPU (torch.cuda.set_device) before constructing the rank, and
    its weights live there.
    """

    def __init__(self, group=None, *, D, E, top_k, F, T, w_router, w_gate_up_local, w_down_local,
                 expert_bias=None, ws_gate_up=None, ws_down=None, act="swiglu", renormalize=True,
                 x_dtype="bf16", ipc=None):
        import socket
        self.group = group
        on = dist.is_initialized()
        P = dist.get_world_size(group) if on else 1
        r = dist.get_rank(group) if on else 0
        if E % P:
            raise ValueError("num_experts must be divisible by the number of ranks")
        dev = w_router.device
        self.D, self.E, self.P, self.rank, self.k, self.F, self.T = D, E, P, r, top_k, F, T
        self.El = El = E // P
        self.S = 0 if ws_gate_up is None else ws_gate_up.shape[0]
        self.Fs = 0 if ws_gate_up is None else ws_down.shape[1]
        self.cap = cap = P * T * min(top_k, El)
        self.w_router = w_router.contiguous()
        self.bias = None if expert_bias is None else expert_bias.contiguous()
        self.tok_cfg = make_config(T, D, E, P, top_k, F, act, renormalize, x_dtype, self.S, self.Fs)
        self.loc_cfg = make_config(cap, D, El, 1, 1, F, act, True, "bf16", self.S, self.Fs)
        self.sh_cfg = make_config(T, D, El, 1, 1, F, act, True, "bf16", self.S, self.Fs)
        i32 = lambda n: torch.zeros(n, dtype=torch.int32, device=dev)
        R = T * top_k
        self.packed = torch.empty(B.moe_packed_weights_size(self.loc_cfg), dtype=torch.uint8, device=dev)
        B.moe_prepare_weights(self.loc_cfg, w_gate_up_local.contiguous(), w_down_local.contiguous(),
                              None if ws_gate_up is None else ws_gate_up.contiguous(),
                              None if ws_down is None else ws_down.contiguous(), self.packed)
        self.topk_idx = torch.zeros((T, top_k), dtype=torch.int32, device=dev)
        self.topk_w = torch.zeros((T, top_k), dtype=torch.float32, device=dev)
        self.counts, self.offsets = i32(E), i32(E + 1)
        self.splits, self.rank_offsets = i32(P), i32(P + 1)
        self.pos, self.src = i32(R), i32(R)
        self.ws_tok = torch.empty(max(B.moe_workspace_size(self.tok_cfg), 256), dtype=torch.uint8, device=dev)
        # the exchange buffers: one zeroed allocation (flags start at 0, the epoch never is)
        self.offsets_x, sizes, total = exchange_layout(P, E, D, T, top_k, cap)
        self.xbuf = torch.zeros(total, dtype=torch.uint8, device=dev)
        view = lambda name, dt, shape: self.xbuf[self.offsets_x[name]:self.offsets_x[name] + sizes[name]] \
            .view(dt).view(shape)
        self.recv_x = view("recv_x", torch.bfloat16, (cap, D))
        self.recv_src = view("recv_src", torch.int32, (cap,))
        self.recv_rank = view("recv_rank", torch.int32, (cap,))
        self.y_back = view("y_back", torch.bfloat16, (R, D))
        self.local_off = i32(El + 1)
        self.act = torch.zeros((cap, F), dtype=torch.bfloat16, device=dev)
        self.y_recv = torch.zeros((cap, D), dtype=torch.bfloat16, device=dev)
        self.ws_loc = torch.empty(max(B.moe_workspace_size(self.loc_cfg), 256), dtype=torch.uint8, device=dev)
        self.ws_sh = torch.empty(max(B.moe_workspace_size(self.sh_cfg), 256), dtype=torch.uint8, device=dev)
        xdt = torch.float32 if x_dtype in ("f32", torch.float32) else torch.bfloat16
        self.shared_out = torch.zeros((T, D), dtype=torch.bfloat16, device=dev) if self.S else None
        self.out = torch.empty((T, D), dtype=xdt, device=dev)
        self.done, self.status = i32(1), i32(1)
        # map the peers' exchange allocations; the handles travel as host bytes
        self.ipc = ipc if ipc is not None else CudaIpc()
        props = torch.cuda.get_device_properties(dev)
        info = {"host": socket.gethostname(), "device": str(getattr(props, "uuid", dev)),
                "export": self.ipc.export(self.xbuf) if P > 1 else None}
        infos = gather_infos(info, group)
        check_peer_devices(infos)
        tables, self._opened = peer_tables(r, self.xbuf.data_ptr(), self.offsets_x, infos, self.ipc)
        self._tables = [torch.tensor(tables[name], dtype=torch.int64, device=dev) for name in EXCHANGE_BUFFERS]
        self.peers = B.MoeEpPeers(P, cap, *[t.data_ptr() for t in self._tables])
        self.epoch = 0
        torch.cuda.synchronize(dev)
        if on:
            dist.barrier(group)     # every rank's flags are zero before any rank's first store

    def forward(self, x, stream=None):
        c, r = self.tok_cfg, self.rank
        self.epoch = self.epoch % 0xFFFFFFFF + 1          # never 0, the flags' initial value
        e = self.epoch
        B.moe_route(c, x, self.w_router, self.bias, None, self.topk_idx, self.topk_w, self.ws_tok, stream)
        B.moe_preprocess(c, self.topk_idx, self.counts, self.offsets, self.splits, self.rank_offsets,
                         self.pos, self.src, self.ws_tok, self.status, stream)
        # counts, then the token pre-all-to-all into the owners' buffers
        B.moe_ep_send_counts(c, self.peers, r, 1, self.counts, e, stream)
        B.moe_ep_send_rows(c, self.peers, r, 1, x, self.topk_idx, self.pos, self.offsets, e, self.done,
                           self.status, stream)
        # the shared experts need only this rank's tokens: they run while the other ranks'
        # rows are still on their way (the wait below then finds them there)
        sh = None
        if self.S:
            sh = self.shared_out
            B.moe_shared_ffn(self.sh_cfg, x, self.packed, sh, self.ws_sh, self.status, stream)
        B.moe_ep_recv_layout(c, self.peers, r, 1, self.local_off, e, self.status, stream)
        # the local experts; the down GEMM's epilogue stores each output row straight into
        # its sender's y_back (the token post-all-to-all, tile by tile)
        B.moe_ep_expert_ffn_return(c, self.loc_cfg, self.peers, r, self.recv_x, self.recv_src,
                                   self.recv_rank, self.local_off, self.packed, self.act, self.y_recv,
                                   self.ws_loc, e, self.done, self.status, stream)
        B.moe_ep_wait_returned(c, self.peers, r, 1, e, self.status, stream)
        B.moe_combine_unpermute(c, self.y_back, self.pos, self.topk_w, x, sh, self.out, stream)
        return self.out

    __call__ = forward

    def check_status(self):
        v = int(self.status.item())
        if v != B.MOE_OK:
            raise B.MoeError("device status", v)

    def close(self):
        """Unmap the peers' buffers once every rank is done with the exchange (all ranks
        call it; the rank's own allocation stays valid until the object is dropped)."""
        torch.cuda.synchronize(self.xbuf.device)
        if dist.is_initialized():
            dist.barrier(self.group)
        for ptr, off in self._opened:
            self.ipc.close(ptr, off)
        self._opened = []
