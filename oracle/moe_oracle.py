"""Plain float64 CPU definition of the expert-parallel MoE-layer forward.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module, and this module imports nothing from the product.

Sources (page title, section):
  [EP]   "Expert Parallel (EP)" (twinkle-kit docs): Configuration (router_dtype,
         keep_router_logits, ignore_shared_experts), Communication Pattern (the
         four-stage pipeline), Requirements (num_experts divisible by ep_size,
         fused gate_up_proj/down_proj experts, shared experts).
  [GATE] "How does the gate coordinate across ranks in expert parallelism?"
         (Tutel issue 278): every rank's gate scores all E experts for its own
         local tokens; gate weights are one replicated set.
  [TRACE] "Worked Example: Tracing a Token Through Expert Parallelism": Step 1
         (softmax over all experts, top-2 picks 2 and 11 with weights 0.6/0.4),
         Step 2 (expert 11 lives on device 2 as local expert 11 mod 4 = 3),
         Step 3 (two-layer FFN per expert, devices hold contiguous expert ranges,
         e.g. 8-11 on device 2), Step 4 (weighted sum 0.6*out_2 + 0.4*out_11),
         Step 5 (residual add).
  [SHARED] torchtitan issue 5554 (shared-expert overlap), description: the
         shared FFN is an independent always-on branch, joined with the routed
         branch before the outputs are combined.

Readings where the pages are silent (each also listed in the design notes):
  * Router logits are fp32: the dot product is formed in float64 and rounded
    once to fp32; an optional per-expert fp32 bias is added in fp32.
  * Top-k order: logit descending, ties to the lower expert index.
  * Weights: softmax over the k chosen logits (renormalised, so the k weights
    sum to 1, as 0.6 + 0.4 does in [TRACE] Step 1); optionally the plain
    softmax over all E, restricted to the k chosen.
  * Expert placement: contiguous ranges, rank = e // (E/ep), local = e % (E/ep).
  * Permuted buffer: rows sorted by expert (equivalently rank-major, then local
    expert), tokens ascending inside an expert; no capacity, no dropping.
  * Expert FFN: no biases; SwiGLU with gate = first F columns of gate_up, up =
    last F; GELU uses the exact erf form.
  * Shared experts: unit weight, summed, applied to every token.
  * Expert inputs and weights are bf16 values; an fp32 x is rounded to bf16
    (round-to-nearest-even) for the expert FFN only; residual and router use x
    as given.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "bf16_round", "bf16_bits_to_f64", "router_logits", "topk_select", "expert_placement",
    "preprocess", "permute", "unpermute", "gelu", "silu", "expert_ffn",
    "shared_experts", "combine", "moe_layer", "route_gaps",
]


# ----------------------------------------------------------------------------
# bf16 storage helpers
# ----------------------------------------------------------------------------

def bf16_round(a) -> np.ndarray:
    """Round fp32 values to the nearest bf16 value, ties to even; returns float64.

    bf16 keeps the top 16 bits of an IEEE fp32.  Round-to-nearest-even on the
    dropped 16 bits: add 0x7FFF plus the lowest kept bit, then truncate.
    Finite inputs only (the workloads hold no inf/NaN).
    """
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Interpret uint16 bf16 bit patterns as numbers (exact)."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# Stage 0: router  ([EP] Configuration: router_dtype='fp32'; [GATE]; [TRACE] Step 1)
# ----------------------------------------------------------------------------

def router_logits(x, w_router, bias=None) -> np.ndarray:
    """fp32 router logits over all E experts for every local token.

    l[t, e] = fl32( sum_d x[t, d] * W_r[e, d] )  (+ b_e, added in fp32)

    [GATE]: the gate output spans all experts globally and each rank scores its
    own local tokens.  [EP] Configuration: router computed in fp32.
    """
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_router, dtype=np.float64)
    logits = (x64 @ w64.T).astype(np.float32)
    if bias is not None:
        logits = (logits + np.asarray(bias, dtype=np.float32)).astype(np.float32)
    return logits


def topk_select(logits, k: int, renormalize: bool = True):
    """Softmax over the experts, then keep the k most probable ([TRACE] Step 1).

    Order: logit descending, equal logits broken toward the lower expert index
    (softmax is monotone, so ordering logits orders probabilities).
    Weights, in float64 from the fp32 logits, with m = the largest logit:
      renormalize:  w_j = exp(l_j - m) / sum_{j' in top-k} exp(l_j' - m)
      otherwise:    w_j = exp(l_j - m) / sum_{e < E}     exp(l_e  - m)
    Returns (topk_idx int32 [T, k], topk_w float64 [T, k]).
    """
    l32 = np.asarray(logits, dtype=np.float32)
    T, E = l32.shape
    if not (1 <= k <= E):
        raise ValueError("top_k must be in [1, E]")
    # A stable sort of the negated logits keeps equal logits in index order.
    order = np.argsort(-l32, axis=1, kind="stable")
    idx = order[:, :k]
    l64 = l32.astype(np.float64)
    chosen = np.take_along_axis(l64, idx, axis=1)
    m = chosen[:, :1]
    num = np.exp(chosen - m)
    if renormalize:
        den = num.sum(axis=1, keepdims=True)
    else:
        den = np.exp(l64 - m).sum(axis=1, keepdims=True)
    return idx.astype(np.int32), num / den


def route_gaps(logits, k: int):
    """Per-token fp32 logit gaps that decide how exactly routing can be compared.

    gap_k[t]     = l_(k) - l_(k+1): the margin of the top-k *set* (inf if k == E).
    inner_gap[t] = the smallest gap between adjacent chosen logits: the margin of
                   the *order* inside the top-k (inf if k == 1).
    """
    l32 = np.asarray(logits, dtype=np.float32)
    T, E = l32.shape
    s = -np.sort(-l32.astype(np.float64), axis=1)
    gap_k = (s[:, k - 1] - s[:, k]) if k < E else np.full(T, np.inf)
    inner = np.diff(-s[:, :k], axis=1).min(axis=1) if k > 1 else np.full(T, np.inf)
    return gap_k, inner


# ----------------------------------------------------------------------------
# Stage 1: preprocess  ([EP] Overview shard_experts, Communication Pattern 1)
# ----------------------------------------------------------------------------

def expert_placement(e, E: int, ep_size: int):
    """Even contiguous split of E experts over ep_size ranks.

    [EP] Requirements: E must be divisible by ep_size.  [TRACE] Step 2:
    expert 11 of 16 on 4 devices is on device 2 as local expert 11 mod 4 = 3;
    Step 3: device 2 holds experts 8-11.
    Returns (rank, local) = (e // El, e % El) with El = E / ep_size.
    """
    if E % ep_size != 0:
        raise ValueError("num_experts must be divisible by ep_size")
    El = E // ep_size
    e = np.asarray(e)
    return e // El, e % El


def preprocess(topk_idx, E: int, ep_size: int) -> dict:
    """Per-expert token counts, split sizes and the dispatch order.

    [EP] Communication Pattern stage 1 (counts and split sizes) and stage 2
    (permute tokens by expert assignment before the exchange).

      counts[e]          number of (token, slot) pairs routed to e
      expert_offsets     exclusive prefix sum of counts, length E+1
      rank_splits[r]     sum of counts over rank r's experts (the exchange's
                         per-destination split size)
      rank_offsets       exclusive prefix sum of rank_splits, length ep+1
      src[row]           flat index t*k + j of the pair stored at permuted row
      pos[t*k + j]       permuted row of pair (t, j); pos and src are inverse

    Rows are ordered by expert (= rank-major, then local expert, since experts
    are contiguous per rank), then by flat index, i.e. token ascending.
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert index out of range")
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    expert_offsets = np.concatenate([[0], np.cumsum(counts)])
    rank, _ = expert_placement(np.arange(E), E, ep_size)
    rank_splits = np.zeros(ep_size, dtype=np.int64)
    np.add.at(rank_splits, rank, counts)
    rank_offsets = np.concatenate([[0], np.cumsum(rank_splits)])
    src = np.argsort(flat, kind="stable")          # stable: flat index ascending per expert
    pos = np.empty_like(src)
    pos[src] = np.arange(src.size)
    i32 = lambda a: np.asarray(a, dtype=np.int32)
    return dict(counts=i32(counts), expert_offsets=i32(expert_offsets),
                rank_splits=i32(rank_splits), rank_offsets=i32(rank_offsets),
                pos=i32(pos), src=i32(src))


def permute(x_rows, src, k: int) -> np.ndarray:
    """Token pre-all-to-all: row `row` of the dispatch buffer is a copy of token
    src[row] // k ([EP] Communication Pattern 2; [TRACE] Step 2: each chosen
    expert gets its own copy of the token)."""
    x_rows = np.asarray(x_rows)
    return x_rows[np.asarray(src, dtype=np.int64) // k]


def unpermute(rows, pos, T: int, k: int) -> np.ndarray:
    """Inverse of ``permute``: gather each token's k rows back, shape [T, k, ...]
    ([EP] Communication Pattern 4, unpermute)."""
    rows = np.asarray(rows)
    return rows[np.asarray(pos, dtype=np.int64).reshape(T, k)]


# ----------------------------------------------------------------------------
# Stage 2: expert compute  ([EP] Communication Pattern 3; [TRACE] Step 3)
# ----------------------------------------------------------------------------

def gelu(h):
    """Exact GELU: h * Phi(h) = 0.5 * h * (1 + erf(h / sqrt 2))."""
    h = np.asarray(h, dtype=np.float64)
    return 0.5 * h * (1.0 + _erf(h / math.sqrt(2.0)))


def silu(g):
    """SiLU: g * sigmoid(g) = g / (1 + exp(-g))."""
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def expert_ffn(x_rows, w_up, w_down, act: str) -> np.ndarray:
    """One expert's two-layer feed-forward network on a block of rows, float64.

    [TRACE] Step 3: the expert transforms the token through its two-layer FFN.
    [EP] Requirements: fused experts are gate_up_proj [D, 2F] and down_proj [F, D].
      swiglu: h = x @ gate_up;  a = silu(h[:, :F]) * h[:, F:];  y = a @ down
      gelu:   y = gelu(x @ W1) @ W2
    No biases.
    """
    x = np.asarray(x_rows, dtype=np.float64)
    wu = np.asarray(w_up, dtype=np.float64)
    wd = np.asarray(w_down, dtype=np.float64)
    h = x @ wu
    if act == "swiglu":
        F = wu.shape[1] // 2
        a = silu(h[:, :F]) * h[:, F:]
    elif act == "gelu":
        a = gelu(h)
    else:
        raise ValueError(act)
    return a @ wd


def shared_experts(x_rows, ws_gate_up, ws_down) -> np.ndarray:
    """Sum of the always-on shared SwiGLU experts, unit weight, every token.

    [EP] Configuration/Requirements: shared experts are handled unless
    ignore_shared_experts; [SHARED]: an independent branch joined with the
    routed branch before the combination.
    """
    x = np.asarray(x_rows, dtype=np.float64)
    s = np.zeros((x.shape[0], x.shape[1]), dtype=np.float64)
    if ws_gate_up is None:
        return s
    for i in range(len(ws_gate_up)):
        s += expert_ffn(x, ws_gate_up[i], ws_down[i], "swiglu")
    return s


# ----------------------------------------------------------------------------
# Stage 3: combine  ([EP] Communication Pattern 4; [TRACE] Steps 4-5)
# ----------------------------------------------------------------------------

def combine(y_tok, topk_w, residual, shared=None) -> np.ndarray:
    """out[t] = x[t] + shared[t] + sum_j w[t, j] * y[t, j]   (float64)

    [TRACE] Step 4: weighted sum of the chosen experts' outputs; Step 5: plus
    the original token representation (residual).  y_tok is [T, k, D].
    """
    y = np.asarray(y_tok, dtype=np.float64)
    w = np.asarray(topk_w, dtype=np.float64)
    out = np.asarray(residual, dtype=np.float64) + np.einsum("tk,tkd->td", w, y)
    if shared is not None:
        out = out + np.asarray(shared, dtype=np.float64)
    return out


# ----------------------------------------------------------------------------
# Whole layer
# ----------------------------------------------------------------------------

def moe_layer(x, w_router, bias, w_up, w_down, ws_gate_up, ws_down, *, E: int,
              ep_size: int, top_k: int, act: str, renormalize: bool = True,
              x_is_f32: bool = False, tokens=None, expert_weights=None) -> dict:
    """Forward of the MoE layer, stage by stage ([EP] Communication Pattern).

    x, w_router, bias: float arrays holding the exact input values.
    w_up [E, D, 2F or F], w_down [E, F, D], ws_*: float arrays of bf16 values;
    ``expert_weights`` may instead be a callable e -> (w_up[e], w_down[e]) so a
    caller can stream large expert tensors one at a time.
    ``tokens``: optional subset of token indices; routing is then evaluated for
    those tokens only (tokens are independent: no capacity, no dropping), and
    the dispatch bookkeeping below covers just that subset.
    Returns the router logits, selection, bookkeeping, per-token expert outputs
    and the layer output, all float64 except the integer arrays and fp32 logits.
    """
    x = np.asarray(x, dtype=np.float64)
    if tokens is not None:
        x = x[np.asarray(tokens)]
    T = x.shape[0]
    logits = router_logits(x, w_router, bias)
    idx, w = topk_select(logits, top_k, renormalize)
    pre = preprocess(idx, E, ep_size)
    # Expert inputs are bf16 values; an fp32 x is rounded for the FFN only.
    x_ffn = bf16_round(x) if x_is_f32 else x
    x_perm = permute(x_ffn, pre["src"], top_k)
    y_perm = np.zeros_like(x_perm)
    off = pre["expert_offsets"]
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue                      # an empty expert is never evaluated
        wu, wd = expert_weights(e) if expert_weights is not None else (w_up[e], w_down[e])
        y_perm[lo:hi] = expert_ffn(x_perm[lo:hi], wu, wd, act)
    y_tok = unpermute(y_perm, pre["pos"], T, top_k)
    shared = shared_experts(x_ffn, ws_gate_up, ws_down) if ws_gate_up is not None else None
    out = combine(y_tok, w, x, shared)
    return dict(logits=logits, topk_idx=idx, topk_w=w, x_perm=x_perm, y_perm=y_perm,
                shared=shared, out=out, **pre)
