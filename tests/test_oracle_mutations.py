"""Plant plausible mistakes in the oracle (on the CPU) and show the pins catch each.

Each mutation patches one function of ``oracle.moe_oracle`` for the duration of
the test; ``moe_layer`` calls its stages through the module namespace, so the
patched stage is what the whole-layer checks see too.
"""
import math

import numpy as np
import pytest

import oracle.moe_oracle as O
from test_oracle_pins import ALL_CHECKS

_orig = {name: getattr(O, name) for name in
         ("combine", "expert_ffn", "topk_select", "gelu", "expert_placement", "preprocess",
          "router_logits", "shared_experts", "bf16_round", "permute", "route_gaps")}


def _combine_no_residual(y_tok, topk_w, residual, shared=None):
    return _orig["combine"](y_tok, topk_w, np.zeros_like(np.asarray(residual, dtype=np.float64)), shared)


def _ffn_swapped(x_rows, w_up, w_down, act):
    if act == "swiglu":
        wu = np.asarray(w_up)
        F = wu.shape[1] // 2
        w_up = np.concatenate([wu[:, F:], wu[:, :F]], axis=1)
    return _orig["expert_ffn"](x_rows, w_up, w_down, act)


def _topk_ties_high(logits, k, renormalize=True):
    l = np.asarray(logits, dtype=np.float32)[:, ::-1]
    idx, w = _orig["topk_select"](l, k, renormalize)
    return (l.shape[1] - 1 - idx).astype(np.int32), w


def _topk_no_renorm(logits, k, renormalize=True):
    return _orig["topk_select"](logits, k, False)


def _gelu_tanh(h):
    h = np.asarray(h, dtype=np.float64)
    return 0.5 * h * (1 + np.tanh(math.sqrt(2 / math.pi) * (h + 0.044715 * h ** 3)))


def _placement_modulo(e, E, ep_size):
    e = np.asarray(e)
    return e % ep_size, e // ep_size


def _preprocess_tokens_descending(topk_idx, E, ep_size):
    pre = _orig["preprocess"](topk_idx, E, ep_size)
    src = pre["src"].copy()
    off = pre["expert_offsets"]
    for e in range(E):
        src[off[e]:off[e + 1]] = src[off[e]:off[e + 1]][::-1]
    pos = np.empty_like(src)
    pos[src] = np.arange(src.size)
    pre.update(src=src, pos=pos.astype(np.int32))
    return pre


def _preprocess_inclusive_scan(topk_idx, E, ep_size):
    pre = _orig["preprocess"](topk_idx, E, ep_size)
    off = pre["expert_offsets"].copy()
    off[:-1] = off[1:]
    pre.update(expert_offsets=off)
    return pre


def _logits_ignore_bias(x, w_router, bias=None):
    return _orig["router_logits"](x, w_router, None)


def _logits_fp32_accumulate(x, w_router, bias=None):
    x32 = np.asarray(x, dtype=np.float32)
    w32 = np.asarray(w_router, dtype=np.float32)
    T, D = x32.shape
    acc = np.zeros((T, w32.shape[0]), dtype=np.float32)
    for d in range(D):                      # naive fp32 accumulation, one term at a time
        acc = (acc + (x32[:, d:d + 1] * w32[:, d][None, :]).astype(np.float32)).astype(np.float32)
    if bias is not None:
        acc = (acc + np.asarray(bias, dtype=np.float32)).astype(np.float32)
    return acc


def _shared_half(x_rows, ws_gate_up, ws_down):
    return 0.5 * _orig["shared_experts"](x_rows, ws_gate_up, ws_down)


def _bf16_truncate(a):
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return (f.view(np.uint32) & 0xFFFF0000).view(np.float32).astype(np.float64)


def _permute_off_by_one(x_rows, src, k):
    return np.asarray(x_rows)[(np.asarray(src, dtype=np.int64) + 1) % (len(src)) // k]


def _gaps_one_neighbour_early(logits, k):
    s = -np.sort(-np.asarray(logits, dtype=np.float64), axis=1)
    gap, inner = _orig["route_gaps"](logits, k)
    if 2 <= k:
        gap = s[:, k - 2] - s[:, k - 1]
    return gap, inner


def _gaps_inner_includes_next(logits, k):
    s = -np.sort(-np.asarray(logits, dtype=np.float64), axis=1)
    gap, inner = _orig["route_gaps"](logits, k)
    if k < s.shape[1]:
        inner = np.diff(-s[:, :k + 1], axis=1).min(axis=1)
    return gap, inner


def _gaps_unsorted(logits, k):
    l = np.asarray(logits, dtype=np.float64)
    T, E = l.shape
    gap = l[:, k - 1] - l[:, k] if k < E else np.full(T, np.inf)
    inner = np.abs(np.diff(l[:, :k], axis=1)).min(axis=1) if k > 1 else np.full(T, np.inf)
    return gap, inner


MUTATIONS = {
    "combine drops the residual": ("combine", _combine_no_residual),
    "SwiGLU gate/up halves swapped": ("expert_ffn", _ffn_swapped),
    "ties broken toward the higher index": ("topk_select", _topk_ties_high),
    "top-k weights not renormalised": ("topk_select", _topk_no_renorm),
    "tanh-approximate GELU": ("gelu", _gelu_tanh),
    "experts placed round-robin": ("expert_placement", _placement_modulo),
    "tokens descending inside an expert": ("preprocess", _preprocess_tokens_descending),
    "inclusive instead of exclusive scan": ("preprocess", _preprocess_inclusive_scan),
    "router bias ignored": ("router_logits", _logits_ignore_bias),
    "router accumulated term by term in fp32": ("router_logits", _logits_fp32_accumulate),
    "shared experts weighted by 1/2": ("shared_experts", _shared_half),
    "bf16 by truncation": ("bf16_round", _bf16_truncate),
    "permute gathers the wrong row": ("permute", _permute_off_by_one),
    "set gap taken one neighbour early": ("route_gaps", _gaps_one_neighbour_early),
    "inner gap includes the (k+1)-th logit": ("route_gaps", _gaps_inner_includes_next),
    "gaps read from unsorted logits": ("route_gaps", _gaps_unsorted),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(O, attr, bad)
    failed = []
    for check in ALL_CHECKS:
        try:
            check(O)
        except (AssertionError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, f"no pin caught: {name}"
