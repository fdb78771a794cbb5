"""Plain, slow, fp64 CPU oracle of the Grok-1-style sparse MoE layer (forward and backward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports or calls this
module: only the tests, the smoke check and the benchmark's CPU-baseline leg
do.  It shares no code with the CUDA path; both sides receive the same input
bits from the ``synth`` generator.

Source of every step: the page "How does Grok-1 use a mixture-of-experts
design?" (n4n.ai).  Sections cited below:
  [Arch]    "The high-level architecture"          (GrokMoELayer.forward)
  [Routing] "Routing: top-2 without auxiliary loss" (grok_router_forward and
            the capacity-factor paragraph after it)
  [Expert]  "Expert implementation: SwiGLU at scale" (SwiGLUExpert,
            FusedSwiGLUExpert)
  [EP]      "Expert parallelism vs. tensor parallelism" (moe_layer_ep_forward:
            each expert's output is scaled by its routing weight)
  [Trade]   "Tradeoffs: when MoE wins and when it doesn't" (expert_batch_size)
  [Dyn]     "Training dynamics: expert specialization" (utilization statistic)
and the page "Let Grok spill the beans on Grok" (Medium), whose feature list
states that the layer output is the weighted sum of the active experts'
outputs.

Readings taken where the pages leave a step open (each one is listed, with its
reason, in the design notes of the repository):
  * capacity = ceil(capacity_factor * T * top_k / E) evaluated in double in that
    order; capacity_factor = +inf (or E/top_k) means no drop;
  * overflow is dropped lowest-token-index-first: an assignment (t, e) is kept
    iff fewer than `capacity` earlier tokens were routed to e;
  * the softmax runs over the two selected logits only and is not renormalised
    after a drop; a token whose two assignments are both dropped outputs 0;
  * equal logits rank the lower expert index first;
  * silu(z) = z * sigmoid(z);
  * an optional per-expert logit bias is added to the logits before top-k.
The method is exact (no approximation), so every function below is the plain
definition, in float64, with numpy's matmul as the only library primitive.
Parity unpinned: none (each function is pinned by tests/test_oracle_pins.py).
"""
from __future__ import annotations

import math
import sys

import numpy as np


# ----------------------------------------------------------------------------
# input decoding (storage format only)
# ----------------------------------------------------------------------------
def to_f64(a: np.ndarray) -> np.ndarray:
    """Widen stored inputs to float64 (exact): uint16 arrays hold bf16 bit patterns.

    A bf16 value is the high half of the fp32 with the same bits, so the bf16
    bits are written into the high 16 bits of zeroed 32-bit words (little-endian
    layout) and the result is read as fp32 and widened to fp64.
    """
    a = np.asarray(a)
    if a.dtype == np.uint16:
        assert sys.byteorder == "little"
        w = np.zeros(a.shape, dtype=np.uint32)
        w.view(np.uint16)[..., 1::2] = a
        return w.view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# [Routing] router logits, top-2, softmax over the two selected logits
# ----------------------------------------------------------------------------
def router_logits(x, w_router, logit_bias=None) -> np.ndarray:
    """logits[t, e] = sum_i x[t, i] * w_router[e, i]  (hidden @ W_r.T), [Routing].

    w_router is stored [E, d] as on the page.  ``logit_bias`` (length E) is
    added to every token's logits before top-k when given.
    """
    lg = to_f64(x) @ to_f64(w_router).T
    if logit_bias is not None:
        lg = lg + np.asarray(logit_bias, dtype=np.float64)[None, :]
    return lg


def top2_softmax(logits: np.ndarray, top_k: int = 2):
    """Top-k experts per token ordered by logit, then softmax over the k values.

    [Arch] / [Routing]: topk over the E logits, then softmax of the selected
    values only.  Ordering: descending logit; equal logits keep the lower
    expert index first (stable sort of the negated logits).
    Returns idx int32 [T, k] and w float64 [T, k].
    """
    lg = np.asarray(logits, dtype=np.float64)
    order = np.argsort(-lg, axis=1, kind="stable")[:, :top_k]
    sel = np.take_along_axis(lg, order, axis=1)
    m = sel.max(axis=1, keepdims=True)
    ex = np.exp(sel - m)
    w = ex / ex.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w


def near_tie_gap(logits: np.ndarray, top_k: int = 2) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest logit of each token."""
    s = -np.sort(-np.asarray(logits, dtype=np.float64), axis=1)
    return s[:, top_k - 1] - s[:, top_k]


# ----------------------------------------------------------------------------
# [Routing] capacity-factor dispatch
# ----------------------------------------------------------------------------
def capacity(T: int, top_k: int, E: int, capacity_factor: float) -> int:
    """Per-expert capacity ceil(cf * T * k / E); +inf means every assignment fits."""
    if math.isinf(capacity_factor):
        return int(T)
    return int(math.ceil(capacity_factor * float(T * top_k) / float(E)))


def dispatch(idx: np.ndarray, w: np.ndarray, E: int, cap: int):
    """Group assignments by expert with the capacity rule.

    Tokens are visited in index order; assignment (t, j) to e = idx[t, j] is
    kept iff fewer than ``cap`` assignments to e were kept before it.  Kept
    assignments of expert e occupy consecutive slots offsets[e] + rank, in token
    order (the grouping step of ``_dispatch_and_combine``, [Arch]).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    kept = np.zeros(E, dtype=np.int64)
    rank = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if kept[e] < cap:
                rank[t, j] = kept[e]
                kept[e] += 1
    counts_raw = np.bincount(idx.ravel().astype(np.int64), minlength=E)[:E]
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    n_kept = int(offsets[E])
    slot_of = np.full((T, k), -1, dtype=np.int64)
    perm = np.full(n_kept, -1, dtype=np.int64)
    row_scale = np.zeros(n_kept, dtype=np.float64)
    for t in range(T):
        for j in range(k):
            if rank[t, j] >= 0:
                s = offsets[int(idx[t, j])] + rank[t, j]
                slot_of[t, j] = s
                perm[s] = t
                row_scale[s] = w[t, j]
    return {
        "counts_raw": counts_raw.astype(np.int64),
        "counts_kept": kept,
        "offsets": offsets,
        "perm": perm,
        "slot_of": slot_of,
        "row_scale": row_scale,
        "n_kept": n_kept,
        "dropped": int(T * k - n_kept),
    }


# ----------------------------------------------------------------------------
# [Expert] SwiGLU expert
# ----------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def swiglu_hidden(x_rows, w_gate_e, w_up_e) -> np.ndarray:
    """H = silu(x @ W_gate) * (x @ W_up)   (SwiGLUExpert.forward, [Expert]).

    Weights are stored [d, f] so that x @ W maps hidden -> expert_dim.
    """
    x = to_f64(x_rows)
    return silu(x @ to_f64(w_gate_e)) * (x @ to_f64(w_up_e))


def swiglu_expert(x_rows, w_gate_e, w_up_e, w_down_e) -> np.ndarray:
    """y = (silu(x @ W_gate) * (x @ W_up)) @ W_down   ([Expert]); W_down is [f, d]."""
    return swiglu_hidden(x_rows, w_gate_e, w_up_e) @ to_f64(w_down_e)


# ----------------------------------------------------------------------------
# [Arch] the whole layer
# ----------------------------------------------------------------------------
def layer_forward(x, w_router, w_gate, w_up, w_down, capacity_factor, logit_bias=None,
                  top_k: int = 2, tokens=None, keep_hidden: bool = False):
    """Forward pass of one MoE layer, returning every intermediate.

    Router, top-k and dispatch run over all T tokens.  The expert FFN and the
    combine run for the tokens in ``tokens`` (default: all), so large layers
    can be checked on a subsample.  out[t] = sum over kept (t, j) of
    w[t, j] * expert_{idx[t, j]}(x[t])  ([Arch] combine, [EP] weight scaling);
    a token with no kept assignment outputs zero.
    """
    x = np.asarray(x)
    T = x.shape[0]
    E = np.asarray(w_router).shape[0]
    lg = router_logits(x, w_router, logit_bias)
    idx, w = top2_softmax(lg, top_k)
    cap = capacity(T, top_k, E, capacity_factor)
    disp = dispatch(idx, w, E, cap)
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    d = x.shape[1]
    out = np.zeros((tok.size, d), dtype=np.float64)
    hidden = {}
    for e in range(E):
        rows = [(i, j) for i, t in enumerate(tok) for j in range(top_k)
                if idx[t, j] == e and disp["slot_of"][t, j] >= 0]
        if not rows:
            continue
        xr = x[[tok[i] for i, _ in rows]]
        h = swiglu_hidden(xr, w_gate[e], w_up[e])
        y = h @ to_f64(w_down[e])
        for r, (i, j) in enumerate(rows):
            out[i] += w[tok[i], j] * y[r]
            if keep_hidden:
                hidden[int(disp["slot_of"][tok[i], j])] = h[r]
    res = dict(disp)
    res.update({"logits": lg, "idx": idx, "w": w, "cap": cap, "tokens": tok, "out": out})
    if keep_hidden:
        res["hidden"] = hidden
    return res


# ----------------------------------------------------------------------------
# Backward pass (training).  The pages give only the forward pass; the
# capacity drop is described as a training-time rule ([Routing], capacity
# paragraph), so training differentiates this same forward.  Reading: the
# gradient of L = sum(out * dout) with respect to x, W_r, the logit bias and
# the expert weights, with the discrete steps (the top-2 choice and the
# capacity mask) held fixed: they are piecewise constant, so their derivative
# is zero wherever it exists.  The gradient reaches the router only through
# the softmax weights of the two selected logits.
# ----------------------------------------------------------------------------
def silu_grad(z: np.ndarray) -> np.ndarray:
    """d/dz [z * sigmoid(z)] = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def layer_backward(x, w_router, w_gate, w_up, w_down, capacity_factor, dout, logit_bias=None, top_k: int = 2,
                   tokens=None):
    """Gradients of sum(out * dout) for the layer of layer_forward.

    Per kept assignment (t, j) with expert e and weight w = w[t, j]:
      g = x_t W_gate[e], u = x_t W_up[e], h = silu(g) * u, y = h W_down[e]
      out_t += w * y                                   ([Arch], [EP])
    so, with dy = w * dout_t:
      dweight[t, j] = <dout_t, y>
      dW_down[e] += h^T dy,   dh = dy W_down[e]^T
      dg = dh * u * silu'(g), du = dh * silu(g)
      dW_gate[e] += x_t^T dg, dW_up[e] += x_t^T du,  dx_t += dg W_gate[e]^T + du W_up[e]^T
    Dropped assignments contribute nothing (dweight = 0).  The softmax over the
    selected logits w_j = exp(l_j) / sum_i exp(l_i) gives
      dlogits[t, idx[t, j]] = w_j * (dweight_j - sum_i w_i * dweight_i)
    and the router logits l = x W_r^T + bias give
      dW_r = dlogits^T x,  dx += dlogits W_r,  dbias = sum_t dlogits[t].
    Returns the forward intermediates of layer_forward plus dx [T, d],
    dw_router [E, d], dbias [E], dw_gate [E, d, f], dw_up [E, d, f],
    dw_down [E, f, d], dlogits [T, E] and dweight [T, k], all float64.
    With ``tokens`` (a subset), routing and capacity still run over all T, but
    only the listed tokens' assignments are differentiated: their rows of dx,
    dlogits and dweight are exact, the other rows are zero, and the parameter
    gradients hold only those tokens' contributions.
    """
    x64 = to_f64(x)
    T, d = x64.shape
    wr = to_f64(w_router)
    E = wr.shape[0]
    g_dout = to_f64(dout)
    lg = router_logits(x, w_router, logit_bias)
    idx, w = top2_softmax(lg, top_k)
    cap = capacity(T, top_k, E, capacity_factor)
    disp = dispatch(idx, w, E, cap)
    f = np.asarray(w_gate[0]).shape[1]
    dx = np.zeros((T, d))
    dwg = np.zeros((E, d, f))
    dwu = np.zeros((E, d, f))
    dwd = np.zeros((E, f, d))
    dweight = np.zeros((T, top_k))
    tok = range(T) if tokens is None else sorted(set(int(t) for t in tokens))
    for e in range(E):
        pairs = [(t, j) for t in tok for j in range(top_k) if idx[t, j] == e and disp["slot_of"][t, j] >= 0]
        if not pairs:
            continue
        ts = np.array([t for t, _ in pairs])
        js = np.array([j for _, j in pairs])
        wg, wu, wd = to_f64(w_gate[e]), to_f64(w_up[e]), to_f64(w_down[e])
        xr = x64[ts]
        g = xr @ wg
        u = xr @ wu
        h = silu(g) * u
        y = h @ wd
        dy = w[ts, js][:, None] * g_dout[ts]
        dweight[ts, js] = np.sum(g_dout[ts] * y, axis=1)
        dwd[e] = h.T @ dy
        dh = dy @ wd.T
        dg = dh * u * silu_grad(g)
        du = dh * silu(g)
        dwg[e] = xr.T @ dg
        dwu[e] = xr.T @ du
        np.add.at(dx, ts, dg @ wg.T + du @ wu.T)
    dlogits = np.zeros((T, E))
    mean = np.sum(w * dweight, axis=1)
    for t in tok:
        for j in range(top_k):
            dlogits[t, idx[t, j]] += w[t, j] * (dweight[t, j] - mean[t])
    dx += dlogits @ wr
    res = dict(disp)
    res.update({"logits": lg, "idx": idx, "w": w, "cap": cap, "dx": dx, "dw_router": dlogits.T @ x64,
                "dbias": dlogits.sum(axis=0), "dw_gate": dwg, "dw_up": dwu, "dw_down": dwd, "dlogits": dlogits,
                "dweight": dweight})
    return res


def expert_weight_grad_slices(x, w_router, w_gate, w_up, w_down, capacity_factor, dout, e, cols,
                              logit_bias=None, top_k: int = 2):
    """Slices of layer_backward's weight gradients for one expert, for layers too
    large to differentiate whole: columns ``cols`` of dW_gate[e] and dW_up[e]
    ([d, n]) and rows ``cols`` of dW_down[e] ([n, d]).  The same formulas
    restricted to those hidden units: every hidden unit m of expert e only needs
    g[:, m], u[:, m] and W_down[e][m, :], so
      dW_down[e][m, :] = sum_r h[r, m] * dy[r, :]
      dW_gate[e][:, m] = sum_r x_r * dg[r, m],  dW_up[e][:, m] = sum_r x_r * du[r, m]
    over the kept rows r of expert e (routing and capacity over all tokens)."""
    x64 = to_f64(x)
    T = x64.shape[0]
    E = np.asarray(w_router).shape[0]
    lg = router_logits(x, w_router, logit_bias)
    idx, w = top2_softmax(lg, top_k)
    disp = dispatch(idx, w, E, capacity(T, top_k, E, capacity_factor))
    pairs = [(t, j) for t in range(T) for j in range(top_k) if idx[t, j] == e and disp["slot_of"][t, j] >= 0]
    cols = np.asarray(cols, dtype=np.int64)
    d = x64.shape[1]
    if not pairs:
        return {"dw_gate_cols": np.zeros((d, cols.size)), "dw_up_cols": np.zeros((d, cols.size)),
                "dw_down_rows": np.zeros((cols.size, d))}
    ts = np.array([t for t, _ in pairs])
    js = np.array([j for _, j in pairs])
    xr = x64[ts]
    wg = to_f64(np.asarray(w_gate[e])[:, cols])
    wu = to_f64(np.asarray(w_up[e])[:, cols])
    wd = to_f64(np.asarray(w_down[e])[cols, :])
    g = xr @ wg
    u = xr @ wu
    h = silu(g) * u
    dy = w[ts, js][:, None] * to_f64(dout)[ts]
    dh = dy @ wd.T
    dg = dh * u * silu_grad(g)
    du = dh * silu(g)
    return {"dw_gate_cols": xr.T @ dg, "dw_up_cols": xr.T @ du, "dw_down_rows": h.T @ dy}


# ----------------------------------------------------------------------------
# 8-bit expert weights ("weights in the official release were quantized":
# "Benchmarking xAI's Grok-1", section "Grok-1: In Practice"; "8-Bit
# Quantization" in the feature list of "Let Grok spill the beans on Grok";
# the n4n.ai page's "Tradeoffs" section on quantising the weights to cut
# their memory).  The pages name no scheme; the reading taken is symmetric
# int8 per output channel, weights only (activations stay in the layer dtype).
# ----------------------------------------------------------------------------
def quantize_int8(w):
    """Per-output-channel symmetric int8 of weights stored [..., K, N] (channel = N).

    An encoding, so every decision is stated in fp32 (IEEE, round to nearest even):
      amax[n]  = max_k |w[k, n]|          (exact: w is bf16 or fp32)
      scale[n] = amax[n] / 127            (fp32 division)
      q[k, n]  = clamp(rint(w[k, n] / scale[n]), -127, 127)   (fp32 division)
    A column of zeros gets scale 0 and codes 0.  Returns (q int8, scale float32).
    """
    a = np.asarray(w)
    if a.dtype == np.uint16:
        wf = np.zeros(a.shape, dtype=np.uint32)
        wf.view(np.uint16)[..., 1::2] = a
        wf = wf.view(np.float32)
    else:
        wf = a.astype(np.float32)
    amax = np.max(np.abs(wf), axis=-2)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    r = (wf / safe[..., None, :]).astype(np.float32)
    q = np.clip(np.rint(r), -127, 127)
    q = np.where(scale[..., None, :] > 0, q, 0).astype(np.int8)
    return q, scale


def dequantize_int8(q, scale):
    """w'[k, n] = q[k, n] * scale[n], in float64 (exact)."""
    return np.asarray(q, dtype=np.float64) * np.asarray(scale, dtype=np.float64)[..., None, :]


ROW_CODE_MAX = 32512  # 127 * 256: a row code splits into two int8 halves


def quantize_rows(v):
    """15-bit symmetric code of each activation row, decisions in IEEE fp32:
      scale[r] = max_k |v[r, k]| / 32512                    (fp32 division)
      code[r, k] = clamp(rint(v[r, k] / scale[r]), -32512, 32512)
      hi = floor((code + 128) / 256),  lo = code - 256 * hi  (both in [-128, 127])
    so that code = 256 * hi + lo exactly.  A row of zeros gets scale 0.
    Input values are taken as fp32 (bf16 bit patterns are widened exactly).
    Returns (hi int8, lo int8, scale float32)."""
    a = np.asarray(v)
    if a.dtype == np.uint16:
        vf = np.zeros(a.shape, dtype=np.uint32)
        vf.view(np.uint16)[..., 1::2] = a
        vf = vf.view(np.float32)
    else:
        vf = a.astype(np.float32)
    amax = np.max(np.abs(vf), axis=-1)
    scale = (amax / np.float32(ROW_CODE_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    code = np.clip(np.rint((vf / safe[..., None]).astype(np.float32)), -ROW_CODE_MAX, ROW_CODE_MAX)
    code = np.where(scale[..., None] > 0, code, 0).astype(np.int64)
    hi = np.floor_divide(code + 128, 256)
    lo = code - 256 * hi
    return hi.astype(np.int8), lo.astype(np.int8), scale


def dequantize_rows(hi, lo, scale):
    """v'[r, k] = (256 * hi + lo) * scale[r], in float64 (exact)."""
    code = 256 * np.asarray(hi, dtype=np.int64) + np.asarray(lo, dtype=np.int64)
    return code.astype(np.float64) * np.asarray(scale, dtype=np.float64)[..., None]


def layer_forward_w8(x, w_router, q_gate, s_gate, q_up, s_up, q_down, s_down, capacity_factor, logit_bias=None,
                     top_k: int = 2, tokens=None):
    """The layer with int8 expert weights, as the 8-bit path defines it.

    Routing, capacity and combine are those of layer_forward.  Each expert sees
    its rows through quantize_rows (x rows, then the fp32-rounded H rows), and
    its weights as q * scale; every product is then exact, so the expert output
    is computed exactly (in float64) from those codes:
      g = rows(x) @ (q_gate * s_gate),  u = rows(x) @ (q_up * s_up)
      H = silu(g) * u,   y = rows(fp32(H)) @ (q_down * s_down)
    """
    x = np.asarray(x)
    T = x.shape[0]
    E = np.asarray(w_router).shape[0]
    lg = router_logits(x, w_router, logit_bias)
    idx, w = top2_softmax(lg, top_k)
    cap = capacity(T, top_k, E, capacity_factor)
    disp = dispatch(idx, w, E, cap)
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    out = np.zeros((tok.size, x.shape[1]), dtype=np.float64)
    for e in range(E):
        rows = [(i, j) for i, t in enumerate(tok) for j in range(top_k)
                if idx[t, j] == e and disp["slot_of"][t, j] >= 0]
        if not rows:
            continue
        xr = dequantize_rows(*quantize_rows(x[[tok[i] for i, _ in rows]]))
        h = silu(xr @ dequantize_int8(q_gate[e], s_gate[e])) * (xr @ dequantize_int8(q_up[e], s_up[e]))
        hr = dequantize_rows(*quantize_rows(h.astype(np.float32)))
        y = hr @ dequantize_int8(q_down[e], s_down[e])
        for r, (i, j) in enumerate(rows):
            out[i] += w[tok[i], j] * y[r]
    res = dict(disp)
    res.update({"logits": lg, "idx": idx, "w": w, "cap": cap, "tokens": tok, "out": out})
    return res


class DequantizedExperts:
    """Expert weights given as (q [E, K, N] int8, scale [E, N]); indexing an expert
    returns its dequantized float64 matrix, so layer_forward can run on them
    without materialising every expert at once."""

    def __init__(self, q, scale):
        self.q, self.scale = q, scale
        self.shape = q.shape

    def __getitem__(self, e):
        return dequantize_int8(self.q[e], self.scale[e])


# ----------------------------------------------------------------------------
# statistics the pages define
# ----------------------------------------------------------------------------
def expert_batch_size(global_batch: int, seq_len: int, num_experts: int = 8, top_k: int = 2) -> float:
    """Average tokens per expert = batch * seq * k / E   ([Trade])."""
    return global_batch * seq_len * top_k / num_experts


def expert_utilization(counts, num_experts: int = 8, top_k: int = 2) -> np.ndarray:
    """Assignments per expert normalised so that a balanced router gives 1.0 ([Dyn]).

    utilization[e] = counts[e] / n_tokens * E / k with n_tokens = sum(counts) / k.
    The page's snippet divides by the number of assignments (tokens * k) instead,
    which would give 0.5 for a balanced router; its own comment says 1.0, and
    that is the reading taken here.
    """
    c = np.asarray(counts, dtype=np.float64)
    n_tokens = c.sum() / top_k
    return c / n_tokens * num_experts / top_k
