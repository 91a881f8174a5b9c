"""CPU oracle for the forward pass of a Laguna-style token-choice MoE layer.

TEST INFRASTRUCTURE.  This module is the independent checker of the CUDA
library, not part of it.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
It shares no code with the CUDA path: it takes plain numpy arrays (bfloat16
inputs as uint16 bit patterns, or float arrays) and computes in float64.

What the layer computes, and where the pages say so:

* Router: sigmoid scores over the experts, token-choice top-k, and
  normalisation of the selected scores to sum to one
  (Laguna M.1/XS.2 Technical Report summary, Key claims, report §3.1: a
  sigmoid router whose top-k scores are normalised after the selection;
  Laguna-M.1-base spec sheet, Mixture of experts: sigmoid router scores,
  top-k renormalisation on).
* Experts: SwiGLU feed-forward blocks without bias
  (Laguna-M.1-base spec sheet, Feed-forward: SwiGLU activation, no FFN
  bias, gate_proj / up_proj / down_proj projections).
* Combine: the routed sum is multiplied by the modulation factor 2.5 and then
  added to an always-on shared expert
  (Laguna M.1/XS.2 Technical Report summary, Key claims, report §3.1;
  Laguna-M.1-base spec sheet, Mixture of experts, "Routed scaling factor":
  1 for M.1, 2.5 introduced in XS.2).
* Expert order: tokens are laid out expert by expert before the grouped GEMM
  (Laguna M.1/XS.2 Technical Report summary, Key claims, report §3.1.2,
  Fig. 2: the tokens are copied so that each expert's rows are contiguous).

Readings where the pages are silent:

* SwiGLU(x) = W_down (silu(W_gate x) * (W_up x)), silu(z) = z * sigmoid(z).
* One shared expert of the same SwiGLU form, ungated, added after the 2.5.
* An optional router bias b (a workload device) is added to the logits
  before the sigmoid; it changes selection and weights alike.
* Top-k is taken on the scores; since the sigmoid is strictly increasing this
  is the same as taking it on the logits.  Exact ties go to the lower expert
  index.  The selected list is ordered by descending score.
* Normalisation runs over the k selected experts only, with no epsilon.
* A padding token (token mask 0) is not routed: no expert, weight 0, no row
  in the expert order; the shared expert still applies to it.
* Auxiliary-loss-free balancing: a per-expert bias is added to the sigmoid
  scores for the choice of the experts only; the weights stay the
  normalised unbiased scores.

Every function is a direct transcription of these definitions; numpy's
matmul is the only library step.
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(a):
    """Exact widening of bfloat16 bit patterns (uint16) to float64.

    Float arrays are passed through as float64 unchanged.
    """
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def sigmoid(z):
    """Logistic function 1 / (1 + exp(-z)), float64."""
    z = np.asarray(z, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    """SiLU (swish) z * sigmoid(z), the gate nonlinearity of SwiGLU."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def router_logits(x, w_router, bias=None):
    """l[t, e] = sum_i x[t, i] * W_r[e, i]  (+ b[e]).

    x: [T, d]; w_router: [E, d] (nn.Linear [out, in] layout); bias: [E] or None.
    """
    X = bf16_to_f64(x)
    W = bf16_to_f64(w_router)
    logits = X @ W.T
    if bias is not None:
        logits = logits + np.asarray(bias, dtype=np.float64)[None, :]
    return logits


def select_topk(logits, k):
    """Indices of the k largest logits per row, largest first.

    Equal values keep ascending expert order, so an exact tie at the k-th
    place goes to the lower expert index.
    """
    logits = np.asarray(logits, dtype=np.float64)
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def normalise(selected_scores, norm_topk_prob=True):
    """w_j = s_j / sum_j' s_j' over the selected experts (no epsilon)."""
    s = np.asarray(selected_scores, dtype=np.float64)
    if not norm_topk_prob:
        return s.copy()
    return s / s.sum(axis=1, keepdims=True)


# Expert id of a (token, slot) pair that is not routed (a padding token).
NOT_ROUTED = -1


def route(x, w_router, bias, k, norm_topk_prob=True, token_mask=None, selection_bias=None):
    """Sigmoid router with post-top-k normalisation.

    token_mask ([T], 0 = padding token) leaves padding tokens unrouted: their
    k slots get expert id NOT_ROUTED and weight 0 (Laguna training notes:
    padding tokens are best neither routed nor load-balanced).

    selection_bias ([E]): the auxiliary-loss-free balancing variant (Laguna-
    M.1-base spec sheet, Mixture of experts, "Load balancing: auxiliary-loss-
    free").  The bias is added to the sigmoid scores for the choice of the k
    experts only; the weights are the normalised unbiased scores.  (``bias``
    and ``selection_bias`` are not combined: pass one of them.)

    Returns (topk_idx [T,k] int64, topk_w [T,k] f64, scores [T,E] f64, logits [T,E] f64).
    For selection_bias, ``scores`` are the selection keys sigmoid(l) + b.
    """
    logits = router_logits(x, w_router, bias)
    scores = sigmoid(logits)
    if selection_bias is None:
        idx = select_topk(logits, k)
    else:
        keys = scores + np.asarray(selection_bias, dtype=np.float64)[None, :]
        idx = select_topk(keys, k)
    sel = np.take_along_axis(scores, idx, axis=1)
    if selection_bias is not None:
        scores = keys
    w = normalise(sel, norm_topk_prob)
    if token_mask is not None:
        pad = np.asarray(token_mask) == 0
        idx[pad, :] = NOT_ROUTED
        w[pad, :] = 0.0
    return idx, w, scores, logits


def swiglu_ffn(x, w_gate, w_up, w_down):
    """down(silu(gate x) * (up x)) without bias, float64.

    x: [n, d]; w_gate, w_up: [F, d]; w_down: [d, F]  (nn.Linear layouts).
    """
    X = bf16_to_f64(x)
    g = X @ bf16_to_f64(w_gate).T
    u = X @ bf16_to_f64(w_up).T
    h = silu(g) * u
    return h @ bf16_to_f64(w_down).T


def expert_order(topk_idx, E):
    """Layout of the (token, slot) pairs in expert order.

    counts[e]  = number of tokens that selected expert e;
    offsets    = exclusive prefix sum of counts, length E + 1;
    perm[r]    = t * k + j for the r-th row in expert order, where rows of
                 one expert are sorted by token t, then by slot j.
    Pairs with expert id NOT_ROUTED are left out: perm has offsets[E] rows.
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    for e in idx.reshape(-1):
        if e != NOT_ROUTED:
            counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.empty(offsets[E], dtype=np.int64)
    fill = offsets[:-1].copy()
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            if e == NOT_ROUTED:
                continue
            perm[fill[e]] = t * k + j
            fill[e] += 1
    return counts, offsets, perm


def moe_forward(x, w_router, w_gate, w_up, w_down, k, *, router_bias=None,
                ws_gate=None, ws_up=None, ws_down=None,
                routed_scaling_factor=2.5, norm_topk_prob=True, routing=None,
                token_mask=None, selection_bias=None):
    """y_t = S(x_t) + scale * sum_j w_{t,j} * E_{e_{t,j}}(x_t), in float64.

    x: [T, d]; w_router: [E, d]; w_gate, w_up: [E, F, d]; w_down: [E, d, F];
    ws_gate, ws_up: [Fs, d]; ws_down: [d, Fs] (None: no shared expert).
    ``routing`` may pass a precomputed (topk_idx, topk_w) pair from ``route``.
    ``token_mask`` ([T], 0 = padding): a padding token is not routed, so its
    routed sum is empty and y_t = S(x_t); the shared expert, which involves no
    routing, still applies.

    Returns a dict with y, the routed sum R (before the scale), the shared
    output Sh, and the routing (topk_idx, topk_w, scores, logits).
    """
    X = bf16_to_f64(x)
    T, d = X.shape
    if routing is None:
        idx, w, scores, logits = route(x, w_router, router_bias, k, norm_topk_prob, token_mask,
                                       selection_bias)
    else:
        idx, w = routing
        scores = logits = None
    E = np.asarray(w_gate).shape[0]
    # contrib[t, j] = w_{t,j} * E_{e_{t,j}}(x_t); each expert evaluated on its tokens.
    contrib = np.zeros((T, k, d), dtype=np.float64)
    for e in range(E):
        tt, jj = np.nonzero(idx == e)
        if tt.size == 0:
            continue
        o = swiglu_ffn(X[tt], w_gate[e], w_up[e], w_down[e])
        contrib[tt, jj, :] = w[tt, jj][:, None] * o
    R = contrib.sum(axis=1)
    if ws_gate is not None:
        Sh = swiglu_ffn(X, ws_gate, ws_up, ws_down)
    else:
        Sh = np.zeros((T, d), dtype=np.float64)
    y = routed_scaling_factor * R + Sh
    return {"y": y, "R": R, "Sh": Sh, "topk_idx": idx, "topk_w": w,
            "scores": scores, "logits": logits}


# ---------------------------------------------------------------- FP8 experts
# FP8 expert weights for decode (the pages name FP8 deployment of the weights
# but no scale layout; this build defines one): every row of every expert
# matrix (an output channel), every token row of x and every row of h gets
# its own float32 scale, s = amax(|row|) / 448 (s = 1 for an all-zero row;
# for h rounded up to a power of two), and the row is stored as e4m3 codes
# q = e4m3(v * r) with r = 1 / s, every step one correctly rounded float32
# operation.  Products of codes are exact;
# the GEMMs accumulate in float32 and apply the row and column scales to the
# accumulator.  h is held in fp16 before it is quantized, as in the 16-bit
# path.

E4M3_MAX = 448.0


def e4m3_value(code):
    """Value of e4m3 codes (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits; exponent 0 is subnormal, 2^-6 * m/8; code S.1111.111 is NaN; no
    infinities)."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    v = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return s * v


def e4m3_round(v):
    """Round float32 values to e4m3 codes: nearest representable value, ties to
    the even code, magnitudes beyond 448 saturate to 448, NaN to the NaN code.

    Returns uint8 codes.
    """
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    _, ex = np.frexp(a)                  # a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex - 1
    e = np.maximum(ex - 1, -6)           # binade; below 2^-6 the subnormal quantum applies
    q = np.ldexp(1.0, e - 3)             # spacing of the 3-bit mantissa in that binade
    r = np.rint(a / q) * q               # round half to even (exact in float64)
    r = np.minimum(r, E4M3_MAX)
    # encode the (representable) magnitude
    _, rx = np.frexp(r)
    re = np.maximum(rx - 1, -6)
    sub = r < 2.0 ** -6
    mant = np.where(sub, np.rint(r / 2.0 ** -9), np.rint((r / np.ldexp(1.0, re) - 1.0) * 8.0))
    code = np.where(sub, mant, ((re + 7) << 3) + mant).astype(np.int64)
    code = np.where(nan, 0x7F, code) | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def pow2_ceil_f32(t):
    """Smallest power of two >= t for positive normal float32 t (2^-126 below the normal
    range), by the float32 bit pattern."""
    t = np.asarray(t, dtype=np.float32)
    u = t.view(np.uint32)
    up = ((u & np.uint32(0x7F800000)) + np.uint32(0x00800000)).astype(np.uint32)
    r = np.where((u & np.uint32(0x007FFFFF)) != 0, up, u).astype(np.uint32)
    r = np.where(u < np.uint32(0x00800000), np.uint32(0x00800000), r).astype(np.uint32)
    return r.view(np.float32)


def quantize_rows_e4m3(a, pow2=False):
    """Per-row e4m3 quantization of a float32 matrix [..., K] (last axis = row).

    Returns (codes uint8 [..., K], scales float32 [...]): s = amax / 448 in
    float32 (1 for an all-zero row), rounded up to a power of two when pow2
    (h rows: then every code depends on its own element only), r = 1 / s in
    float32, codes = e4m3_round(float32(a * r)).
    """
    a = np.asarray(a, dtype=np.float32)
    amax = np.max(np.abs(a), axis=-1)
    t = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    if pow2:
        t = pow2_ceil_f32(np.where(amax > 0, t, np.float32(1.0)))
    s = np.where(amax > 0, t, np.float32(1.0)).astype(np.float32)
    r = (np.float32(1.0) / s).astype(np.float32)
    codes = e4m3_round((a * r[..., None]).astype(np.float32))
    return codes, s


def dequantize_rows_e4m3(codes, scales):
    return e4m3_value(codes) * np.asarray(scales, dtype=np.float64)[..., None]


def quantize_experts_fp8(w_gate, w_up, w_down, ws_gate=None, ws_up=None, ws_down=None):
    """FP8 copies of the expert weights (bf16 bit patterns or floats in), one
    scale per output row: gate/up [E, F] (rows of [E, F, d]), down [E, d]."""
    def f(w):
        if w is None:
            return None
        w = np.asarray(w)
        if w.ndim == 2:
            return quantize_rows_e4m3(bf16_to_f64(w).astype(np.float32))
        parts = [quantize_rows_e4m3(bf16_to_f64(w[e]).astype(np.float32))  # expert by expert
                 for e in range(w.shape[0])]
        return np.stack([c for c, _ in parts]), np.stack([sc for _, sc in parts])
    return {"gate": f(w_gate), "up": f(w_up), "down": f(w_down),
            "s_gate": f(ws_gate), "s_up": f(ws_up), "s_down": f(ws_down)}


def moe_forward_fp8(x, w_router, fp8, k, *, router_bias=None, routed_scaling_factor=2.5,
                    norm_topk_prob=True):
    """The layer with FP8 expert weights: routing as in ``route`` (bf16 router),
    x quantized per token, h = SwiGLU(x_q W_g,q^T, x_q W_u,q^T) rounded to fp16 and
    quantized per row, o = h_q W_d,q^T; combine as in ``moe_forward``.  Every
    product of dequantized values is evaluated in float64."""
    X = bf16_to_f64(x)
    T, d = X.shape
    idx, w, scores, logits = route(x, w_router, router_bias, k, norm_topk_prob)
    xq = dequantize_rows_e4m3(*quantize_rows_e4m3(X.astype(np.float32)))

    def expert(xrows, g, u, dn):
        G = xrows @ dequantize_rows_e4m3(*g).T
        U = xrows @ dequantize_rows_e4m3(*u).T
        h = (silu(G) * U).astype(np.float16).astype(np.float32)
        hq = dequantize_rows_e4m3(*quantize_rows_e4m3(h, pow2=True))
        return hq @ dequantize_rows_e4m3(*dn).T

    gq, gs = fp8["gate"]
    uq, us = fp8["up"]
    dq, ds = fp8["down"]
    E = gq.shape[0]
    contrib = np.zeros((T, k, d), dtype=np.float64)
    for e in range(E):
        tt, jj = np.nonzero(idx == e)
        if tt.size == 0:
            continue
        o = expert(xq[tt], (gq[e], gs[e]), (uq[e], us[e]), (dq[e], ds[e]))
        contrib[tt, jj, :] = w[tt, jj][:, None] * o
    R = contrib.sum(axis=1)
    if fp8["s_gate"] is not None:
        Sh = expert(xq, fp8["s_gate"], fp8["s_up"], fp8["s_down"])
    else:
        Sh = np.zeros((T, d), dtype=np.float64)
    y = routed_scaling_factor * R + Sh
    return {"y": y, "R": R, "Sh": Sh, "topk_idx": idx, "topk_w": w, "scores": scores,
            "logits": logits}
