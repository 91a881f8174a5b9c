"""Comparison rules between the CUDA path and the CPU oracle.

Selection (expert indices, counts): bit-exact, except for tokens whose
oracle scores at places k and k+1 differ by less than EXEMPT (1e-6, absolute
difference of sigmoid scores).  For such a token the GPU's index set is
accepted if every expert it has that the oracle lacks, and every one the
oracle has that it lacks, scores within EXEMPT of the oracle's k-th score.
Index sets are compared sorted (the order among near-equal interior scores is
not graded); there is no exemption when k = E.

Weights: |dw| <= W_TOL per weight, matched by expert id.  Order inside the
selected list: descending score up to ORDER_TOL (1e-5 in score, i.e. the
kernels' fp32 logit error of up to 4e-5 times the sigmoid's largest slope).
Output: relative Frobenius error <= 1e-2 and per element
|dy| <= 2e-2 * (|y_ref| + 0.05).
"""
import numpy as np

EXEMPT = 1e-6
W_TOL = 1e-5
ORDER_TOL = 1e-5
Y_REL_FRO = 1e-2
Y_ELEM_A = 2e-2
Y_ELEM_B = 0.05


def to_numpy_bf16(t):
    """torch bfloat16 tensor -> numpy uint16 bit patterns (host copy)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def compare_routing(gpu_idx, gpu_w, ref_idx, ref_w, ref_scores, k):
    """Returns (n_exempt_tokens, n_differing_tokens, list of hard failures)."""
    gpu_idx = np.asarray(gpu_idx)
    ref_idx = np.asarray(ref_idx)
    T, E = ref_scores.shape
    fails = []
    n_exempt = 0
    n_diff = 0
    srt = np.sort(ref_scores, axis=1)[:, ::-1]
    kth = srt[:, k - 1]
    gap = srt[:, k - 1] - srt[:, k] if k < E else np.full(T, np.inf)
    exempt = gap < EXEMPT
    n_exempt = int(exempt.sum())
    for t in range(T):
        gs = set(gpu_idx[t].tolist())
        rs = set(ref_idx[t].tolist())
        if len(gs) != k or min(gs) < 0 or max(gs) >= E:
            fails.append((t, "invalid index set", sorted(gs)))
            continue
        if gs != rs:
            n_diff += 1
            sym = gs ^ rs
            if not exempt[t] or any(abs(ref_scores[t, e] - kth[t]) >= EXEMPT for e in sym):
                fails.append((t, "selection", sorted(gs), sorted(rs)))
            continue
        # same set: weights matched by expert id
        gw = dict(zip(gpu_idx[t].tolist(), np.asarray(gpu_w[t]).tolist()))
        rw = dict(zip(ref_idx[t].tolist(), np.asarray(ref_w[t]).tolist()))
        for e in rs:
            if abs(gw[e] - rw[e]) > W_TOL:
                fails.append((t, "weight", e, gw[e], rw[e]))
                break
        # listed in descending score order (near-equal scores may swap)
        sc = ref_scores[t, gpu_idx[t]]
        if np.any(np.diff(sc) > ORDER_TOL):
            fails.append((t, "order", gpu_idx[t].tolist()))
    return n_exempt, n_diff, fails


def same_selection_mask(gpu_idx, ref_idx):
    return np.array([set(a) == set(b) for a, b in zip(np.asarray(gpu_idx).tolist(),
                                                       np.asarray(ref_idx).tolist())])


def compare_output(got, ref, rows=None):
    """Returns (rel_fro, max_violation_ratio); ok iff rel_fro <= 1e-2 and ratio <= 1."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if rows is not None:
        got, ref = got[rows], ref[rows]
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    bound = Y_ELEM_A * (np.abs(ref) + Y_ELEM_B)
    ratio = float(np.max(np.abs(got - ref) / bound)) if got.size else 0.0
    return rel, ratio


def output_ok(got, ref, rows=None):
    rel, ratio = compare_output(got, ref, rows)
    return rel <= Y_REL_FRO and ratio <= 1.0, rel, ratio
