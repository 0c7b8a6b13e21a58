"""Oracle of the sparse MoE layer forward (test infrastructure only; see package docstring).

Notation: T tokens, H hidden (5120 in [P1] "Status": router GEMM (5120, 256)), E routed
experts (256), k chosen per token (8; [P2] "Overview"), I expert intermediate size.

Steps, in order ([P1] "Status"/"Remaining work", [P2] "Overview"/"Variants", [P3]
"Agents worked on the serving path"):
  1. router logits l = x W_r^T, x BF16 and W_r FP32 taken exactly, accumulated in FP64
  2. p = softmax over all E logits
  3. the k experts of largest p (equal p: lower expert index first), in descending p
  4. w_j = p_j / sum of the chosen p (renormalisation over the chosen k)
  5. token -> expert histogram, exclusive prefix sum (offsets), and the permutation
     that lists the rows of expert e in [offsets[e], offsets[e+1]) in ascending token order
  6. A1 = Q(x, alpha_a1)                              (NVFP4 activation, W4A4)
     (MXFP8 variant: A1 = MX(x), no tensor scale; see mxfp8.py for the reading)
  7. G = deq(A1) deq(W_gate)^T, U = deq(A1) deq(W_up)^T  per expert (FP64)
  8. h = G * sigmoid(G) * U                           (SwiGLU), rounded to FP32
  9. A2 = Q(h, alpha_a2)                              (MXFP8 variant: A2 = MX(h))
 10. y = deq(A2) deq(W_down)^T                        (FP64)
 11. m = sum_j w_j y_j                                (weighted un-permute, MoE finalize)
 12. n = m / sqrt(mean(m^2) + eps) * gamma            (post-RMSNorm of the sandwich norm)
 13. out = bf16_rne(residual + n)                     (residual add)
Readings where the pages are silent: gate rows are the first I rows of the stored
gate/up weight, up rows the last I; no bias, no clamp, no shared expert; RMSNorm is the
plain gamma * x_hat form; the output is rounded to BF16 once, from the exact sum.
"""

from __future__ import annotations

import numpy as np

from .mxfp8 import dequantize_mxfp8, quantize_mxfp8
from .nvfp4 import dequantize_nvfp4, quantize_nvfp4, tensor_scale

FORMATS = ("nvfp4", "mxfp8")


# ----------------------------------------------------------------------------- routing
def router_logits(x: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    """Step 1: l[t, e] = sum_h x[t, h] * W_r[e, h] in FP64 ([P1] "Status": (5120, 256))."""
    return np.asarray(x, np.float64) @ np.asarray(router_w, np.float64).T


def route_topk(logits: np.ndarray, k: int):
    """Steps 2-4 ([P2] "Overview": each token goes to 8 of 256 experts).

    Returns ids [T, k] (int64, descending p, ties to the lower index), w [T, k] (FP64,
    renormalised over the chosen k) and p [T, E] (softmax over all experts).
    """
    l = np.asarray(logits, np.float64)
    z = np.exp(l - l.max(axis=1, keepdims=True))
    p = z / z.sum(axis=1, keepdims=True)
    # A stable sort of -p keeps equal probabilities in ascending index order.
    order = np.argsort(-p, axis=1, kind="stable")
    ids = order[:, :k]
    psel = np.take_along_axis(p, ids, axis=1)
    w = psel / psel.sum(axis=1, keepdims=True)
    return ids.astype(np.int64), w, p


def near_tie_mask(logits: np.ndarray, k: int, rel: float = 1e-5) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest logits differ by less than
    rel * max(|l_k|, |l_k+1|, 1); their choice of expert is not unique at FP32-class
    precision, so exact-match checks of routing skip and count them."""
    l = np.asarray(logits, np.float64)
    if k >= l.shape[1]:
        return np.zeros(l.shape[0], dtype=bool)
    srt = -np.sort(-l, axis=1)
    a, b = srt[:, k - 1], srt[:, k]
    return (a - b) < rel * np.maximum(np.maximum(np.abs(a), np.abs(b)), 1.0)


def permute(ids: np.ndarray, num_experts: int):
    """Step 5: histogram, exclusive scan and the stable (expert, token) permutation.

    Returns counts [E], offsets [E+1], perm_src [T*k] (token of permuted row r),
    perm_slot [T*k] (slot j of that row) and inv [T, k] (permuted row of (t, j)).
    """
    ids = np.asarray(ids, np.int64)
    t_count, k = ids.shape
    flat_e = ids.reshape(-1)
    flat_t = np.repeat(np.arange(t_count), k)
    flat_j = np.tile(np.arange(k), t_count)
    counts = np.bincount(flat_e, minlength=num_experts).astype(np.int64)
    offsets = np.zeros(num_experts + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    # Sort by expert, then by token (lexsort: last key is primary).
    order = np.lexsort((flat_t, flat_e))
    perm_src = flat_t[order]
    perm_slot = flat_j[order]
    inv = np.empty((t_count, k), np.int64)
    inv[perm_src, perm_slot] = np.arange(t_count * k)
    return dict(counts=counts, offsets=offsets, perm_src=perm_src, perm_slot=perm_slot, inv=inv)


# ----------------------------------------------------------------------------- experts
def quantize_expert(w_gu: np.ndarray, w_d: np.ndarray, fmt: str = "nvfp4"):
    """Quantised weights of one expert ([P2] "Variants": routed experts are NVFP4; the FP8
    checkpoint is the second variant, MXFP8 here).

    w_gu: FP32 [2I, H] (rows 0..I-1 gate, I..2I-1 up); w_d: FP32 [H, I].
    NVFP4: one tensor scale for gate+up together and one for down, each amax / 2688.
    MXFP8: E4M3 codes with one UE8M0 scale per 32 values of a row, no tensor scale.
    """
    if fmt == "mxfp8":
        gu_c, gu_s = quantize_mxfp8(w_gu)
        d_c, d_s = quantize_mxfp8(w_d)
        return dict(fmt="mxfp8", w_gu=gu_c, w_gu_sf=gu_s, w_d=d_c, w_d_sf=d_s)
    if fmt != "nvfp4":
        raise ValueError(f"unknown expert format {fmt!r}")
    a_gu = tensor_scale(w_gu)
    a_d = tensor_scale(w_d)
    gu_p, gu_s = quantize_nvfp4(w_gu, a_gu)
    d_p, d_s = quantize_nvfp4(w_d, a_d)
    return dict(w_gu=gu_p, w_gu_sf=gu_s, w_gu_alpha=a_gu, w_d=d_p, w_d_sf=d_s, w_d_alpha=a_d)


def dequantize_expert(q):
    """FP64 gate/up [2I, H] and down [H, I] of a quantised expert."""
    if q.get("fmt") == "mxfp8":
        return dequantize_mxfp8(q["w_gu"], q["w_gu_sf"]), dequantize_mxfp8(q["w_d"], q["w_d_sf"])
    return (
        dequantize_nvfp4(q["w_gu"], q["w_gu_sf"], q["w_gu_alpha"]),
        dequantize_nvfp4(q["w_d"], q["w_d_sf"], q["w_d_alpha"]),
    )


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Step 8 before rounding: silu(g) * u = g * sigmoid(g) * u, FP64."""
    return g / (1.0 + np.exp(-g)) * u


def quantize_act(v, alpha, fmt: str = "nvfp4"):
    """Activation quantiser of steps 6 and 9: NVFP4 Q(v, alpha), or MXFP8 (alpha unused).
    Returns (codes, scale codes): packed E2M1 [.., K/2] + E4M3 [.., K/16], or E4M3 [.., K]
    + UE8M0 [.., K/32]."""
    if fmt == "mxfp8":
        return quantize_mxfp8(v)
    return quantize_nvfp4(v, alpha)


def dequantize_act(codes, sf, alpha, fmt: str = "nvfp4"):
    if fmt == "mxfp8":
        return dequantize_mxfp8(codes, sf)
    return dequantize_nvfp4(codes, sf, alpha)


def expert_forward(a1_packed, a1_sf, alpha_a1, deq_w, alpha_a2, fmt: str = "nvfp4"):
    """Steps 7-10 for the rows routed to one expert.

    a1_packed/a1_sf: quantised rows of that expert's inputs (format fmt); deq_w: (gate/up,
    down) in FP64.  Returns dict(h32 [R, I] FP32, a2_packed, a2_sf, y [R, H] FP64); for
    MXFP8 a2_packed holds one E4M3 code per value.
    """
    w_gu, w_d = deq_w
    inter = w_gu.shape[0] // 2
    a1 = dequantize_act(a1_packed, a1_sf, alpha_a1, fmt)
    g = a1 @ w_gu[:inter].T
    u = a1 @ w_gu[inter:].T
    h32 = swiglu(g, u).astype(np.float32)
    a2_packed, a2_sf = quantize_act(h32, alpha_a2, fmt)
    a2 = dequantize_act(a2_packed, a2_sf, alpha_a2, fmt)
    y = a2 @ w_d.T
    return dict(h32=h32, a2_packed=a2_packed, a2_sf=a2_sf, y=y)


# ----------------------------------------------------------------------------- finalize
def bf16_round(z: np.ndarray) -> np.ndarray:
    """Round FP64 values to the nearest BF16 (8 significant bits), ties to even; returns
    the rounded values as FP64 (finite inputs within the BF16 range)."""
    z = np.asarray(z, np.float64)
    f, ex = np.frexp(z)  # z = f * 2**ex, |f| in [0.5, 1)
    q = np.ldexp(1.0, ex - 8)  # step of an 8-bit significand in that binade
    out = np.rint(z / q) * q
    # BF16 keeps the FP32 exponent range; below 2^-126 the step stays 2^-133.
    tiny = np.abs(z) < 2.0 ** -126
    if np.any(tiny):
        out[tiny] = np.rint(z[tiny] / 2.0 ** -133) * 2.0 ** -133
    return out


def finalize(y_sel: np.ndarray, w: np.ndarray, residual: np.ndarray, gamma: np.ndarray, eps: float):
    """Steps 11-13 ([P1] "Remaining work": MoE finalize; "Status": sandwich norms).

    y_sel: [T, k, H] expert outputs of each token's chosen experts, w: [T, k].
    Returns (pre-rounding FP64 output [T, H], BF16-rounded output as FP64 [T, H], m).
    """
    m = np.einsum("tk,tkh->th", np.asarray(w, np.float64), np.asarray(y_sel, np.float64))
    rms = np.sqrt(np.mean(m * m, axis=1, keepdims=True) + eps)
    n = m / rms * np.asarray(gamma, np.float64)[None, :]
    pre = np.asarray(residual, np.float64) + n
    return pre, bf16_round(pre), m


def next_prenorm(out_bf16: np.ndarray, gamma_next: np.ndarray, eps: float):
    """The next sublayer's sandwich pre-norm on the updated residual stream ([PR] "Status":
    Beam's sandwich norms; "Remaining work": fused with the MoE finalize).

    out_bf16: the layer output as it leaves the layer (BF16 values, as FP64) [T, H].
    Returns (pre-rounding FP64, BF16-rounded as FP64) of out / sqrt(mean(out^2) + eps) * gamma_next.
    Reading: the norm reads the BF16 residual the next layer receives, not the FP32 sum.
    """
    o = np.asarray(out_bf16, np.float64)
    pre = o / np.sqrt(np.mean(o * o, axis=1, keepdims=True) + eps) * np.asarray(gamma_next, np.float64)[None, :]
    return pre, bf16_round(pre)


# ----------------------------------------------------------------------------- forward
class ExpertCache:
    """Quantises (with this oracle's quantiser) and dequantises experts on first use.

    get_fp32(e) must return the FP32 weights (w_gu [2I, H], w_d [H, I]) of expert e;
    fmt is the experts' format ("nvfp4" or "mxfp8").
    """

    def __init__(self, get_fp32, keep: int = 64, fmt: str = "nvfp4"):
        if fmt not in FORMATS:
            raise ValueError(f"unknown expert format {fmt!r}")
        self.get_fp32 = get_fp32
        self.keep = keep
        self.fmt = fmt
        self._deq = {}
        self._q = {}

    def quantized(self, e: int):
        if e not in self._q:
            w_gu, w_d = self.get_fp32(e)
            self._q[e] = quantize_expert(w_gu, w_d, self.fmt)
        return self._q[e]

    def dequantized(self, e: int):
        if e not in self._deq:
            if len(self._deq) >= self.keep:
                self._deq.pop(next(iter(self._deq)))
            self._deq[e] = dequantize_expert(self.quantized(e))
        return self._deq[e]


def moe_forward_tokens(x, residual, router_w, gamma, experts: ExpertCache, top_k, alpha_a1, alpha_a2,
                       eps=1e-6):
    """Steps 1-4 and 6-13 for a set of tokens (each token's output depends on that token
    only, so any subset of a batch gives the same rows as the whole batch).  The
    activations use the experts' format; alpha_a1 / alpha_a2 are unused for MXFP8.

    x, residual: FP64 [T, H] (exact BF16 values).  Returns dict with logits, ids, w,
    near_tie, a1 (packed, sf), h32 [T, k, I], y [T, k, H], out_pre, out (BF16 as FP64).
    """
    x = np.asarray(x, np.float64)
    t_count, hidden = x.shape
    logits = router_logits(x, router_w)
    ids, w, _ = route_topk(logits, top_k)
    fmt = experts.fmt
    a1_packed, a1_sf = quantize_act(x.astype(np.float32), alpha_a1, fmt)
    y = np.zeros((t_count, top_k, hidden), np.float64)
    h32 = None
    for e in np.unique(ids):
        tt, jj = np.nonzero(ids == e)
        r = expert_forward(a1_packed[tt], a1_sf[tt], alpha_a1, experts.dequantized(int(e)), alpha_a2, fmt)
        if h32 is None:
            h32 = np.zeros((t_count, top_k, r["h32"].shape[1]), np.float32)
        h32[tt, jj] = r["h32"]
        y[tt, jj] = r["y"]
    out_pre, out, m = finalize(y, w, residual, gamma, eps)
    return dict(logits=logits, ids=ids, w=w, near_tie=near_tie_mask(logits, top_k),
                a1_packed=a1_packed, a1_sf=a1_sf, h32=h32, y=y, m=m, out_pre=out_pre, out=out)


def moe_forward(x, residual, router_w, gamma, experts: ExpertCache, num_experts, top_k, alpha_a1, alpha_a2,
                eps=1e-6):
    """The whole layer for a batch: moe_forward_tokens plus the permutation of step 5."""
    r = moe_forward_tokens(x, residual, router_w, gamma, experts, top_k, alpha_a1, alpha_a2, eps)
    r.update(permute(r["ids"], num_experts))
    return r


# ----------------------------------------------------------------------------- tensor parallel
def shard_dequantized(deq_w, rank: int, world: int):
    """Rank `rank`'s slice of one expert under tensor parallelism over the intermediate size:
    the gate and up rows of features [r s, (r+1) s) and the same columns of down, s = I / world
    ([PR] "Status": Beam's TP all-reduce; [RECIPE] "Launching the server": NVFP4 with TP4).
    deq_w: (gate/up [2I, H], down [H, I]) FP64.  Returns the shard's (gate/up [2s, H], down [H, s])."""
    w_gu, w_d = deq_w
    inter = w_gu.shape[0] // 2
    if inter % world:
        raise ValueError("the intermediate size must split evenly over the ranks")
    s = inter // world
    lo, hi = rank * s, (rank + 1) * s
    return np.concatenate([w_gu[lo:hi], w_gu[inter + lo:inter + hi]]), w_d[:, lo:hi]


def moe_forward_tp(x, residual, router_w, gamma, experts: ExpertCache, top_k, alpha_a1, alpha_a2, world: int,
                   eps=1e-6):
    """The layer with its experts split over `world` tensor-parallel ranks ([PR] "Status": the
    TP all-reduce fused with the sandwich norms and the MoE finalize).  Every rank routes
    the same tokens and quantises the same A1; rank r runs its shard of every expert and
    forms its partial m_r = sum_j w_j y_r; the all-reduce gives m = sum_r m_r (ranks in
    order), then the post-RMSNorm and the residual add as in finalize.  The activation
    quantisation blocks (16 or 32 values along I) never straddle a shard boundary when
    I / world is a multiple of them, so each rank's A2 is the matching slice of the
    unsharded A2.  Returns dict(ids, w, m_parts [world, T, H], m, out_pre, out)."""
    x = np.asarray(x, np.float64)
    t_count, hidden = x.shape
    logits = router_logits(x, router_w)
    ids, w, _ = route_topk(logits, top_k)
    fmt = experts.fmt
    a1_packed, a1_sf = quantize_act(x.astype(np.float32), alpha_a1, fmt)
    m_parts = np.zeros((world, t_count, hidden), np.float64)
    for r in range(world):
        y = np.zeros((t_count, top_k, hidden), np.float64)
        for e in np.unique(ids):
            tt, jj = np.nonzero(ids == e)
            shard = shard_dequantized(experts.dequantized(int(e)), r, world)
            y[tt, jj] = expert_forward(a1_packed[tt], a1_sf[tt], alpha_a1, shard, alpha_a2, fmt)["y"]
        m_parts[r] = np.einsum("tk,tkh->th", w, y)
    m = np.zeros((t_count, hidden), np.float64)
    for r in range(world):
        m = m + m_parts[r]
    rms = np.sqrt(np.mean(m * m, axis=1, keepdims=True) + eps)
    out_pre = np.asarray(residual, np.float64) + m / rms * np.asarray(gamma, np.float64)[None, :]
    return dict(ids=ids, w=w, near_tie=near_tie_mask(logits, top_k), m_parts=m_parts, m=m, out_pre=out_pre,
                out=bf16_round(out_pre))


# ----------------------------------------------------------------------------- expert parallel
def moe_forward_ep(x_ranks, residual_ranks, router_w, gamma, experts: ExpertCache, num_experts, top_k, alpha_a1,
                   alpha_a2, world: int, eps=1e-6):
    """The layer with its experts split over `world` expert-parallel ranks, each with its own
    batch (attention data parallelism: [PR] "Status", Attention DP + MegaMoE; [RECIPE]
    "Overview": 8 of 256 experts).  Rank q holds experts [q E/W, (q+1) E/W).  In order:
      1. every rank routes its own tokens (steps 1-4) and quantises each of them once (step 6);
      2. dispatch: the quantised row of slot (t, j) of rank s goes to the rank that holds
         expert ids_s[t, j]; rank q's rows of expert e are ordered by (source rank, token);
      3. every rank runs its experts on the rows it received (steps 7-10);
      4. combine: each output row y goes back to its source rank, into slot (t, j);
      5. every rank finalizes its own tokens from the returned rows (steps 11-13).
    Only routed rows travel: no rank routes or quantises another rank's tokens.  Returns dict
    with, per rank: ids, w, near_tie, y (returned rows [T, k, H]), m, out_pre, out; and
    counts [world][E] (rows each rank sends to each expert) and received [world] (rows
    each rank computes)."""
    if num_experts % world or len(x_ranks) != world:
        raise ValueError("one batch per rank, and the experts must split evenly over the ranks")
    fmt = experts.fmt
    e_loc = num_experts // world
    routed = []
    for xs in x_ranks:  # step 1 on every rank, its own tokens only
        xs = np.asarray(xs, np.float64)
        logits = router_logits(xs, router_w)
        ids, w, _ = route_topk(logits, top_k)
        a1p, a1s = quantize_act(xs.astype(np.float32), alpha_a1, fmt)
        routed.append(dict(ids=ids, w=w, near_tie=near_tie_mask(logits, top_k), a1p=a1p, a1s=a1s,
                           y=np.zeros((xs.shape[0], top_k, xs.shape[1]), np.float64)))
    counts = np.array([np.bincount(r["ids"].reshape(-1), minlength=num_experts) for r in routed], np.int64)
    received = np.zeros(world, np.int64)
    for q in range(world):  # steps 2-4: rank q computes the rows of its experts
        for e in range(q * e_loc, (q + 1) * e_loc):
            src, tok, slot = [], [], []
            for sr, r in enumerate(routed):  # rows ordered by (source rank, token)
                tt, jj = np.nonzero(r["ids"] == e)
                src += [sr] * len(tt)
                tok += list(tt)
                slot += list(jj)
            if not src:
                continue
            a1p = np.concatenate([routed[sr]["a1p"][t][None] for sr, t in zip(src, tok)])
            a1s = np.concatenate([routed[sr]["a1s"][t][None] for sr, t in zip(src, tok)])
            y = expert_forward(a1p, a1s, alpha_a1, experts.dequantized(e), alpha_a2, fmt)["y"]
            received[q] += len(src)
            for i, (sr, t, j) in enumerate(zip(src, tok, slot)):
                routed[sr]["y"][t, j] = y[i]
    ranks = []
    for r, res in zip(routed, residual_ranks):  # step 5 on every rank
        pre, out, m = finalize(r["y"], r["w"], res, gamma, eps)
        ranks.append(dict(ids=r["ids"], w=r["w"], near_tie=r["near_tie"], y=r["y"], m=m, out_pre=pre, out=out))
    return dict(ranks=ranks, counts=counts, received=received, out_pre=[q["out_pre"] for q in ranks],
                out=[q["out"] for q in ranks], near_tie=np.concatenate([q["near_tie"] for q in ranks]))
