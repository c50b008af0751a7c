"""Plain CPU oracle of the MoE expert-parallel token shuffle: route -> dispatch -> SwiGLU FFN -> combine.

TEST INFRASTRUCTURE ONLY.  Nothing under ``oracle/`` is part of the product path: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``
may import it.  It shares no code with the CUDA library and never takes inputs from it.

Sources (web pages on expert-parallel MoE communication):

* "大模型MoE稀疏激活原理与硬件适配实战" (MoE sparse activation and hardware fit), section 3.2
  (fine ranking: sort the router logits, take the top experts), section 4.1 (the heat map's diagonal
  is zero: one token's experts are distinct), section 5.3 scenario 3 (the router runs in FP32),
  section 2.3 (mean expert load (B*S*K)/E, per-expert capacity).
* The ThunderEP page, section 2.1, redundancy 1 (pack every token bound for one destination into
  one contiguous buffer on the sender) and section 2.2 (each rank keeps only its own slice of the
  routing table).
* "NCCL EP架构解析" (NCCL EP architecture), section 2.1 (expert-major layout for the expert compute;
  FP8 payload with a scale tensor; the combine weights expert outputs by the token's routing
  weights, looping over the top-k slots), section 2.2 (high-throughput layout: one packed
  [sum T x H] buffer), section 5.1 (INVALID_TOPK when a routing index is out of range).
* "细粒度专家并行方案对比：MegaMoE与传统方案" (MegaMoE vs non-fused expert parallelism), section
  "核心差异分析 1" (two linear layers with a SwiGLU activation per expert), and
  "DWDP: 在NVL72上的高性能分布式权重数据并行", the ``NvFp4WeightView`` / ``run_moe`` passage
  (fused ``w3_w1`` first projection with SwiGLU, ``w2`` second projection, finalize = weighted
  scatter back to token order).

Readings where the pages are silent (each is listed with its reason in the design notes):
selection is on fp32 logits, ties to the lower expert id, slots ordered by descending logit; NaN
ranks below -inf; weights are the softmax over the selected k (``renormalize``) or the full-E
softmax; h = silu(x W_gate^T) * (x W_up^T) rounded to bf16, y = h W_down^T rounded to bf16; rows of
one expert are in ascending token order and overflow past the capacity is dropped in token order;
capacity C = ceil(cf * T * k / E); FP8 scale = amax / 448 per 128-element block (1 when amax = 0),
q = e4m3 round-to-nearest-even, saturating, of x / scale in fp32.

Precision: fp64 for the router weights and the FFN, as the pages fix neither.  The FP8 scale and
quotient are taken in fp32 (IEEE division), because they decide the quantised codes and the GPU
takes that decision in fp32.  The combine accumulates in fp32 in the fixed slot order, because the
pages' combine loop is written in float.
"""
from __future__ import annotations

import math

import numpy as np

from .numerics import bf16_bits, bf16_from_bits, bf16_round, e4m3_decode, e4m3_encode_satfinite

__all__ = ["capacity", "route", "dispatch_plan", "dispatch_payload", "expert_ffn", "combine",
           "pipeline", "QBLOCK", "quantize_rows_fp8", "dequantize_rows_fp8", "expert_ffn_w8",
           "ep_segment_rows", "ep_regroup", "ep_pipeline", "backward", "combine_backward",
           "router_backward", "expert_backward"]

QBLOCK = 128   # elements per FP8 scale block
E4M3_MAX_F32 = np.float32(448.0)


def capacity(cf: float, T: int, k: int, E: int) -> int:
    """Per-expert capacity ceil(cf * T * k / E); 0 means no limit (cf == 0).

    Mean load per expert is T*k/E (MoE sparse activation page, section 2.3: (B*S*K)/E, printed
    example 32*2048*2/128 = 1024)."""
    if cf <= 0:
        return 0
    return int(math.ceil(cf * (T * k) / E))


def _as_f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def route(logits, k: int, renormalize: bool = True):
    """Top-k selection and routing weights per token.

    For each token the experts are sorted by (logit descending, expert id ascending), NaN after
    every number (including -inf); the first k are the token's experts, in that order.  Weights are
    the softmax of the selected logits (``renormalize``) or their full softmax over all E experts,
    computed in fp64 and stored as fp32.  Limits of the softmax define the non-finite cases: NaN
    counts as -inf; if any +inf is present the +inf entries share the mass equally; if every entry
    of the denominator is -inf the mass is shared equally among them.

    Returns ``(topk_idx int32 [T,k], topk_w fp32 [T,k], expert_routed int32 [E])``.
    """
    l = _as_f32(logits)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    nan = np.isnan(l)
    neg = np.where(nan, 0.0, -l.astype(np.float64))
    ids = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((ids, neg, nan), axis=-1)        # primary: NaN last; then logit desc; then id
    idx = order[:, :k].astype(np.int32)

    lv = np.where(nan, -np.inf, l.astype(np.float64))    # NaN counts as -inf in the weights
    sel = np.take_along_axis(lv, idx.astype(np.int64), axis=1)
    den_src = sel if renormalize else lv
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        s, d = sel[t], den_src[t]
        n_pinf = np.count_nonzero(d == np.inf)
        if n_pinf:
            w[t] = np.where(s == np.inf, 1.0 / n_pinf, 0.0)
        elif np.all(d == -np.inf):
            w[t] = 1.0 / d.size
        else:
            m = np.max(d)
            w[t] = np.exp(s - m) / np.sum(np.exp(d - m))
    routed = np.bincount(idx.ravel(), minlength=E).astype(np.int32)
    return idx, w.astype(np.float32), routed


def dispatch_plan(topk_idx, E: int, R: int, cap: int = 0):
    """Positions of every routed slot in the packed expert-major send buffer.

    Walking the slots in token order, a slot's position inside its expert is the number of earlier
    slots routed to the same expert.  A slot is kept when there is no capacity (``cap == 0``) or its
    position is below ``cap``; kept slots of expert e occupy rows
    ``expert_offsets[e] .. expert_offsets[e+1]`` in ascending token order, experts in ascending id.
    Rank r owns experts [r*E/R, (r+1)*E/R), so the buffer is also rank-major and
    ``rank_offsets[r] = expert_offsets[r*E/R]``.

    Returns a dict with int32 arrays ``expert_routed`` [E], ``expert_counts`` (kept) [E],
    ``expert_offsets`` [E+1], ``rank_offsets`` [R+1], ``slot_row`` [T,k] (-1 = dropped),
    ``row_token`` [S] and the kept total ``S``.
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    T, k = idx.shape
    if E % R:
        raise ValueError("E must be a multiple of R")
    if idx.size and (idx.min() < 0 or idx.max() >= E):
        raise ValueError("routing index out of range")
    pos = np.empty((T, k), dtype=np.int64)
    running = [0] * E
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            pos[t, j] = running[e]
            running[e] += 1
    routed = np.array(running, dtype=np.int64)
    kept = np.minimum(routed, cap) if cap > 0 else routed
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    S = int(offsets[E])
    slot_row = np.full((T, k), -1, dtype=np.int64)
    row_token = np.empty(S, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if cap == 0 or pos[t, j] < cap:
                row = int(offsets[e] + pos[t, j])
                slot_row[t, j] = row
                row_token[row] = t
    per_rank = E // R
    rank_offsets = offsets[::per_rank][: R + 1]
    return {
        "expert_routed": routed.astype(np.int32),
        "expert_counts": kept.astype(np.int32),
        "expert_offsets": offsets.astype(np.int32),
        "rank_offsets": rank_offsets.astype(np.int32),
        "slot_row": slot_row.astype(np.int32),
        "row_token": row_token.astype(np.int32),
        "S": S,
    }


def quantize_row_fp8(x_row_f32: np.ndarray):
    """One token row -> (e4m3 codes [H], fp32 scales [H/128]).

    Per 128-element block: amax = max |x| (exact in fp32); scale = amax / 448 in fp32 (1 when
    amax = 0); code = e4m3 round-to-nearest-even, saturating, of the fp32 quotient x / scale."""
    x = x_row_f32.astype(np.float32).reshape(-1, QBLOCK)
    amax = np.max(np.abs(x), axis=1)
    scale = np.where(amax == 0, np.float32(1.0), amax / np.float32(E4M3_MAX_F32)).astype(np.float32)
    q = (x / scale[:, None]).astype(np.float32)            # fp32 IEEE division
    return e4m3_encode_satfinite(q).reshape(-1), scale



def dispatch_payload(x_bf16_bits, plan, fp8: bool = False):
    """Packed send buffer: ``send[row] = payload(x[row_token[row]])`` for every kept row.

    bf16 payload: the token's bytes.  FP8 payload: per-block e4m3 codes plus one fp32 scale per
    128-element block.  Returns ``(send, send_scales or None)`` with S rows."""
    xb = np.asarray(x_bf16_bits, dtype=np.uint16)
    T, H = xb.shape
    rt = plan["row_token"]
    S = plan["S"]
    if not fp8:
        return xb[rt].copy(), None
    if H % QBLOCK:
        raise ValueError("FP8 payload needs H % 128 == 0")
    xf = bf16_from_bits(xb)
    codes = np.empty((T, H), dtype=np.uint8)
    scales = np.empty((T, H // QBLOCK), dtype=np.float32)
    for t in range(T):
        codes[t], scales[t] = quantize_row_fp8(xf[t])
    return codes[rt].copy(), scales[rt].copy()


def dequantize_fp8_rows(codes, scales) -> np.ndarray:
    """bf16 values (as float64) of the FFN input rows of an FP8 payload: bf16(fp32(q) * scale)."""
    q = e4m3_decode(codes).astype(np.float32)
    s = np.repeat(np.asarray(scales, dtype=np.float32), QBLOCK, axis=1)
    prod = (q * s).astype(np.float32)                       # one fp32 product per element
    return bf16_round(prod)


def expert_ffn(send_rows_f64: np.ndarray, expert_offsets, w_gate_bits, w_up_bits, w_down_bits,
               rows=None):
    """Grouped SwiGLU FFN on the packed rows, expert by expert.

    For expert e and each of its rows x: g = x W_gate[e]^T, u = x W_up[e]^T (fp64 accumulate),
    h = bf16(g * sigmoid(g) * u), y = bf16(h W_down[e]^T) (fp64 accumulate).

    ``send_rows_f64`` holds the FFN input values (bf16 values as float64) of every packed row.
    ``rows`` optionally restricts the computation to those packed row indices (the other output
    rows are left as NaN).  Returns (h, y) as bf16 bit patterns; h has F columns, y has H.
    """
    off = np.asarray(expert_offsets, dtype=np.int64)
    E = off.size - 1
    S = int(off[E])
    H = w_gate_bits.shape[2]
    F = w_gate_bits.shape[1]
    want = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    h_out = np.full((S, F), 0x7FC0, dtype=np.uint16)
    y_out = np.full((S, H), 0x7FC0, dtype=np.uint16)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        r = want[(want >= lo) & (want < hi)]
        if r.size == 0:
            continue
        x = np.asarray(send_rows_f64[r], dtype=np.float64)
        wg = bf16_from_bits(w_gate_bits[e]).astype(np.float64)
        wu = bf16_from_bits(w_up_bits[e]).astype(np.float64)
        g = x @ wg.T
        u = x @ wu.T
        del wg, wu
        h = bf16_round(g / (1.0 + np.exp(-g)) * u)
        wd = bf16_from_bits(w_down_bits[e]).astype(np.float64)
        y = h @ wd.T
        h_out[r] = bf16_bits(h)
        y_out[r] = bf16_bits(y)
    return h_out, y_out


def quantize_rows_fp8(values):
    """Rows -> (e4m3 codes, one fp32 scale per row): scale = amax / 448 of the row's fp32 values
    (1 when amax = 0), code = e4m3 round-to-nearest-even, saturating, of the fp32 quotient
    value / scale.  The per-block quantiser of the FP8 payload, with the whole row as the block
    (used for FP8 expert weights, one scale per output row, and for the FFN's own FP8 input rows).

    ``values``: float array [rows, K] whose entries are fp32 values (e.g. bf16 values)."""
    x = np.asarray(values, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], dtype=np.float32)
    scale = np.where(amax == 0, np.float32(1.0), amax / np.float32(E4M3_MAX_F32)).astype(np.float32)
    q = (x / scale[:, None]).astype(np.float32)            # fp32 IEEE division
    return e4m3_encode_satfinite(q), scale


def dequantize_rows_fp8(codes, scales) -> np.ndarray:
    """Exact values (float64) of e4m3 codes times their row's fp32 scale."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[..., None]


def expert_ffn_w8(send_rows_f64: np.ndarray, expert_offsets, wg_codes, wg_scales, wu_codes,
                  wu_scales, w_down_bits, rows=None):
    """Grouped SwiGLU FFN with FP8 gate / up weights (W8A8 first projection).

    Per packed row x (its FFN input values, as for ``expert_ffn``): the row is quantised on its own,
    (qx, sx) = quantize_rows_fp8(x); the gate and up weights are e4m3 codes with one fp32 scale per
    output row.  For expert e: g = sx * sg[f] * sum_h qx[h] qg[f, h] (exact values, fp64), the same
    for u; h = bf16(g * sigmoid(g) * u); y = bf16(h W_down[e]^T) with bf16 down weights (fp64
    accumulate).  Returns (h, y) as bf16 bit patterns like ``expert_ffn``."""
    off = np.asarray(expert_offsets, dtype=np.int64)
    E = off.size - 1
    S = int(off[E])
    F, H = wg_codes.shape[1], wg_codes.shape[2]
    want = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    h_out = np.full((S, F), 0x7FC0, dtype=np.uint16)
    y_out = np.full((S, H), 0x7FC0, dtype=np.uint16)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        r = want[(want >= lo) & (want < hi)]
        if r.size == 0:
            continue
        qx, sx = quantize_rows_fp8(np.asarray(send_rows_f64[r], dtype=np.float64))
        xq = dequantize_rows_fp8(qx, sx)
        g = xq @ dequantize_rows_fp8(wg_codes[e], wg_scales[e]).T
        u = xq @ dequantize_rows_fp8(wu_codes[e], wu_scales[e]).T
        h = bf16_round(g / (1.0 + np.exp(-g)) * u)
        wd = bf16_from_bits(w_down_bits[e]).astype(np.float64)
        y = h @ wd.T
        h_out[r] = bf16_bits(h)
        y_out[r] = bf16_bits(y)
    return h_out, y_out


def combine(expert_out_bits, slot_row, topk_w, T: int, H: int):
    """y[t] = bf16( sum over j in 0..k-1 with slot_row[t,j] >= 0 of w[t,j] * expert_out[row] ).

    The sum is taken in fp32 in slot order j = 0, 1, ..., starting from 0, with each product and
    each addition rounded to fp32 separately.  A token whose slots were all dropped gives 0.
    Returns bf16 bit patterns [T,H]."""
    eo = bf16_from_bits(np.asarray(expert_out_bits, dtype=np.uint16))
    sr = np.asarray(slot_row, dtype=np.int64)
    w = _as_f32(topk_w)
    k = sr.shape[1]
    acc = np.zeros((T, H), dtype=np.float32)
    for j in range(k):
        rows = sr[:, j]
        valid = rows >= 0
        prod = (w[valid, j][:, None] * eo[rows[valid]]).astype(np.float32)
        acc[valid] = (acc[valid] + prod).astype(np.float32)
    return bf16_bits(acc)


def ffn_inputs(send, send_scales, fp8: bool) -> np.ndarray:
    """FFN input values (float64) of the packed rows: the bf16 rows, or the dequantised FP8 rows."""
    if fp8:
        return dequantize_fp8_rows(send, send_scales)
    return bf16_from_bits(send).astype(np.float64)


def pipeline(logits, x_bf16_bits, w_gate_bits, w_up_bits, w_down_bits, k: int, R: int,
             cf: float = 0.0, fp8: bool = False, renormalize: bool = True, ffn_rows=None):
    """The whole path on the CPU.  Returns every intermediate as a dict."""
    T, E = np.asarray(logits).shape
    H = np.asarray(x_bf16_bits).shape[1]
    idx, w, routed = route(logits, k, renormalize)
    cap = capacity(cf, T, k, E)
    plan = dispatch_plan(idx, E, R, cap)
    send, scales = dispatch_payload(x_bf16_bits, plan, fp8)
    xin = ffn_inputs(send, scales, fp8)
    h, y_e = expert_ffn(xin, plan["expert_offsets"], w_gate_bits, w_up_bits, w_down_bits, ffn_rows)
    out = dict(plan)
    out.update(topk_idx=idx, topk_w=w, routed=routed, cap=cap, send=send, send_scales=scales,
               h=h, expert_out=y_e)
    if ffn_rows is None:
        out["y"] = combine(y_e, plan["slot_row"], w, T, H)
    return out


# ---- expert parallelism across ranks ------------------------------------------------------------

def ep_segment_rows(counts, order: int, stride: int):
    """Row position of every row of a segmented layout: {(a, b, q): row}.

    ``counts`` [A, B]: segment (a, b) holds counts[a][b] rows.  Order 0 (a-major): for a = 0..A-1,
    for b = 0..B-1, the segment's rows in turn; block a (all of its b) starts at row a*stride, or
    right after block a-1 when stride is 0.  Order 1 (b-major): the same with the roles of a and b
    swapped (for b, for a).  This is the layout of a sender's per-destination blocks (the ThunderEP
    page, section 2.1: one contiguous block per destination, expert-major inside) and of a
    receiver's per-source blocks (the NCCL EP page, section 2.2: packed blocks in the high-throughput
    mode, fixed-size per-peer blocks in the low-latency mode)."""
    c = np.asarray(counts, dtype=np.int64)
    A, B = c.shape
    pos = {}
    outer, inner = (A, B) if order == 0 else (B, A)
    row = 0
    for o in range(outer):
        if stride > 0:
            row = o * stride
        for i in range(inner):
            a, b = (o, i) if order == 0 else (i, o)
            for q in range(int(c[a, b])):
                pos[(a, b, q)] = row
                row += 1
    return pos


def ep_regroup(counts, src, src_order: int, src_stride: int, dst, dst_order: int,
               dst_stride: int):
    """Move every row of every segment from its position in the source layout to its position in
    the destination layout (``ep_segment_rows``); other rows of ``dst`` are left as they are.
    Returns ``dst`` and the packed b-major start of every b (the total at [B])."""
    c = np.asarray(counts, dtype=np.int64)
    ps = ep_segment_rows(c, src_order, src_stride)
    pd = ep_segment_rows(c, dst_order, dst_stride)
    for key, r in ps.items():
        dst[pd[key]] = src[r]
    col = c.sum(axis=0)
    offsets = np.zeros(c.shape[1] + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(col)
    return dst, offsets


def ep_pipeline(logits_ranks, x_ranks, w_gate_bits, w_up_bits, w_down_bits, k: int,
                fp8: bool = False, renormalize: bool = True):
    """The path with expert parallelism over R = len(logits_ranks) ranks, each with its own tokens.

    Rank r owns experts [r*E/R, (r+1)*E/R).  Every rank routes its own tokens and packs its send
    buffer for R destinations (``dispatch_plan`` with R); destination d receives, from every source
    s in rank order, the rows of block d of s, expert-major over d's experts (the NCCL EP page,
    sections 1 and 2: a dispatch exchange to the experts' owners); it regroups them expert-major and
    runs the grouped FFN over its own experts; each output row goes back to the slot of its sender
    that it came from (the combine exchange), and every rank combines its own tokens.
    Returns the list of per-rank outputs y (bf16 bit patterns [T_r, H])."""
    R = len(logits_ranks)
    E = np.asarray(logits_ranks[0]).shape[1]
    E_loc = E // R
    per = []
    for r in range(R):
        idx, w, _ = route(logits_ranks[r], k, renormalize)
        plan = dispatch_plan(idx, E, R, 0)
        send, scales = dispatch_payload(x_ranks[r], plan, fp8)
        per.append((idx, w, plan, send, scales))
    H = per[0][3].shape[1]
    back = [np.zeros((p[2]["S"], H), dtype=np.uint16) for p in per]
    for d in range(R):
        # counts[s][e]: rows source s sends to local expert e of rank d
        counts = np.array([p[2]["expert_counts"][d * E_loc:(d + 1) * E_loc] for p in per])
        blocks = [p[3][p[2]["rank_offsets"][d]:p[2]["rank_offsets"][d + 1]] for p in per]
        recv = np.concatenate(blocks, axis=0)
        grouped, off = ep_regroup(counts, recv, 0, 0, np.zeros_like(recv), 1, 0)
        if fp8:
            sblocks = [p[4][p[2]["rank_offsets"][d]:p[2]["rank_offsets"][d + 1]] for p in per]
            rs = np.concatenate(sblocks, axis=0)
            gs, _ = ep_regroup(counts, rs, 0, 0, np.zeros_like(rs), 1, 0)
        else:
            gs = None
        xin = ffn_inputs(grouped, gs, fp8)
        _, y_e = expert_ffn(xin, off, w_gate_bits[d * E_loc:(d + 1) * E_loc],
                            w_up_bits[d * E_loc:(d + 1) * E_loc],
                            w_down_bits[d * E_loc:(d + 1) * E_loc])
        ret, _ = ep_regroup(counts, y_e, 1, 0, np.zeros_like(y_e), 0, 0)
        # source s's rows sit at [sum of earlier sources' block sizes, ...) of ret
        base = 0
        for s, p in enumerate(per):
            n = int(counts[s].sum())
            lo = p[2]["rank_offsets"][d]
            back[s][lo:lo + n] = ret[base:base + n]
            base += n
    out = []
    for r, (idx, w, plan, _, _) in enumerate(per):
        out.append(combine(back[r], plan["slot_row"], w, idx.shape[0], H))
    return out


# ---- backward ------------------------------------------------------------------------------------

def combine_backward(dy_bits, slot_row, topk_w, expert_out_f64, S: int, exact: bool = False):
    """Step 1 of the backward (the gradient of the combine), for every kept slot (t, j) -> row:
    d_eo[row] = bf16(fp32(w[t,j] * dy[t])) (the bf16 rounding of y taken as the identity) and
    d_w[t,j] = sum_h dy[t,h] eo[row,h] (exact); a dropped slot has d_w = 0.  ``expert_out_f64`` holds
    the expert outputs' values [S,H].  ``exact`` keeps d_eo in fp64.  Returns (d_eo float64 [S,H],
    d_w float64 [T,k])."""
    sr = np.asarray(slot_row, dtype=np.int64)
    w = np.asarray(topk_w, dtype=np.float32)
    dy = bf16_from_bits(np.asarray(dy_bits, dtype=np.uint16)).astype(np.float64)
    T, k = sr.shape
    H = dy.shape[1]
    d_eo = np.zeros((S, H), dtype=np.float64)
    d_w = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            row = sr[t, j]
            if row < 0:
                continue
            prod = dy[t] * float(w[t, j])
            d_eo[row] = prod if exact else prod.astype(np.float32)
            d_w[t, j] = float(np.dot(dy[t], expert_out_f64[row]))
    return (d_eo if exact else bf16_round(d_eo)), d_w


def router_backward(logits, topk_idx, topk_w, d_w, renormalize: bool = True):
    """Step 4: the router's logit gradient from the routing-weight gradient.  With ``renormalize``
    the weights are the softmax of the selected logits, so for a selected expert i of token t
    d_logits[t,i] = w_i (d_w_i - sum_j w_j d_w_j), 0 elsewhere; otherwise they are the full-E
    softmax p, and d_logits[t,i] = p_i (d_i - sum_e p_e d_e) with d_i = d_w of the slot that
    selected i (0 for unselected experts).  fp64 [T,E]."""
    L = np.asarray(logits, dtype=np.float64)
    idx = np.asarray(topk_idx, dtype=np.int64)
    w = np.asarray(topk_w, dtype=np.float32)
    T, k = idx.shape
    d_logits = np.zeros_like(L)
    for t in range(T):
        if renormalize:
            wt = w[t].astype(np.float64)
            c = float(np.dot(wt, d_w[t]))
            for j in range(k):
                d_logits[t, idx[t, j]] = wt[j] * (d_w[t, j] - c)
        else:
            p = np.exp(L[t] - L[t].max())
            p /= p.sum()
            d = np.zeros(L.shape[1])
            for j in range(k):
                d[idx[t, j]] = d_w[t, j]
            d_logits[t] = p * (d - float(np.dot(p, d)))
    return d_logits


def expert_backward(xin, d_eo, expert_offsets, w_gate_bits, w_up_bits, w_down_bits,
                    exact: bool = False):
    """Step 2: the experts' backward on their packed rows, x = the FFN input values (as in the
    forward) and d_eo = the output gradient of the rows (float64 [S,H]).  For expert e:
    g = x Wg^T, u = x Wu^T, s = sigmoid(g), h = bf16(g s u) (recomputed as the forward made it),
    dh = d_eo Wd, dg = bf16(dh u s (1 + g (1 - s))), du = bf16(dh g s),
    dx_rows = bf16(dg Wg + du Wu), dWd = d_eo^T h, dWg = dg^T x, dWu = du^T x (fp64 sums).
    ``exact`` skips the bf16 roundings.  Returns a dict of float64 arrays dg, du [S,F], dx_rows
    [S,H], d_w_gate, d_w_up [E,F,H], d_w_down [E,H,F]."""
    rnd = (lambda a: np.asarray(a, dtype=np.float64)) if exact else bf16_round
    off = np.asarray(expert_offsets, dtype=np.int64)
    E = off.size - 1
    S = int(off[E])
    H = w_gate_bits.shape[2]
    F = w_gate_bits.shape[1]
    dg_all = np.zeros((S, F))
    du_all = np.zeros((S, F))
    dxr = np.zeros((S, H))
    dWg = np.zeros((E, F, H))
    dWu = np.zeros((E, F, H))
    dWd = np.zeros((E, H, F))
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        x = np.asarray(xin[lo:hi], dtype=np.float64)
        wg = bf16_from_bits(w_gate_bits[e]).astype(np.float64)
        wu = bf16_from_bits(w_up_bits[e]).astype(np.float64)
        wd = bf16_from_bits(w_down_bits[e]).astype(np.float64)
        g = x @ wg.T
        u = x @ wu.T
        sg = 1.0 / (1.0 + np.exp(-g))
        h = rnd(g * sg * u)
        de = d_eo[lo:hi]
        dh = de @ wd
        dg = rnd(dh * u * sg * (1.0 + g * (1.0 - sg)))
        du = rnd(dh * g * sg)
        dxr[lo:hi] = rnd(dg @ wg + du @ wu)
        dWd[e] = de.T @ h
        dWg[e] = dg.T @ x
        dWu[e] = du.T @ x
        dg_all[lo:hi] = dg
        du_all[lo:hi] = du
    return {"dg": dg_all, "du": du_all, "dx_rows": dxr, "d_w_gate": dWg, "d_w_up": dWu,
            "d_w_down": dWd}


def backward(fwd, dy_bits, logits, w_gate_bits, w_up_bits, w_down_bits, renormalize: bool = True,
             fp8: bool = False, exact: bool = False):
    """Gradients of the path for an output gradient dy [T,H] (bf16 bit patterns), given the forward
    intermediates ``fwd`` of ``pipeline`` (routing, plan, payload, expert outputs).

    The training step of the NCCL EP page (section 3.2) reuses the forward's routing: the gradient is
    dispatched through the same plan, the experts run backward, and the gradients are combined back.
    In that order: ``combine_backward`` (step 1), ``expert_backward`` (step 2), the combine of the
    input gradients dx[t] = bf16(sum over kept j of dx_rows[slot_row[t,j]]), fp32 in slot order (the
    forward combine with unit weights; step 3), and ``router_backward`` (step 4).

    ``exact`` skips every bf16 rounding and uses the expert outputs without their rounding (all
    fp64), for checks against finite differences.
    Returns a dict of dx (bf16 bits [T,H], or float64 when exact), d_logits fp32 [T,E], d_w fp32
    [T,k], d_w_gate / d_w_up fp32 [E,F,H], d_w_down fp32 [E,H,F], and the intermediates d_eo,
    dg, du, dx_rows (bf16 bits, or float64 when exact) in packed row order."""
    slot_row = np.asarray(fwd["slot_row"], dtype=np.int64)
    w = np.asarray(fwd["topk_w"], dtype=np.float32)
    off = np.asarray(fwd["expert_offsets"], dtype=np.int64)
    T, k = slot_row.shape
    E = off.size - 1
    S = int(off[E])
    H = np.asarray(dy_bits).shape[1]
    xin = ffn_inputs(fwd["send"], fwd["send_scales"], fp8)
    if exact:
        # the expert outputs without their bf16 roundings
        eo = np.zeros((S, H))
        for e in range(E):
            lo, hi = off[e], off[e + 1]
            if hi == lo:
                continue
            x = np.asarray(xin[lo:hi], dtype=np.float64)
            g = x @ bf16_from_bits(w_gate_bits[e]).astype(np.float64).T
            u = x @ bf16_from_bits(w_up_bits[e]).astype(np.float64).T
            eo[lo:hi] = (g / (1.0 + np.exp(-g)) * u) @ bf16_from_bits(w_down_bits[e]).astype(
                np.float64).T
    else:
        eo = bf16_from_bits(np.asarray(fwd["expert_out"], dtype=np.uint16)).astype(np.float64)
    d_eo, d_w = combine_backward(dy_bits, slot_row, w, eo, S, exact)
    ex = expert_backward(xin, d_eo, off, w_gate_bits, w_up_bits, w_down_bits, exact)
    dxr = ex["dx_rows"]
    if exact:
        dx = np.zeros((T, H))
        for t in range(T):
            for j in range(k):
                if slot_row[t, j] >= 0:
                    dx[t] += dxr[slot_row[t, j]]
    else:
        dx = combine(bf16_bits(dxr), slot_row, np.ones((T, k), dtype=np.float32), T, H)
    d_logits = router_backward(logits, fwd["topk_idx"], w, d_w, renormalize)
    out = {"dx": dx, "d_logits": d_logits.astype(np.float32),
           "d_w": d_w.astype(np.float32),
           "d_w_gate": ex["d_w_gate"] if exact else ex["d_w_gate"].astype(np.float32),
           "d_w_up": ex["d_w_up"] if exact else ex["d_w_up"].astype(np.float32),
           "d_w_down": ex["d_w_down"] if exact else ex["d_w_down"].astype(np.float32)}
    if exact:
        out.update(d_eo=d_eo, dg=ex["dg"], du=ex["du"], dx_rows=dxr, d_logits=d_logits, d_w=d_w)
    else:
        out.update(d_eo=bf16_bits(d_eo), dg=bf16_bits(ex["dg"]), du=bf16_bits(ex["du"]),
                   dx_rows=bf16_bits(dxr))
    return out
