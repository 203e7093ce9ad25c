"""CPU oracle for the DeepSeek-V3-style MoE layer forward pass (test infrastructure).

This is the plain, slow, obviously-correct statement of what the layer
computes, in float64 numpy. It exists only to check the CUDA library: only the
tests, the package's smoke check and the benchmark's CPU-baseline leg may import
it. It shares no code with the CUDA path and imports nothing from the package;
callers hand it plain numpy arrays.

Sources (the pages this follows):
  * "DeepSeek-V3.2-Exp - Expert scores" (router): the Gate constructor fields
    and the Gate.forward excerpt - fp32 logits x.W_r^T, softmax or sigmoid,
    a selection-only bias, group scores (top-2 sum with a bias, max without),
    the top-`topk_groups` groups, masking the rest to -inf, expert top-k,
    gathering the UNBIASED scores, renormalising them for sigmoid, and scaling
    by route_scale.
  * "DeepSeek-V3.2-Exp - Weighted expert sum" (combine): y_routed =
    sum_i G_i E_i, accumulated in float32 and cast back at the end; the
    MoE.forward excerpt (bincount of the indices, a loop over experts in
    ascending order, rows found in row-major order, y[rows] += E(x[rows]) *
    weight, then the shared expert added to every token).
  * hackaday "time to jump right in and swim with the big fish", MoE class:
    routed experts Expert(dim, moe_inter_dim) and one shared MLP of width
    n_shared_experts * moe_inter_dim.
  * The expert body is not on the pages; the layer's definition takes it as
    SwiGLU, E(x) = w2 (silu(w1 x) * (w3 x)), silu(u) = u / (1 + e^-u), no
    biases, weights stored [out, in] like the router weight.

Readings where the pages are silent:
  * ties in any top-k: the lower index wins; top-k output is ordered by
    descending score, then ascending index;
  * the accumulator is fp32 (the V3.2 page) and the shared expert is added
    before the single final cast;
  * the CUDA path rounds h = silu(a)*b to the activation dtype (it is the
    input of the w2 product) and each expert's and the shared MLP's output to
    the activation dtype (an expert returns the activation dtype, which is then
    scaled by the fp32 weight); `round_to` reproduces exactly those roundings
    from the fp64 values, and `round_to=None` skips them.

Pins: every function here is checked by tests/test_oracle_*.py against
brute-force enumeration, invariants, closed forms and library routines;
see those tests for the list.
"""

from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# Number formats


def to_f64(a) -> np.ndarray:
    """Exact widening of float32 / bfloat16 values to float64. A bfloat16
    array is accepted as its raw uint16 bit pattern (the top 16 bits of a
    float32)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits), ties
    to even, returned as float64. Written from the format: v = m * 2^e with
    0.5 <= |m| < 1, keep m to 1/256 with round-half-even."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def round_f32(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(v: np.ndarray, dtype) -> np.ndarray:
    if dtype is None:
        return np.asarray(v, dtype=np.float64)
    if dtype == "bf16":
        return round_bf16(v)
    if dtype == "f32":
        return round_f32(v)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# FP8 (e4m3) block-scaled numbers. The pages say only that the block's other
# linears are FP8 ("Expert scores", dtype note); the layout here is this
# library's: e4m3 values (1 sign, 4 exponent bits with bias 7, 3 mantissa
# bits, largest finite 448, subnormals down to 2^-9) with one power-of-two
# scale per block -- 128 x 128 for a weight matrix [out, in], 1 x 128 for a row
# of activations. A block's scale 2^s is the smallest with amax <= 448 * 2^s,
# and its values are q = e4m3(v / 2^s) rounded to nearest, ties to even.

E4M3_MAX = 448.0


def round_e4m3(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest e4m3 value, ties to even, returned
    as float64 (|v| <= 448 expected; larger magnitudes saturate to 448).
    Normal range: v = m * 2^e with 0.5 <= |m| < 1 keeps m to 1/16; below
    2^-6 the spacing is the subnormal step 2^-9."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    normal = np.ldexp(np.round(m * 16.0) / 16.0, e)
    sub = np.round(v * 512.0) / 512.0
    out = np.where(np.abs(v) < 2.0 ** -6, sub, normal)
    return np.clip(out, -E4M3_MAX, E4M3_MAX)


SCALE_EXP_MIN = -127   # the smallest power of two a UE8M0 scale byte encodes


def block_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer s >= SCALE_EXP_MIN with amax <= 448 * 2^s (0 for an
    all-zero block). The lower limit keeps every scale encodable as one UE8M0
    byte (2^-127 .. 2^127), the form the tensor core's block scaling reads; a
    block whose largest magnitude is below 448 * 2^-127 keeps 2^-127."""
    amax = np.asarray(amax, dtype=np.float64)
    m, e = np.frexp(np.where(amax > 0, amax, 1.0))   # amax = m 2^e, 0.5 <= m < 1
    # amax = (2m) 2^(e-1) and 448 = 1.75 * 2^8: s = e - 9, one more when 2m > 1.75
    s = np.maximum(e - 9 + (2.0 * m > 1.75), SCALE_EXP_MIN)
    return np.where(amax > 0, s, 0).astype(np.int64)


def quantize_blocks(a: np.ndarray, block_rows: int, block_cols: int):
    """Quantize a 2D array to e4m3 with one power-of-two scale per block
    (blocks of block_rows x block_cols, partial at the edges). Returns
    (q [R, C] float64 e4m3 values, scale [ceil(R/br), ceil(C/bc)] powers of two)."""
    a = to_f64(a)
    R, C = a.shape
    nr, nc = -(-R // block_rows), -(-C // block_cols)
    q = np.empty_like(a)
    scale = np.empty((nr, nc))
    for i in range(nr):
        for j in range(nc):
            blk = a[i * block_rows:(i + 1) * block_rows, j * block_cols:(j + 1) * block_cols]
            s = float(np.ldexp(1.0, int(block_exponent(np.abs(blk).max()))))
            scale[i, j] = s
            q[i * block_rows:(i + 1) * block_rows, j * block_cols:(j + 1) * block_cols] = \
                round_e4m3(blk / s)
    return q, scale


def dequantize_blocks(q: np.ndarray, scale: np.ndarray, block_rows: int, block_cols: int):
    """q * the scale of its block."""
    q = np.asarray(q, dtype=np.float64)
    full = np.repeat(np.repeat(np.asarray(scale, np.float64), block_rows, 0), block_cols, 1)
    return q * full[:q.shape[0], :q.shape[1]]


def fp8_act(a: np.ndarray) -> np.ndarray:
    """Activations as the FP8 experts see them: quantized per 1 x 128 block
    and dequantized."""
    q, s = quantize_blocks(a, 1, 128)
    return dequantize_blocks(q, s, 1, 128)


def swiglu_fp8(xr, w1, w3, w2, round_out=None) -> np.ndarray:
    """E(x) with FP8 block-scaled weights (given dequantized, [out, in]) and
    FP8 activations: x and h are each quantized per 1 x 128 block before
    their product; the products accumulate exactly (fp64 here); the output is
    rounded to `round_out`."""
    xq = fp8_act(xr)
    a = xq @ to_f64(w1).T
    c = xq @ to_f64(w3).T
    h = fp8_act(silu(a) * c)
    return round_to(np.matmul(h, to_f64(w2).T), round_out)


# --------------------------------------------------------------------------
# Step 1: router logits and scores ("Expert scores": z = x W_r, applied in
# float32 -- here float64, which is the exact value up to rounding)


def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """z[t, e] = sum_d x[t, d] * W_r[e, d]; W_r is stored [out, in]."""
    return to_f64(x) @ to_f64(w_router).T


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


def softmax(z: np.ndarray) -> np.ndarray:
    """softmax over experts (last axis), with the row max subtracted first."""
    m = z.max(axis=-1, keepdims=True)
    p = np.exp(z - m)
    return p / p.sum(axis=-1, keepdims=True)


def scores(z: np.ndarray, score_func: str) -> np.ndarray:
    if score_func == "softmax":
        return softmax(z)
    if score_func == "sigmoid":
        return sigmoid(z)
    raise ValueError(score_func)


# --------------------------------------------------------------------------
# Step 2: group-limited top-k routing ("Expert scores", Gate.forward)


def _order_desc(v: np.ndarray) -> np.ndarray:
    """Indices of the last axis sorted by descending value, ties broken by the
    lower index (a stable sort of -v). -inf sorts last."""
    return np.argsort(-v, axis=-1, kind="stable")


def route(z: np.ndarray, bias, *, n_groups: int, topk_groups: int, topk: int,
          score_func: str, route_scale: float) -> dict:
    """Route every token from its logits z [T, E].

    Returns a dict with
      weights [T, k] float64  - route_scale * unbiased scores at idx
                                 (renormalised over the k picks for sigmoid)
      idx     [T, k] int64    - chosen experts, descending biased score
      groups  [T, TG] int64   - kept groups (sorted ascending), or None if G == 1
      biased  [T, E] float64  - selection scores after masking (-inf outside)
      margin  [T] float64     - smallest gap that decided this token's routing
    """
    T, E = z.shape
    s = scores(z, score_func)                       # original (unbiased) scores
    b = s + np.asarray(bias, dtype=np.float64)[None, :] if bias is not None else s.copy()

    margin = np.full(T, np.inf)
    groups = None
    if n_groups > 1:
        per = E // n_groups
        blocks = b.reshape(T, n_groups, per)        # contiguous blocks of experts
        if bias is None:
            gscore = blocks.max(axis=-1)
        else:
            top2 = -np.sort(-blocks, axis=-1)[:, :, :2]
            gscore = top2.sum(axis=-1)
        gorder = _order_desc(gscore)
        keep = gorder[:, :topk_groups]
        groups = np.sort(keep, axis=-1)
        masked = np.full((T, n_groups), True)
        np.put_along_axis(masked, keep, False, axis=-1)
        b = np.where(np.repeat(masked, per, axis=-1), -np.inf, b)
        if topk_groups < n_groups:
            gs = np.take_along_axis(gscore, gorder, axis=-1)
            margin = np.minimum(margin, gs[:, topk_groups - 1] - gs[:, topk_groups])

    order = _order_desc(b)
    idx = order[:, :topk]
    # decisive gaps: between consecutive picks (their order) and between the
    # k-th pick and the best expert left out
    ranked = np.take_along_axis(b, order[:, :min(topk + 1, E)], axis=-1)
    gaps = ranked[:, :-1] - ranked[:, 1:]
    gaps = np.where(np.isnan(gaps), np.inf, gaps)  # -inf - -inf never decides
    if gaps.shape[1]:
        margin = np.minimum(margin, gaps.min(axis=-1))

    w = np.take_along_axis(s, idx, axis=-1)         # unbiased scores
    if score_func == "sigmoid":
        w = w / w.sum(axis=-1, keepdims=True)
    w = w * route_scale
    return dict(weights=w, idx=idx.astype(np.int64), groups=groups, biased=b, margin=margin)


# --------------------------------------------------------------------------
# Step 3: dispatch (the bincount and the per-expert row lists of MoE.forward)


def dispatch(idx: np.ndarray, n_experts: int) -> dict:
    """Expert-contiguous order of the (token, slot) pairs.

    counts[e]  = number of pairs routed to e (bincount, minlength E)
    offsets    = exclusive scan of counts, offsets[E] = T*k
    src[p]     = token of the p-th row of the expert-contiguous order
    pos[t, j]  = row p that holds pair (t, j)
    Within an expert, rows follow the row-major order of idx (ascending token),
    which is the order the rows of `where(indices == e)` come in.
    """
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    src = np.empty(T * k, dtype=np.int64)
    pos = np.empty(T * k, dtype=np.int64)
    fill = offsets[:-1].copy()
    for q in range(T * k):                         # row-major over (t, j)
        e = flat[q]
        p = fill[e]
        fill[e] += 1
        src[p] = q // k
        pos[q] = p
    return dict(counts=counts, offsets=offsets, src=src, pos=pos.reshape(T, k))


# --------------------------------------------------------------------------
# Step 4: the SwiGLU experts


def silu(u: np.ndarray) -> np.ndarray:
    return u / (1.0 + np.exp(-u))


def swiglu(xr: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray,
           round_h=None, round_out=None) -> np.ndarray:
    """E(x) = w2 (silu(w1 x) * (w3 x)) for rows xr [n, D]; w1, w3 [I, D] and
    w2 [D, I] in [out, in] layout. h and the output are rounded to `round_h` /
    `round_out` ("bf16", "f32" or None)."""
    xr = to_f64(xr)
    a = xr @ to_f64(w1).T
    c = xr @ to_f64(w3).T
    h = round_to(silu(a) * c, round_h)
    return round_to(h @ to_f64(w2).T, round_out)


# --------------------------------------------------------------------------
# Step 5: the weighted combine, and the whole layer


def moe_layer(x: np.ndarray, weights: np.ndarray, idx: np.ndarray, experts, shared,
              *, act_dtype=None, tokens=None, fp8=False) -> np.ndarray:
    """y[t] = sum_j weights[t, j] * E_{idx[t, j]}(x[t]) + S(x[t]).

    `experts(e)` returns (w1, w3, w2) of routed expert e; `shared` is
    (ws1, ws3, ws2) or None. Experts are visited in ascending order and each
    adds its weighted rows into an fp64 accumulator, then the shared MLP is
    added and the sum is rounded once to `act_dtype` (None keeps fp64).
    `tokens` restricts the computation to a subset of token rows (a token's
    output depends only on its own row); the result then has len(tokens) rows.
    With `fp8`, the expert weights are FP8 block-scaled (given dequantized)
    and every expert, the shared MLP included, runs as swiglu_fp8.
    """
    x = to_f64(x)
    T, D = x.shape
    rows = np.arange(T) if tokens is None else np.asarray(tokens)
    xs, ws, ids = x[rows], np.asarray(weights, np.float64)[rows], np.asarray(idx)[rows]
    y = np.zeros((len(rows), D))
    for e in np.unique(ids):
        r, j = np.nonzero(ids == e)                 # row-major, as where() gives
        w1, w3, w2 = experts(int(e))
        if fp8:
            out = swiglu_fp8(xs[r], w1, w3, w2, round_out=act_dtype)
        else:
            out = swiglu(xs[r], w1, w3, w2, round_h=act_dtype, round_out=act_dtype)
        y[r] += out * ws[r, j][:, None]
    if shared is not None:
        ws1, ws3, ws2 = shared
        if fp8:
            y += swiglu_fp8(xs, ws1, ws3, ws2, round_out=act_dtype)
        else:
            y += swiglu(xs, ws1, ws3, ws2, round_h=act_dtype, round_out=act_dtype)
    return round_to(y, act_dtype)


# --------------------------------------------------------------------------
# Expert parallelism (the MoE class on the hackaday page and DeepseekV3MoE on
# the thataiguy page: rank r of world_size holds the contiguous block of
# n_routed / world_size experts starting at r * n_routed / world_size; every
# rank routes all tokens, runs only its own experts, and the ranks' partial
# outputs are summed by one all_reduce of y. The V3.2 listing ("Weighted
# expert sum", MoE.forward) adds the shared MLP into y before that all_reduce,
# so each rank holds a slice of the shared MLP -- a block of its inner width
# -- whose outputs add up to the whole MLP.)


def expert_block(n_experts: int, world_size: int, rank: int) -> range:
    """Experts held by `rank`: a contiguous block of n_experts / world_size."""
    if n_experts % world_size:
        raise ValueError("n_routed_experts must divide by world_size")
    per = n_experts // world_size
    return range(rank * per, (rank + 1) * per)


def shared_block(shared_inter: int, world_size: int, rank: int) -> range:
    """Inner features of the shared MLP held by `rank` (a contiguous block)."""
    if shared_inter % world_size:
        raise ValueError("the shared MLP's width must divide by world_size")
    per = shared_inter // world_size
    return range(rank * per, (rank + 1) * per)


def moe_layer_partial(x: np.ndarray, weights: np.ndarray, idx: np.ndarray, experts, shared,
                      *, expert_range: range, shared_range: range, act_dtype=None,
                      tokens=None) -> np.ndarray:
    """One rank's contribution to y before the all_reduce, in fp64 (not
    rounded at the end): the weighted outputs of the experts in
    `expert_range` for the tokens routed to them, plus the shared MLP
    restricted to the inner features `shared_range` (rows of ws1 and ws3,
    columns of ws2). Each expert's output and the shared slice's output are
    rounded to `act_dtype` as in moe_layer."""
    x = to_f64(x)
    T, D = x.shape
    rows = np.arange(T) if tokens is None else np.asarray(tokens)
    xs, ws, ids = x[rows], np.asarray(weights, np.float64)[rows], np.asarray(idx)[rows]
    y = np.zeros((len(rows), D))
    for e in np.unique(ids):
        if int(e) not in expert_range:
            continue
        r, j = np.nonzero(ids == e)
        w1, w3, w2 = experts(int(e))
        out = swiglu(xs[r], w1, w3, w2, round_h=act_dtype, round_out=act_dtype)
        y[r] = y[r] + out * ws[r, j][:, None]
    if shared is not None and len(shared_range):
        ws1, ws3, ws2 = shared
        f = np.asarray(shared_range)
        y += swiglu(xs, np.asarray(ws1)[f], np.asarray(ws3)[f], np.asarray(ws2)[:, f],
                    round_h=act_dtype, round_out=act_dtype)
    return y


def moe_layer_ep(x, weights, idx, experts, shared, *, n_experts, world_size, act_dtype=None,
                 tokens=None) -> np.ndarray:
    """The layer over `world_size` expert-parallel ranks: every rank's
    partial output (its expert block and its slice of the shared MLP),
    summed as the all_reduce does, then rounded once to `act_dtype`."""
    Is = 0 if shared is None else np.asarray(shared[0]).shape[0]
    y = 0.0
    for r in range(world_size):
        y = y + moe_layer_partial(x, weights, idx, experts, shared,
                                  expert_range=expert_block(n_experts, world_size, r),
                                  shared_range=shared_block(Is, world_size, r) if Is else range(0),
                                  act_dtype=act_dtype, tokens=tokens)
    return round_to(y, act_dtype)


def moe_forward(x, w_router, bias, experts, shared, *, n_groups, topk_groups, topk,
                score_func, route_scale, act_dtype=None, tokens=None) -> dict:
    """The whole layer: route every token, then combine (for `tokens`)."""
    n_experts = np.asarray(w_router).shape[0]
    r = route(router_logits(x, w_router), bias, n_groups=n_groups, topk_groups=topk_groups,
              topk=topk, score_func=score_func, route_scale=route_scale)
    d = dispatch(r["idx"], n_experts)
    y = moe_layer(x, r["weights"], r["idx"], experts, shared, act_dtype=act_dtype, tokens=tokens)
    return dict(y=y, **r, **d)
