"""CPU oracle for the packed-sequence pre-norm encoder layer (numpy, float64).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module;
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code, table or helper with the CUDA
path: it is a plain, slow, direct restatement of what the layer computes,
written so that it can be checked against the pages by eye.

Sources (web pages, cited by title and section):
  * "Days-gone/cti2026" README -- TransformerEncoder section (per-layer
    pseudo-code: LayerNorm, Linear_qkv, FlashAttention_Varlen(qkv,
    user_offsets), residual + Linear_out, LayerNorm, Gate -> (topk_idx,
    topk_weight), FusedMoE, residual), the FlashAttention_Varlen operator
    design (segment boundaries from cu_seqlens, query i sees keys 0..i of its
    own user, online softmax in fp32), the SMoE structure (Gate Linear(512->8)
    then softmax -> top-2 -> renormalise; 8 experts Linear(512->1024) + ReLU
    + Linear(1024->512); each token weighted over its 2 experts), the fused
    MoE routing notes (per-expert counts, token reordering, route-major rows
    token_id*top_k + k_idx, per-token weighted sum) and the Prediction Head
    section (Linear(512->1) -> clamp(-15, 15) -> sigmoid, pred_mask select),
    and the RepEncoder section (28-slot embedding bag with sum pooling,
    LayerNorm over the 14336 concatenated values, Linear(14336->512)).
  * "CTI-Inference-Opt" optimisation plan -- attention as softmax(QK^T/sqrt(d))V.
  * "cry-daniel/recsys" README -- the HSTU attention mask logic (contextual,
    historical and candidate segments; mask types none, local, causal,
    context + causal, target + causal), for the masked-attention variants.
  * "CTI-Inference-Opt" AUC-recovery plan -- the dense block-diagonal causal
    mask built from user_offsets (same user AND lower triangle), the
    FlexAttention mask_mod restatement of it, and the vectorised SMoE that
    evaluates all experts for all tokens and then gathers the top-k.

Readings taken where the pages are silent:
  * every Linear has a bias; LayerNorm eps = 1e-5 with biased variance;
  * QKV columns split as [Q | K | V], head h = 64-column block h of each;
  * softmax scale 1/sqrt(64) = 0.125;
  * top-2 ties go to the lower expert index, slot 0 holds the larger weight;
  * renormalised weights w_k = p_k / (p_e0 + p_e1) with no epsilon;
  * route id r = 2 t + k; within an expert, routes are ordered by ascending r
    (a stable counting sort);
  * the head applies a final LayerNorm before Linear(512->1).

Parity status: every function below is pinned by tests/test_oracle_pins.py
(closed forms, library routines, brute force and invariants); the composed
random layer beyond those pins is checked only through its pinned parts.
"""
from __future__ import annotations

import numpy as np

LN_EPS = 1e-5
N_HEADS = 8
D_HEAD = 64
TOP_K = 2
LOGIT_CLAMP = 15.0


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def round_bf16(a):
    """Round to the nearest bfloat16 value (ties to even), returned as float64:
    keep the top 16 bits of the float32 encoding after adding half of the
    dropped part (0x7FFF plus the lowest kept bit, which breaks ties to even).
    Used only by the storage='bf16' mode below."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    keep = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return keep.astype(np.uint32).view(np.float32).astype(np.float64).reshape(f.shape)


def _storage(storage):
    """Rounding applied where the bf16 pipeline stores an activation: the
    identity for the exact fp64 oracle (storage=None), bfloat16 rounding for
    storage='bf16' (the cti2026 README runs inference in bf16 with fp32
    accumulation and fp32 softmax statistics, writing results back as bf16)."""
    if storage is None:
        return lambda a: _f64(a)
    if storage == "bf16":
        return round_bf16
    raise ValueError(storage)


# --------------------------------------------------------------------------
# LayerNorm and Linear (cti2026 README, TransformerEncoder section)
# --------------------------------------------------------------------------
def layer_norm(x, gamma, beta, eps=LN_EPS):
    """Per-row LayerNorm: (x - mean) / sqrt(biased var + eps) * gamma + beta."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * _f64(gamma) + _f64(beta)


def linear(x, weight, bias=None):
    """nn.Linear: y = x W^T + b with W stored [out, in]."""
    y = _f64(x) @ _f64(weight).T
    if bias is not None:
        y = y + _f64(bias)
    return y


def split_qkv(qkv):
    """[T, 3*H*Dh] -> q, k, v each [T, H, Dh]; columns are [Q | K | V] and
    head h owns columns h*Dh .. h*Dh+Dh-1 of each block."""
    qkv = _f64(qkv)
    T = qkv.shape[0]
    hd = qkv.shape[1] // 3
    H = hd // D_HEAD
    q = qkv[:, :hd].reshape(T, H, D_HEAD)
    k = qkv[:, hd:2 * hd].reshape(T, H, D_HEAD)
    v = qkv[:, 2 * hd:].reshape(T, H, D_HEAD)
    return q, k, v


# --------------------------------------------------------------------------
# Attention (cti2026 README, FlashAttention_Varlen operator design)
# --------------------------------------------------------------------------
def _softmax_rows(s):
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=-1, keepdims=True)


def jagged_causal_attention(q, k, v, cu_seqlens, scale=None):
    """Block-diagonal causal attention over a packed stream.

    q, k, v: [T, H, Dh].  For user u (tokens cu[u] .. cu[u+1]-1) and head h,
    S = Q_u K_u^T * scale with S[i, j] = -inf for j > i, P = row softmax(S),
    O_u = P V_u.  Tokens of other users are never seen.  Returns [T, H, Dh].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, Dh = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(Dh)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    out = np.zeros_like(q)
    for u in range(len(cu) - 1):
        s, e = int(cu[u]), int(cu[u + 1])
        L = e - s
        if L <= 0:
            continue
        future = np.triu(np.ones((L, L), dtype=bool), k=1)
        for h in range(H):
            S = q[s:e, h, :] @ k[s:e, h, :].T * scale
            S[future] = -np.inf
            out[s:e, h, :] = _softmax_rows(S) @ v[s:e, h, :]
    return out


def dense_block_causal_mask(cu_seqlens):
    """[T, T] boolean mask: key j visible to query i iff same user and j <= i
    (the AUC-recovery plan's dense mask and its FlexAttention mask_mod)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lengths = np.diff(cu)
    user_of = np.repeat(np.arange(len(lengths)), lengths)
    T = int(cu[-1])
    same = user_of[:, None] == user_of[None, :]
    causal = np.tril(np.ones((T, T), dtype=bool))
    return same & causal


def dense_masked_attention(q, k, v, cu_seqlens, scale=None):
    """Second formulation: one [T, T] score matrix per head with the dense
    block-diagonal causal mask applied (tiny inputs only)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, Dh = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(Dh)
    mask = dense_block_causal_mask(cu_seqlens)
    out = np.zeros_like(q)
    for h in range(H):
        S = q[:, h, :] @ k[:, h, :].T * scale
        S = np.where(mask, S, -np.inf)
        out[:, h, :] = _softmax_rows(S) @ v[:, h, :]
    return out


# --------------------------------------------------------------------------
# HSTU-style attention masks (cry-daniel/recsys README: HSTU attention mask
# logic and the attention function's mask types).  Not on the encoder layer's
# path; a second workload for the same jagged attention.
# --------------------------------------------------------------------------
def hstu_user_mask(L, causal=True, num_contexts=0, num_targets=0, target_group_size=1, window=0):
    """[L, L] boolean visibility for one user's sequence laid out as
    [contextual tokens][historical tokens][candidate tokens].

    Readings of the README's segment picture (it gives no formulas):
      * base: key j is visible to query i when j <= i (causal), or always
        (causal=False, the 'no mask' type);
      * contextual tokens (the first C = num_contexts) attend to one another
        in both directions;
      * candidate tokens (the last N = num_targets, starting at Hs = L - N)
        form groups of target_group_size in order; a candidate sees every
        non-candidate token and the candidates of its own group (subject to
        the base rule), never another group; non-candidates never see a
        candidate;
      * the local (sliding-window) type: with window W > 0 only keys with
        |i - j| < W are visible.
    Every query sees itself."""
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    vis = (j <= i) if causal else np.ones((L, L), dtype=bool)
    C = int(num_contexts)
    if C > 0:
        vis = vis | ((i < C) & (j < C))
    N = int(num_targets)
    if N > 0:
        Hs = L - N
        G = int(target_group_size)
        cand_i, cand_j = i >= Hs, j >= Hs
        same_group = ((i - Hs) // G) == ((j - Hs) // G)
        vis = vis & ~(cand_j & ~cand_i)            # non-candidates never see candidates
        vis = vis & ~(cand_i & cand_j & ~same_group)  # candidates see only their own group
    if window > 0:
        vis = vis & (np.abs(i - j) < window)
    return vis


def jagged_hstu_attention(q, k, v, cu_seqlens, causal=True, num_contexts=None, num_targets=None,
                          target_group_size=1, window=0, scale=None):
    """softmax(Q K^T * scale) V per user and head under hstu_user_mask.
    num_contexts / num_targets: per-user counts ([U]) or None (all zero)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, Dh = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(Dh)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    U = len(cu) - 1
    ctx = np.zeros(U, np.int64) if num_contexts is None else np.asarray(num_contexts, np.int64)
    tgt = np.zeros(U, np.int64) if num_targets is None else np.asarray(num_targets, np.int64)
    out = np.zeros_like(q)
    for u in range(U):
        s, e = int(cu[u]), int(cu[u + 1])
        L = e - s
        if L <= 0:
            continue
        if not (0 <= ctx[u] and 0 <= tgt[u] and ctx[u] + tgt[u] <= L):
            raise ValueError(f"user {u}: contexts + targets exceed its length")
        vis = hstu_user_mask(L, causal, ctx[u], tgt[u], target_group_size, window)
        for h in range(H):
            S = q[s:e, h, :] @ k[s:e, h, :].T * scale
            S = np.where(vis, S, -np.inf)
            out[s:e, h, :] = _softmax_rows(S) @ v[s:e, h, :]
    return out


# --------------------------------------------------------------------------
# RepEncoder front end (cti2026 README, RepEncoder section: a batched
# embedding bag over 28 slots with sum pooling, the [tokens, 28, 512] result
# flattened to [tokens, 14336], LayerNorm over the 14336 values, then
# Linear(14336 -> 512) into the encoder's input rows)
# --------------------------------------------------------------------------
REP_SLOTS = 28


def embedding_bags(tables, ids, bag_offsets, num_tokens):
    """Sum pooling per (token, slot): bag (t, s) holds ids[off[t*28+s] ..
    off[t*28+s+1]) of slot s's table; an empty bag gives zeros.  Returns
    [T, 28*dim] with slot s in columns s*dim .. s*dim+dim-1."""
    off = np.asarray(bag_offsets, np.int64)
    ids = np.asarray(ids, np.int64)
    dim = np.asarray(tables[0]).shape[1]
    out = np.zeros((num_tokens, REP_SLOTS * dim))
    for t in range(num_tokens):
        for sl in range(REP_SLOTS):
            b = t * REP_SLOTS + sl
            rows = ids[off[b]:off[b + 1]]
            if rows.size:
                out[t, sl * dim:(sl + 1) * dim] = _f64(np.asarray(tables[sl])[rows]).sum(axis=0)
    return out


def rep_encoder(tables, ids, bag_offsets, num_tokens, ln_g, ln_b, w, b=None, storage=None):
    """The front end: embedding bags -> LayerNorm(28*512) -> Linear to 512.
    storage='bf16' rounds the normalised rows as a bf16 pipeline stores them."""
    st = _storage(storage)
    bags = embedding_bags(tables, ids, bag_offsets, num_tokens)
    normed = st(layer_norm(bags, ln_g, ln_b))
    return linear(normed, w, b)


# --------------------------------------------------------------------------
# FP8 (e4m3) GEMM operands (cry-daniel/recsys README: FP8 among the listed
# optimisations; CTI-Inference-Opt optimisation plan, INT8 quantisation
# section, as the motivation for low-precision expert and QKV GEMMs)
# --------------------------------------------------------------------------
E4M3_MAX = 448.0


def quantize_e4m3(x):
    """Nearest e4m3 value (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits, no infinities: largest finite 448), ties to even, saturating at
    +-448.  Normal binade [2^E, 2^(E+1)) for E >= -6 has spacing 2^(E-3);
    below 2^-6 the subnormal spacing is 2^-9."""
    x = _f64(x)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        E = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    quantum = np.where(a >= 2.0 ** -6, 2.0 ** (np.maximum(E, -6) - 3), 2.0 ** -9)
    q = np.round(a / quantum) * quantum  # numpy rounds half to even
    q = np.minimum(q, E4M3_MAX)
    return np.sign(x) * q


def quantize_rows_e4m3(x, precision=None):
    """Per-row scaled e4m3: s = max|row| / 448 (1 for an all-zero row),
    codes = quantize_e4m3(row / s); returns (codes, s) with row ~ codes * s.

    precision=None computes s and the quotient in float64.  precision='f32'
    computes both as IEEE float32 operations (numpy's float32 division is
    correctly rounded): the code is an integer decided by floating point, and
    this is the precision a float32 kernel decides it in, so both sides pick
    the same code (the float64 quotient can fall on the other side of an e4m3
    rounding boundary when it lies within a float32 rounding of it)."""
    if precision == "f32":
        x32 = np.asarray(x, dtype=np.float32)
        amax = np.abs(x32).max(axis=-1, keepdims=True)
        s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        return quantize_e4m3((x32 / s).astype(np.float32)), s[..., 0].astype(np.float64)
    x = _f64(x)
    amax = np.abs(x).max(axis=-1, keepdims=True)
    s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return quantize_e4m3(x / s), s[..., 0]


def linear_fp8(x, weight, bias=None, precision=None):
    """y = x W^T + b with both operands quantised per row (rows of x = tokens,
    rows of W = output channels) to e4m3; the products of the codes are summed
    exactly (fp64 here; fp32 on the tensor cores) and scaled by s_x[i] s_w[j].
    precision: where the codes are decided (see quantize_rows_e4m3)."""
    qx, sx = quantize_rows_e4m3(x, precision)
    qw, sw = quantize_rows_e4m3(weight, precision)
    y = (qx @ qw.T) * sx[:, None] * sw[None, :]
    if bias is not None:
        y = y + _f64(bias)
    return y


# --------------------------------------------------------------------------
# Gate (cti2026 README, SMoE structure: softmax -> top-2 -> renormalise)
# --------------------------------------------------------------------------
def gate_probs(xn2, w_gate, b_gate):
    """p = softmax(xn2 Wg^T + bg) over the experts, [T, E]."""
    return _softmax_rows(linear(xn2, w_gate, b_gate))


def top2(p):
    """Top-2 experts by descending probability (ties: lower expert index
    first), and their renormalised weights.  Returns idx [T,2] int64, w [T,2]."""
    p = _f64(p)
    order = np.argsort(-p, axis=-1, kind="stable")
    idx = order[:, :TOP_K]
    pt = np.take_along_axis(p, idx, axis=-1)
    w = pt / pt.sum(axis=-1, keepdims=True)
    return idx.astype(np.int64), w


def top2_gap(p):
    """p_(2) - p_(3): how far the chosen pair sits from the first left out."""
    ps = -np.sort(-_f64(p), axis=-1)
    return ps[:, 1] - ps[:, 2]


def top1_gap(p):
    """p_(1) - p_(2): how far apart the two chosen experts are (slot order)."""
    ps = -np.sort(-_f64(p), axis=-1)
    return ps[:, 0] - ps[:, 1]


# --------------------------------------------------------------------------
# Route builder (cti2026 README, fused MoE routing preparation)
# --------------------------------------------------------------------------
def route_build(idx, num_experts):
    """Counting sort of the routes r = 2 t + k by expert.

    Returns cnt [E] (routes per expert), off [E+1] (exclusive prefix of cnt),
    perm [2T] (perm[off[e] + j] = j-th route of expert e, ascending r) and
    pos [2T] (the inverse: the slot of route r).
    """
    r_expert = np.asarray(idx, dtype=np.int64).reshape(-1)
    cnt = np.bincount(r_expert, minlength=num_experts).astype(np.int64)
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)
    perm = np.argsort(r_expert, kind="stable").astype(np.int64)
    pos = np.empty_like(perm)
    pos[perm] = np.arange(perm.size)
    return cnt, off, perm, pos


# --------------------------------------------------------------------------
# Experts and combine (cti2026 README, SMoE + fused MoE; AUC-recovery plan)
# --------------------------------------------------------------------------
def expert_ffn(x, w1, b1, w2, b2):
    """One expert: Linear(D->F) + ReLU + Linear(F->D)."""
    return linear(np.maximum(linear(x, w1, b1), 0.0), w2, b2)


def moe_routed(xn2, idx, w, w1, b1, w2, b2, hidden_round=None):
    """Sparse top-2 MoE.  Routes are grouped per expert with ``route_build``;
    each expert runs its FFN on its gathered tokens; route r's result is kept
    in route-major row r = 2 t + k; token t's output is w[t,0] y[2t] +
    w[t,1] y[2t+1].  Returns (moe_out [T, D], y [2T, D], hidden per route
    [2T, F] in slot order).  hidden_round, if given, is applied to the
    hidden layer and to each route's output before the weighted sum (the
    bf16 storage mode of layer_forward)."""
    xn2 = _f64(xn2)
    T, D = xn2.shape
    E = np.asarray(w1).shape[0]
    F = np.asarray(w1).shape[1]
    cnt, off, perm, _ = route_build(idx, E)
    y = np.zeros((2 * T, D))
    hidden = np.zeros((2 * T, F))
    for e in range(E):
        routes = perm[off[e]:off[e + 1]]
        if routes.size == 0:
            continue
        tok = routes // TOP_K
        h = np.maximum(linear(xn2[tok], w1[e], b1[e]), 0.0)
        if hidden_round is not None:
            h = hidden_round(h)
        hidden[off[e]:off[e + 1]] = h
        ye = linear(h, w2[e], b2[e])
        y[routes] = ye if hidden_round is None else hidden_round(ye)
    w = _f64(w)
    out = w[:, 0:1] * y[0::2] + w[:, 1:2] * y[1::2]
    return out, y, hidden


def moe_dense_all_experts(xn2, idx, w, w1, b1, w2, b2):
    """Second formulation: every expert on every token, then gather the two
    selected outputs and weight them."""
    xn2 = _f64(xn2)
    E = np.asarray(w1).shape[0]
    allout = np.stack([expert_ffn(xn2, w1[e], b1[e], w2[e], b2[e]) for e in range(E)], axis=1)
    sel = np.take_along_axis(allout, np.asarray(idx)[:, :, None], axis=1)  # [T, 2, D]
    return (sel * _f64(w)[:, :, None]).sum(axis=1)


# --------------------------------------------------------------------------
# Layer, stack, head (cti2026 README, TransformerEncoder + Prediction Head)
# --------------------------------------------------------------------------
def layer_forward(x, cu_seqlens, wts, return_intermediates=False, storage=None, choose=None):
    """One pre-norm layer over the packed stream x [T, D].

    storage=None computes everything in float64.  storage='bf16' rounds to
    bfloat16 the activations a bf16 pipeline stores between its steps -- the
    LayerNorm1 output, q/k/v, the attention output, the LayerNorm2 output fed
    to the experts, the expert hidden layer, each route's expert output and
    the layer output -- while the
    residual x1 inside the layer stays unrounded (an fp32 buffer in such a
    pipeline), the gate sees the unrounded LayerNorm2 output and all
    arithmetic stays float64.  It follows the same definition; only the stored values
    carry the bf16 rounding.

    choose(p, idx) -> idx, if given, may replace the top-2 pairs before
    routing (the weights are renormalised from p for the pairs it returns).
    Tests use it to follow another valid branch where two experts tie."""
    rnd = _storage(storage)
    x = _f64(x)
    T, D = x.shape
    xn = rnd(layer_norm(x, wts["ln1_g"], wts["ln1_b"]))
    qkv = rnd(linear(xn, wts["w_qkv"], wts.get("b_qkv")))
    q, k, v = split_qkv(qkv)
    attn = rnd(jagged_causal_attention(q, k, v, cu_seqlens).reshape(T, D))
    x1 = x + linear(attn, wts["w_o"], wts.get("b_o"))
    xn2_exact = layer_norm(x1, wts["ln2_g"], wts["ln2_b"])
    xn2 = rnd(xn2_exact)
    p = gate_probs(xn2_exact, wts["w_gate"], wts.get("b_gate"))
    idx, w = top2(p)
    if choose is not None:
        idx = np.asarray(choose(p, idx), dtype=np.int64)
        pt = np.take_along_axis(p, idx, axis=-1)
        w = pt / pt.sum(axis=-1, keepdims=True)
    moe, y, hidden = moe_routed(xn2, idx, w, wts["w1"], wts["b1"], wts["w2"], wts["b2"],
                                hidden_round=rnd)
    out = rnd(x1 + moe)
    if not return_intermediates:
        return out
    E = np.asarray(wts["w1"]).shape[0]
    cnt, off, perm, pos = route_build(idx, E)
    return out, dict(xn=xn, qkv=qkv, attn=attn, x1=x1, xn2=xn2, p=p, idx=idx, w=w,
                     gap=top2_gap(p), gap12=top1_gap(p), cnt=cnt, off=off, perm=perm, pos=pos,
                     y=y, hidden=hidden, moe=moe, out=out)


def head_forward(x, head, pred_mask=None):
    """Final LayerNorm, Linear(D->1), clamp to [-15, 15], sigmoid; keep the
    tokens whose pred_mask is set, in ascending token order."""
    z = linear(layer_norm(x, head["lnf_g"], head["lnf_b"]),
               _f64(head["w"]).reshape(1, -1), head.get("b")).reshape(-1)
    z = np.clip(z, -LOGIT_CLAMP, LOGIT_CLAMP)
    probs = 1.0 / (1.0 + np.exp(-z))
    if pred_mask is None:
        return probs
    return probs[np.asarray(pred_mask).astype(bool)]


def stack_forward(x, cu_seqlens, layers, head=None, pred_mask=None, storage=None,
                  return_intermediates=False, choose=None):
    """L layers in sequence, each with its own weights, then the optional head.
    With return_intermediates, also returns each layer's intermediates.
    choose(layer, p, idx) -> idx is passed to each layer (see layer_forward)."""
    h = _f64(x)
    per_layer = []
    for li, wts in enumerate(layers):
        ch = None if choose is None else (lambda p, idx, li=li: choose(li, p, idx))
        if return_intermediates:
            h, it = layer_forward(h, cu_seqlens, wts, return_intermediates=True, storage=storage,
                                  choose=ch)
            per_layer.append(it)
        else:
            h = layer_forward(h, cu_seqlens, wts, storage=storage, choose=ch)
    res = (h,) if head is None else (h, head_forward(h, head, pred_mask))
    if return_intermediates:
        res = res + (per_layer,)
    return res[0] if len(res) == 1 else res
