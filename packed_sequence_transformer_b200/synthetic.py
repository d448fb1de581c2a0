"""Seeded synthetic workloads for the packed-sequence encoder layer.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic.  Both the CUDA path (through the binding) and the CPU
oracle consume what it returns, so every parity comparison starts from the
same values.

Workload shapes follow the cti2026 README (Days-gone/cti2026): d_model 512,
8 heads x 64, QKV 512->1536, 8 ReLU experts 512->1024->512, top-2 gating,
many users packed end to end with ``user_offsets`` boundaries, 1221-10793
tokens per batch and about 44k tokens as the point where a dense [S,S] mask
no longer fits.  The competition data the README measured on is not
available; these generators stand in for it.

Draw order for one case (all from ``numpy.random.default_rng(seed)``, PCG64,
in float32):
  1. user lengths (lognormal, clipped, rescaled to the target total),
  2. x [T, 512] ~ N(0, 1),
  3. per layer: Wqkv, Wo, Wg, W1, W2 ~ N(0, sigma^2) (sigma 0.02; the gate
     may use its own sigma),
  4. biases (zero unless the case asks for random biases),
  5. head weight ~ N(0, 0.02^2),
  6. pred_mask ~ Bernoulli(0.3).
LayerNorm gamma = 1, beta = 0.  For bfloat16 cases every float array is
rounded to the bfloat16 grid (round to nearest even) before it is returned,
so the GPU receives exactly the values the oracle sees.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

D_MODEL = 512
N_HEADS = 8
D_HEAD = 64
D_FF = 1024
N_EXPERTS = 8
TOP_K = 2


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    r = ((u + bias) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(np.shape(a))


def lognormal_lengths(rng: np.random.Generator, num_users: int, total: int,
                      median: float, sigma: float, lmin: int, lmax: int) -> np.ndarray:
    """Per-user lengths: lognormal, clipped to [lmin, lmax], rescaled to sum to ``total``.

    1. L = clip(rint(lognormal(ln median, sigma)), lmin, lmax)
    2. rescale once: L = clip(rint(L * total / sum L), lmin, lmax)
    3. fix the remainder one token at a time, round robin over users in a
       stable descending-length order, skipping users that sit at a bound.
    """
    if not (lmin * num_users <= total <= lmax * num_users):
        raise ValueError("total tokens not reachable with the given bounds")
    raw = rng.lognormal(mean=np.log(median), sigma=sigma, size=num_users)
    L = np.clip(np.rint(raw), lmin, lmax).astype(np.int64)
    L = np.clip(np.rint(L * (total / L.sum())), lmin, lmax).astype(np.int64)
    order = np.argsort(-L, kind="stable")
    rem = int(total - L.sum())
    step = 1 if rem > 0 else -1
    i = 0
    guard = 0
    while rem != 0:
        u = order[i % num_users]
        if lmin <= L[u] + step <= lmax:
            L[u] += step
            rem -= step
            guard = 0
        else:
            guard += 1
            if guard > num_users:
                raise RuntimeError("cannot distribute remainder")
        i += 1
    return L


def offsets_from_lengths(lengths) -> np.ndarray:
    """cu_seqlens / user_offsets = [0, L0, L0+L1, ..., T] as int64."""
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


@dataclass
class Case:
    """One synthetic workload.  All float arrays are float32 (bf16-rounded
    when ``dtype == 'bf16'``); ``layers`` holds one weight dict per layer in
    nn.Linear [out, in] layout."""
    name: str
    dtype: str
    cu_seqlens: np.ndarray
    x: np.ndarray
    layers: List[Dict[str, np.ndarray]]
    head: Optional[Dict[str, np.ndarray]] = None
    pred_mask: Optional[np.ndarray] = None
    meta: Dict[str, object] = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def num_users(self) -> int:
        return int(len(self.cu_seqlens) - 1)

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.cu_seqlens)


def _normal(rng, shape, std):
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


# Parameters kept in float32 in both builds: LayerNorm affine parameters, the
# gate weight, and every bias (they feed fp32 arithmetic in the epilogues).
# The big matrices (Wqkv, Wo, W1, W2) and the activations use the build dtype.
FP32_PARAMS = ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "w_gate", "b_gate",
               "b_qkv", "b_o", "b1", "b2")


def _round_case(c: Case) -> Case:
    if c.dtype != "bf16":
        return c
    c.x = round_to_bf16(c.x)
    for lw in c.layers:
        for k in list(lw):
            if k not in FP32_PARAMS:
                lw[k] = round_to_bf16(lw[k])
    return c


def make_case(name: str, *, lengths=None, num_users=None, total=None, median=None,
              sigma=None, lmin=1, lmax=None, seed=0, len_seed=None, dtype="bf16",
              num_layers=1, w_std=0.02, gate_std=None, random_bias=False,
              gate_bias=None, with_head=False, pred_p=0.3) -> Case:
    """Build a case.  ``lengths`` fixes the packing; otherwise it is drawn
    with ``lognormal_lengths`` from ``len_seed`` (default: ``seed``)."""
    rng = np.random.default_rng(seed)
    if lengths is None:
        lrng = rng if len_seed is None or len_seed == seed else np.random.default_rng(len_seed)
        lengths = lognormal_lengths(lrng, num_users, total, median, sigma, lmin, lmax)
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = offsets_from_lengths(lengths)
    T = int(cu[-1])
    x = rng.standard_normal(size=(T, D_MODEL), dtype=np.float32)
    layers = [dict() for _ in range(num_layers)]
    for li in range(num_layers):
        D, F, E = D_MODEL, D_FF, N_EXPERTS
        gs = w_std if gate_std is None else gate_std
        layers[li]["w_qkv"] = _normal(rng, (3 * D, D), w_std)
        layers[li]["w_o"] = _normal(rng, (D, D), w_std)
        layers[li]["w_gate"] = _normal(rng, (E, D), gs)
        layers[li]["w1"] = _normal(rng, (E, F, D), w_std)
        layers[li]["w2"] = _normal(rng, (E, D, F), w_std)
    for li in range(num_layers):
        D, F, E = D_MODEL, D_FF, N_EXPERTS
        lw = layers[li]
        if random_bias:
            lw["b_qkv"] = _normal(rng, (3 * D,), 0.02)
            lw["b_o"] = _normal(rng, (D,), 0.02)
            lw["b_gate"] = _normal(rng, (E,), 0.02)
            lw["b1"] = _normal(rng, (E, F), 0.02)
            lw["b2"] = _normal(rng, (E, D), 0.02)
        else:
            lw["b_qkv"] = np.zeros(3 * D, np.float32)
            lw["b_o"] = np.zeros(D, np.float32)
            lw["b_gate"] = np.zeros(E, np.float32)
            lw["b1"] = np.zeros((E, F), np.float32)
            lw["b2"] = np.zeros((E, D), np.float32)
        if gate_bias is not None:
            lw["b_gate"] = (lw["b_gate"] + np.asarray(gate_bias, np.float32)).astype(np.float32)
        lw["ln1_g"] = np.ones(D, np.float32)
        lw["ln1_b"] = np.zeros(D, np.float32)
        lw["ln2_g"] = np.ones(D, np.float32)
        lw["ln2_b"] = np.zeros(D, np.float32)
    head = None
    pred_mask = None
    if with_head:
        hw = _normal(rng, (D_MODEL,), 0.02)
        head = {"lnf_g": np.ones(D_MODEL, np.float32), "lnf_b": np.zeros(D_MODEL, np.float32),
                "w": hw, "b": np.zeros(1, np.float32)}
        pred_mask = (rng.random(T) < pred_p).astype(np.uint8)
    c = Case(name=name, dtype=dtype, cu_seqlens=cu, x=x, layers=layers, head=head,
             pred_mask=pred_mask,
             meta={"seed": seed, "num_layers": num_layers, "lengths_median": float(np.median(lengths)),
                   "lengths_max": int(lengths.max()) if len(lengths) else 0,
                   "pairs": int((lengths * (lengths + 1) // 2).sum())})
    return _round_case(c)


def replicate_batch(case: Case, copies: int, seed: int) -> Case:
    """One batch of `copies` copies of the case's packing laid end to end:
    copy 0 is the case's own activations (and prediction mask), copy r > 0
    draws them afresh from ``default_rng(seed + r)`` with the same
    distributions; the layer weights and the head are shared (a replicated
    model serving a larger batch)."""
    if copies == 1:
        return case
    xs, masks = [case.x], [case.pred_mask]
    T = case.total_tokens
    for r in range(1, copies):
        rng = np.random.default_rng(seed + r)
        x = rng.standard_normal(size=(T, D_MODEL), dtype=np.float32)
        xs.append(round_to_bf16(x) if case.dtype == "bf16" else x)
        if case.pred_mask is not None:
            masks.append((rng.random(T) < 0.3).astype(np.uint8))
    lengths = np.tile(case.lengths, copies)
    return Case(name=f"{case.name}_x{copies}", dtype=case.dtype, cu_seqlens=offsets_from_lengths(lengths),
                x=np.concatenate(xs), layers=case.layers, head=case.head,
                pred_mask=None if case.pred_mask is None else np.concatenate(masks),
                meta=dict(case.meta, copies=copies))


# The five workloads.  Sizes, seeds and distributions as stated for each.
def config0() -> Case:
    """fp32, 1 layer, 4 users of {3,7,12,20} tokens (42), seed 0."""
    return make_case("config0_fp32_42tok", lengths=[3, 7, 12, 20], seed=0, dtype="fp32")


def config1_lengths() -> np.ndarray:
    rng = np.random.default_rng(1)
    return lognormal_lengths(rng, 60, 6823, 80.0, 1.0, 1, 1024)


def config1() -> Case:
    """bf16, 1 layer, 60 users / 6823 tokens, lognormal median 80 in [1,1024],
    gate weights N(0, 0.1^2), seed 1."""
    return make_case("config1_bf16_6823tok_60u", num_users=60, total=6823, median=80.0,
                     sigma=1.0, lmax=1024, seed=1, dtype="bf16", gate_std=0.1)


def config2() -> Case:
    """bf16, 8-layer stack + final LN + Linear(512->1) + sigmoid on a
    Bernoulli(0.3) pred_mask; same packing as config 1; weights from seed 2."""
    return make_case("config2_bf16_stack8_6823tok_60u", lengths=config1_lengths(), seed=2,
                     dtype="bf16", num_layers=8, with_head=True)


def config3() -> Case:
    """bf16, 8-layer stack, 390 users / 44,000 tokens, median 90 in [1,2048], seed 3."""
    return make_case("config3_bf16_stack8_44000tok_390u", num_users=390, total=44000,
                     median=90.0, sigma=0.8, lmax=2048, seed=3, dtype="bf16", num_layers=8)


def config4() -> Case:
    """bf16, 1 layer, 16 users x 4096 tokens, gate bias +2 on expert 0 and +1
    on expert 1, seed 4."""
    gb = np.zeros(N_EXPERTS, np.float32)
    gb[0], gb[1] = 2.0, 1.0
    return make_case("config4_bf16_16x4096_skewed_gate", lengths=[4096] * 16, seed=4,
                     dtype="bf16", gate_bias=gb)


CONFIGS = {0: config0, 1: config1, 2: config2, 3: config3, 4: config4}


def random_bf16_array(rng: np.random.Generator, shape, std=1.0) -> np.ndarray:
    """N(0, std^2) float32 values rounded to the bfloat16 grid."""
    return round_to_bf16(_normal(rng, shape, std))


# ------------------------------------------------------------ RepEncoder
REP_SLOTS = 28
REP_DIM = 512


@dataclass
class RepCase:
    """Inputs of the RepEncoder front end: 28 embedding tables, the id bags
    (bag (t, s) = ids[bag_offsets[t*28+s] .. bag_offsets[t*28+s+1])) and the
    LayerNorm / Linear parameters."""
    name: str
    dtype: str
    num_tokens: int
    tables: List[np.ndarray]   # 28 x [vocab_s, 512]
    ids: np.ndarray            # int64 [n_ids]
    bag_offsets: np.ndarray    # int64 [T*28 + 1]
    ln_g: np.ndarray           # [14336] f32
    ln_b: np.ndarray
    w: np.ndarray              # [512, 14336]
    b: Optional[np.ndarray]    # [512] or None


def make_rep_case(name: str, num_tokens: int, *, vocab=1000, max_bag=4, empty_p=0.1, seed=0,
                  dtype="bf16", table_std=1.0, w_std=0.02, random_affine=False) -> RepCase:
    """Seeded synthetic front-end inputs: per slot a table of `vocab` rows
    (a slot index that differs per slot, so that mixing up slots shows),
    bag sizes uniform in 1..max_bag with a share `empty_p` of empty bags,
    ids uniform over the slot's table."""
    rng = np.random.default_rng(seed)
    vocabs = [int(vocab) + 7 * s for s in range(REP_SLOTS)]
    tables = [_normal(rng, (v, REP_DIM), table_std) for v in vocabs]
    n_bags = num_tokens * REP_SLOTS
    sizes = rng.integers(1, max_bag + 1, size=n_bags)
    sizes[rng.random(n_bags) < empty_p] = 0
    off = np.zeros(n_bags + 1, np.int64)
    np.cumsum(sizes, out=off[1:])
    slot_of_bag = np.arange(n_bags) % REP_SLOTS
    ids = np.concatenate([rng.integers(0, vocabs[s], size=int(n)) for s, n in zip(slot_of_bag, sizes)]
                         if n_bags else [np.zeros(0, np.int64)]).astype(np.int64)
    width = REP_SLOTS * REP_DIM
    ln_g = np.ones(width, np.float32)
    ln_b = np.zeros(width, np.float32)
    b = None
    if random_affine:
        ln_g = (1.0 + 0.1 * rng.standard_normal(width)).astype(np.float32)
        ln_b = (0.1 * rng.standard_normal(width)).astype(np.float32)
        b = (0.02 * rng.standard_normal(REP_DIM)).astype(np.float32)
    w = _normal(rng, (REP_DIM, width), w_std)
    if dtype == "bf16":
        tables = [round_to_bf16(t) for t in tables]
        w = round_to_bf16(w)
    return RepCase(name, dtype, num_tokens, tables, ids, off, ln_g, ln_b, w, b)
