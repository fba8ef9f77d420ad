"""CPU oracle for the fused Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module: only the tests, `__graft_entry__.smoke()`
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code, table or helper with the CUDA library and imports nothing
from it.

What it computes
----------------
The layer the pages describe: "a token usually activates only a selected
subset" of the experts, and the work is "routing tokens to experts, moving data
and combining expert outputs" (toolboxkart.tech, "AWS SageMaker MoE kernel
optimizations H200", section "Why MoE inference needs specialized kernels").
The pages do not spell the arithmetic out; this module takes the plain reading
of a top-k softmax MoE layer with SwiGLU experts:

1. route   - per token, the k largest logits (ties to the lower expert id),
             weights = full softmax restricted to those k and renormalised;
2. permute - pair ids p = t*k + j grouped by expert, ascending p inside each
             expert, optionally padded to a tile of BT rows;
3. FP8     - per-tensor e4m3 (or e5m2) quantisation of weights (one scale per
             expert and tensor), of x and of the intermediate h ("FP8
             tensor-quantized fused MoE", same page, section "2. FP8 backend
             routing changes which kernel path runs"; E4M3 = 4 exponent and 3
             mantissa bits, E5M2 = 5 and 2, kongchang.com, "MoE Kernel
             Engineering Optimization Practices on Amazon SageMaker AI", section
             "Triton Backend Routing");
4. experts - h = silu(W_gate x) * (W_up x), y = W_down h;
5. combine - out_t = sum_j w_tj * y_(t,j), the routing-weight scale applied
             after the down projection ("fuses scaling, matrix multiplication,
             and expert aggregation into one GPU pass", aib.vote, "AWS
             SageMaker MoE kernel optimizations", third paragraph).

Swap-AB (computing C^T = B^T A^T, kongchang.com page, section "Swap-AB:
Making WGMMA Run at Full Utilization") changes no arithmetic, so the oracle has
a single GEMM orientation.

Precision: fp64 throughout, except that every step that turns a float into an
integer code (the FP8 quantisation of weights, x and h) is taken in IEEE fp32,
the precision in which the kernels take it.

Every function here is pinned by the CPU tests in ``tests/test_oracle_*.py``
against brute force, closed forms, invariants or an independent library
routine; no function is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0          # largest finite e4m3 magnitude (exponent 1111, mantissa 110)
E4M3_MIN_NORMAL_EXP = -6  # 2^-6 is the smallest normal e4m3 magnitude
E4M3_SUBNORMAL_STEP = 2.0 ** -9

E5M2_MAX = 57344.0        # largest finite e5m2 magnitude (exponent 11110, mantissa 11)
E5M2_MIN_NORMAL_EXP = -14
E5M2_SUBNORMAL_STEP = 2.0 ** -16


# --------------------------------------------------------------------------- routing
def route(logits: np.ndarray, k: int):
    """Top-k selection on the logits and the renormalised softmax weights.

    Selection is on the logits themselves (exp is monotone, so this is the
    same set as selection on probabilities, and it keeps ties exact). Order
    within a token: descending logit, equal logits by ascending expert id;
    -0.0 and +0.0 compare equal. The weights are the literal definition: a
    softmax over all E logits in fp64 (max subtracted), restricted to the
    selected experts and divided by their sum.

    A row whose logits are all -inf has no finite softmax; it takes the limit
    of a row of k equal logits, i.e. weight 1/k for each selected expert (the
    k lowest ids, by the tie rule).

    Returns (ids [M,k] int32, w [M,k] float64).
    """
    logits = np.asarray(logits, dtype=np.float32)
    M, E = logits.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    # a stable sort of -logit keeps equal logits in ascending id order
    order = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")
    ids = order[:, :k].astype(np.int32)
    l64 = logits.astype(np.float64)
    mx = l64.max(axis=1, keepdims=True)
    all_neg_inf = np.isneginf(mx[:, 0])
    p = np.exp(l64 - np.where(all_neg_inf[:, None], 0.0, mx))
    p = np.where(all_neg_inf[:, None], 1.0, p)
    p /= p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return ids, w


# --------------------------------------------------------------------------- permutation
def permute(ids: np.ndarray, E: int):
    """Group (token, slot) pairs by expert.

    Pair id p = t*k + j. For e = 0..E-1 in order, list the pairs routed to e in
    ascending p. Returns (counts [E], offsets [E+1], sorted_pairs [P]) with
    offsets the exclusive prefix sum of counts.
    """
    flat = np.asarray(ids, dtype=np.int64).ravel()
    groups = [np.nonzero(flat == e)[0] for e in range(E)]
    counts = np.array([g.size for g in groups], dtype=np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_pairs = (np.concatenate(groups) if groups else np.zeros(0, np.int64))
    return counts, offsets, sorted_pairs.astype(np.int64)


def pad_permutation(counts: np.ndarray, sorted_pairs: np.ndarray, BT: int, sentinel: int):
    """Pad every expert's group of pairs up to a multiple of BT rows.

    Pad slots hold ``sentinel`` (the pair count P). Returns
    (padded_offsets [E+1], padded_pairs [sum ceil(n_e/BT)*BT]).
    """
    counts = np.asarray(counts, dtype=np.int64)
    E = counts.size
    padded = ((counts + BT - 1) // BT) * BT
    poff = np.zeros(E + 1, dtype=np.int64)
    poff[1:] = np.cumsum(padded)
    out = np.full(int(poff[-1]), sentinel, dtype=np.int64)
    src = 0
    for e in range(E):
        n = int(counts[e])
        out[poff[e]:poff[e] + n] = sorted_pairs[src:src + n]
        src += n
    return poff, out


# --------------------------------------------------------------------------- e4m3 codec
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each e4m3 code: 1 sign, 4 exponent (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; there is no
    infinity. Returns float64.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    man = c & 0x7
    normal = (1.0 + man / 8.0) * np.exp2(ex - 7.0)
    sub = man * E4M3_SUBNORMAL_STEP
    mag = np.where(ex == 0, sub, normal)
    mag = np.where((ex == 15) & (man == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to e4m3: round to nearest, ties to even, saturating.

    Magnitudes above 448 (infinity included) become 448; NaN becomes the NaN
    code with the input's sign bit. Works on the exact value of each fp32
    input (held in fp64, which represents every fp32 exactly).
    """
    f = np.asarray(v, dtype=np.float32)
    neg = np.signbit(f)
    nan = np.isnan(f)
    a = np.abs(f.astype(np.float64))
    a = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))
    # binade of a: a = m * 2^ex with m in [0.5, 1)  =>  floor(log2 a) = ex - 1
    _, ex = np.frexp(a)
    e = ex.astype(np.int64) - 1
    subnormal = (a < 2.0 ** E4M3_MIN_NORMAL_EXP)
    # quantum of the grid at a: 2^-9 below the normal range, 2^(e-3) above
    step = np.where(subnormal, E4M3_SUBNORMAL_STEP, np.exp2((e - 3).astype(np.float64)))
    q = np.rint(a / step).astype(np.int64)  # np.rint rounds half to even
    # subnormal: the code is q itself (q == 8 lands exactly on 2^-6, code 0x08)
    code_sub = q
    # normal: q in [8, 16]; 16 carries into the next binade
    carry = q == 16
    e_n = np.where(carry, e + 1, e)
    q_n = np.where(carry, 8, q)
    code_norm = ((e_n + 7) << 3) | (q_n - 8)
    code = np.where(subnormal, code_sub, code_norm)
    code = np.where(a == 0.0, 0, code)
    code = np.where(nan, 0x7F, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------- e5m2 codec
# The second FP8 variant the kongchang.com page names ("MoE Kernel Engineering
# Optimization Practices on Amazon SageMaker AI", section "Triton Backend Routing: A
# Practical Path to FP8 Quantization"): 5 exponent bits and 2 mantissa bits, a wider
# range than E4M3 at lower precision. Bias 15 (the IEEE-style layout of the OCP 8-bit
# floating-point definition): exponent field 0 is subnormal (m * 2^-16), field 31 is
# infinity (m = 0) or NaN; the largest finite magnitude is 1.75 * 2^15 = 57344.
def e5m2_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each e5m2 code: 1 sign, 5 exponent (bias 15), 2 mantissa bits. Returns float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 2) & 0x1F
    man = c & 0x3
    normal = (1.0 + man / 4.0) * np.exp2(ex - 15.0)
    sub = man * E5M2_SUBNORMAL_STEP
    mag = np.where(ex == 0, sub, normal)
    mag = np.where(ex == 31, np.where(man == 0, np.inf, np.nan), mag)
    return sign * mag


def e5m2_encode(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to e5m2: round to nearest, ties to even, saturating.

    Magnitudes above 57344 (infinity included) become 57344 (code 0x7B); NaN
    becomes the NaN code 0x7F with the input's sign bit. Works on the exact value
    of each fp32 input (held in fp64).
    """
    f = np.asarray(v, dtype=np.float32)
    neg = np.signbit(f)
    nan = np.isnan(f)
    a = np.abs(f.astype(np.float64))
    a = np.where(nan, 0.0, np.minimum(a, E5M2_MAX))
    _, ex = np.frexp(a)
    e = ex.astype(np.int64) - 1                      # a in [2^e, 2^(e+1))
    subnormal = a < 2.0 ** E5M2_MIN_NORMAL_EXP
    # quantum of the grid at a: 2^-16 below the normal range, 2^(e-2) above
    step = np.where(subnormal, E5M2_SUBNORMAL_STEP, np.exp2((e - 2).astype(np.float64)))
    q = np.rint(a / step).astype(np.int64)           # ties to even
    code_sub = q                                     # q == 4 lands on 2^-14, code 0x04
    carry = q == 8                                   # normal q in [4, 8]; 8 is the next binade
    e_n = np.where(carry, e + 1, e)
    q_n = np.where(carry, 4, q)
    code_norm = ((e_n + 15) << 2) | (q_n - 4)
    code = np.where(subnormal, code_sub, code_norm)
    code = np.where(a == 0.0, 0, code)
    code = np.where(nan, 0x7F, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


# name -> (encode, decode, largest finite magnitude)
FP8_FORMATS = {"e4m3": (e4m3_encode, e4m3_decode, E4M3_MAX), "e5m2": (e5m2_encode, e5m2_decode, E5M2_MAX)}


def per_tensor_scale(t: np.ndarray, fmt: str = "e4m3") -> np.float32:
    """s = amax(|t|) / (largest finite value of the format) in fp32; an all-zero
    tensor takes s = 1."""
    fmax = FP8_FORMATS[fmt][2]
    a = np.float32(np.max(np.abs(np.asarray(t, dtype=np.float32)))) if np.size(t) else np.float32(0)
    if a == 0:
        return np.float32(1.0)
    return np.float32(a) / np.float32(fmax)


def quantize(t: np.ndarray, s: np.float32, fmt: str = "e4m3") -> np.ndarray:
    """FP8 codes of t / s, the division in IEEE fp32."""
    q = np.asarray(t, dtype=np.float32) / np.float32(s)
    return FP8_FORMATS[fmt][0](q.astype(np.float32))


_DECODE_TABLES = {}


def dequantize(codes: np.ndarray, s, fmt: str = "e4m3") -> np.ndarray:
    """decode(code) * s in fp64; the decode goes through a 256-entry table of the
    format's decode function, which is the same function evaluated once per code."""
    if fmt not in _DECODE_TABLES:
        _DECODE_TABLES[fmt] = FP8_FORMATS[fmt][1](np.arange(256, dtype=np.uint8))
    return _DECODE_TABLES[fmt][np.asarray(codes, dtype=np.uint8)] * float(s)


def quantize_expert_weights(W: np.ndarray, fmt: str = "e4m3"):
    """One scale per expert for a stacked weight tensor W [E, rows, cols].

    Returns (scales [E] float32, codes [E, rows, cols] uint8).
    """
    W = np.asarray(W, dtype=np.float32)
    E = W.shape[0]
    scales = np.zeros(E, dtype=np.float32)
    codes = np.zeros(W.shape, dtype=np.uint8)
    for e in range(E):
        s = per_tensor_scale(W[e], fmt)
        scales[e] = s
        codes[e] = quantize(W[e], s, fmt)
    return scales, codes


# --------------------------------------------------------------------------- experts
def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + e^-z), in fp64."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


class _Weights:
    """Per-expert weight access in fp64: plain arrays or a callable e -> (Wg, Wu, Wd)."""

    def __init__(self, w_gate=None, w_up=None, w_down=None, provider=None):
        self.provider = provider
        self.wg, self.wu, self.wd = w_gate, w_up, w_down

    def get(self, e: int):
        if self.provider is not None:
            g, u, d = self.provider(e)
        else:
            g, u, d = self.wg[e], self.wu[e], self.wd[e]
        return (np.asarray(g, dtype=np.float32), np.asarray(u, dtype=np.float32),
                np.asarray(d, dtype=np.float32))


def _map_experts(fn, experts, threads):
    """fn(e) for every e, in expert order; threads only overlap independent experts."""
    if threads <= 1 or len(experts) <= 1:
        return [fn(e) for e in experts]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, experts))


def moe_forward(x, logits, k, w_gate=None, w_up=None, w_down=None, *, fp8=False,
                provider=None, tokens=None, return_intermediates=False, threads=None,
                weight_cache=None, fp8_format="e4m3", expert_fp8=None):
    """The layer's output in fp64.

    x       [M, H]  bf16 values (any float array holding them)
    logits  [M, E]  fp32
    w_gate  [E, I, H], w_up [E, I, H], w_down [E, H, I] (bf16 values), or
    provider(e) -> (w_gate[e], w_up[e], w_down[e]) for weights too large to
            hold on the host at once.
    fp8     emulate the per-tensor FP8 path: each weight tensor of each
            expert quantised with its own scale, x quantised with one scale
            over all M*H elements, h quantised with one scale over all valid
            (token, slot) rows; dequantised values feed the fp64 arithmetic.
    expert_fp8  optional [E] booleans, a precision per expert instead of one for
            the layer (the per-expert choice of FP8 or higher precision the
            kongchang.com page describes, "MoE Kernel Engineering Optimization
            Practices on Amazon SageMaker AI", section "Triton Backend Routing: A
            Practical Path to FP8 Quantization"): FP8 experts take the FP8
            path above, the others the bf16 path. s_x is over all of x; s_h is
            over the valid h rows of the FP8 experts only (the rows that feed an
            FP8 down projection). When given, `fp8` is ignored.
    tokens  optional list of token indices whose output rows are wanted; the
            other rows come back as NaN. Routing, the permutation, s_x and
            (FP8) s_h are still computed over the whole batch, as defined.
    threads experts are independent, so they may be evaluated on several
            threads (default: the CPU count); no result depends on it.
    fp8_format  "e4m3" (default) or "e5m2": the code format of every FP8 tensor.
    weight_cache  optional dict reused across calls with the same weights: it
            keeps each expert's FP8 scales and codes so that they are not
            recomputed (the values are identical either way).

    Returns out [M, H] float64, or (out, dict of intermediates).
    """
    x = np.asarray(x, dtype=np.float32)
    logits = np.asarray(logits, dtype=np.float32)
    M, H = x.shape
    E = logits.shape[1]
    W = _Weights(w_gate, w_up, w_down, provider)
    ids, w = route(logits, k)
    counts, offsets, sorted_pairs = permute(ids, E)
    P = M * k

    inter = {"ids": ids, "w": w, "counts": counts, "offsets": offsets,
             "sorted_pairs": sorted_pairs}

    if expert_fp8 is None:
        expert_fp8 = np.full(E, bool(fp8))
    expert_fp8 = np.asarray(expert_fp8, dtype=bool)
    any_fp8 = bool(expert_fp8.any())

    fmt = fp8_format
    x64 = x.astype(np.float64)
    xq = None
    if any_fp8:
        s_x = per_tensor_scale(x, fmt)
        x_codes = quantize(x, s_x, fmt)
        xq = dequantize(x_codes, s_x, fmt)
        inter["s_x"] = s_x
        inter["x_codes"] = x_codes
        inter["w_scales"] = np.zeros((E, 3), dtype=np.float32)

    want = np.ones(M, dtype=bool) if tokens is None else np.zeros(M, dtype=bool)
    if tokens is not None:
        want[np.asarray(tokens, dtype=np.int64)] = True

    if threads is None:
        import os
        threads = os.cpu_count() or 1

    def expert_weights(e):
        if not expert_fp8[e]:
            g_w, u_w, d_w = W.get(e)
            return g_w.astype(np.float64), u_w.astype(np.float64), d_w.astype(np.float64)
        q = weight_cache.get(e) if weight_cache is not None else None
        if q is None:
            q = []
            for t in W.get(e):
                st = per_tensor_scale(t, fmt)
                q.append((st, quantize(t, st, fmt)))
            if weight_cache is not None:
                weight_cache[e] = q
        return tuple(dequantize(c, st, fmt) for st, c in q), tuple(st for st, _ in q)

    active = [e for e in range(E) if counts[e] > 0]

    # pass 1: gate/up projections and SwiGLU. An FP8 expert needs every valid h row
    # for the amax behind s_h; a bf16 expert only needs the wanted tokens' pairs.
    def pass1(e):
        f8 = bool(expert_fp8[e])
        n = int(counts[e])
        pairs = sorted_pairs[offsets[e]:offsets[e] + n]
        sel = want[pairs // k]
        if not f8 and not sel.any():
            return e, None
        if f8:
            (g_w, u_w, d_w), sc = expert_weights(e)
            inter["w_scales"][e] = sc
        else:
            g_w, u_w, d_w = expert_weights(e)
        rows = pairs if f8 else pairs[sel]
        X = (xq if f8 else x64)[rows // k]
        Hh = silu(X @ g_w.T) * (X @ u_w.T)
        amax = np.float32(np.max(np.abs(Hh.astype(np.float32)))) if f8 else None
        keep = {int(p): Hh[i] for i, p in enumerate(rows) if want[p // k]}
        Ym = None if f8 else Hh @ d_w.T       # bf16 expert: down projection right away
        return e, (rows, keep, amax, Ym)

    h_rows, Y = {}, {}
    h_amax = np.float32(0.0)
    for e, res in _map_experts(pass1, active, threads):
        if res is None:
            continue
        rows, keep, amax, Ym = res
        h_rows.update(keep)
        if expert_fp8[e]:
            h_amax = max(h_amax, amax)
        else:
            for i, p in enumerate(rows):
                Y[int(p)] = Ym[i]

    if any_fp8:
        s_h = np.float32(1.0) if h_amax == 0 else np.float32(h_amax) / np.float32(FP8_FORMATS[fmt][2])
        inter["s_h"] = s_h

        # pass 2: quantised h of the FP8 experts through their dequantised down projection
        def pass2(e):
            n = int(counts[e])
            pairs = [int(p) for p in sorted_pairs[offsets[e]:offsets[e] + n] if want[int(p) // k]]
            if not pairs:
                return []
            d_w = expert_weights(e)[0][2]
            Hm = np.stack([h_rows[p] for p in pairs])
            Hm = dequantize(quantize(Hm.astype(np.float32), s_h, fmt), s_h, fmt)
            Ym = Hm @ d_w.T
            return [(p, Ym[i]) for i, p in enumerate(pairs)]

        for res in _map_experts(pass2, [e for e in active if expert_fp8[e]], threads):
            for p, y in res:
                Y[p] = y

    out = np.full((M, H), np.nan, dtype=np.float64)
    for t in range(M):
        if not want[t]:
            continue
        acc = np.zeros(H, dtype=np.float64)
        for j in range(k):            # combine in slot order
            acc += w[t, j] * Y[t * k + j]
        out[t] = acc
    if return_intermediates:
        inter["h_rows"] = h_rows
        return out, inter
    return out


# --------------------------------------------------------------------------- tensor parallelism
def shard_weights(w_gate, w_up, w_down, shard: int, num_shards: int):
    """Slice `shard` of `num_shards` over the intermediate dimension I: rows
    [g*I/G, (g+1)*I/G) of every W_gate[e] and W_up[e], the same columns of every
    W_down[e] (the eight-way tensor parallelism the pages deploy the layer with,
    toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "3.
    Removing repeat compilation can reduce first-token delay")."""
    I = np.asarray(w_gate).shape[1]
    if I % num_shards:
        raise ValueError("I must divide into the shards")
    a, b = shard * I // num_shards, (shard + 1) * I // num_shards
    return (np.asarray(w_gate)[:, a:b, :], np.asarray(w_up)[:, a:b, :], np.asarray(w_down)[:, :, a:b])


def moe_forward_tp(x, logits, k, w_gate=None, w_up=None, w_down=None, *, num_shards: int, provider=None,
                   fp8=False, fp8_format="e4m3"):
    """The layer split over `num_shards` ranks by the intermediate dimension: each rank
    is a layer of its slice (routing is the same everywhere: it reads only the logits),
    and the combine adds the ranks' outputs. SwiGLU acts per intermediate feature and
    the down projection sums over features, so in exact arithmetic the bf16 result is
    the unsharded layer's. FP8 ranks quantise their own slice (weights) and their own
    h, so the FP8 result is the sum of the ranks' FP8 layers. Weights as stacked
    arrays, or provider(e) -> (w_gate[e], w_up[e], w_down[e]) of the FULL layer."""
    out = None
    for g in range(num_shards):
        if provider is None:
            kw = dict(zip(("w_gate", "w_up", "w_down"), shard_weights(w_gate, w_up, w_down, g, num_shards)))
        else:
            def sliced(e, g=g):
                gw, uw, dw = (np.asarray(t) for t in provider(e))
                sub = shard_weights(gw[None], uw[None], dw[None], g, num_shards)
                return sub[0][0], sub[1][0], sub[2][0]
            kw = {"provider": sliced}
        part = moe_forward(x, logits, k, fp8=fp8, fp8_format=fp8_format, **kw)
        out = part if out is None else out + part
    return out
