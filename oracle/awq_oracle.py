"""CPU oracle for AWQ's activation-aware scale search and group-wise INT4 quantization.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links this module; only the
test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use it. It shares no
code with the CUDA library (no kernels, headers, helpers, tables or constants).

Plain, slow, step-by-step restatement of the method, one operation at a time:

* float32 steps use numpy float32 element-wise operations (IEEE-754 round-to-nearest-even, one rounding
  per operation, never fused); ``np.rint`` rounds half to even like ``torch.round`` in the pages' code;
* the correctly rounded power uses ``decimal`` at 60 significant digits;
* sums that define the activation statistic are fp64, in a fixed order;
* the reconstruction loss is evaluated in fp64 (the weight error ``w - w_hat`` is exact in fp64).

Sources (web pages about AWQ and weight quantization, cited by title and section):

[P1] "AWQ 离群激活平滑实操逐通道等价缩放与 4-bit 精度无损转换" (gsyq.cn): section 一 (the equivalence
     ``Y = (X diag(s)^-1)(diag(s) W)``), section 二 (the asymmetric group-128 INT4 pseudo-quantizer and the
     scale-search loop with a strict ``<`` best-loss update).
[P2] bjdmk.com.cn AWQ article: section "显著权重的识别" (importance ``S_X(i) = (1/N) sum_j |X_ji|``), section
     "数学等价变换与通道自适应缩放" (loss ``L(s) = ||W X - Q(W diag(s)) diag(s)^-1 X||^2``, grid search),
     section "GPU 硬件级反量化算子内联融合" (4-bit codes packed two per byte).
[P4] "AWQ：激活感知权重量化算法说明" (msModelSlim docs): section 原理 (``scales = act_mean.pow(ratio)
     .clamp(min=1e-4)``, ``scales = scales / sqrt(scales.max() * scales.min())``, ratio in [0, 1) with step
     1/n_grid, n_grid = 20), section 缩放因子搜索流程 (scale, quantize, unscale, MSE, keep the minimum),
     section NormLinearSubgraph (several linears on one input share one scale; outputs concatenated).
[P5] "大模型量化中的离群值：成因、解法与部署实战" (hncyxsy.com): section 1.1 (outlier channels sit at nearly
     fixed positions), sections 2.1-2.2 (symmetric per-channel INT8, ``s = max|x| / 127``, codes clamped to
     [-127, 127], and the worked figures of one outlier wiping out small values), used by the INT8 option.

Readings where the pages are silent or disagree (each is listed with its reason in the design notes):
the mean statistic (P2/P4) rather than P1's max formula; P4's clamp-then-normalise with the geometric
normaliser; a step clamp of 1e-5 after ``(max - min) / 15``; the zero point is not clamped and is stored
as float32 with -0 turned into +0; codes of in-feature k sit in word k // 8 at bits 4*(k % 8); the
activation statistic sums |x| in fp64 over consecutive 256-row chunks (rows in increasing order inside a
chunk, chunk totals in chunk order) and rounds S / N to fp64 and then to fp32; the power is the correctly
rounded fp32 value of the real power.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py`` (closed forms, brute
force, exact rational checks and an independent multiprecision library). The per-ratio loss has no
closed form; it is pinned through its invariants (ratio 0 gives plain round-to-nearest, an on-grid W
gives zero loss, the scaling identity, and the two-GEMM form of the loss).
"""
from __future__ import annotations

from decimal import Decimal, localcontext

import numpy as np

F32 = np.float32
F64 = np.float64

GROUP = 128                 # group size along the input dimension [P1 section 二]
ACT_CHUNK = 256             # rows per chunk of the fixed-order activation sum (reading, see module doc)
SCALE_FLOOR = F32(1e-4)     # clamp(min=1e-4) on the powered statistic [P4 原理]
STEP_FLOOR = F32(1e-5)      # clamp(min=1e-5) on the quantization step
LEVELS = F32(15)            # 4-bit: 16 levels, 15 intervals [P1 section 二]
QMAX = F32(15)
QMIN = F32(0)
POW_DIGITS = 60


def widen_bf16(bits) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32, exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------------------------------
# (1) activation statistic   act_mean[k] = mean_i |X[i, k]|        [P2 显著权重的识别; P4 原理]
# ---------------------------------------------------------------------------------------------------
def act_mean(x_bits, chunk: int = ACT_CHUNK) -> np.ndarray:
    """Per-channel mean absolute activation, float32 [K].

    S_k is accumulated in fp64: inside a chunk of ``chunk`` consecutive rows one row at a time in
    increasing row order, then the chunk totals one at a time in chunk order. The result is
    RN32(RN64(S_k / N))."""
    x_bits = np.asarray(x_bits)
    N, K = x_bits.shape
    if N < 1:
        raise ValueError("need at least one calibration row")
    S = np.zeros(K, F64)
    for c0 in range(0, N, chunk):
        part = np.zeros(K, F64)
        rows = widen_bf16(x_bits[c0:min(N, c0 + chunk)]).astype(F64)
        for i in range(rows.shape[0]):
            part = part + np.abs(rows[i])
        S = S + part
    return (S / F64(N)).astype(F32)


# ---------------------------------------------------------------------------------------------------
# (2) candidate scales        s = clamp(act_mean^ratio, 1e-4);  s /= sqrt(max(s) * min(s))   [P4 原理]
# ---------------------------------------------------------------------------------------------------
def ratio(j: int, n_grid: int) -> np.float32:
    """Grid point j of [0, 1) with step 1/n_grid, as the fp32 quotient RN32(j / n_grid)."""
    return F32(F32(j) / F32(n_grid))


def _decimal_to_f32(y: Decimal) -> np.float32:
    """Round a (positive, finite) Decimal to the nearest float32, ties to even, by exact comparison."""
    f = F32(float(y))
    if not np.isfinite(f):
        return f
    best, best_d = None, None
    with localcontext() as ctx:
        ctx.prec = 400                     # wide enough that these differences are exact
        for c in (np.nextafter(f, F32(-np.inf)), f, np.nextafter(f, F32(np.inf))):
            d = abs(Decimal(float(c)) - y)  # Decimal(float) is exact
            if best is None or d < best_d or (d == best_d and (int(c.view(np.uint32)) & 1) == 0):
                best, best_d = c, d
    return F32(best)


def cr_pow(a, r) -> np.float32:
    """Correctly rounded float32 of the real number a ** r (a >= 0 float32, r float32 in [0, 1)).

    0 ** 0 = 1 and 0 ** r = 0 for r > 0."""
    a = F32(a)
    r = F32(r)
    if r == 0:
        return F32(1.0)
    if a == 0:
        return F32(0.0)
    with localcontext() as ctx:
        ctx.prec = POW_DIGITS
        y = (Decimal(float(r)) * Decimal(float(a)).ln()).exp()
    return _decimal_to_f32(y)


def _cr_pow_row(a_vec: np.ndarray, r: np.float32, ln_cache: dict) -> np.ndarray:
    out = np.empty(a_vec.shape[0], F32)
    if r == 0:
        out[:] = F32(1.0)
        return out
    rd = Decimal(float(r))
    with localcontext() as ctx:
        ctx.prec = POW_DIGITS
        for i, a in enumerate(a_vec):
            if a == 0:
                out[i] = F32(0.0)
                continue
            key = float(a)
            ln = ln_cache.get(key)
            if ln is None:
                ln = Decimal(key).ln()
                ln_cache[key] = ln
            out[i] = _decimal_to_f32((rd * ln).exp())
    return out


def scale_candidates(act: np.ndarray, r: np.float32, ln_cache: dict | None = None) -> np.ndarray:
    """One row of the scale table at ratio r: t = CR32(act^r); t = max(t, 1e-4);
    d = RN32(sqrt(RN32(max(t) * min(t)))); s = RN32(t / d)."""
    act = np.asarray(act, F32)
    t = _cr_pow_row(act, F32(r), {} if ln_cache is None else ln_cache)
    t = np.maximum(t, SCALE_FLOOR)
    d = np.sqrt(F32(t.max() * t.min()))
    return (t / d).astype(F32)


def scale_table(act: np.ndarray, n_grid: int) -> np.ndarray:
    """float32 [n_grid, K]: row j holds the candidate scales at ratio j / n_grid."""
    act = np.asarray(act, F32)
    cache: dict = {}
    return np.stack([scale_candidates(act, ratio(j, n_grid), cache) for j in range(n_grid)])


# ---------------------------------------------------------------------------------------------------
# (3) asymmetric 4-bit group quantizer on W' = W diag(s)           [P1 section 二 pseudo-quantizer]
# ---------------------------------------------------------------------------------------------------
def quantize_groups(wp: np.ndarray, group: int = GROUP):
    """Quantize the scaled weight ``wp`` (float32 [O, K]) group-wise along K.

    Per group of ``group`` consecutive in-features of one output row:
      step = max(RN32(RN32(max - min) / 15), 1e-5);   z = rint(RN32(-min / step));
      q = min(max(RN32(rint(RN32(w' / step)) + z), 0), 15);   deq = RN32(RN32(q - z) * step).
    Returns (q float32 [O,K], step float32 [O,K/g], z float32 [O,K/g] with -0 -> +0, deq float32 [O,K])."""
    wp = np.asarray(wp, F32)
    O, K = wp.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    g = wp.reshape(O, K // group, group)
    mx = g.max(axis=2)
    mn = g.min(axis=2)
    step = np.maximum((mx - mn) / LEVELS, STEP_FLOOR).astype(F32)
    z = np.rint(-mn / step).astype(F32)
    q = np.minimum(np.maximum(np.rint(g / step[..., None]) + z[..., None], QMIN), QMAX).astype(F32)
    deq = ((q - z[..., None]) * step[..., None]).astype(F32)
    z = (z + F32(0.0)).astype(F32)
    return q.reshape(O, K), step, z, deq.reshape(O, K)


def pseudo_quantize(w_bits_or_f32, s: np.ndarray, group: int = GROUP):
    """Scale, quantize, dequantize and unscale one weight matrix at per-channel scales ``s``.

    w' = RN32(w * s_k); quantize_groups(w'); w_hat = RN32(deq / s_k).
    Returns (w_hat float32 [O,K], q, step, z)."""
    w = _as_f32_weight(w_bits_or_f32)
    s = np.asarray(s, F32)
    wp = (w * s[None, :]).astype(F32)
    q, step, z, deq = quantize_groups(wp, group)
    w_hat = (deq / s[None, :]).astype(F32)
    return w_hat, q, step, z


def _as_f32_weight(w):
    w = np.asarray(w)
    if w.dtype == np.uint16:
        return widen_bf16(w)
    return w.astype(F32)


# ---------------------------------------------------------------------------------------------------
# (4) reconstruction loss and the grid search          [P2 数学等价变换; P1 section 二; P4 搜索流程]
# ---------------------------------------------------------------------------------------------------
def loss_of(x_bits, w_bits, w_hat) -> float:
    """mean over all N*O outputs of (X W^T - X W_hat^T)^2, evaluated as mean((X (W - W_hat)^T)^2) in fp64."""
    x = widen_bf16(x_bits).astype(F64) if np.asarray(x_bits).dtype == np.uint16 else np.asarray(x_bits, F64)
    w = _as_f32_weight(w_bits).astype(F64)
    dw = w - np.asarray(w_hat, F32).astype(F64)
    E = x @ dw.T
    return float((E * E).sum() / F64(E.size))


def argmin_first(losses) -> int:
    """Index of the first minimum: scan in order, replace the best only on a strictly smaller loss."""
    best_j, best = 0, None
    for j, l in enumerate(losses):
        if best is None or l < best:
            best_j, best = j, l
    return best_j


def search(x_bits, w_bits, n_grid: int = 20, group: int = GROUP, act=None, table=None, mode: str = "p4",
           quant: str = "int4"):
    """The whole search for one linear (or several sharing X, rows of W concatenated).

    mode selects the candidate scales: "p4" (default), "weight_aware" or "rms" (see the variants below).
    quant selects the weight quantizer: "int4" (asymmetric, groups of ``group``) or "int8" (symmetric
    per output channel, section (9); zeros is then None and codes are int8).
    Returns dict(act_mean, table [n_grid,K], losses [n_grid] fp64, best_j, scales, codes, steps, zeros)."""
    if act is None:
        act = act_mean(x_bits)
    if table is None:
        if mode == "p4":
            table = scale_table(act, n_grid)
        elif mode == "weight_aware":
            table = scale_table_weight_aware(act, weight_mean(w_bits), n_grid)
        elif mode == "rms":
            table = scale_table_rms(act, n_grid)
        else:
            raise ValueError(mode)
    losses = np.empty(n_grid, F64)
    if quant not in ("int4", "int8"):
        raise ValueError(quant)
    pq = pseudo_quantize if quant == "int4" else (lambda w, s, g: pseudo_quantize_int8(w, s) + (None,))
    for j in range(n_grid):
        w_hat = pq(w_bits, table[j], group)[0]
        losses[j] = loss_of(x_bits, w_bits, w_hat)
    best = argmin_first(losses)
    _, q, step, z = pq(w_bits, table[best], group)
    return dict(act_mean=act, table=table, losses=losses, best_j=best, scales=table[best].copy(),
                codes=q.astype(np.uint8 if quant == "int4" else np.int8), steps=step, zeros=z)


# ---------------------------------------------------------------------------------------------------
# (5) packed codes: 8 codes per uint32, code of in-feature k at bits 4*(k % 8) of word k // 8
# ---------------------------------------------------------------------------------------------------
def pack_codes(q) -> np.ndarray:
    q = np.asarray(q).astype(np.uint32)
    O, K = q.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    words = np.zeros((O, K // 8), np.uint32)
    for i in range(8):
        words |= q[:, i::8] << np.uint32(4 * i)
    return words


def unpack_codes(words, K: int) -> np.ndarray:
    words = np.asarray(words, np.uint32)
    O = words.shape[0]
    q = np.empty((O, K), np.uint8)
    for i in range(8):
        q[:, i::8] = ((words >> np.uint32(4 * i)) & np.uint32(0xF)).astype(np.uint8)
    return q


def quantize_pack(w_bits, s, group: int = GROUP):
    """Codes, steps and zeros of W at scales s, codes packed (the artefact of the search)."""
    _, q, step, z = pseudo_quantize(w_bits, s, group)
    return pack_codes(q.astype(np.uint32)), step, z


# ---------------------------------------------------------------------------------------------------
# (6) applying the scales to the subgraph            [P4 缩放因子搜索流程 (SubgraphFusionFactory), 支持的子图类型]
#     forward scaling of the target linears' input columns, inverse scaling of the producer of that input
#     (norm weight, or the rows and bias of the source linear); outputs are bfloat16.
# ---------------------------------------------------------------------------------------------------
def round_f32_to_bf16(x) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    keep = u >> np.uint64(16)
    rest = u & np.uint64(0xFFFF)
    up = (rest > 0x8000) | ((rest == 0x8000) & ((keep & np.uint64(1)) == 1))
    return (keep + up.astype(np.uint64)).astype(np.uint16)


def fold_columns(a_bits, s, divide: bool) -> np.ndarray:
    """out[r, c] = bf16(RN32(a[r, c] * s[c])) or bf16(RN32(a[r, c] / s[c]))."""
    a = widen_bf16(a_bits)
    s = np.asarray(s, F32)[None, :]
    r = (a / s) if divide else (a * s)
    return round_f32_to_bf16(r.astype(F32))


def fold_rows(a_bits, s, divide: bool) -> np.ndarray:
    """out[r, c] = bf16(RN32(a[r, c] * s[r])) or bf16(RN32(a[r, c] / s[r]))."""
    a = widen_bf16(a_bits)
    s = np.asarray(s, F32)[:, None]
    r = (a / s) if divide else (a * s)
    return round_f32_to_bf16(r.astype(F32))


# ---------------------------------------------------------------------------------------------------
# (7) deployment GEMM of the quantized linear (W4A16)   [P2 GPU 硬件级反量化算子内联融合]
#     the weights are restored from the packed codes with the group step and zero, to a 16-bit float
#     (bfloat16 here), and multiplied with the activations; here exactly, in fp64.
# ---------------------------------------------------------------------------------------------------
def dequant_w4(words, steps, zeros, group: int = GROUP) -> np.ndarray:
    """float32 [O, K]: RN32(RN32(q - z) * step) per element, q unpacked from the words."""
    q = unpack_codes(words, np.asarray(words).shape[1] * 8).astype(F32)
    st = np.repeat(np.asarray(steps, F32), group, axis=1)
    z = np.repeat(np.asarray(zeros, F32), group, axis=1)
    return ((q - z) * st).astype(F32)


def w4a16_matmul(x_bits, words, steps, zeros, group: int = GROUP, weights: str = "bf16") -> np.ndarray:
    """fp64 [M, O] = X' @ deq(W)^T with the weights restored to bfloat16 (weights="bf16": the 16-bit
    operand of a kernel that dequantizes into its tensor-core tiles) or kept at their fp32 dequantized
    value RN32((q - z) * step) (weights="fp32": a kernel that applies the step and zero point after the
    products of each group)."""
    deq = dequant_w4(words, steps, zeros, group)
    if weights == "bf16":
        deq = widen_bf16(round_f32_to_bf16(deq))
    elif weights != "fp32":
        raise ValueError("weights must be 'bf16' or 'fp32'")
    x = widen_bf16(x_bits).astype(F64)
    return x @ deq.astype(F64).T


# ---------------------------------------------------------------------------------------------------
# (8) variants of the candidate scales
#   weight-aware [P2 数学等价变换与通道自适应缩放, AWQChannelScaler]: s = clamp(act^p / (wmean^(1-p) + 1e-6),
#       1e-4), s /= sqrt(max(s) min(s)), p over linspace(0, 1, n): p_j = RN32(j / (n - 1)) (1.0 included);
#       wmean[k] = mean_o |W[o, k]| (the same fixed-order mean as the activation statistic).
#   RMS-normalised [P1 section 二, search_smooth_scaling_factors]: a = clamp(act, 1e-5); s = a^alpha;
#       s /= sqrt(mean(s^2)); s = clamp(s, 1e-4); alpha_j = RN32(j / (n - 1)) (n = 11 gives 0, 0.1, ..., 1.0).
#       mean(s^2) = RN32(RN64(S / K)) with S the fp64 sum of RN32(s_k^2) in 256-column chunks (columns in
#       order inside a chunk, chunk totals in order); the root and the division are single fp32 operations.
# The quantizer and the loss are the ones above in both cases.
# ---------------------------------------------------------------------------------------------------
WEIGHT_EPS = F32(1e-6)
RMS_ACT_FLOOR = F32(1e-5)


def weight_mean(w_bits) -> np.ndarray:
    """mean over output rows of |W[o, k]|, float32 [K] (same fixed order as act_mean)."""
    return act_mean(w_bits)


def closed_grid(j: int, n_grid: int) -> np.float32:
    """Point j of linspace(0, 1, n_grid): RN32(j / (n_grid - 1)); a single point is 0."""
    if n_grid == 1:
        return F32(0)
    return F32(F32(j) / F32(n_grid - 1))


def scale_table_weight_aware(act, wmean, n_grid: int) -> np.ndarray:
    act = np.asarray(act, F32)
    wmean = np.asarray(wmean, F32)
    cache_a: dict = {}
    cache_w: dict = {}
    rows = []
    for j in range(n_grid):
        p = closed_grid(j, n_grid)
        q = F32(F32(1) - p)
        t = _cr_pow_row(act, p, cache_a)
        u = _cr_pow_row(wmean, q, cache_w)
        s = np.maximum((t / (u + WEIGHT_EPS)).astype(F32), SCALE_FLOOR)
        d = np.sqrt(F32(s.max() * s.min()))
        rows.append((s / d).astype(F32))
    return np.stack(rows)


def _sum_sq_fixed(t: np.ndarray, chunk: int = 256) -> np.float64:
    sq = (t * t).astype(F32).astype(F64)
    total = F64(0)
    for c0 in range(0, sq.shape[0], chunk):
        part = F64(0)
        for v in sq[c0:c0 + chunk]:
            part = part + v
        total = total + part
    return total


def scale_table_rms(act, n_grid: int) -> np.ndarray:
    act = np.maximum(np.asarray(act, F32), RMS_ACT_FLOOR)
    K = act.shape[0]
    cache: dict = {}
    rows = []
    for j in range(n_grid):
        t = _cr_pow_row(act, closed_grid(j, n_grid), cache)
        m = F32(_sum_sq_fixed(t) / F64(K))
        d = np.sqrt(m)
        rows.append(np.maximum((t / d).astype(F32), SCALE_FLOOR))
    return np.stack(rows)


# ---------------------------------------------------------------------------------------------------
# (9) INT8 symmetric per-channel quantizer for the search   [P4 YAML weight_qconfig: per_channel, int8,
#     symmetric, minmax; P5 section 2.1: q = clamp(round(x / s), -127, 127), s = max|x| / 127]
#     per output row o of W' = W diag(s): step = max(RN32(max_k |w'| / 127), 1e-5) (the 1e-5 floor as in the
#     INT4 quantizer, so an all-zero row stays finite); q = min(max(rint(RN32(w' / step)), -127), 127);
#     deq = RN32(q * step).
# ---------------------------------------------------------------------------------------------------
QMAX8 = F32(127)


def quantize_rows_int8(wp):
    wp = np.asarray(wp, F32)
    amax = np.abs(wp).max(axis=1)
    step = np.maximum((amax / QMAX8).astype(F32), STEP_FLOOR).astype(F32)
    q = np.minimum(np.maximum(np.rint(wp / step[:, None]), -QMAX8), QMAX8).astype(F32)
    deq = (q * step[:, None]).astype(F32)
    return q, step, deq


def pseudo_quantize_int8(w_bits_or_f32, s):
    """w_hat = RN32(deq / s) with the INT8 per-channel quantizer on W diag(s). Returns (w_hat, q, step)."""
    w = _as_f32_weight(w_bits_or_f32)
    s = np.asarray(s, F32)
    q, step, deq = quantize_rows_int8((w * s[None, :]).astype(F32))
    return (deq / s[None, :]).astype(F32), q, step


def quantize_pack_int8(w_bits, s):
    """(codes int8 [O, K], steps float32 [O]) of W at scales s."""
    _, q, step = pseudo_quantize_int8(w_bits, s)
    return q.astype(np.int8), step
