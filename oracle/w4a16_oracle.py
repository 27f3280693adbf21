"""CPU oracle for group-wise low-bit weight quantization and the W4A16 GEMV.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code,
constant table or helper with the CUDA library, and never calls it.

It is the plain, slow, obviously correct statement of what the hot path
computes: numpy in float64, following the pages step by step.

Pages cited (by title and section):

* [L13] "MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading guide
  (quidproquo.cc).  §AWQ "why scaling lowers the error" (slides 26, 28):
  Q(w) = Delta * Round(w / Delta), Delta = max|w| / 2^(N-1), expected Round
  error about 0.25; the search objective with s = s_X^alpha, s_X the mean
  activation magnitude; scaling salient channels by s and folding 1/s into the
  previous op (slides 25-27).  §TinyChat: offline packing so that one AND and
  one shift unpack the codes (slide 36); dequantization fused into the matmul
  (slide 37).  §"why W8A8 is not enough": decode is memory-bound (slides 19-20).
* [CMU] "CMU 11-868 LLM Systems: Model Quantization (L19/L20)" reading guide
  (quidproquo.cc).  §"absmax and zero-point" and the two PyTorch functions of
  lecture slide 10: zero-point scale from (max - min) / (2^8 - 1), a rounded
  zero point, clipping to the code range, dequant = (q - zp) * step, and a
  zero range replaced by 1.  §"back to the question": batch-1 decode is a GEMV
  and memory-bound.  §L20 "GPTQ": the layer objective ||WX - W_hat X||^2;
  quantize one column block at a time and push each column's rounding error
  onto the columns not yet quantized; the four steps (G = Cholesky((2XX^T +
  lambda I)^-1)^T computed first; quantize one column; divide its error by
  G's diagonal element; update the rest of the block, then everything right
  of the block at once); a fixed column order (slide 18); the Cholesky factor
  precomputed instead of updating H^-1 (slide 20); the AutoGPTQ example uses
  4 bits and group size 128.
* [Lab4] "MIT 6.5940 Lab 4 + Lab 5" reading guide (quidproquo.cc).  §Lab 4
  setup: calibration statistic = mean |X| per input channel over 512-token
  blocks; pseudo quantization (quantize, then dequantize at once); 3-bit,
  group 128.
* [L13] §QServe (slides 47-57; also the lecture summary of the same guide):
  the W4A8 setting -- 4-bit per-group weights, 8-bit per-token activations,
  INT8 tensor cores with the float conversion delayed to the end of the
  accumulation -- and progressive quantization, whose dequantization
  multiplies by the group scale before subtracting the zero point so that the
  register-level (packed byte) arithmetic cannot overflow.
* [ML11] "Learning-ML-DL ch. 11: Quantization for LLMs"
  (hoangvt2501.github.io).  §11.3: Y = (X diag(s)^-1)(W diag(s))^T;
  §11.4: AWQ's s = s_X^alpha with s_X the mean channel magnitude; GPTQ's
  Hessian H = 2XX^T of the output error per weight row, the OBS correction
  of the later columns after quantizing column q, damping by a fraction of
  the mean diagonal of H, the upper Cholesky factor of H^-1, and the
  qualitative result that GPTQ raises the weight error but lowers the output
  error.

Readings of points the pages leave open:

1. Symmetric step Delta = max|w| / 2^(N-1) as in [L13]; the signed code is
   clamped to [-2^(N-1), 2^(N-1)-1] and stored as u = q + 2^(N-1), z = 2^(N-1).
2. Round = round half to even (numpy ``rint``), matching the pages' ``round``.
3. Asymmetric codes are u = clamp(Round(w / Delta) + z, 0, 2^N - 1), so that an
   unclamped element dequantizes to exactly Delta * Round(w / Delta).
4. Asymmetric step Delta = fp16(fp64((max - min) / (2^N - 1))); zero point
   z = clamp(Round(-min / Delta), 0, 2^N - 1), stored as an fp16 integer.
5. A step that would be zero in fp16 (zero range included) is computed as if
   the range were 1, extending [CMU]'s "range 0 -> 1" rule.
6. The AWQ-scaled weight is rounded to fp16 once, w' = fp16(W * s), before
   the group statistics are taken.
7. s = fp16(s_X ** alpha) with s_X the fp64 mean of |X| over tokens; no other
   normalisation.
8. Packed layout v1 (our own design, stated in include/w4a16.h): qweight is
   u32[N, K/8]; word (n, j) holds k = 8j + i, i = 0..7; nibble slot p (bits
   4p..4p+3) holds i = [0, 2, 4, 6, 1, 3, 5, 7][p].
9. Search objective ([L13] slide 28): the norm is not named; the loss is the
   mean squared output error, which has the same minimiser as the Frobenius
   norm.  The divided activation is rounded to fp16 once, x' = fp16(x / s); the
   quantized output is taken as the W4A16 GEMM delivers it, rounded to fp16;
   the target W X is exact.  The grid of alphas is the caller's.
10. GPTQ Hessian: H = 2 X^T X over calibration tokens X[T, K] (the pages'
   2 X X^T with tokens as columns), plus lambda I with lambda = 0.01 *
   mean(diag(2 X^T X)) ([ML11] §11.4 damps by a fraction of the mean
   diagonal; 0.01 is its default; [CMU] L20 writes lambda I without a value).
11. GPTQ blocks are the quantization groups (128 columns), swept left to
   right.  Delta and z of a group come from the group's weights as they stand
   when the sweep reaches its first column (the rounding errors of earlier
   groups already pushed into them), by the RTN formulas of readings 1-5
   applied to those float64 values: Delta = fp16(fp64(fp64(max - min) /
   (2^N - 1))).  GPTQ here takes no AWQ scale (s = 1).
12. GPTQ arithmetic order (float64, each product and each sum rounded once):
   for column i of a block, u = clamp(Round(w / Delta) + z), q = (u - z) Delta,
   e = (w - q) / G[i, i]; every later column j of the block becomes
   w_j - e G[i, j].  After the block, every column j right of it becomes
   w_j - A_j with A_j = sum of e_i G[i, j] over the block's columns i, added
   in column order starting from 0.
13. G = Cholesky(H^-1)^T is the upper-triangular factor with H^-1 = G^T G and
   a positive diagonal ([CMU] L20 step 1); it is computed by numpy's Cholesky
   of numpy's inverse.
14. W4A8 level 1 (per output channel, symmetric INT8): s1 = fp16(max|W| / 119),
   w8 = clamp(Round(W / s1), -119, 119); a zero row takes s1 = fp16(1/119).
   119 is the largest R with R + ceil(2R / 15) / 2 <= 127: the level-2 values
   of a range within [-R, R] then dequantize inside int8 (see 15).  The pages
   ask only that the dequantization not overflow.
15. W4A8 level 2 (per group of 128 along K, asymmetric INT4 with integer
   step), over the group's range widened to include 0 (mn = min(min w8, 0),
   mx = max(max w8, 0)): s2 = max(1, ceil((mx - mn) / 15)) <= 16,
   z2 = Round(-mn / s2) (in [0, 15] without clamping), u = clamp(Round(w8 / s2)
   + z2, 0, 15).  Without the widening, a group far from zero (all values near
   -119, say) would take a small step and a clamped zero point and dequantize
   far from its values; with it every value lands within half a step.
   stored as layout-v1 codes, s2 (uint8) and the scaled zero zs = z2 * s2
   (uint8 <= 240).  Progressive dequantization: w8_hat = u * s2 - zs, where
   u * s2 <= 240 fits an unsigned byte, so four codes packed in a 32-bit word
   are scaled by one integer multiply and the zero removed by a bytewise
   subtraction.
16. W4A8 activations (per token, symmetric INT8): s_x = fp16(max|x| / 127),
   x8 = clamp(Round(x / s_x), -127, 127); a zero row takes s_x = fp16(1/127).
   The quotient of two fp16 values never lies within 2^-19 (relative) of a
   half-integer unless it is one, so an fp32 quotient rounds to the same x8.
17. W4A8 output: acc = sum_k x8 * w8_hat exactly (int64 here; it fits int32
   for K < 133,000), y = fp16(acc * s_x * s1) with the product exact (fp64).

Every function here is pinned by tests marked ``not gpu`` against closed
forms, brute force, invariants the pages state, or special cases.
"""
from __future__ import annotations

import numpy as np

F16 = np.float16
F64 = np.float64

ASYM = 0
SYM = 1

# layout v1: which element i of an 8-element k-block sits in nibble slot p
SLOT_TO_ELEM = (0, 2, 4, 6, 1, 3, 5, 7)


# ---------------------------------------------------------------------------
# a0: AWQ activation-aware scale  ([L13] slide 28, [Lab4] setup, [ML11] §11.4)
# ---------------------------------------------------------------------------
def act_scale(X: np.ndarray, alpha: float) -> np.ndarray:
    """s_k = fp16( (mean_t |X[t, k]|) ** alpha ) for calibration tokens X[T, K].

    s_X is the per-input-channel mean activation magnitude ([L13] slide 28,
    [ML11] §11.4) averaged over the calibration tokens ([Lab4] setup).
    """
    X = np.asarray(X)
    sx = np.abs(X.astype(F64)).mean(axis=0)
    return (sx ** F64(alpha)).astype(F16)


# ---------------------------------------------------------------------------
# a1: scaled weight  ([L13] slides 25-27, [ML11] §11.3)
# ---------------------------------------------------------------------------
def scale_weight(W: np.ndarray, s: np.ndarray | None) -> np.ndarray:
    """w'[n, k] = fp16(W[n, k] * s[k]): input channel k of the weight times s_k.

    The matching activation is divided by s_k in the previous op, so that
    (X diag(s)^-1)(W diag(s))^T = X W^T ([ML11] §11.3).
    """
    W = np.asarray(W, dtype=F16)
    if s is None:
        return W.copy()
    s = np.asarray(s, dtype=F16)
    return (W.astype(F64) * s.astype(F64)[None, :]).astype(F16)


# ---------------------------------------------------------------------------
# a2 + a3: group statistics, step Delta and zero point z
# ---------------------------------------------------------------------------
def group_params(wp: np.ndarray, bits: int, mode: int, group: int = 128):
    """Per (row, group) step Delta and zero point z, both returned as fp16.

    Asymmetric ([CMU] zero-point function): Delta = fp16((max - min) / (2^N-1)),
    z = clamp(Round(-min / Delta), 0, 2^N - 1).
    Symmetric ([L13] slide 26): Delta = fp16(max|w| / 2^(N-1)), z = 2^(N-1).
    A zero step is replaced by the step of a unit range (reading 5).
    """
    N, K = wp.shape
    g = wp.astype(F64).reshape(N, K // group, group)
    qmax = 2 ** bits - 1
    if mode == ASYM:
        mx = g.max(axis=-1)
        mn = g.min(axis=-1)
        delta = ((mx - mn) / F64(qmax)).astype(F16)
        delta[delta == 0] = F16(1.0 / qmax)
        # an integer zero point has no sign of zero: -0.0 (from min = 0) becomes +0.0
        z = np.clip(np.rint(-mn / delta.astype(F64)), 0, qmax) + 0.0
    elif mode == SYM:
        amax = np.abs(g).max(axis=-1)
        half = 2 ** (bits - 1)
        delta = (amax / F64(half)).astype(F16)
        delta[delta == 0] = F16(1.0 / half)
        z = np.full(delta.shape, F64(half))
    else:
        raise ValueError("mode must be ASYM or SYM")
    return delta, z.astype(F16)


# ---------------------------------------------------------------------------
# a4: round-to-nearest codes  ([L13] slide 26, [CMU] zero-point function)
# ---------------------------------------------------------------------------
def quantize_codes(wp: np.ndarray, delta: np.ndarray, z: np.ndarray, bits: int, group: int = 128) -> np.ndarray:
    """u = clamp(Round(w' / Delta) + z, 0, 2^N - 1) as uint8 [N, K]."""
    N, K = wp.shape
    g = wp.astype(F64).reshape(N, K // group, group)
    d = delta.astype(F64)[..., None]
    zz = z.astype(F64)[..., None]
    u = np.clip(np.rint(g / d) + zz, 0, 2 ** bits - 1)
    return u.reshape(N, K).astype(np.uint8)


# ---------------------------------------------------------------------------
# a5: pack / unpack, layout v1  ([L13] slide 36: offline reordering)
# ---------------------------------------------------------------------------
def pack_v1(u: np.ndarray) -> np.ndarray:
    """Pack codes u[N, K] (values < 16) into qweight u32[N, K/8] (layout v1)."""
    N, K = u.shape
    blocks = u.astype(np.uint32).reshape(N, K // 8, 8)
    words = np.zeros((N, K // 8), dtype=np.uint32)
    for p, i in enumerate(SLOT_TO_ELEM):
        words |= blocks[:, :, i] << np.uint32(4 * p)
    return words


def unpack_v1(qweight: np.ndarray) -> np.ndarray:
    """Inverse of pack_v1: qweight u32[N, K/8] -> codes uint8[N, K]."""
    qweight = np.asarray(qweight, dtype=np.uint32)
    N, KW = qweight.shape
    u = np.zeros((N, KW, 8), dtype=np.uint8)
    for p, i in enumerate(SLOT_TO_ELEM):
        u[:, :, i] = (qweight >> np.uint32(4 * p)) & np.uint32(0xF)
    return u.reshape(N, KW * 8)


# ---------------------------------------------------------------------------
# The quantizer end to end: awq_quantize_pack
# ---------------------------------------------------------------------------
def quantize_pack(W: np.ndarray, s: np.ndarray | None, group: int = 128, bits: int = 4, mode: int = ASYM):
    """(qweight u32[N,K/8], scales fp16[N,K/group], zeros fp16[N,K/group])."""
    wp = scale_weight(W, s)
    delta, z = group_params(wp, bits, mode, group)
    u = quantize_codes(wp, delta, z, bits, group)
    return pack_v1(u), delta, z


# ---------------------------------------------------------------------------
# a6: dequantization  ([CMU] dequant = (q - zp) * step; [Lab4] pseudo quant)
# ---------------------------------------------------------------------------
def dequant(qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int = 128) -> np.ndarray:
    """w_hat[n, k] = (u[n, k] - z[n, g]) * Delta[n, g] in float64 (exact)."""
    u = unpack_v1(qweight).astype(F64)
    N, K = u.shape
    d = np.repeat(scales.astype(F64), group, axis=1)
    z = np.repeat(zeros.astype(F64), group, axis=1)
    return (u - z) * d


# ---------------------------------------------------------------------------
# a7 / a8: the GEMV / skinny GEMM  ([L13] slides 19-20, 37; [CMU] slide 23)
# ---------------------------------------------------------------------------
def gemm_ref(x: np.ndarray, w_hat: np.ndarray):
    """y = x @ w_hat^T in float64 and the per-element bound B = |x| @ |w_hat|^T.

    The tolerance the CUDA result must meet is |y - y_ref| <= 2e-3 * B + 1e-3.
    """
    x64 = np.asarray(x).astype(F64)
    y = x64 @ w_hat.T
    bound = np.abs(x64) @ np.abs(w_hat).T
    return y, bound


def gemm(x, qweight, scales, zeros, group: int = 128):
    """Pseudo-quantized reference of w4a16_gemm: dequantize, then fp64 matmul."""
    return gemm_ref(x, dequant(qweight, scales, zeros, group))


def gemm_rows(x, qweight, scales, zeros, rows, group: int = 128):
    """The reference restricted to output channels ``rows`` (for sampled checks)."""
    rows = np.asarray(rows)
    w_hat = dequant(qweight[rows], scales[rows], zeros[rows], group)
    return gemm_ref(x, w_hat)


# ---------------------------------------------------------------------------
# search for the scaling strength  ([L13] slide 28; [YT]: a small grid search
# on calibration data picks it)
# ---------------------------------------------------------------------------
def divide_activation(X: np.ndarray, s: np.ndarray) -> np.ndarray:
    """x'[t, k] = fp16(X[t, k] / s[k]): the activation that meets the scaled
    weight, the 1/s folded into the previous op ([ML11] §11.3, [L13] slide 27)."""
    X = np.asarray(X, dtype=F16).astype(F64)
    return (X / np.asarray(s, dtype=F16).astype(F64)[None, :]).astype(F16)


def awq_loss(W: np.ndarray, X: np.ndarray, alpha: float, group: int = 128, bits: int = 4, mode: int = ASYM) -> float:
    """L(alpha) = mean over outputs of (Q(W s)(s^-1 X) - W X)^2 with s = s_X^alpha
    ([L13] slide 28), for weights W[N, K] and calibration tokens X[T, K].

    Q(W s)(s^-1 X) is the W4A16 product of the divided activation with the
    packed, scaled weight, rounded to fp16 (reading 9); W X is exact.
    """
    s = act_scale(X, alpha)
    q, sc, z = quantize_pack(W, s, group, bits, mode)
    w_hat = dequant(q, sc, z, group)
    y_q = (divide_activation(X, s).astype(F64) @ w_hat.T).astype(F16).astype(F64)
    y = np.asarray(X, dtype=F16).astype(F64) @ np.asarray(W, dtype=F16).astype(F64).T
    return float(np.mean((y_q - y) ** 2))


def awq_search(W: np.ndarray, X: np.ndarray, alphas, group: int = 128, bits: int = 4, mode: int = ASYM):
    """alpha* = argmin over the grid of L(alpha) ([L13] slide 28): (losses, index of the minimum)."""
    losses = [awq_loss(W, X, float(a), group, bits, mode) for a in alphas]
    return losses, int(np.argmin(losses))


# ---------------------------------------------------------------------------
# GPTQ: error-compensating column sweep  ([CMU] §L20 "GPTQ"; [ML11] §11.4)
# ---------------------------------------------------------------------------
GPTQ_DAMP = 0.01


def gptq_hessian(X: np.ndarray, damp: float = GPTQ_DAMP) -> np.ndarray:
    """H = 2 X^T X + lambda I for calibration tokens X[T, K], lambda = damp * mean
    of the diagonal of 2 X^T X (reading 10).  H is K x K, independent of T."""
    Xf = np.asarray(X, dtype=F16).astype(F64)
    H = 2.0 * (Xf.T @ Xf)
    lam = damp * float(np.mean(np.diag(H)))
    return H + lam * np.eye(H.shape[0])


def gptq_factor(H: np.ndarray) -> np.ndarray:
    """G = Cholesky(H^-1)^T: upper triangular, H^-1 = G^T G (reading 13)."""
    return np.linalg.cholesky(np.linalg.inv(np.asarray(H, dtype=F64))).T


def gptq_sweep(W: np.ndarray, G: np.ndarray, group: int = 128, bits: int = 4, mode: int = ASYM):
    """The column sweep of [CMU] §L20 in the order of readings 11-12.

    Returns (u uint8[N, K], Delta fp16[N, K/group], z fp16[N, K/group], wq
    float64[N, K]), where wq[:, i] is column i as it stood when it was
    quantized (the value its code rounds).
    """
    Wc = np.asarray(W, dtype=F16).astype(F64).copy()
    G = np.asarray(G, dtype=F64)
    N, K = Wc.shape
    qmax = 2 ** bits - 1
    u = np.zeros((N, K), dtype=np.uint8)
    wq = np.zeros((N, K), dtype=F64)
    deltas = np.zeros((N, K // group), dtype=F16)
    zeros = np.zeros((N, K // group), dtype=F16)
    for gi, b0 in enumerate(range(0, K, group)):
        b1 = b0 + group
        # group parameters from the block as the sweep finds it (reading 11)
        d16, z16 = group_params(Wc[:, b0:b1], bits, mode, group)
        deltas[:, gi], zeros[:, gi] = d16[:, 0], z16[:, 0]
        d, z = d16[:, 0].astype(F64), z16[:, 0].astype(F64)
        errs = np.zeros((N, group), dtype=F64)
        for i in range(b0, b1):
            w = Wc[:, i].copy()
            wq[:, i] = w
            ui = np.clip(np.rint(w / d) + z, 0, qmax)
            u[:, i] = ui.astype(np.uint8)
            e = (w - (ui - z) * d) / G[i, i]
            errs[:, i - b0] = e
            # the rest of the block, one column's correction at a time
            Wc[:, i + 1:b1] = Wc[:, i + 1:b1] - e[:, None] * G[i, i + 1:b1][None, :]
        # everything right of the block at once: the block's corrections summed in column order
        if b1 < K:
            acc = np.zeros((N, K - b1), dtype=F64)
            for i in range(b0, b1):
                acc = acc + errs[:, i - b0][:, None] * G[i, b1:][None, :]
            Wc[:, b1:] = Wc[:, b1:] - acc
    return u, deltas, zeros, wq


def gptq_quantize(W: np.ndarray, X: np.ndarray, group: int = 128, bits: int = 4, mode: int = ASYM,
                  damp: float = GPTQ_DAMP):
    """GPTQ end to end: (qweight u32[N, K/8] in layout v1, scales fp16, zeros fp16),
    the same format awq_quantize_pack produces, for the same GEMV."""
    G = gptq_factor(gptq_hessian(X, damp))
    u, d, z, _ = gptq_sweep(W, G, group, bits, mode)
    return pack_v1(u), d, z


# ---------------------------------------------------------------------------
# W4A8 with progressive group quantization  ([L13] §QServe; readings 14-17)
# ---------------------------------------------------------------------------
W4A8_L1 = 119   # level-1 range (reading 14)
W4A8_ACT = 127  # activation range (reading 16)


def w4a8_level2_params(w8: np.ndarray, group: int = 128):
    """Integer step s2 and zero point z2 of each group of int8 values (reading 15)."""
    N, K = w8.shape
    g = np.asarray(w8, dtype=np.int64).reshape(N, K // group, group)
    mx, mn = np.maximum(g.max(axis=-1), 0), np.minimum(g.min(axis=-1), 0)
    s2 = np.maximum(1, -((mn - mx) // 15))            # ceil((mx - mn) / 15) in integers
    z2 = np.clip(np.rint(-mn / s2), 0, 15).astype(np.int64)  # exact rationals of small integers, ties to even
    return s2, z2


def w4a8_quantize_weight(W: np.ndarray, group: int = 128):
    """(qweight u32[N, K/8] layout v1, s1 fp16[N], s2 uint8[N, K/group], zs uint8[N, K/group])."""
    W64 = np.asarray(W, dtype=F16).astype(F64)
    N, K = W64.shape
    amax = np.abs(W64).max(axis=1)
    s1 = (amax / W4A8_L1).astype(F16)
    s1[s1 == 0] = F16(1.0 / W4A8_L1)
    w8 = np.clip(np.rint(W64 / s1.astype(F64)[:, None]), -W4A8_L1, W4A8_L1).astype(np.int64)
    s2, z2 = w4a8_level2_params(w8, group)
    g = w8.reshape(N, K // group, group)
    u = np.clip(np.rint(g / s2[..., None]) + z2[..., None], 0, 15).astype(np.uint8).reshape(N, K)
    return pack_v1(u), s1, s2.astype(np.uint8), (z2 * s2).astype(np.uint8)


def w4a8_dequant_int8(qweight: np.ndarray, s2: np.ndarray, zs: np.ndarray, group: int = 128) -> np.ndarray:
    """w8_hat = u * s2 - zs as int64 [N, K] (the progressive order of reading 15)."""
    u = unpack_v1(qweight).astype(np.int64)
    return u * np.repeat(s2.astype(np.int64), group, axis=1) - np.repeat(zs.astype(np.int64), group, axis=1)


def w4a8_quantize_act(x: np.ndarray):
    """(x8 int8 [M, K], s_x fp16 [M]) per token (reading 16)."""
    x64 = np.asarray(x, dtype=F16).astype(F64)
    sx = (np.abs(x64).max(axis=1) / W4A8_ACT).astype(F16)
    sx[sx == 0] = F16(1.0 / W4A8_ACT)
    x8 = np.clip(np.rint(x64 / sx.astype(F64)[:, None]), -W4A8_ACT, W4A8_ACT).astype(np.int8)
    return x8, sx


def w4a8_gemm(x8, sx, qweight, s1, s2, zs, group: int = 128):
    """(y fp16 [M, N], acc int64 [M, N]): acc = x8 . w8_hat^T exactly, y = fp16(acc s_x s1) (reading 17)."""
    acc = np.asarray(x8, dtype=np.int64) @ w4a8_dequant_int8(qweight, s2, zs, group).T
    y = (acc.astype(F64) * np.asarray(sx, dtype=F16).astype(F64)[:, None]
         * np.asarray(s1, dtype=F16).astype(F64)[None, :]).astype(F16)
    return y, acc
