"""Plain, slow, fp64 CPU oracle of the SVDQuant linear layer.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline may use it; the C-ABI library never does.  It shares no code with
the CUDA path (no kernels, headers, tables or helpers); only the seeded input
generator in `synth` serves both.

What it computes follows "SVDQuant: How a Small High-Precision Branch Makes
4-Bit Diffusion Practical" (technical review of arXiv:2411.05007v4):

  * smoothing  X~ = X D^-1, W~ = D W, D = diag(lambda)        (section 3.1, eq. 3)
  * lambda_i = max|X_:,i|^a / max|W_i,:|^(1-a)                 (section 3.1, eq. 4)
  * rank-r SVD  L1 = U_r S_r, L2 = V_r^T, R = W~ - L1 L2       (section 5, eq. 10)
  * symmetric INT4 group quantiser s = max|Z|/7,
    Q(Z) = s round(Z/s)                                        (section 2.2, eq. 1)
  * two-branch output  Y = (X~ L1) L2 + Q(X~) Q(R)            (section 4.2, eq. 7)
  * LoRA in smoothed coordinates  [L1 | D A] [L2 ; B]          (section 7, eq. 13)
  * MAC and storage ratios                                     (section 6, eqs. 11-12)
  * calibration refinement: alpha search by the calibrated layer-output
    error, factors re-fitted to W~ - Q(R)                        (section 5)
  * GPTQ rounding of the residual on the calibration Hessian   (section 8)
  * W8A8 comparator: int8 operands, one scale per token / output channel
    applied once          (section 8, the eight-bit setting; section 9.3, INT8)
  * NVFP4 variant: E2M1 codes in groups of 16 with E4M3 group scales and
    an fp32 scale per row                         (section 8; section 9.1)

Readings taken where the pages leave a step open (each is listed in the
design notes of the repository):
  * group size 64 along K on both operands, scales stored as fp32
    s = fl32(max|z| / 7); codes round-half-even of the exact quotient z/s,
    then clamped to [-8, 7] (the clamp only acts when s is subnormal);
    an all-zero group, or one whose scale underflows to 0, has s = 0, codes 0;
  * lambda_k = 1 when either statistic is zero;  inv_lambda = fl32(1/lambda);
  * x~ = fl32(x * inv_lambda) (one fp32 rounding of the exact product);
  * the 16-bit branch is bf16: L1, L2 stored as bf16, Z = bf16(bf16(x~) L1)
    with exact (fp64) accumulation;
  * R is taken against the stored bf16 factors, summed j = 0..r-1 in order;
  * Y = bf16(sum_g s_x s_w P_g + Z L2 + b), optional exact-erf GELU before
    the final rounding.
Every function is pinned by the tests in tests/test_oracle_*.py; none is
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "GROUP", "bf16_bits_to_f64", "round_bf16_bits", "round_bf16", "round_f32",
    "smoothing_lambda", "quantize_groups", "pack_nibbles", "unpack_nibbles",
    "calib_absmax", "pack_weights", "quantize_act", "group_partials",
    "linear", "gelu", "layer_forward", "mac_ratio", "storage_ratio",
    "two_branch_unquantized", "dequantize_groups", "residual_quantize",
    "leading_svd", "layer_output_error", "refine_factors", "pack_weights_calibrated",
    "quantize_rows_int8", "pack_weights_w8a8", "quantize_act_w8a8", "linear_w8a8",
    "gptq_hessian", "gptq_quantize_residual",
    "NVFP4_GROUP", "E2M1_VALUES", "round_e4m3", "e4m3_bits", "e2m1_codes", "e2m1_values",
    "quantize_nvfp4_rows", "dequantize_nvfp4", "pack_weights_nvfp4", "quantize_act_nvfp4",
    "linear_nvfp4",
]

GROUP = 64


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def bf16_bits_to_f64(b):
    """bf16 bit patterns -> exactly equal float64 values."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_bf16(x):
    """Round float64 values to the nearest bf16 value, ties to even, in ONE
    rounding (no detour through fp32).  Returns float64 values.

    bf16 keeps 8 significant bits and fp32's exponent range; its subnormal
    quantum is 2^-133.  Values whose rounded magnitude reaches 2^128
    overflow to +-inf."""
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    xf = x[fin]
    _, e = np.frexp(xf)                     # xf = m 2^e, 0.5 <= |m| < 1
    qexp = np.maximum(e - 8, -133)          # quantum exponent
    y = np.ldexp(np.rint(np.ldexp(xf, -qexp)), qexp)
    y[np.abs(y) >= 2.0 ** 128] = np.copysign(np.inf, y[np.abs(y) >= 2.0 ** 128])
    out[fin] = y
    return out


def round_bf16_bits(x):
    """Round float64 values to bf16 (one rounding) and return the bits."""
    y = round_bf16(x).astype(np.float32)    # exact: y is a bf16 value
    return (np.ascontiguousarray(y).view(np.uint32) >> 16).astype(np.uint16)


def round_f32(x):
    """Round float64 values to fp32 (IEEE round-to-nearest-even), as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# eq. 4: smoothing factors
# --------------------------------------------------------------------------
def calib_absmax(X):
    """Calibration statistic max_i |X_ik| per input channel k (eq. 4's
    max|X_:,i|), over the rows of X (float64 values)."""
    return np.max(np.abs(np.asarray(X, dtype=np.float64)), axis=0)


def smoothing_lambda(act_absmax, w_absmax, alpha=0.5):
    """lambda_k = a_k^alpha / w_k^(1-alpha) (eq. 4); lambda_k = 1 where either
    statistic is zero (the pages name no safeguard; this is the reading).
    alpha = 0.5 is evaluated as sqrt(a)/sqrt(w) (correctly rounded)."""
    a = np.asarray(act_absmax, dtype=np.float64)
    w = np.asarray(w_absmax, dtype=np.float64)
    lam = np.ones_like(a)
    ok = (a > 0) & (w > 0)
    if alpha == 0.5:
        lam[ok] = np.sqrt(a[ok]) / np.sqrt(w[ok])
    else:
        lam[ok] = np.power(a[ok], alpha) / np.power(w[ok], 1.0 - alpha)
    return lam


# --------------------------------------------------------------------------
# eq. 1: symmetric INT4 group quantiser
# --------------------------------------------------------------------------
def quantize_groups(z):
    """Quantise groups of fp32 values (given as float64, last axis = one
    group of 64) with eq. 1: s = fl32(max|z| / 7), q = round(z / s).

    The rounding is round-half-even of the EXACT real quotient z/s, decided
    by exact fp64 comparisons of z with (q +- 1/2) s: q*s has at most 28
    significant bits and z - q*s at most 29, so every quantity below is
    exact.  fl32(m/7) is taken as the fp64 quotient rounded to fp32, which
    equals the correctly rounded fp32 quotient (53 >= 2*24 + 2).
    Codes are clamped to [-8, 7]; with a normal s they already lie in
    [-7, 7].  s = 0 (all-zero group, or a scale that underflows) gives
    codes 0.  Returns (codes int64 like z, scales float64 [..., G])."""
    z = np.asarray(z, dtype=np.float64)
    m = np.max(np.abs(z), axis=-1)
    s = round_f32(m / 7.0)
    codes = np.zeros(z.shape, dtype=np.int64)
    nz = s > 0
    if np.any(nz):
        zz = z[nz]
        ss = np.broadcast_to(s[nz][..., None], zz.shape)
        q = np.rint(zz / ss)
        for _ in range(3):                  # converges in one pass
            d = zz - q * ss                 # exact
            two_d = 2.0 * d
            q = np.where(two_d > ss, q + 1, np.where(two_d < -ss, q - 1, q))
        d = zz - q * ss
        tie = (2.0 * np.abs(d) == ss) & (np.mod(q, 2) != 0)
        q = np.where(tie, q + np.sign(d), q)
        codes[nz] = np.clip(q, -8, 7).astype(np.int64)
    return codes, s


def dequantize_groups(codes, scales):
    """codes [rows, K], scales [G, rows] -> float64 [rows, K] = q * s."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    G = K // GROUP
    s = np.asarray(scales, dtype=np.float64).T.reshape(rows, G, 1)
    return (codes.reshape(rows, G, GROUP) * s).reshape(rows, K)


def pack_nibbles(codes):
    """Two's-complement nibbles, two per byte: byte b of a row holds
    k = 2b in the low nibble and k = 2b+1 in the high nibble (the review's
    companion explainer describes packing two 4-bit values per byte)."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    p = np.asarray(packed, dtype=np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out)


def _quantize_rows(v):
    """v float64 [rows, K] of fp32 values -> codes [rows, K], scales [G, rows]."""
    rows, K = v.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of the group size 64")
    codes, s = quantize_groups(v.reshape(rows, K // GROUP, GROUP))
    return codes.reshape(rows, K), np.ascontiguousarray(s.T)


# --------------------------------------------------------------------------
# offline pack: eqs. 3, 4, 10, 13 and eq. 1 on the residual
# --------------------------------------------------------------------------
def residual_quantize(Wt, L1b, L2b):
    """R = W~ - L1b L2b (fp64; the product of two bf16 values is exact and the
    rank-one terms are subtracted j = 0..r-1 in order, each step rounded),
    then eq. 1 per group of 64 input channels of each output column.
    Wt is the smoothed weight [K, N].  Returns (R, codes [N, K], s_w [G, N])."""
    R = np.array(Wt, dtype=np.float64, copy=True)
    for j in range(L1b.shape[1]):
        R -= np.outer(L1b[:, j], L2b[j, :])
    codes, s_w = _quantize_rows(round_f32(R.T))
    return R, codes, s_w


def leading_svd(Wt, k):
    """Leading k singular triplets of W~ (fp64) with ARPACK (scipy's svds),
    returned like np.linalg.svd's truncated output (descending order)."""
    from scipy.sparse.linalg import svds
    k = min(k, min(Wt.shape) - 1)
    U, S, Vt = svds(Wt, k=k, tol=0, which="LM", random_state=0)
    order = np.argsort(S)[::-1]
    return U[:, order], S[order], Vt[order]


def pack_weights(W_bits, act_absmax, rank, alpha=0.5, bias_bits=None,
                 lora_A_bits=None, lora_B_bits=None, lora_scale=1.0,
                 smooth=True, svd=None):
    """Offline transform of one linear layer (the review's offline procedure,
    section 5, with alpha fixed and no refinement / GPTQ).

    W_bits: bf16 bits [N, K] (nn.Linear layout; the math weight W is its
    transpose, K x N, rows = input channels).  act_absmax: [K] calibration
    statistic.  smooth=False uses lambda = 1 (plain W4A4, for ablations).
    svd=None runs the full LAPACK SVD (np.linalg.svd); svd="leading" takes
    only the leading rank+1 triplets from ARPACK (same definition, for large
    layers)."""
    Wl = bf16_bits_to_f64(W_bits)                      # [N, K]
    N, K = Wl.shape
    W = Wl.T                                           # [K, N]
    w_absmax = np.max(np.abs(W), axis=1)
    if smooth:
        lam = smoothing_lambda(act_absmax, w_absmax, alpha)
    else:
        lam = np.ones(K)
    inv_lam = round_f32(1.0 / lam)
    Wt = lam[:, None] * W                              # eq. 3, W~ = D W
    if svd is None:
        U, S, Vt = np.linalg.svd(Wt, full_matrices=False)
    elif svd == "leading":
        U, S, Vt = leading_svd(Wt, int(rank) + 1)
    else:
        raise ValueError(svd)
    r = int(rank)
    L1 = U[:, :r] * S[None, :r]                        # eq. 10
    L2 = Vt[:r, :]
    L1b = round_bf16(L1)
    L2b = round_bf16(L2)
    R, codes, s_w = residual_quantize(Wt, L1b, L2b)
    if lora_A_bits is not None and lora_A_bits.shape[1] > 0:
        A = bf16_bits_to_f64(lora_A_bits)              # [K, k]
        B = bf16_bits_to_f64(lora_B_bits)              # [k, N]
        DA = (lam[:, None] * A) * float(np.float32(lora_scale))
        L1b = np.hstack([L1b, round_bf16(DA)])         # eq. 13: [L1 | D A]
        L2b = np.vstack([L2b, B])                      #          [L2 ; B]
    bias = (np.zeros(N) if bias_bits is None else bf16_bits_to_f64(bias_bits))
    return dict(lam=lam, inv_lambda=inv_lam, Wt=Wt, U=U, S=S, Vt=Vt,
                L1=L1, L2=L2, L1b=L1b, L2b=L2b, R=R, wcodes=codes,
                wq=pack_nibbles(codes), s_w=s_w, sigma=S[:r + 1].copy(),
                bias=bias, rank=L1b.shape[1], K=K, N=N)


# --------------------------------------------------------------------------
# runtime: activation quantise + down-projection, then the two-branch product
# --------------------------------------------------------------------------
def quantize_act(X_bits, inv_lambda, L1b):
    """Review section 6.1, activation side: x~ = fl32(x * inv_lambda) (eq. 3),
    eq. 1 per (token, group of 64), and the 16-bit down-projection
    Z = bf16(bf16(x~) L1) with exact accumulation.
    Returns (codes [M, K], s_x [G, M], Z [M, r] float64 bf16 values, xhat)."""
    X = bf16_bits_to_f64(X_bits)
    xhat = round_f32(X * np.asarray(inv_lambda, dtype=np.float64)[None, :])
    codes, s_x = _quantize_rows(xhat)
    r = L1b.shape[1]
    if r:
        Z = round_bf16(round_bf16(xhat) @ L1b)
    else:
        Z = np.zeros((X.shape[0], 0))
    return codes, s_x, Z, xhat


def group_partials(xcodes, wcodes, rows=None, cols=None):
    """P_g[i, n] = sum_{k in group g} q_x[i, k] q_w[n, k] for every group g.
    Computed as an fp64 matmul of integer-valued arrays: every product and
    partial sum is an integer below 2^13, so the result is exact.
    Returns int64 [G, len(rows), len(cols)]."""
    xc = np.asarray(xcodes)
    wc = np.asarray(wcodes)
    if rows is not None:
        xc = xc[rows]
    if cols is not None:
        wc = wc[cols]
    m, K = xc.shape
    n = wc.shape[0]
    G = K // GROUP
    xg = xc.reshape(m, G, GROUP).astype(np.float64)
    wg = wc.reshape(n, G, GROUP).astype(np.float64)
    P = np.empty((G, m, n), dtype=np.int64)
    for g in range(G):
        P[g] = np.rint(xg[:, g, :] @ wg[:, g, :].T).astype(np.int64)
    return P


def gelu(y):
    """GELU with the exact error function: 0.5 y (1 + erf(y / sqrt 2))."""
    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * (1.0 + _erf(y / math.sqrt(2.0)))


def linear(xcodes, s_x, Z, wcodes, s_w, L2b, bias, apply_gelu=False,
           rows=None, cols=None):
    """Review section 6.1, product side / eq. 7:
    Y = sum_g s_x[g, i] s_w[g, n] P_g[i, n] + Z L2 + b (fp64), optional GELU,
    then one bf16 rounding.  Returns (Y float64, Y_bf16 float64 values)."""
    xc = np.asarray(xcodes)
    M = xc.shape[0]
    N = np.asarray(wcodes).shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    cols = np.arange(N) if cols is None else np.asarray(cols)
    P = group_partials(xc, wcodes, rows, cols)
    sx = np.asarray(s_x, dtype=np.float64)[:, rows]
    sw = np.asarray(s_w, dtype=np.float64)[:, cols]
    Y = np.zeros((len(rows), len(cols)))
    for g in range(P.shape[0]):
        Y += (sx[g][:, None] * sw[g][None, :]) * P[g]
    if np.asarray(L2b).shape[0]:
        Y += np.asarray(Z)[rows] @ np.asarray(L2b)[:, cols]
    Y += np.asarray(bias, dtype=np.float64)[cols][None, :]
    if apply_gelu:
        Y = gelu(Y)
    return Y, round_bf16(Y)


def layer_forward(X_bits, packed, apply_gelu=False, rows=None, cols=None):
    """quantize_act then linear for one packed layer (oracle end to end)."""
    xc, s_x, Z, _ = quantize_act(X_bits, packed["inv_lambda"], packed["L1b"])
    Y, Yb = linear(xc, s_x, Z, packed["wcodes"], packed["s_w"], packed["L2b"],
                   packed["bias"], apply_gelu, rows, cols)
    return dict(xcodes=xc, s_x=s_x, Z=Z, Y=Y, Ybf16=Yb)


# --------------------------------------------------------------------------
# calibration refinement (review section 5, the offline procedure): search
# the migration strength alpha by the calibrated layer-output error, with
# alternating updates of the protected factors from W~ - Q(R)
# --------------------------------------------------------------------------
def layer_output_error(X_bits, packed, W_bits):
    """Relative Frobenius error of the quantised layer (both branches, no
    bias, before the bf16 output rounding) against X W on the tokens X:
    ||Y_q - X W||_F / ||X W||_F, all in fp64."""
    X = bf16_bits_to_f64(X_bits)
    W = bf16_bits_to_f64(W_bits).T                       # [K, N]
    ref = X @ W
    no_bias = dict(packed, bias=np.zeros(W.shape[1]))
    Yq = layer_forward(X_bits, no_bias)["Y"]
    return float(np.linalg.norm(Yq - ref) / np.linalg.norm(ref))


def gptq_hessian(X_bits, inv_lambda):
    """H = X~^T X~ (fp64) on the calibration tokens, X~ = fl32(x * inv_lambda):
    the second moment of the smoothed activations the residual multiplies."""
    X = bf16_bits_to_f64(X_bits)
    Xh = round_f32(X * np.asarray(inv_lambda, dtype=np.float64)[None, :])
    return Xh.T @ Xh


def gptq_quantize_residual(R, H, damp=0.01):
    """GPTQ rounding of the residual R [K, N] (the review's offline procedure,
    section 8: "residual weights use GPTQ"; the published algorithm of
    Frantar et al.).  H is dampened by damp * mean(diag H) (a channel the
    calibration never activates gets H_kk = 1); U is the upper Cholesky
    factor of H^-1.  Input channels are taken in order; on entering a group
    of 64 the eq. 1 scale of every output column is taken from the current
    (updated) group; then each channel k is quantised (eq. 1 on fl32 of the
    updated value) and its error err = (w - q s) / U_kk is pushed onto the
    later channels: R[j] -= U_kj err.  Returns (codes [N, K], s_w [G, N])."""
    R = np.array(R, dtype=np.float64, copy=True)
    K, N = R.shape
    Hd = np.array(H, dtype=np.float64, copy=True)
    dead = np.diag(Hd) == 0
    Hd[dead, dead] = 1.0
    Hd += damp * np.mean(np.diag(Hd)) * np.eye(K)
    U = np.linalg.cholesky(np.linalg.inv(Hd)).T            # upper, H^-1 = U^T U
    G = K // GROUP
    codes = np.zeros((N, K), dtype=np.int64)
    s_w = np.zeros((G, N))
    for k in range(K):
        g = k // GROUP
        if k % GROUP == 0:
            _, s_w[g] = quantize_groups(round_f32(R[k:k + GROUP].T))
        s = s_w[g]
        w32 = round_f32(R[k])
        q = np.zeros(N, dtype=np.int64)
        nz = s > 0
        if np.any(nz):
            c, _ = _round_with_scale(w32[nz], s[nz])
            q[nz] = c
        codes[:, k] = q
        err = (R[k] - q * s) / U[k, k]
        R[k + 1:] -= np.outer(U[k, k + 1:], err)
    return codes, s_w


def _round_with_scale(z, s):
    """Codes of eq. 1 for values z with given scales s (exact round-half-even
    of z / s by fp64 comparisons, clamped to [-8, 7])."""
    z = np.asarray(z, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    q = np.rint(z / s)
    for _ in range(3):
        two_d = 2.0 * (z - q * s)
        q = np.where(two_d > s, q + 1, np.where(two_d < -s, q - 1, q))
    d = z - q * s
    tie = (2.0 * np.abs(d) == s) & (np.mod(q, 2) != 0)
    q = np.where(tie, q + np.sign(d), q)
    return np.clip(q, -8, 7).astype(np.int64), s


def _set_factors(p, Wt, L1, L2):
    """New protected factors for a packed layer: store them as bf16, take R
    against the stored factors and quantise it again (eqs. 10, 1)."""
    L1b = round_bf16(L1)
    L2b = round_bf16(L2)
    R, codes, s_w = residual_quantize(Wt, L1b, L2b)
    q = dict(p)
    q.update(L1=L1, L2=L2, L1b=L1b, L2b=L2b, R=R, wcodes=codes, wq=pack_nibbles(codes), s_w=s_w)
    return q


def refine_factors(p, svd=None):
    """One alternating step: the rank-r SVD of W~ - deq(Q(R)) gives the new
    factors, then R is recomputed against W~ and quantised."""
    Wt = p["Wt"]
    r = p["L1b"].shape[1]
    T = Wt - dequantize_groups(p["wcodes"], p["s_w"]).T   # deq(Q(R)) is [N, K]
    if svd is None:
        U, S, Vt = np.linalg.svd(T, full_matrices=False)
    else:
        U, S, Vt = leading_svd(T, r + 1)
    return _set_factors(p, Wt, U[:, :r] * S[None, :r], Vt[:r, :])


def _with_gptq(p, H):
    """The packed layer with its residual R quantised by GPTQ instead."""
    codes, s_w = gptq_quantize_residual(p["R"], H)
    return dict(p, wcodes=codes, wq=pack_nibbles(codes), s_w=s_w)


def pack_weights_calibrated(W_bits, X_cal_bits, rank, alphas=(0.3, 0.4, 0.5, 0.6, 0.7),
                            iters=1, bias_bits=None, lora_A_bits=None, lora_B_bits=None,
                            lora_scale=1.0, svd=None, gptq=False):
    """For every candidate alpha: smoothing, SVD, residual quantisation, then
    `iters` alternating refinements; keep the candidate with the smallest
    calibrated layer-output error (the first one on ties).  The statistics
    and the error use the calibration tokens X_cal.  gptq=True quantises
    every residual (the first and each refined one) with GPTQ on the
    calibration Hessian of the candidate's smoothed activations.  LoRA joins
    the branch afterwards, as in pack_weights.  Returns (packed, errors)."""
    a = calib_absmax(bf16_bits_to_f64(X_cal_bits))
    best, best_err, errs = None, None, []
    for alpha in alphas:
        p = pack_weights(W_bits, a, rank, alpha=alpha, svd=svd)
        H = gptq_hessian(X_cal_bits, p["inv_lambda"]) if gptq else None
        if gptq:
            p = _with_gptq(p, H)
        for _ in range(iters):
            p = refine_factors(p, svd=svd)
            if gptq:
                p = _with_gptq(p, H)
        e = layer_output_error(X_cal_bits, p, W_bits)
        errs.append(e)
        if best is None or e < best_err:
            best, best_err = dict(p, alpha=alpha), e
    p = best
    bias = np.zeros(p["N"]) if bias_bits is None else bf16_bits_to_f64(bias_bits)
    p = dict(p, bias=bias)
    if lora_A_bits is not None and lora_A_bits.shape[1] > 0:
        A = bf16_bits_to_f64(lora_A_bits)
        B = bf16_bits_to_f64(lora_B_bits)
        DA = (p["lam"][:, None] * A) * float(np.float32(lora_scale))
        p["L1b"] = np.hstack([p["L1b"], round_bf16(DA)])
        p["L2b"] = np.vstack([p["L2b"], B])
        p["rank"] = p["L1b"].shape[1]
    return p, errs


# --------------------------------------------------------------------------
# W8A8 comparator: the same two-branch layer with 8-bit operands and one
# scale per token (activations) and per output channel (residual), applied
# once (review section 8: the eight-bit setting with rank 16, dynamic
# per-token activation and per-channel weight scales; section 9.3, INT8)
# --------------------------------------------------------------------------
def quantize_rows_int8(v):
    """Symmetric int8 quantisation with one scale per row (last axis):
    s = fl32(max|v| / 127), q = round-half-even of the exact quotient v/s
    (exact fp64 comparisons, as in quantize_groups: q*s has at most 31
    significant bits), clamped to [-128, 127] (|q| <= 127 for a normal s).
    s = 0 gives codes 0.  Returns (codes int64 like v, scales [...])."""
    v = np.asarray(v, dtype=np.float64)
    m = np.max(np.abs(v), axis=-1)
    s = round_f32(m / 127.0)
    codes = np.zeros(v.shape, dtype=np.int64)
    nz = s > 0
    if np.any(nz):
        zz = v[nz]
        ss = np.broadcast_to(s[nz][..., None], zz.shape)
        q = np.rint(zz / ss)
        for _ in range(3):
            two_d = 2.0 * (zz - q * ss)
            q = np.where(two_d > ss, q + 1, np.where(two_d < -ss, q - 1, q))
        d = zz - q * ss
        tie = (2.0 * np.abs(d) == ss) & (np.mod(q, 2) != 0)
        q = np.where(tie, q + np.sign(d), q)
        codes[nz] = np.clip(q, -128, 127).astype(np.int64)
    return codes, s


def pack_weights_w8a8(W_bits, act_absmax, rank, alpha=0.5, bias_bits=None, lora_A_bits=None,
                      lora_B_bits=None, lora_scale=1.0, svd=None):
    """pack_weights' smoothing, factors and residual R, with R quantised to
    int8 per output channel (over all K): wcodes8 [N, K], s_w8 [N]."""
    p = pack_weights(W_bits, act_absmax, rank, alpha=alpha, bias_bits=bias_bits,
                     lora_A_bits=lora_A_bits, lora_B_bits=lora_B_bits, lora_scale=lora_scale,
                     svd=svd)
    codes8, s_w8 = quantize_rows_int8(round_f32(p["R"].T))
    return dict(p, wcodes8=codes8, s_w8=s_w8)


def quantize_act_w8a8(X_bits, inv_lambda, L1b):
    """x~ = fl32(x * inv_lambda), int8 codes and one scale per token, and
    the same 16-bit down-projection as quantize_act.
    Returns (codes [M, K], s_x [M], Z [M, r], xhat)."""
    X = bf16_bits_to_f64(X_bits)
    xhat = round_f32(X * np.asarray(inv_lambda, dtype=np.float64)[None, :])
    codes, s_x = quantize_rows_int8(xhat)
    r = L1b.shape[1]
    Z = round_bf16(round_bf16(xhat) @ L1b) if r else np.zeros((X.shape[0], 0))
    return codes, s_x, Z, xhat


def linear_w8a8(xcodes, s_x, Z, wcodes, s_w, L2b, bias, apply_gelu=False, rows=None, cols=None):
    """Y = s_x[i] s_w[n] sum_k q_x q_w + Z L2 + b (fp64; the integer sum is
    an fp64 matmul of integers below 2^53 in magnitude, exact), optional
    GELU, one bf16 rounding.  Returns (Y, Y_bf16)."""
    xc = np.asarray(xcodes)
    rows = np.arange(xc.shape[0]) if rows is None else np.asarray(rows)
    cols = np.arange(np.asarray(wcodes).shape[0]) if cols is None else np.asarray(cols)
    P = xc[rows].astype(np.float64) @ np.asarray(wcodes)[cols].astype(np.float64).T
    Y = (np.asarray(s_x, dtype=np.float64)[rows][:, None] *
         np.asarray(s_w, dtype=np.float64)[cols][None, :]) * P
    if np.asarray(L2b).shape[0]:
        Y += np.asarray(Z)[rows] @ np.asarray(L2b)[:, cols]
    Y += np.asarray(bias, dtype=np.float64)[cols][None, :]
    if apply_gelu:
        Y = gelu(Y)
    return Y, round_bf16(Y)


# --------------------------------------------------------------------------
# NVFP4 variant: FP4 (E2M1) codes in groups of 16 along K with FP8 (E4M3)
# group scales (review section 8: "NVFP4 uses group size 16 with FP8
# scales"; section 9.1 on the nonuniform FP4 grid).  Reading: each row (a
# token of x~, or an output column of R, over all K) also has an fp32 scale
# s = fl32(max|row| / (6 * 448)), so that the group scales use E4M3's range:
#     b = e4m3(fl32(max|group| / fl32(6 s))),  q = e2m1(z / (b s)),
# both rounded to nearest, ties to even, saturating at 448 and 6.
# --------------------------------------------------------------------------
NVFP4_GROUP = 16
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
E4M3_MAX = 448.0


def round_e4m3(t):
    """Round non-negative float64 values to FP8 E4M3 (4 significant bits,
    exponent bias 7, subnormal quantum 2^-9, largest finite 448), nearest
    with ties to even, saturating at 448.  Returns float64 values."""
    t = np.asarray(t, dtype=np.float64)
    out = np.zeros_like(t)
    pos = t > 0
    if np.any(pos):
        tp = t[pos]
        _, e = np.frexp(tp)                        # tp = m 2^e, 0.5 <= m < 1
        qexp = np.maximum(e - 4, -9)               # quantum exponent: 3 fraction bits, min 2^-9
        v = np.ldexp(np.rint(np.ldexp(tp, -qexp)), qexp)
        out[pos] = np.minimum(v, E4M3_MAX)
    return out


def e4m3_bits(v):
    """Bit patterns (uint8) of non-negative E4M3 values (as from round_e4m3)."""
    v = np.asarray(v, dtype=np.float64)
    bits = np.zeros(v.shape, dtype=np.uint8)
    nz = v > 0
    if np.any(nz):
        m, e = np.frexp(v[nz])                     # v = m 2^e
        ebias = e - 1 + 7                          # exponent field of a normal
        sub = ebias <= 0
        man = np.where(sub, np.rint(v[nz] * 2.0 ** 9), np.rint((m * 2 - 1) * 8))
        field = np.where(sub, 0, ebias)
        bits[nz] = ((field << 3) | man.astype(np.int64)).astype(np.uint8)
    return bits


def e2m1_codes(z, d):
    """FP4 E2M1 codes (bit 3 = sign, bits 0-2 = index into E2M1_VALUES) of the
    exact quotients z / d, d > 0 (float64, z / d decided by exact fp64
    comparisons of |z| with the grid midpoints times d), nearest with ties
    to the even index, saturating at 6.  A zero magnitude has no sign."""
    z = np.asarray(z, dtype=np.float64)
    d = np.broadcast_to(np.asarray(d, dtype=np.float64), z.shape)
    a = np.abs(z)
    mids = _E2M1_MIDS[None, :] * d.reshape(-1)[:, None]      # exact: <= 31 bits
    af = a.reshape(-1)
    idx = np.sum(mids < af[:, None], axis=1)
    tie = np.zeros_like(af, dtype=bool)
    ok = idx < 7
    tie[ok] = af[ok] == mids[ok, idx[ok]]
    idx = np.where(tie & (idx % 2 == 1), idx + 1, idx).reshape(z.shape)
    sign = (z < 0) & (idx > 0)
    return (idx | (sign.astype(np.int64) << 3)).astype(np.int64)


def e2m1_values(codes):
    c = np.asarray(codes, dtype=np.int64)
    v = E2M1_VALUES[c & 7]
    return np.where(c & 8, -v, v)


def quantize_nvfp4_rows(v):
    """v float64 [rows, K] of fp32 values (K % 16 == 0) -> (codes [rows, K],
    group scales b [rows, K/16] as E4M3 values, row scales s [rows])."""
    v = np.asarray(v, dtype=np.float64)
    rows, K = v.shape
    if K % NVFP4_GROUP:
        raise ValueError("K must be a multiple of 16")
    s = round_f32(np.max(np.abs(v), axis=1) / (6.0 * E4M3_MAX))
    d6 = round_f32(6.0 * s)
    g = v.reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    mg = np.max(np.abs(g), axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(d6[:, None] > 0, round_f32(mg / d6[:, None]), 0.0)
    b = round_e4m3(t)
    d = b * s[:, None]                             # exact: 4 x 24 bits
    codes = np.zeros(g.shape, dtype=np.int64)
    live = d > 0
    if np.any(live):
        codes[live] = e2m1_codes(g[live], d[live][:, None])
    return codes.reshape(rows, K), b, s


def dequantize_nvfp4(codes, b, s):
    rows, K = np.asarray(codes).shape
    v = e2m1_values(codes).reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    return (v * (np.asarray(b)[:, :, None] * np.asarray(s)[:, None, None])).reshape(rows, K)


def pack_weights_nvfp4(W_bits, act_absmax, rank, alpha=0.5, bias_bits=None, svd=None):
    """pack_weights' smoothing, factors and residual R, with R quantised by
    the NVFP4 rule per output column: wcodes4 [N, K], wb4 [N, K/16], ws4 [N]."""
    p = pack_weights(W_bits, act_absmax, rank, alpha=alpha, bias_bits=bias_bits, svd=svd)
    codes, b, s = quantize_nvfp4_rows(round_f32(p["R"].T))
    return dict(p, wcodes4=codes, wb4=b, ws4=s)


def quantize_act_nvfp4(X_bits, inv_lambda, L1b):
    """x~ = fl32(x * inv_lambda), its NVFP4 codes, group and row scales, and
    the 16-bit down-projection of quantize_act.
    Returns (codes [M, K], b [M, K/16], s [M], Z [M, r], xhat)."""
    X = bf16_bits_to_f64(X_bits)
    xhat = round_f32(X * np.asarray(inv_lambda, dtype=np.float64)[None, :])
    codes, b, s = quantize_nvfp4_rows(xhat)
    r = L1b.shape[1]
    Z = round_bf16(round_bf16(xhat) @ L1b) if r else np.zeros((X.shape[0], 0))
    return codes, b, s, Z, xhat


def linear_nvfp4(xcodes, xb, xs, Z, wcodes, wb, ws, L2b, bias, apply_gelu=False, rows=None,
                 cols=None):
    """Y = deq(X) deq(W)^T + Z L2 + b with deq = code value x group scale x
    row scale (every dequantised value is exact in fp64), fp64 sums,
    optional GELU, one bf16 rounding.  Returns (Y, Y_bf16)."""
    xc = np.asarray(xcodes)
    rows = np.arange(xc.shape[0]) if rows is None else np.asarray(rows)
    cols = np.arange(np.asarray(wcodes).shape[0]) if cols is None else np.asarray(cols)
    Xq = dequantize_nvfp4(xc[rows], np.asarray(xb)[rows], np.asarray(xs)[rows])
    Wq = dequantize_nvfp4(np.asarray(wcodes)[cols], np.asarray(wb)[cols], np.asarray(ws)[cols])
    Y = Xq @ Wq.T
    if np.asarray(L2b).shape[0]:
        Y += np.asarray(Z)[rows] @ np.asarray(L2b)[:, cols]
    Y += np.asarray(bias, dtype=np.float64)[cols][None, :]
    if apply_gelu:
        Y = gelu(Y)
    return Y, round_bf16(Y)


def two_branch_unquantized(X, lam, L1, L2, R, bias):
    """Eq. 7 with quantisation switched off, all in fp64:
    (X~ L1) L2 + X~ R + b with X~ = X D^-1 (exact-lambda smoothing)."""
    Xt = np.asarray(X, dtype=np.float64) / np.asarray(lam)[None, :]
    out = Xt @ R + np.asarray(bias)[None, :]
    if np.asarray(L1).shape[1]:
        out += (Xt @ L1) @ L2
    return out


# --------------------------------------------------------------------------
# eqs. 11-12: cost accounting of the protected branch
# --------------------------------------------------------------------------
def mac_ratio(m, n, r):
    """Low-rank MACs over dense MACs: (b m r + b r n) / (b m n) (eq. 11)."""
    return (m * r + r * n) / (m * n)


def storage_ratio(m, n, r):
    """(m n / 2 + 2 r (m + n)) / (2 m n) bytes vs bf16 (eq. 12)."""
    return (m * n / 2 + 2 * r * (m + n)) / (2 * m * n)
