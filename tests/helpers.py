"""Shared helpers of the parity tests (comparison rules only; no method
arithmetic beyond what the oracle provides)."""
import numpy as np

import oracle

# Final output: relative Frobenius error against the oracle's bf16 Y.
Y_REL_FRO = 2e-3


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def column_signs(L1_lib_bits, L1_oracle):
    """+-1 per branch column: singular vectors are defined up to sign, so the
    library's L1 column j equals the oracle's up to a sign (decided by their
    inner product)."""
    A = oracle.bf16_bits_to_f64(L1_lib_bits)
    s = np.sign(np.sum(A * L1_oracle, axis=0))
    s[s == 0] = 1.0
    return s


def z_tolerance(xhat, L1b, K):
    """Bound for |Z_gpu - Z_oracle|: one bf16 ulp of the value plus the fp32
    accumulation error bound K 2^-24 sum_k |bf16(x~_k) L1_kj|."""
    terms = np.abs(oracle.round_bf16(xhat)) @ np.abs(L1b)
    return terms * (K * 2.0 ** -24)


def check_z(Zg_bits, Zo, xhat, L1b, signs):
    Zg = oracle.bf16_bits_to_f64(Zg_bits) * signs[None, :]
    tol = 2.0 ** -7 * np.abs(Zo) + z_tolerance(xhat, L1b, xhat.shape[1]) + 1e-30
    bad = np.abs(Zg - Zo) > tol
    assert not bad.any(), f"{bad.sum()} Z entries out of tolerance"
    return Zg
