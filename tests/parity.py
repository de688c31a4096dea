"""Shared parity helpers of the GPU tests: tolerances, the near-tie routing rule, token sampling.

Tolerances (fp32 output of the MoE forward against the fp64 oracle): max-abs 2e-2 and relative
Frobenius 1e-2, for bf16 inputs with fp32 accumulation. The derivation: h is rounded once to bf16
(relative 2^-9), GEMM2 sums F such terms with random signs, so the output error is about
2^-9 / sqrt(3) * rms(h) * 0.02 * sqrt(F) per expert; at the Mixtral shape that is ~3e-3 std and
~1.1e-2 at the tail, and ~1e-3 relative in the Frobenius norm. fp32 inputs run as tf32 (10-bit
mantissa) and land in the same range.
"""
import numpy as np

MAX_ABS = 2e-2
REL_FROB = 1e-2
U_FP32 = 2.0 ** -24


def rel_frob(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def fp32_dot_bound(D, absdot, safety=2.0):
    """Higham's bound gamma_D * sum|x_d w_d| for an fp32 evaluation (any order) of a dot product
    of exact inputs; `safety` covers the bias addition and FMA contraction."""
    g = D * U_FP32 / (1.0 - D * U_FP32)
    return safety * g * absdot + 4 * U_FP32 * np.abs(absdot)


def check_routing(gpu_te, oracle_te, logits, absdot, D):
    """The GPU's top-k must equal the oracle's, except where the oracle's logits are within the
    fp32 rounding bound of each other; there the GPU's order must still be consistent with some
    logits inside the bound. Returns the number of tokens that differ (all of them justified)."""
    gpu_te = np.asarray(gpu_te)
    oracle_te = np.asarray(oracle_te)
    n, k = gpu_te.shape
    E = logits.shape[1]
    b = fp32_dot_bound(D, absdot)
    diff = 0
    for t in range(n):
        if np.array_equal(gpu_te[t], oracle_te[t]):
            continue
        diff += 1
        g = gpu_te[t]
        assert len(set(g.tolist())) == k, f"token {t}: repeated expert {g}"
        assert np.all((g >= 0) & (g < E))
        lo = logits[t] - b[t]
        hi = logits[t] + b[t]
        for j in range(k - 1):
            assert hi[g[j]] >= lo[g[j + 1]], f"token {t}: order {g} not within rounding"
        rest = [e for e in range(E) if e not in set(g.tolist())]
        for e in rest:
            assert hi[g[k - 1]] >= lo[e], (
                f"token {t}: gpu {g} vs oracle {oracle_te[t]}: expert {e} beats the k-th choice "
                f"by more than the rounding bound")
    return diff


def sample_tokens(S, n, seed=0, must=()):
    rng = np.random.default_rng(seed)
    n = min(n, S)
    base = rng.choice(S, size=n, replace=False) if n < S else np.arange(S)
    toks = np.unique(np.concatenate([base, np.asarray(must, dtype=np.int64)])).astype(np.int32)
    return toks
