"""Reference GEMM on dequantized operands (oracle; test infrastructure only).

"Can you explain the role of FP8 precision in DeepSeek-V3 training", sections
"Mixed-precision framework" (the compute-heavy GEMMs run in FP8) and "Increased
accumulation precision" (partial results are promoted to FP32 at fixed intervals):
whatever the promotion interval, the exact value the GEMM approximates is the product of
the dequantized operands, C = A_dq . B_dq^T.  That product is computed here in FP64 (a
library matmul as the one step), together with the bound T = |A_dq| . |B_dq|^T used by
the acceptance test

    |C_gpu - C_ref| <= 2^-7 |C_ref| + 1e-4 T      (elementwise).

Operand conventions (both K-major, C = A . B^T, C row-major M x N):

* blockwise A: codes (M, K), decode scales s_a (K/128, >= M) with s_a[kb, m];
* blockwise B, FPROP: codes (N, K), block scales s_b (N/128, K/128) -> s_b[nb, kb];
* blockwise B, DGRAD: codes (N, K), block scales s_b (K/128, N/128) -> s_b[kb, nb];
* blockwise B, WGRAD: codes (N, K), 1x128 scales s_b (K/128, >= N) -> s_b[kb, n];
* MX: codes (R, K), E8M0 (R, K/32); per-tensor: codes and one scalar;
* NVFP4: packed E2M1 (R, K/2), E4M3 scales (R, K/16), one FP32 decode scale.
"""
import numpy as np

from .formats import e2m1_decode, e4m3_decode, e5m2_decode, e8m0_decode, unpack_e2m1

FPROP, DGRAD, WGRAD = 0, 1, 2
TOL_REL = 2.0 ** -7
TOL_ABS_T = 1e-4


def dequant_a_1x128(q, s, rows=None):
    """A_dq[m, k] = decode(q[m, k]) * s[k // 128, m] (FP64)."""
    q = np.asarray(q)
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    K = q.shape[1]
    sc = np.asarray(s, dtype=np.float64)[:, rows].T            # (len(rows), K/128)
    return e4m3_decode(q[rows]) * np.repeat(sc, 128, axis=1)[:, :K]


def dequant_b_blockwise(q, s, layout, rows=None):
    """B_dq[n, k] for the three scale modes (FP64)."""
    q = np.asarray(q)
    s = np.asarray(s, dtype=np.float64)
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    K = q.shape[1]
    kb = np.arange(K) // 128
    if layout == FPROP:
        sc = s[rows[:, None] // 128, kb[None, :]]
    elif layout == DGRAD:
        sc = s[kb[None, :], rows[:, None] // 128]
    elif layout == WGRAD:
        sc = s[kb[None, :], rows[:, None]]
    else:
        raise ValueError(layout)
    return e4m3_decode(q[rows]) * sc


def dequant_mx(q, e8m0, rows=None):
    """X_dq[r, k] = decode(q[r, k]) * 2^(e8m0[r, k // 32] - 127) (FP64)."""
    q = np.asarray(q)
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    K = q.shape[1]
    return e4m3_decode(q[rows]) * np.repeat(e8m0_decode(np.asarray(e8m0)[rows]), 32,
                                            axis=1)[:, :K]


def dequant_tensor(q, s, rows=None, fmt="e4m3"):
    """Per-tensor operand: X_dq = fmt(q) * s (FP64); fmt "e4m3" or "e5m2"."""
    q = np.asarray(q)
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    return (e4m3_decode(q[rows]) if fmt == "e4m3" else e5m2_decode(q[rows])) * float(s)


def dequant_nvfp4(packed, sf, g_dec, rows=None):
    """X_dq[r, k] = e2m1(q[r, k]) * e4m3(sf[r, k // 16]) * g_dec (FP64)."""
    packed = np.asarray(packed)
    rows = np.arange(packed.shape[0]) if rows is None else np.asarray(rows)
    codes = unpack_e2m1(packed[rows])
    K = codes.shape[1]
    return (e2m1_decode(codes) * np.repeat(e4m3_decode(np.asarray(sf)[rows]), 16,
                                           axis=1)[:, :K] * float(g_dec))


def reference(a_dq, b_dq):
    """C_ref = A_dq . B_dq^T and T = |A_dq| . |B_dq|^T, both FP64."""
    return a_dq @ b_dq.T, np.abs(a_dq) @ np.abs(b_dq).T


def tolerance_violation(c_gpu, c_ref, t):
    """Elementwise excess over the bound (<= 0 everywhere means pass)."""
    c_gpu = np.asarray(c_gpu, dtype=np.float64)
    return np.abs(c_gpu - c_ref) - (TOL_REL * np.abs(c_ref) + TOL_ABS_T * t)


def sample_tiles(M, N, n_tiles=64, seed=0, tile=128):
    """n_tiles distinct (m0, n0) output tiles, drawn with default_rng(seed + 1000)."""
    tm, tn = -(-M // tile), -(-N // tile)
    total = tm * tn
    rng = np.random.default_rng(seed + 1000)
    pick = rng.choice(total, size=min(n_tiles, total), replace=False)
    return [(int(p // tn) * tile, int(p % tn) * tile) for p in sorted(pick)]


def sample_band_tiles(M, N, n_row_bands=8, n_col_bands=8, seed=0, tile=128):
    """Every pairing of n_row_bands distinct random row bands with n_col_bands distinct
    random column bands (drawn with default_rng(seed + 2000)): n_row_bands * n_col_bands
    distinct (m0, n0) tiles whose operand bands are few, for operands that are costly to
    quantize band by band."""
    tm, tn = -(-M // tile), -(-N // tile)
    rng = np.random.default_rng(seed + 2000)
    rb = np.sort(rng.choice(tm, size=min(n_row_bands, tm), replace=False))
    cb = np.sort(rng.choice(tn, size=min(n_col_bands, tn), replace=False))
    return [(int(r) * tile, int(c) * tile) for r in rb for c in cb]


def sample_group_tiles(m_offsets, N, n_tiles=64, seed=0, tile=128):
    """Tiles across experts in proportion to their row counts, at least one per
    non-empty expert when n_tiles allows.  Returns (group, m0_global, m1_global, n0)."""
    rng = np.random.default_rng(seed + 1000)
    m_offsets = np.asarray(m_offsets, dtype=np.int64)
    G = len(m_offsets) - 1
    counts = np.diff(m_offsets)
    tn = -(-N // tile)
    cand = []
    for g in range(G):
        for mt in range(-(-int(counts[g]) // tile)):
            for nt in range(tn):
                m0 = int(m_offsets[g]) + mt * tile
                cand.append((g, m0, min(m0 + tile, int(m_offsets[g + 1])), nt * tile))
    if len(cand) <= n_tiles:
        return cand
    chosen = set()
    nonempty = [g for g in range(G) if counts[g] > 0]
    for g in nonempty[:n_tiles]:
        idx = [i for i, c in enumerate(cand) if c[0] == g]
        chosen.add(int(rng.choice(idx)))
    rest = [i for i in range(len(cand)) if i not in chosen]
    extra = rng.choice(rest, size=n_tiles - len(chosen), replace=False)
    chosen.update(int(i) for i in extra)
    return [cand[i] for i in sorted(chosen)]
