"""Quantizers, written step by step from the pages' recipe (oracle; test infrastructure only).

Pages (cited by title and section):

* [DSV3] "Can you explain the role of FP8 precision in DeepSeek-V3 training":
  "Fine-grained quantization" - activations in 1x128 tiles, weights in 128x128 blocks,
  each with its own scale; "Online quantization" - the scale comes from the live amax of
  the tile or block, not from a history; "Unified E4M3 format" - E4M3 for every tensor.
* [NeMo] "Accelerating FP8 training performance with the NVIDIA NeMo framework":
  per-tensor scaling (the coarse recipe) and MXFP8 (blocks of 32 values).
* [NVFP4] "NVIDIA developed a method to train neural networks in 4-bit precision",
  "How it works": 4-bit values, 16x16 random Hadamard transforms on gradient inputs,
  stochastic rounding.

The pages give no formula for any scale.  Readings taken (each listed with its reason in
the design notes):

* 1x128 / 128x128 / per-tensor: amax = max |x| over the tile, block or tensor (FP32).
  amax == 0 -> sf = 1; else sf = fp32(448 / amax), and sf = FLT_MAX if that overflows.
  Codes q = E4M3_RNE_SAT(fp32(x * sf)); the stored (decode) scale is s = fp32(1 / sf).
* MX: per 32 elements, the E8M0 exponent e is the smallest integer with amax <= 448 * 2^e
  (no element saturates); amax == 0 -> e = -127; e clamped to [-127, 127]; stored code
  e + 127; q = E4M3_RNE_SAT(fp32(x * 2^-e)).
* NVFP4: G = amax of the (transformed) tensor; S_g = fp32(2688 / G) (448 * 6; G == 0 ->
  1; overflow -> FLT_MAX).  Per 16 elements: sb = E4M3_RNE_SAT(fp32(fp32(amax_b / 6) *
  S_g)); enc = 0 if sb == 0 else fp32(S_g / decode(sb)); y = fp32(x * enc); q = E2M1 of y
  by round-to-nearest-even or by stochastic rounding; stored g_dec = fp32(1 / S_g).
* NVFP4 weights for the forward path: one E4M3 scale per 16x16 block, from the amax over
  its 256 elements by the same formula, round-to-nearest-even codes, emitted rowwise and
  colwise (the same codes transposed), so fprop and dgrad read one quantized matrix.
* Delayed (per-tensor, amax history; the recipe [DSV3] "Online quantization" contrasts
  with): sf = fp32(fmt_max / max(history)) (max 0 -> 1, overflow -> FLT_MAX), fmt_max 448
  for E4M3 or 57344 for E5M2; q = FMT_RNE_SAT(fp32(x * sf)); s = fp32(1 / sf); the
  tensor's own amax is returned for the caller's history and does not affect its codes.
* Stochastic rounding: a = |y|; a >= 6 -> 6; else lo <= a < hi adjacent E2M1 values,
  p = (a - lo) / (hi - lo) (exact in FP32); r = word (idx & 3) of Philox4x32-10 with
  counter (idx >> 2 low 32 bits, idx >> 2 high 32 bits, 0, tag) and key sr_seed, where
  idx is the element's linear index in the quantized output and tag is 0 for the
  rowwise output, 1 for the colwise one; u = (r >> 8) * 2^-24; round up iff u < p.

All arithmetic that decides a code is done in FP32 (NumPy float32 is IEEE binary32 with
round-to-nearest-even and gradual underflow), the precision the GPU uses.

"Rowwise" quantizes along the last (column) axis.  "Colwise" quantizes along rows and is
returned transposed: colwise(x) == rowwise(x.T), with the transposed layout K-major in
the original row index (the wgrad operands).
"""
import numpy as np

from .formats import (E4M3_MAX, E5M2_MAX, FLT_MAX, bf16_bits_to_f32, e2m1_encode_rne, e2m1_grid_neighbours,
                      e4m3_decode, e4m3_encode, e5m2_encode, pack_e2m1)
from .philox import philox4x32_10, seed_to_key
from .rht import rht16_lastdim, rht_signs

_F448 = np.float32(448.0)
_F2688 = np.float32(2688.0)
_CHUNK = 1 << 21      # elements per row chunk, to bound temporaries


def as_f32(x):
    """BF16 bit patterns (uint16/int16) or float arrays -> float32."""
    x = np.asarray(x)
    if x.dtype in (np.uint16, np.int16):
        return bf16_bits_to_f32(x)
    return x.astype(np.float32)


def _row_chunks(R, C):
    step = max(1, _CHUNK // max(C, 1))
    for r0 in range(0, R, step):
        yield r0, min(R, r0 + step)


def e4m3_scale_from_amax(amax):
    """sf = 448 / amax in FP32 with the zero and overflow rules.  Parity unpinned for
    the zero / overflow rules (the spec's own reading); 448 / amax is pinned by the
    scaled-amax invariant."""
    amax = np.asarray(amax, dtype=np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        sf = np.where(amax == 0, np.float32(1.0), _F448 / np.where(amax == 0, 1, amax))
    sf = sf.astype(np.float32)
    return np.where(np.isinf(sf), FLT_MAX, sf).astype(np.float32)


# ------------------------------------------------------------------- 1 x 128 tiles
def quantize_1x128_rowwise(x):
    """[DSV3] "Fine-grained quantization": one scale per 1x128 tile along the last axis.

    x: (R, C) BF16 bits or float, C % 128 == 0.
    Returns q (R, C) uint8 E4M3 codes and s (C/128, R) float32 decode scales, stored
    MN-major: s[kb, r] is the scale of tile (r, kb).
    """
    x = np.asarray(x)
    R, C = x.shape
    assert C % 128 == 0
    q = np.empty((R, C), dtype=np.uint8)
    s = np.empty((C // 128, R), dtype=np.float32)
    for r0, r1 in _row_chunks(R, C):
        t = as_f32(x[r0:r1]).reshape(r1 - r0, C // 128, 128)
        amax = np.max(np.abs(t), axis=-1)
        sf = e4m3_scale_from_amax(amax)
        y = (t * sf[..., None]).astype(np.float32)
        q[r0:r1] = e4m3_encode(y).reshape(r1 - r0, C)
        s[:, r0:r1] = (np.float32(1.0) / sf).T
    return q, s


def quantize_1x128_colwise(x):
    """1x128 tiles along rows (the token dimension), output transposed: returns
    q_col (C, R) and s_col (R/128, C) == quantize_1x128_rowwise(x.T)."""
    return quantize_1x128_rowwise(np.ascontiguousarray(np.asarray(x).T))


# ------------------------------------------------------------------- 128 x 128 blocks
def quantize_128x128(w):
    """[DSV3] "Fine-grained quantization": one scale per 128x128 weight block.

    w: (K, N) BF16 bits or float, K % 128 == N % 128 == 0.
    Returns q (K, N), q_t (N, K) == q.T (the same codes) and s (N/128, K/128) float32,
    s[j, i] being the decode scale of block (rows 128i.., cols 128j..).
    """
    w = np.asarray(w)
    K, N = w.shape
    assert K % 128 == 0 and N % 128 == 0
    q = np.empty((K, N), dtype=np.uint8)
    s = np.empty((N // 128, K // 128), dtype=np.float32)
    for i in range(K // 128):
        blk = as_f32(w[128 * i:128 * (i + 1)]).reshape(128, N // 128, 128)
        amax = np.max(np.abs(blk), axis=(0, 2))                 # (N/128,)
        sf = e4m3_scale_from_amax(amax)
        y = (blk * sf[None, :, None]).astype(np.float32)
        q[128 * i:128 * (i + 1)] = e4m3_encode(y).reshape(128, N)
        s[:, i] = np.float32(1.0) / sf
    return q, np.ascontiguousarray(q.T), s


# ------------------------------------------------------------------- per tensor
def quantize_tensor(x):
    """[NeMo] per-tensor current scaling: one amax over the whole tensor.

    Returns q (R, C) uint8 and the float32 decode scale s_dec = 1 / sf.
    """
    x = np.asarray(x)
    R, C = x.shape
    amax = np.float32(0.0)
    for r0, r1 in _row_chunks(R, C):
        amax = max(amax, np.max(np.abs(as_f32(x[r0:r1]))) if r1 > r0 else 0)
    sf = e4m3_scale_from_amax(np.float32(amax))
    q = np.empty((R, C), dtype=np.uint8)
    for r0, r1 in _row_chunks(R, C):
        q[r0:r1] = e4m3_encode((as_f32(x[r0:r1]) * sf).astype(np.float32))
    return q, np.float32(np.float32(1.0) / sf)


# ------------------------------------------------------------ delayed scaling (history)
def quantize_tensor_delayed(x, amax_history, fmt="e4m3"):
    """Per-tensor delayed scaling, the recipe "Can you explain the role of FP8 precision in
    DeepSeek-V3 training" (section "Online quantization") contrasts with its own: the scale
    comes from the amaxes of previous iterations, not from the tensor being cast.

    sf = fmt_max / max(amax_history) in FP32 (max 0 -> 1, overflow -> FLT_MAX); codes
    fmt(x * sf) with saturation (values beyond the historical range clip); stored decode
    scale fp32(1 / sf).  Also returns this tensor's amax, which the caller records in the
    history for later iterations (it does not affect this cast).  fmt: "e4m3" (448) or
    "e5m2" (57344).
    """
    x = np.asarray(x)
    R, C = x.shape
    fmax = np.float32(E4M3_MAX if fmt == "e4m3" else E5M2_MAX)
    hmax = np.float32(np.max(np.asarray(amax_history, dtype=np.float32))) if np.size(amax_history) else np.float32(0)
    with np.errstate(divide="ignore", over="ignore"):
        sf = np.float32(1.0) if hmax == 0 else np.float32(fmax / hmax)
    if np.isinf(sf):
        sf = FLT_MAX
    enc = e4m3_encode if fmt == "e4m3" else e5m2_encode
    q = np.empty((R, C), dtype=np.uint8)
    amax = np.float32(0.0)
    for r0, r1 in _row_chunks(R, C):
        xf = as_f32(x[r0:r1])
        q[r0:r1] = enc((xf * sf).astype(np.float32))
        if r1 > r0:
            amax = max(amax, np.float32(np.max(np.abs(xf))))
    return q, np.float32(np.float32(1.0) / sf), np.float32(amax)


# ------------------------------------------------------------------- MX (E8M0, 32)
def mx_exponent(amax):
    """Smallest integer e with amax <= 448 * 2^e, from the FP32 bits of amax.

    With amax = 1.f * 2^E: amax / 2^(E-8) = 1.f * 2^8 fits under 448 = 1.75 * 2^8 exactly
    when the 23-bit fraction is at most 0x600000; otherwise one more power of two is
    needed.  amax == 0 -> -127.  Clamped to [-127, 127].
    """
    a = np.asarray(amax, dtype=np.float32).astype(np.float64)
    _, ex = np.frexp(a)
    E = ex.astype(np.int64) - 1
    mant23 = np.where(a > 0, (a / np.exp2(E.astype(np.float64)) - 1.0) * 2.0 ** 23, 0)
    e = E - 8 + (mant23 > 0x600000).astype(np.int64)
    e = np.where(a == 0, -127, e)
    return np.clip(e, -127, 127)


def quantize_mx_rowwise(x, block=32):
    """[NeMo] MXFP8: E8M0 scale per 32 consecutive elements along the last axis.

    Returns q (R, C) uint8 E4M3 and e8m0 (R, C/32) uint8 (code = e + 127), row-major.
    """
    x = np.asarray(x)
    R, C = x.shape
    assert C % block == 0
    q = np.empty((R, C), dtype=np.uint8)
    sc = np.empty((R, C // block), dtype=np.uint8)
    for r0, r1 in _row_chunks(R, C):
        t = as_f32(x[r0:r1]).reshape(r1 - r0, C // block, block)
        e = mx_exponent(np.max(np.abs(t), axis=-1))
        mul = np.exp2(-e.astype(np.float64)).astype(np.float32)   # exact powers of two
        q[r0:r1] = e4m3_encode((t * mul[..., None]).astype(np.float32)).reshape(r1 - r0, C)
        sc[r0:r1] = (e + 127).astype(np.uint8)
    return q, sc


def quantize_mx_colwise(x, block=32):
    """MX blocks along rows, transposed output: == quantize_mx_rowwise(x.T)."""
    return quantize_mx_rowwise(np.ascontiguousarray(np.asarray(x).T), block)


# ------------------------------------------------------------------- NVFP4
def nvfp4_global_scale(G):
    """S_g = 2688 / G in FP32 (G == 0 -> 1, overflow -> FLT_MAX).  Parity unpinned for
    the zero / overflow rules."""
    G = np.float32(G)
    if G == 0:
        return np.float32(1.0)
    with np.errstate(over="ignore"):
        sg = np.float32(_F2688 / G)
    return FLT_MAX if np.isinf(sg) else sg


def sr_words(idx, tag, sr_seed):
    """Philox word for each linear output index idx (int64 array): word idx & 3 of the call
    at counter (idx >> 2, 0, tag).  Pinned statistically (the words of the four elements of
    one call, and of neighbouring calls, give uncorrelated decisions; tags 0 and 1 give
    uncorrelated streams) and by element-wise brute force over output indices."""
    idx = np.asarray(idx, dtype=np.int64)
    blk = (idx >> 2).astype(np.uint64)
    ctr = np.stack([(blk & np.uint64(0xFFFFFFFF)).astype(np.uint32),
                    (blk >> np.uint64(32)).astype(np.uint32),
                    np.zeros(idx.shape, np.uint32),
                    np.full(idx.shape, tag, np.uint32)], axis=-1)
    out = philox4x32_10(ctr, seed_to_key(sr_seed))
    return np.take_along_axis(out, (idx & 3)[..., None], axis=-1)[..., 0]


def e2m1_encode_sr(y, words):
    """Stochastic rounding of float32 y to E2M1 with one random 32-bit word per element.

    The word -> uniform mapping (top 24 bits, round up iff u < p) is a reading: it is pinned
    for unbiasedness over 10^6 draws; which word an element takes is pinned in sr_words.
    """
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y)
    lo, hi, i_lo = e2m1_grid_neighbours(np.minimum(a, np.float32(5.999)).astype(np.float64))
    lo32 = lo.astype(np.float32)
    p = ((a - lo32) / (hi - lo).astype(np.float32)).astype(np.float32)
    u = ((np.asarray(words, np.uint32) >> np.uint32(8)).astype(np.float32)
         * np.float32(2.0 ** -24))
    code = np.where(a >= np.float32(6.0), 7, i_lo + (u < p).astype(np.int64))
    return (code | (np.signbit(y).astype(np.int64) << 3)).astype(np.uint8)


def quantize_nvfp4_rowwise(x, rht=False, rht_seed=0, sr=False, sr_seed=0, tag=0,
                           rows=None):
    """[NVFP4] E2M1 values, one E4M3 scale per 16 elements along the last axis, one FP32
    per-tensor decode scale; optional 16x16 RHT along the same axis; optional SR.

    x: (R, C), C % 16 == 0.  ``rows`` (optional) restricts the *outputs* to a subset of
    row indices (the global amax still covers the whole tensor), for sampled checks.
    Returns q (len(rows), C/2) packed uint8 (even element in the low nibble),
    sf (len(rows), C/16) uint8 E4M3 codes (row-major) and g_dec (float32).
    """
    x = np.asarray(x)
    R, C = x.shape
    assert C % 16 == 0
    signs = rht_signs(rht_seed) if rht else None

    def transformed(r0, r1):
        v = as_f32(x[r0:r1])
        return rht16_lastdim(v, signs) if rht else v

    G = np.float32(0.0)
    for r0, r1 in _row_chunks(R, C):
        if r1 > r0:
            G = max(G, np.float32(np.max(np.abs(transformed(r0, r1)))))
    S_g = nvfp4_global_scale(G)
    rows = np.arange(R) if rows is None else np.asarray(rows, dtype=np.int64)
    q = np.empty((len(rows), C // 2), dtype=np.uint8)
    sfo = np.empty((len(rows), C // 16), dtype=np.uint8)
    step = max(1, _CHUNK // max(C, 1))
    for i0 in range(0, len(rows), step):
        rr = rows[i0:i0 + step]
        v = as_f32(x[rr])
        if rht:
            v = rht16_lastdim(v, signs)
        t = v.reshape(len(rr), C // 16, 16)
        amax_b = np.max(np.abs(t), axis=-1)
        sb = e4m3_encode(((amax_b / np.float32(6.0)).astype(np.float32) * S_g)
                         .astype(np.float32))
        dec = e4m3_decode(sb).astype(np.float32)
        with np.errstate(divide="ignore"):
            enc = np.where(sb == 0, np.float32(0.0),
                           (S_g / np.where(sb == 0, np.float32(1.0), dec)).astype(np.float32))
        y = (t * enc.astype(np.float32)[..., None]).astype(np.float32).reshape(len(rr), C)
        if sr:
            idx = rr[:, None].astype(np.int64) * C + np.arange(C, dtype=np.int64)[None, :]
            codes = e2m1_encode_sr(y, sr_words(idx, tag, sr_seed))
        else:
            codes = e2m1_encode_rne(y)
        q[i0:i0 + len(rr)] = pack_e2m1(codes)
        sfo[i0:i0 + len(rr)] = sb
    return q, sfo, np.float32(np.float32(1.0) / S_g)


def quantize_nvfp4_colwise(x, rht=False, rht_seed=0, sr=False, sr_seed=0, rows=None):
    """NVFP4 along rows (tokens), output transposed (C, R/2 packed), tag 1 for SR."""
    return quantize_nvfp4_rowwise(np.ascontiguousarray(np.asarray(x).T), rht, rht_seed,
                                  sr, sr_seed, tag=1, rows=rows)


def quantize_nvfp4_2d(x, amax=None):
    """NVFP4 weights with one E4M3 scale per 16x16 block, emitted in both operand layouts.

    [NVFP4] "How it works" fixes the per-16 E4M3 scales and the per-tensor FP32 scale but
    not how a weight tensor serves both the forward GEMM (quantized along one axis) and the
    backward-data GEMM (along the other).  Reading taken: the 16 x 16 elements of a block
    share one scale, computed as for a 16-element group with the amax over all 256, and the
    codes are round-to-nearest-even (no transform, no stochastic rounding: these are
    weights, not gradient inputs).  The rowwise and colwise outputs then hold the same codes
    transposed, so both dequantize to one matrix.

    x: (R, C) with R % 16 == C % 16 == 0; ``amax`` (optional) is the global amax G when x
    is a 16-aligned sub-rectangle of a larger tensor (sampled checks).
    Returns q_row (R, C/2), sf_row (R, C/16), q_col (C, R/2), sf_col (C, R/16) (E4M3
    scale codes, row-major, each block's code repeated over its 16 rows or columns) and
    g_dec = fp32(1 / S_g).
    """
    v = as_f32(x)
    R, C = v.shape
    assert R % 16 == 0 and C % 16 == 0
    G = np.float32(np.max(np.abs(v))) if amax is None else np.float32(amax)
    if R * C == 0:
        G = np.float32(0.0) if amax is None else G
    S_g = nvfp4_global_scale(G)
    blocks = v.reshape(R // 16, 16, C // 16, 16)
    amax_b = np.max(np.abs(blocks), axis=(1, 3)) if R * C else np.zeros((R // 16, C // 16), np.float32)
    sb = e4m3_encode(((amax_b / np.float32(6.0)).astype(np.float32) * S_g).astype(np.float32))
    dec = e4m3_decode(sb).astype(np.float32)
    with np.errstate(divide="ignore"):
        enc = np.where(sb == 0, np.float32(0.0),
                       (S_g / np.where(sb == 0, np.float32(1.0), dec)).astype(np.float32)).astype(np.float32)
    y = (blocks * enc[:, None, :, None]).astype(np.float32).reshape(R, C)
    codes = e2m1_encode_rne(y)
    q_row = pack_e2m1(codes)
    q_col = pack_e2m1(np.ascontiguousarray(codes.T))
    sf_row = np.repeat(sb, 16, axis=0).astype(np.uint8)
    sf_col = np.repeat(np.ascontiguousarray(sb.T), 16, axis=0).astype(np.uint8)
    return q_row, sf_row, q_col, sf_col, np.float32(np.float32(1.0) / S_g)


# ------------------------------------------------------------------- scale layouts
def sf_tiled_size(rows, sf_cols):
    """Bytes of the MMA-tiled scale layout: rows padded to 128, scale columns to 4."""
    return (-(-rows // 128) * 128) * (-(-sf_cols // 4) * 4)


def sf_tiled_offset(r, c, sf_cols):
    """Byte offset of scale (row r, scale column c) in the MMA-tiled layout.

    The tensor-core block-scaled MMA reads its scale factors from tensor memory with
    the 128 rows of a tile in four 32-row groups, one 32-bit column per group holding
    four consecutive K-block scales (the scale-factor layout of the block-scaled
    tcgen05.mma in the PTX ISA).  The matching memory image, per 128 rows x 4 scale
    columns, is 512 contiguous bytes: row r % 32 at 16 bytes, group (r % 128) / 32 at 4
    bytes, scale column c % 4 at 1 byte.  Atoms run along the scale columns first.
    Parity unpinned as a layout; the MX and NVFP4 GEMM parity tests exercise it.
    """
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    s4 = -(-sf_cols // 4)
    return (((r // 128) * s4 + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4
            + (c % 4))


def sf_to_tiled(sf):
    """(rows, sf_cols) scale bytes -> flat MMA-tiled image (padding bytes are 0)."""
    sf = np.asarray(sf, dtype=np.uint8)
    R, S = sf.shape
    out = np.zeros(sf_tiled_size(R, S), dtype=np.uint8)
    rr, cc = np.meshgrid(np.arange(R), np.arange(S), indexing="ij")
    out[sf_tiled_offset(rr, cc, S)] = sf
    return out


def sf_from_tiled(flat, rows, sf_cols):
    """Inverse of sf_to_tiled."""
    rr, cc = np.meshgrid(np.arange(rows), np.arange(sf_cols), indexing="ij")
    return np.asarray(flat, dtype=np.uint8)[sf_tiled_offset(rr, cc, sf_cols)]
