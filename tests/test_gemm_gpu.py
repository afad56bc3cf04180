"""Block-scaled GEMMs vs the CPU oracle, through the C ABI.

The GPU GEMM consumes operands produced by the GPU quantize kernels (bit-exact with the
oracle, tested separately); the oracle quantizes the same BF16 inputs itself and computes
the FP64 product of its dequantized operands.  Acceptance, elementwise:
    |C_gpu - C_ref| <= 2^-7 |C_ref| + 1e-4 (|A_dq| |B_dq|^T)
on every element of small shapes (ragged M/N tails, several tiles, many K chunks, more
tiles than SMs) and on 64 sampled 128x128 tiles of the full-size workloads."""
import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import gemm as G
from oracle import quant as Q

pytestmark = pytest.mark.gpu


def host(t):
    return t.detach().cpu().numpy()


def f32bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def check(c_gpu, c_ref, t, what):
    got = host(c_gpu.float()).astype(np.float64) if isinstance(c_gpu, torch.Tensor) else c_gpu
    v = G.tolerance_violation(got, c_ref, t)
    worst = float(v.max())
    if worst > 0:
        i = np.unravel_index(int(np.argmax(v)), v.shape)
        raise AssertionError(f"{what}: {int((v > 0).sum())} elements outside tolerance; worst at {i}: "
                             f"gpu={got[i]} ref={c_ref[i]} T={t[i]}")


def bf(shape, sigma, seed, frac=0.0, fac=1.0):
    return workloads.normal_bf16(shape, sigma, seed, frac, fac)


# ----------------------------------------------------------------------------- blockwise
@pytest.mark.parametrize("M,K,N", [(256, 512, 256), (300, 384, 384), (256, 4096, 512), (1, 128, 128)])
def test_blockwise_fprop(cuda_lib, M, K, N):
    fq = cuda_lib
    X, W = bf((M, K), 1.0, M + K, 1e-3, 50.0), bf((K, N), 0.02, K + N)
    qx = fq.quantize_1x128(X.cuda())
    qw = fq.quantize_128x128(W.cuda())
    c = fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qx["s_row"], b_scale=qw["s"])
    assert fq.device_status() == 0
    ox, osx = Q.quantize_1x128_rowwise(workloads.bf16_bits(X))
    _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(W))
    ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(owt, osw, G.FPROP))
    check(c, ref, t, "fprop")


def test_tiny_config_end_to_end(cuda_lib):
    """The tiny blockwise configuration exactly as specified (A 256x512 N(0,1) with 0.1% x100
    outliers, B 512x256 N(0,0.02), seed 0): quantized codes and scales bit-exact, and every
    element of C = A.B within the tolerance."""
    fq = cuda_lib
    d = workloads.tiny()
    A, B = d["A"], d["B"]
    qa = fq.quantize_1x128(A.cuda())
    qb = fq.quantize_128x128(B.cuda())
    c = fq.gemm(qa["q_row"], qb["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qa["s_row"], b_scale=qb["s"])
    assert fq.device_status() == 0
    oa, osa = Q.quantize_1x128_rowwise(workloads.bf16_bits(A))
    _, obt, osb = Q.quantize_128x128(workloads.bf16_bits(B))
    assert np.array_equal(host(qa["q_row"]), oa)
    assert np.array_equal(host(qa["s_row"]).view(np.uint32), osa.astype(np.float32).view(np.uint32))
    assert np.array_equal(host(qb["q_t"]), obt)
    assert np.array_equal(host(qb["s"]).view(np.uint32), osb.astype(np.float32).view(np.uint32))
    ref, t = G.reference(G.dequant_a_1x128(oa, osa), G.dequant_b_blockwise(obt, osb, G.FPROP))
    assert c.shape == (256, 256)
    check(c, ref, t, "tiny fprop")


@pytest.mark.parametrize("M,Kw,Nw", [(300, 384, 512), (256, 256, 1024)])
def test_blockwise_dgrad(cuda_lib, M, Kw, Nw):
    """dX = dY . W^T with W (Kw x Nw): GEMM N = Kw, K = Nw, B = W's K x N codes."""
    fq = cuda_lib
    dY, W = bf((M, Nw), 1e-3, M + Nw), bf((Kw, Nw), 0.02, Kw * 3 + Nw)
    qd = fq.quantize_1x128(dY.cuda())
    qw = fq.quantize_128x128(W.cuda())
    c = fq.gemm(qd["q_row"], qw["q"], fq.FP8Q_BLOCKWISE, fq.FP8Q_DGRAD, a_scale=qd["s_row"], b_scale=qw["s"],
                ld_sb=Kw // 128)
    od, osd = Q.quantize_1x128_rowwise(workloads.bf16_bits(dY))
    ow, _, osw = Q.quantize_128x128(workloads.bf16_bits(W))
    ref, t = G.reference(G.dequant_a_1x128(od, osd), G.dequant_b_blockwise(ow, osw, G.DGRAD))
    check(c, ref, t, "dgrad")


@pytest.mark.parametrize("layout", ["wgrad", "fprop"])
def test_blockwise_fp32_accumulate(cuda_lib, layout):
    """FP32 main-gradient update: C_out = fp32(C_in + A.B^T) with the FP32 sum unrounded to
    BF16.  Checked elementwise: (C_out - C_in) against the oracle product within the GEMM
    tolerance, plus half an FP32 ulp of C_out for the final addition."""
    fq = cuda_lib
    if layout == "wgrad":
        T, Kf, N = 256, 208, 400                      # tokens, output rows (M), output cols
        X, dY = bf((T, Kf), 1.0, 61, 1e-3, 50.0), bf((T, N), 1e-3, 62)
        qx = fq.quantize_1x128(X.cuda(), rowwise=False, colwise=True)
        qd = fq.quantize_1x128(dY.cuda(), rowwise=False, colwise=True)
        a, b, sa, sb, L, ld_sb = qx["q_col"], qd["q_col"], qx["s_col"], qd["s_col"], fq.FP8Q_WGRAD, None
        ox, osx = Q.quantize_1x128_colwise(workloads.bf16_bits(X))
        od, osd = Q.quantize_1x128_colwise(workloads.bf16_bits(dY))
        ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(od, osd, G.WGRAD))
        M = Kf
    else:
        M, K, N = 300, 384, 384
        X, W = bf((M, K), 1.0, 63, 1e-3, 50.0), bf((K, N), 0.02, 64)
        qx = fq.quantize_1x128(X.cuda())
        qw = fq.quantize_128x128(W.cuda())
        a, b, sa, sb, L, ld_sb = qx["q_row"], qw["q_t"], qx["s_row"], qw["s"], fq.FP8Q_FPROP, None
        ox, osx = Q.quantize_1x128_rowwise(workloads.bf16_bits(X))
        _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(W))
        ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(owt, osw, G.FPROP))
    g = torch.Generator().manual_seed(65)
    c_in = (torch.randn((M, N), generator=g, dtype=torch.float64) * float(np.abs(ref).mean() + 1e-30)).float()
    c = c_in.cuda().clone()
    fq.gemm(a, b, fq.FP8Q_BLOCKWISE, L, a_scale=sa, b_scale=sb, ld_sb=ld_sb, out=c, accumulate_fp32=True)
    assert fq.device_status() == 0
    got = host(c).astype(np.float64)
    cin = c_in.numpy().astype(np.float64)
    excess = G.tolerance_violation(got - cin, ref, t) - np.abs(got) * 2.0 ** -24
    assert float(excess.max()) <= 0, f"{int((excess > 0).sum())} elements outside tolerance"


def _fused_quant_checks(fq, c, q_out, s_out, ref, t, what):
    """The fused 1x128 output quantization (1) equals the standalone 1x128 quantizer run on the
    same BF16 output, bit for bit, and (2) dequantizes to the oracle's product within the GEMM
    tolerance plus E4M3's rounding bound (half an ulp: 2^-4 relative for normal codes, 2^-10
    times the decode scale below them), with decode scales within the GEMM tolerance of the
    oracle's amax / 448 per 128-column group."""
    M, N = ref.shape
    qs = fq.quantize_1x128(c, rowwise=True, colwise=False)
    assert np.array_equal(host(q_out), host(qs["q_row"])), f"{what}: codes differ from the 1x128 quantizer"
    assert np.array_equal(f32bits(host(s_out)), f32bits(host(qs["s_row"])[:, :M])), f"{what}: scales differ"
    q = host(q_out)
    s = host(s_out).astype(np.float64)                       # (N/128, M)
    deq = F.e4m3_decode(q).astype(np.float64) * np.repeat(s.T, 128, axis=1)
    g_ref = np.abs(ref).reshape(M, N // 128, 128).max(axis=2)
    g_t = t.reshape(M, N // 128, 128).max(axis=2)
    s_bound = np.repeat((g_ref + g_t) / 448.0 * (1 + 2.0 ** -20), 128, axis=1)
    bound = t + 2.0 ** -4 * (np.abs(ref) + t) + 2.0 ** -10 * s_bound
    excess = np.abs(deq - ref) - bound
    assert float(excess.max()) <= 0, f"{what}: {int((excess > 0).sum())} dequantized codes outside the bound"
    s_ref = g_ref.T / 448.0
    assert np.all(np.abs(s - s_ref) <= (2.0 ** -7 * s_ref + g_t.T / 448.0) * 1.01 + 1e-30), f"{what}: scales"


@pytest.mark.parametrize("M,K,N", [(300, 512, 640), (256, 384, 256), (1, 1024, 128)])
def test_blockwise_fprop_with_fused_output_quantization(cuda_lib, M, K, N):
    """fprop whose epilogue also emits the next layer's 1x128 E4M3 codes and scales of Y."""
    fq = cuda_lib
    X, W = bf((M, K), 1.0, 71 + M, 1e-3, 50.0), bf((K, N), 0.02, 72 + N)
    qx = fq.quantize_1x128(X.cuda())
    qw = fq.quantize_128x128(W.cuda())
    q_out = torch.empty((M, N), dtype=torch.uint8, device="cuda")
    s_out = torch.empty((N // 128, M), dtype=torch.float32, device="cuda")
    c = fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qx["s_row"], b_scale=qw["s"],
                q_out=q_out, s_out=s_out)
    assert fq.device_status() == 0
    ox, osx = Q.quantize_1x128_rowwise(workloads.bf16_bits(X))
    _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(W))
    ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(owt, osw, G.FPROP))
    check(c, ref, t, "fprop (fused quantization)")
    _fused_quant_checks(fq, c, q_out, s_out, ref, t, "fprop")


def test_blockwise_dgrad_and_wgrad_with_fused_output_quantization(cuda_lib):
    fq = cuda_lib
    M, Kw, Nw = 256, 384, 512            # dgrad: dY (M x Nw) . W^T -> (M x Kw)
    W, dY = bf((Kw, Nw), 0.02, 81), bf((M, Nw), 1e-3, 82)
    qw = fq.quantize_128x128(W.cuda())
    qd = fq.quantize_1x128(dY.cuda())
    q_out = torch.empty((M, Kw), dtype=torch.uint8, device="cuda")
    s_out = torch.empty((Kw // 128, M), dtype=torch.float32, device="cuda")
    c = fq.gemm(qd["q_row"], qw["q"], fq.FP8Q_BLOCKWISE, fq.FP8Q_DGRAD, a_scale=qd["s_row"], b_scale=qw["s"],
                ld_sb=(Kw + 127) // 128, q_out=q_out, s_out=s_out)
    od, osd = Q.quantize_1x128_rowwise(workloads.bf16_bits(dY))
    ow, _, osw = Q.quantize_128x128(workloads.bf16_bits(W))
    ref, t = G.reference(G.dequant_a_1x128(od, osd), G.dequant_b_blockwise(ow, osw, G.DGRAD))
    check(c, ref, t, "dgrad (fused quantization)")
    _fused_quant_checks(fq, c, q_out, s_out, ref, t, "dgrad")
    T, Kf, N = 512, 256, 384             # wgrad: X^T . dY over T tokens -> (Kf x N)
    X, dY2 = bf((T, Kf), 1.0, 83, 1e-3, 50.0), bf((T, N), 1e-3, 84)
    qx = fq.quantize_1x128(X.cuda(), rowwise=False, colwise=True)
    qd2 = fq.quantize_1x128(dY2.cuda(), rowwise=False, colwise=True)
    q_out = torch.empty((Kf, N), dtype=torch.uint8, device="cuda")
    s_out = torch.empty((N // 128, Kf), dtype=torch.float32, device="cuda")
    c = fq.gemm(qx["q_col"], qd2["q_col"], fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, a_scale=qx["s_col"],
                b_scale=qd2["s_col"], q_out=q_out, s_out=s_out)
    ox, osx = Q.quantize_1x128_colwise(workloads.bf16_bits(X))
    od2, osd2 = Q.quantize_1x128_colwise(workloads.bf16_bits(dY2))
    ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(od2, osd2, G.WGRAD))
    check(c, ref, t, "wgrad (fused quantization)")
    _fused_quant_checks(fq, c, q_out, s_out, ref, t, "wgrad")
    assert fq.device_status() == 0


@pytest.mark.parametrize("T,Kf,N", [(256, 208, 400), (1024, 256, 512)])
def test_blockwise_wgrad(cuda_lib, T, Kf, N):
    """dW = X^T . dY: both operands 1x128 along tokens (colwise, transposed)."""
    fq = cuda_lib
    X, dY = bf((T, Kf), 1.0, T + Kf, 1e-3, 50.0), bf((T, N), 1e-3, 2 * T + N)
    qx = fq.quantize_1x128(X.cuda(), rowwise=False, colwise=True)
    qd = fq.quantize_1x128(dY.cuda(), rowwise=False, colwise=True)
    c = fq.gemm(qx["q_col"], qd["q_col"], fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, a_scale=qx["s_col"],
                b_scale=qd["s_col"])
    ox, osx = Q.quantize_1x128_colwise(workloads.bf16_bits(X))
    od, osd = Q.quantize_1x128_colwise(workloads.bf16_bits(dY))
    ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(od, osd, G.WGRAD))
    check(c, ref, t, "wgrad")


@pytest.mark.parametrize("layout", ["fprop", "dgrad", "wgrad", "wgrad_acc32"])
def test_blockwise_partial_last_wave(cuda_lib, layout):
    """80 output tiles of 256 x 256 on the persistent grid (74 CTA pairs on 148 SMs): a second,
    mostly empty wave, in every layout and the FP32-accumulate epilogue.  Every element is
    checked against the oracle."""
    fq = cuda_lib
    M, N, K = 2048, 2560, 1024
    if layout == "fprop":
        X, W = bf((M, K), 1.0, 91, 1e-3, 50.0), bf((K, N), 0.02, 92)
        qx, qw = fq.quantize_1x128(X.cuda()), fq.quantize_128x128(W.cuda())
        c = fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qx["s_row"], b_scale=qw["s"])
        ox, osx = Q.quantize_1x128_rowwise(workloads.bf16_bits(X))
        _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(W))
        ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(owt, osw, G.FPROP))
        check(c, ref, t, "fprop, partial last wave")
    elif layout == "dgrad":
        dY, W = bf((M, K), 1e-3, 93), bf((N, K), 0.02, 94)          # W: N x K codes read along N
        qd, qw = fq.quantize_1x128(dY.cuda()), fq.quantize_128x128(W.cuda())
        c = fq.gemm(qd["q_row"], qw["q"], fq.FP8Q_BLOCKWISE, fq.FP8Q_DGRAD, a_scale=qd["s_row"], b_scale=qw["s"],
                    ld_sb=N // 128)
        od, osd = Q.quantize_1x128_rowwise(workloads.bf16_bits(dY))
        ow, _, osw = Q.quantize_128x128(workloads.bf16_bits(W))
        ref, t = G.reference(G.dequant_a_1x128(od, osd), G.dequant_b_blockwise(ow, osw, G.DGRAD))
        check(c, ref, t, "dgrad, partial last wave")
    else:
        X, dY = bf((K, M), 1.0, 95, 1e-3, 50.0), bf((K, N), 1e-3, 96)   # K tokens
        qx = fq.quantize_1x128(X.cuda(), rowwise=False, colwise=True)
        qd = fq.quantize_1x128(dY.cuda(), rowwise=False, colwise=True)
        ox, osx = Q.quantize_1x128_colwise(workloads.bf16_bits(X))
        od, osd = Q.quantize_1x128_colwise(workloads.bf16_bits(dY))
        ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(od, osd, G.WGRAD))
        if layout == "wgrad":
            c = fq.gemm(qx["q_col"], qd["q_col"], fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, a_scale=qx["s_col"],
                        b_scale=qd["s_col"])
            check(c, ref, t, "wgrad, partial last wave")
        else:
            c_in = torch.full((M, N), 0.5, dtype=torch.float32)
            c = c_in.cuda()
            fq.gemm(qx["q_col"], qd["q_col"], fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, a_scale=qx["s_col"],
                    b_scale=qd["s_col"], out=c, accumulate_fp32=True)
            got = host(c).astype(np.float64)
            excess = G.tolerance_violation(got - 0.5, ref, t) - np.abs(got) * 2.0 ** -24
            assert float(excess.max()) <= 0, f"{int((excess > 0).sum())} elements outside tolerance"
    assert fq.device_status() == 0


def _pairs():
    return torch.cuda.get_device_properties(0).multi_processor_count // 2


def _split_tail_plan(M, N, K, pairs):
    """The launcher's split of the last wave, restated: 256 x 256 pair tiles in its raster
    order (groups of row tiles sweeping the columns when M <= N, else groups of column tiles
    sweeping the rows, each group about 40 MB of the resident operand); the last
    tiles % pairs tiles are split into s = min(pairs // tail, (K / 128) // 4) K ranges when they
    fill at most half a wave, s >= 2 and the split saves at least 16 of the K / 128 chunks.
    Returns the (row, column) origins of the split tiles and the workspace bytes (0: no split)."""
    tm, tn = -(-M // 256), -(-N // 256)
    tiles = tm * tn
    tail = tiles % pairs
    if tail == 0 or 2 * tail > pairs:
        return [], 0
    kb = K // 128
    s = min(pairs // tail, kb // 4)
    if s < 2 or kb - -(-kb // s) < 16:
        return [], 0
    g = (40 << 20) // (256 * K)
    out = []
    for t in range(tiles - tail, tiles):
        if M <= N:
            gm = max(1, min(g, tm))
            per = gm * tn
            grp, loc = divmod(t, per)
            first = grp * gm
            gsz = min(tm - first, gm)
            rt, nt = first + loc % gsz, loc // gsz
        else:
            gn = max(1, min(g, tn))
            per = gn * tm
            grp, loc = divmod(t, per)
            first = grp * gn
            gsz = min(tn - first, gn)
            nt, rt = first + loc % gsz, loc // gsz
        out.append((rt * 256, nt * 256))
    return out, tail * s * 256 * 256 * 4


@pytest.mark.parametrize("layout", ["fprop", "dgrad", "wgrad", "wgrad_acc32"])
def test_blockwise_split_last_wave(cuda_lib, layout):
    """One full wave plus 4 tiles (6 row tiles, the last 240 rows; 13 column tiles, the last
    128 wide; 74 pairs): the 4 tiles run as 12 K ranges of 4 chunks each, after the whole
    tiles in the same launch, with FP32 partial sums in a workspace, in every layout and with
    FP32 accumulation into C.  Every element is checked against the oracle, with and without
    the split; the split result is the same on a second run."""
    fq = cuda_lib
    pairs = _pairs()
    tn = -(-(pairs + 4) // 6)
    M, N, K = 6 * 256 - 16, tn * 256 - 128, 6144     # M % 16 == 0: wgrad's colwise quantization
    tiles, nbytes = _split_tail_plan(M, N, K, pairs)
    assert nbytes > 0 and len(tiles) == 6 * tn - pairs
    acc32 = layout == "wgrad_acc32"
    L = {"fprop": fq.FP8Q_FPROP, "dgrad": fq.FP8Q_DGRAD, "wgrad": fq.FP8Q_WGRAD, "wgrad_acc32": fq.FP8Q_WGRAD}[layout]
    assert fq.gemm_workspace_bytes(M, N, K, fq.FP8Q_BLOCKWISE, L, accumulate_fp32=acc32) == nbytes
    c_in = torch.full((M, N), 0.5, dtype=torch.float32, device="cuda")
    if layout == "fprop":
        X, W = bf((M, K), 1.0, 71, 1e-3, 50.0), bf((K, N), 0.02, 72)
        qx, qw = fq.quantize_1x128(X.cuda()), fq.quantize_128x128(W.cuda())
        run = lambda split: fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, L, a_scale=qx["s_row"],  # noqa: E731
                                    b_scale=qw["s"], split_tail=split)
        ox, osx = Q.quantize_1x128_rowwise(workloads.bf16_bits(X))
        _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(W))
        ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(owt, osw, G.FPROP))
    elif layout == "dgrad":
        dY, W = bf((M, K), 1e-3, 73), bf((N, K), 0.02, 74)
        qd, qw = fq.quantize_1x128(dY.cuda()), fq.quantize_128x128(W.cuda())
        run = lambda split: fq.gemm(qd["q_row"], qw["q"], fq.FP8Q_BLOCKWISE, L, a_scale=qd["s_row"],  # noqa: E731
                                    b_scale=qw["s"], ld_sb=N // 128, split_tail=split)
        od, osd = Q.quantize_1x128_rowwise(workloads.bf16_bits(dY))
        ow, _, osw = Q.quantize_128x128(workloads.bf16_bits(W))
        ref, t = G.reference(G.dequant_a_1x128(od, osd), G.dequant_b_blockwise(ow, osw, G.DGRAD))
    else:
        X, dY = bf((K, M), 1.0, 75, 1e-3, 50.0), bf((K, N), 1e-3, 76)   # K tokens
        qx = fq.quantize_1x128(X.cuda(), rowwise=False, colwise=True)
        qd = fq.quantize_1x128(dY.cuda(), rowwise=False, colwise=True)
        run = lambda split: fq.gemm(qx["q_col"], qd["q_col"], fq.FP8Q_BLOCKWISE, L, a_scale=qx["s_col"],  # noqa: E731
                                    b_scale=qd["s_col"], split_tail=split,
                                    out=c_in.clone() if acc32 else None, accumulate_fp32=acc32)
        ox, osx = Q.quantize_1x128_colwise(workloads.bf16_bits(X))
        od, osd = Q.quantize_1x128_colwise(workloads.bf16_bits(dY))
        ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(od, osd, G.WGRAD))
    c_split = run(True)
    c_again = run(True)
    c_whole = run(False)
    assert fq.device_status() == 0
    for c, what in ((c_split, "split last wave"), (c_whole, "unsplit")):
        if acc32:   # C_out - 0.5 against the product, plus half an FP32 ulp for the one addition
            got = host(c).astype(np.float64)
            excess = G.tolerance_violation(got - 0.5, ref, t) - np.abs(got) * 2.0 ** -24
            assert float(excess.max()) <= 0, f"{layout}, {what}: {int((excess > 0).sum())} elements outside"
        else:
            check(c, ref, t, f"{layout}, {what}")
    bits = torch.int32 if acc32 else torch.int16
    assert torch.equal(c_split.view(bits), c_again.view(bits)), "split result not repeatable"
    # outside the split tiles the two schedules run the same kernel on the same data
    mask = torch.ones((M, N), dtype=torch.bool)
    for m0, n0 in tiles:
        mask[m0:m0 + 256, n0:n0 + 256] = False
    assert torch.equal(c_split.cpu()[mask].view(bits), c_whole.cpu()[mask].view(bits))


def test_llama8b_split_last_wave_tiles_fullsize(cuda_lib):
    """At the bench's sizes fprop (1792 tiles: 24 waves + 16, 32 chunks cut 4 ways) and wgrad
    (896: 12 waves + 8, 64 chunks cut 9 ways) split their last wave; dgrad (512: 6 waves + 68)
    does not.  Every element of every split tile is checked against the oracle."""
    fq = cuda_lib
    pairs = _pairs()
    assert fq.gemm_workspace_bytes(8192, 4096, 14336, fq.FP8Q_BLOCKWISE, fq.FP8Q_DGRAD) == 0
    d = workloads.llama8b(device="cuda")
    X, W, dY = d["X"], d["W"], d["dY"]
    Xb, Wb, dYb = workloads.bf16_bits(X), workloads.bf16_bits(W), workloads.bf16_bits(dY)
    # FPROP (8192, 4096, 14336)
    tiles, nb = _split_tail_plan(8192, 14336, 4096, pairs)
    assert nb > 0 and len(tiles) == 1792 % pairs
    assert fq.gemm_workspace_bytes(8192, 14336, 4096, fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP) == nb
    qx = fq.quantize_1x128(X, rowwise=True, colwise=True)
    qw = fq.quantize_128x128(W)
    c = host(fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qx["s_row"],
                     b_scale=qw["s"]).float())
    for m0, n0 in tiles:
        for r in (m0, m0 + 128):
            oa, sa = Q.quantize_1x128_rowwise(Xb[r:r + 128])
            for q in (n0, n0 + 128):
                _, owt, sw = Q.quantize_128x128(Wb[:, q:q + 128])
                ref, t = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
                check(c[r:r + 128, q:q + 128].astype(np.float64), ref, t, f"fprop split tile {r},{q}")
    # WGRAD (4096, 8192, 14336)
    tiles, nb = _split_tail_plan(4096, 14336, 8192, pairs)
    assert nb > 0 and len(tiles) == 896 % pairs
    assert fq.gemm_workspace_bytes(4096, 14336, 8192, fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD) == nb
    qd = fq.quantize_1x128(dY, rowwise=False, colwise=True)
    c = host(fq.gemm(qx["q_col"], qd["q_col"], fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, a_scale=qx["s_col"],
                     b_scale=qd["s_col"]).float())
    for m0, n0 in tiles:
        for r in (m0, m0 + 128):
            oa, sa = Q.quantize_1x128_colwise(Xb[:, r:r + 128])
            for q in (n0, n0 + 128):
                ob, sb = Q.quantize_1x128_colwise(dYb[:, q:q + 128])
                ref, t = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(ob, sb, G.WGRAD))
                check(c[r:r + 128, q:q + 128].astype(np.float64), ref, t, f"wgrad split tile {r},{q}")
    assert fq.device_status() == 0


def test_blockwise_more_tiles_than_sms(cuda_lib):
    """2048 x 4096 output = 256 tiles: every CTA runs the persistent loop more than once."""
    fq = cuda_lib
    M, K, N = 2048, 256, 4096
    X, W = bf((M, K), 1.0, 91), bf((K, N), 0.02, 92)
    qx = fq.quantize_1x128(X.cuda())
    qw = fq.quantize_128x128(W.cuda())
    c = fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qx["s_row"], b_scale=qw["s"])
    ox, osx = Q.quantize_1x128_rowwise(workloads.bf16_bits(X))
    _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(W))
    ref, t = G.reference(G.dequant_a_1x128(ox, osx), G.dequant_b_blockwise(owt, osw, G.FPROP))
    check(c, ref, t, "fprop persistent")


def test_grouped_fprop_ragged_experts(cuda_lib):
    fq = cuda_lib
    counts = [130, 0, 1, 257, 60, 128]
    K, N, Gn = 384, 256, len(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offs[-1])
    A = bf((M, K), 1.0, 31)
    Ws = [bf((K, N), 0.006, 40 + g) for g in range(Gn)]
    qa = fq.quantize_1x128(A.cuda())
    qws = [fq.quantize_128x128(w.cuda()) for w in Ws]
    B = torch.stack([q["q_t"] for q in qws])              # (G, N, K)
    SB = torch.stack([q["s"] for q in qws])               # (G, N/128, K/128)
    c = fq.gemm(qa["q_row"], B, fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qa["s_row"], b_scale=SB,
                ld_sb=K // 128, m_offsets=torch.from_numpy(offs).cuda())
    oa, osa = Q.quantize_1x128_rowwise(workloads.bf16_bits(A))
    got = host(c.float()).astype(np.float64)
    for g in range(Gn):
        r0, r1 = offs[g], offs[g + 1]
        if r1 == r0:
            continue
        _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(Ws[g]))
        rows = np.arange(r0, r1)
        ref, t = G.reference(G.dequant_a_1x128(oa, osa, rows=rows), G.dequant_b_blockwise(owt, osw, G.FPROP))
        check(got[r0:r1], ref, t, f"grouped expert {g}")


@pytest.mark.parametrize("offs,clamped", [([0, 130, 130, 500], [0, 130, 130, 300]),
                                          ([0, 200, 100, 300], [0, 200, 200, 300])])
def test_grouped_offsets_out_of_rule_are_clamped_on_the_device(cuda_lib, offs, clamped):
    """Expert offsets past M or decreasing: the kernel clamps each to [previous, M], writes
    no row outside C (guard rows below C keep their sentinel), computes the clamped
    experts, and records FP8Q_ERR_DEVICE_ARG in the device status word."""
    fq = cuda_lib
    M, K, N, Gn = 300, 384, 256, 3
    A = bf((M, K), 1.0, 61)
    Ws = [bf((K, N), 0.006, 70 + g) for g in range(Gn)]
    qa = fq.quantize_1x128(A.cuda())
    qws = [fq.quantize_128x128(w.cuda()) for w in Ws]
    B = torch.stack([q["q_t"] for q in qws])
    SB = torch.stack([q["s"] for q in qws])
    assert fq.device_status() == fq.FP8Q_OK
    big = torch.full((M + 256, N), 7.0, dtype=torch.bfloat16, device="cuda")
    fq.gemm(qa["q_row"], B, fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qa["s_row"], b_scale=SB,
            ld_sb=K // 128, m_offsets=torch.tensor(offs, dtype=torch.int32, device="cuda"), out=big[:M])
    assert fq.device_status() == fq.FP8Q_ERR_DEVICE_ARG
    assert fq.device_status() == fq.FP8Q_OK                     # reading the status cleared it
    assert bool((big[M:] == 7.0).all())
    oa, osa = Q.quantize_1x128_rowwise(workloads.bf16_bits(A))
    got = host(big[:M].float()).astype(np.float64)
    for g in range(Gn):
        r0, r1 = clamped[g], clamped[g + 1]
        if r1 == r0:
            continue
        _, owt, osw = Q.quantize_128x128(workloads.bf16_bits(Ws[g]))
        rows = np.arange(r0, r1)
        ref, t = G.reference(G.dequant_a_1x128(oa, osa, rows=rows), G.dequant_b_blockwise(owt, osw, G.FPROP))
        check(got[r0:r1], ref, t, f"clamped expert {g}")


# ----------------------------------------------------------------------------- other recipes
@pytest.mark.parametrize("M,K,N", [(300, 512, 400), (256, 1024, 256)])
def test_mxfp8(cuda_lib, M, K, N):
    fq = cuda_lib
    A, W = bf((M, K), 1.0, M + 7 * K), bf((K, N), 0.02, N + K)
    qa = fq.quantize_mx32(A.cuda(), rowwise=True, sf_layout=fq.FP8Q_SF_MMA_TILED)
    qb = fq.quantize_mx32(W.cuda(), rowwise=False, colwise=True, sf_layout=fq.FP8Q_SF_MMA_TILED)
    c = fq.gemm(qa["q_row"], qb["q_col"], fq.FP8Q_MXFP8, a_scale=qa["e8m0_row"], b_scale=qb["e8m0_col"])
    oa, ea = Q.quantize_mx_rowwise(workloads.bf16_bits(A))
    ob, eb = Q.quantize_mx_colwise(workloads.bf16_bits(W))
    ref, t = G.reference(G.dequant_mx(oa, ea), G.dequant_mx(ob, eb))
    check(c, ref, t, "mxfp8")


@pytest.mark.parametrize("M,K,N", [(300, 512, 400)])
def test_per_tensor(cuda_lib, M, K, N):
    fq = cuda_lib
    A, W = bf((M, K), 1.0, 3 * M + K), bf((K, N), 0.02, 5 * N + K)
    Wt = W.t().contiguous()
    qa = fq.quantize_tensor(A.cuda())
    qb = fq.quantize_tensor(Wt.cuda())
    c = fq.gemm(qa["q"], qb["q"], fq.FP8Q_PERTENSOR, a_global=qa["s_dec"], b_global=qb["s_dec"])
    oa, sa = Q.quantize_tensor(workloads.bf16_bits(A))
    ob, sb = Q.quantize_tensor(workloads.bf16_bits(Wt))
    ref, t = G.reference(G.dequant_tensor(oa, sa), G.dequant_tensor(ob, sb))
    check(c, ref, t, "per-tensor")


def test_per_tensor_e5m2_gradient_times_e4m3_weights(cuda_lib):
    """dgrad of the delayed-scaling recipe: an E5M2 gradient (A) times E4M3 weights (B),
    per-tensor scales, against the FP64 product of the dequantized operands."""
    fq = cuda_lib
    M, K, N = 300, 512, 400
    dY, W = bf((M, K), 1e-3, 81, 5e-4, 100.0), bf((N, K), 0.02, 82)
    ha = torch.tensor([0.0], dtype=torch.float32, device="cuda")
    hb = torch.tensor([0.0], dtype=torch.float32, device="cuda")
    fq.quantize_tensor_delayed(dY.cuda(), ha, 0, fq.FP8Q_E5M2)        # records the amaxes
    fq.quantize_tensor_delayed(W.cuda(), hb, 0, fq.FP8Q_E4M3)
    qa = fq.quantize_tensor_delayed(dY.cuda(), ha, 0, fq.FP8Q_E5M2)   # scaled by them
    qb = fq.quantize_tensor_delayed(W.cuda(), hb, 0, fq.FP8Q_E4M3)
    c = fq.gemm(qa["q"], qb["q"], fq.FP8Q_PERTENSOR, a_global=qa["s_dec"], b_global=qb["s_dec"], a_format=fq.FP8Q_E5M2)
    assert fq.device_status() == 0
    ref, t = G.reference(G.dequant_tensor(host(qa["q"]), host(qa["s_dec"])[0], fmt="e5m2"),
                         G.dequant_tensor(host(qb["q"]), host(qb["s_dec"])[0]))
    check(c, ref, t, "per-tensor e5m2 x e4m3")


@pytest.mark.parametrize("M,K,N,rht", [(300, 512, 400, False), (256, 1024, 256, True)])
def test_nvfp4(cuda_lib, M, K, N, rht):
    fq = cuda_lib
    A, B = bf((M, K), 1e-3, M + 11 * K, 5e-4, 100.0), bf((N, K), 0.02, N + 13 * K)
    flag = fq.FP4Q_ROW if rht else 0
    qa = fq.rht16_quantize_sr(A.cuda(), rht=flag, rht_seed=5, sr=fq.FP4Q_ROW, sr_seed=6,
                              sf_layout=fq.FP8Q_SF_MMA_TILED)
    qb = fq.rht16_quantize_sr(B.cuda(), rht=flag, rht_seed=5, sf_layout=fq.FP8Q_SF_MMA_TILED)
    c = fq.gemm(qa["q_row"], qb["q_row"], fq.FP8Q_NVFP4, a_scale=qa["sf_row"], b_scale=qb["sf_row"],
                a_global=qa["g_row"], b_global=qb["g_row"], K=K)
    oa, sa, ga = Q.quantize_nvfp4_rowwise(workloads.bf16_bits(A), rht=rht, rht_seed=5, sr=True, sr_seed=6)
    ob, sb, gb = Q.quantize_nvfp4_rowwise(workloads.bf16_bits(B), rht=rht, rht_seed=5)
    ref, t = G.reference(G.dequant_nvfp4(oa, sa, ga), G.dequant_nvfp4(ob, sb, gb))
    check(c, ref, t, "nvfp4")


@pytest.mark.parametrize("M,K,N", [(300, 512, 768), (128, 256, 256)])
def test_nvfp4_forward_and_dgrad_with_16x16_weights(cuda_lib, M, K, N):
    """One 16x16-block quantization of W (K x N) feeds both fprop (X . W, W read along K:
    its colwise output) and dgrad (dY . W^T, W read along N: its rowwise output)."""
    fq = cuda_lib
    X, W, dY = bf((M, K), 1.0, M + 3 * K, 1e-3, 50.0), bf((K, N), 0.02, K + 5 * N), bf((M, N), 1e-3, M + 7 * N)
    qw = fq.quantize_nvfp4_2d16(W.cuda())
    qx = fq.rht16_quantize_sr(X.cuda(), sf_layout=fq.FP8Q_SF_MMA_TILED)
    y = fq.gemm(qx["q_row"], qw["q_col"], fq.FP8Q_NVFP4, a_scale=qx["sf_row"], b_scale=qw["sf_col"],
                a_global=qx["g_row"], b_global=qw["g"], K=K)
    qd = fq.rht16_quantize_sr(dY.cuda(), sr=fq.FP4Q_ROW, sr_seed=6, sf_layout=fq.FP8Q_SF_MMA_TILED)
    dx = fq.gemm(qd["q_row"], qw["q_row"], fq.FP8Q_NVFP4, a_scale=qd["sf_row"], b_scale=qw["sf_row"],
                 a_global=qd["g_row"], b_global=qw["g"], K=N)
    ow_row, sw_row, ow_col, sw_col, gw = Q.quantize_nvfp4_2d(workloads.bf16_bits(W))
    ox, sx, gx = Q.quantize_nvfp4_rowwise(workloads.bf16_bits(X))
    ref, t = G.reference(G.dequant_nvfp4(ox, sx, gx), G.dequant_nvfp4(ow_col, sw_col, gw))
    check(y, ref, t, "nvfp4 fprop, 16x16 weights")
    od, sd, gd = Q.quantize_nvfp4_rowwise(workloads.bf16_bits(dY), sr=True, sr_seed=6)
    ref, t = G.reference(G.dequant_nvfp4(od, sd, gd), G.dequant_nvfp4(ow_row, sw_row, gw))
    check(dx, ref, t, "nvfp4 dgrad, 16x16 weights")


def test_k_zero_gives_zeros(cuda_lib):
    fq = cuda_lib
    a = torch.zeros((4, 128), dtype=torch.uint8, device="cuda")
    s = torch.ones((1, 4), dtype=torch.float32, device="cuda")
    out = torch.full((4, 8), 7.0, dtype=torch.bfloat16, device="cuda")
    fq.gemm(a, a[:, :0].new_zeros((8, 128)), fq.FP8Q_BLOCKWISE, a_scale=s, b_scale=s, K=0, out=out)
    assert float(out.abs().max()) == 0.0


# ----------------------------------------------------------------------------- full size, sampled
def amax_bf16(bits, rows=1024):
    """max |x| of a BF16 bit-pattern matrix, by row chunks (no full FP32 copy)."""
    return max(np.float32(np.abs(Q.as_f32(bits[r:r + rows])).max()) for r in range(0, bits.shape[0], rows))


def _tiles(M, N, seed):
    return G.sample_tiles(M, N, 64, seed=seed)


def test_llama8b_fprop_dgrad_wgrad_sampled(cuda_lib):
    """The bench's three GEMMs at M=8192, hidden 4096, FFN 14336 on 64 sampled tiles each."""
    fq = cuda_lib
    d = workloads.llama8b(device="cuda")
    X, W, dY = d["X"], d["W"], d["dY"]
    qx = fq.quantize_1x128(X, rowwise=True, colwise=True)
    qw = fq.quantize_128x128(W)
    qd = fq.quantize_1x128(dY, rowwise=True, colwise=True)
    Xb, Wb, dYb = workloads.bf16_bits(X), workloads.bf16_bits(W), workloads.bf16_bits(dY)
    # FPROP (8192, 4096, 14336)
    c = host(fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qx["s_row"],
                     b_scale=qw["s"]).float())
    for m0, n0 in _tiles(8192, 14336, 2):
        oa, sa = Q.quantize_1x128_rowwise(Xb[m0:m0 + 128])
        _, owt, sw = Q.quantize_128x128(Wb[:, n0:n0 + 128])
        ref, t = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
        check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"fprop tile {m0},{n0}")
    # DGRAD (8192, 14336, 4096): B = W (4096 x 14336)
    c = host(fq.gemm(qd["q_row"], qw["q"], fq.FP8Q_BLOCKWISE, fq.FP8Q_DGRAD, a_scale=qd["s_row"],
                     b_scale=qw["s"], ld_sb=4096 // 128).float())
    for m0, n0 in _tiles(8192, 4096, 3):
        oa, sa = Q.quantize_1x128_rowwise(dYb[m0:m0 + 128])
        ow, _, sw = Q.quantize_128x128(Wb[n0:n0 + 128])            # W rows n0.. (its K), all N
        ref, t = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(ow, sw, G.DGRAD))
        check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"dgrad tile {m0},{n0}")
    # WGRAD (4096, 8192, 14336): A = X^T, B = dY^T, K = tokens
    c = host(fq.gemm(qx["q_col"], qd["q_col"], fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, a_scale=qx["s_col"],
                     b_scale=qd["s_col"]).float())
    for m0, n0 in _tiles(4096, 14336, 4):
        oa, sa = Q.quantize_1x128_colwise(Xb[:, m0:m0 + 128])
        ob, sb = Q.quantize_1x128_colwise(dYb[:, n0:n0 + 128])
        ref, t = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(ob, sb, G.WGRAD))
        check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"wgrad tile {m0},{n0}")
    assert fq.device_status() == 0


def test_llama8b_fprop_fused_quantization_fullsize(cuda_lib):
    """Full-size fprop (8192, 4096, 14336) with the fused 1x128 quantization of Y: codes and
    scales equal the standalone quantizer's on the same Y everywhere; 64 sampled tiles are
    checked against the oracle."""
    fq = cuda_lib
    d = workloads.llama8b(device="cuda")
    X, W = d["X"], d["W"]
    del d
    M, K, N = X.shape[0], X.shape[1], W.shape[1]
    qx = fq.quantize_1x128(X)
    qw = fq.quantize_128x128(W)
    q_out = torch.empty((M, N), dtype=torch.uint8, device="cuda")
    s_out = torch.empty((N // 128, M), dtype=torch.float32, device="cuda")
    c = fq.gemm(qx["q_row"], qw["q_t"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qx["s_row"], b_scale=qw["s"],
                q_out=q_out, s_out=s_out)
    qs = fq.quantize_1x128(c, rowwise=True, colwise=False)
    assert torch.equal(q_out, qs["q_row"]) and torch.equal(s_out.view(torch.int32), qs["s_row"][:, :M].view(torch.int32))
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    q_h, s_h = host(q_out), host(s_out)
    c_h = host(c.float()).astype(np.float64)
    for m0, g0 in _tiles(M, N, 9):           # 128-aligned tiles: one scale group each
        oa, sa = Q.quantize_1x128_rowwise(Xb[m0:m0 + 128])
        _, owt, sw = Q.quantize_128x128(Wb[:, g0:g0 + 128])
        ref, t = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
        check(c_h[m0:m0 + 128, g0:g0 + 128], ref, t, f"fprop tile {m0},{g0}")
        deq = F.e4m3_decode(q_h[m0:m0 + 128, g0:g0 + 128]).astype(np.float64) * s_h[g0 // 128, m0:m0 + 128, None]
        s_bound = (np.abs(ref).max(axis=1, keepdims=True) + t.max(axis=1, keepdims=True)) / 448.0 * (1 + 2.0 ** -20)
        excess = np.abs(deq - ref) - (t + 2.0 ** -4 * (np.abs(ref) + t) + 2.0 ** -10 * s_bound)
        assert float(excess.max()) <= 0, f"fused codes of tile {m0},{g0}"
    assert fq.device_status() == 0


def test_mxfp8_and_per_tensor_fullsize_sampled(cuda_lib):
    """MXFP8 and per-tensor current-scaling GEMMs at the three Llama-3-8B attention/MLP shapes,
    64 sampled output tiles each."""
    fq = cuda_lib
    d = workloads.mxfp8(device="cuda")
    for i, (M, K, N) in enumerate(workloads.MXFP8_GEMMS):
        A, W = d[f"A{i}"], d[f"W{i}"]
        qa = fq.quantize_mx32(A, rowwise=True, sf_layout=1)
        qb = fq.quantize_mx32(W, rowwise=False, colwise=True, sf_layout=1)
        c = host(fq.gemm(qa["q_row"], qb["q_col"], fq.FP8Q_MXFP8, a_scale=qa["e8m0_row"],
                         b_scale=qb["e8m0_col"]).float())
        Ab, Wb = workloads.bf16_bits(A), workloads.bf16_bits(W)
        for m0, n0 in _tiles(M, N, 10 + i):
            oa, ea = Q.quantize_mx_rowwise(Ab[m0:m0 + 128])
            ob, eb = Q.quantize_mx_colwise(Wb[:, n0:n0 + 128])
            ref, t = G.reference(G.dequant_mx(oa, ea), G.dequant_mx(ob, eb))
            check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"mxfp8 {i} tile {m0},{n0}")
        del qa, qb, c
        # per-tensor comparison variant on the same tensors
        Wt = W.t().contiguous()
        qa = fq.quantize_tensor(A)
        qb = fq.quantize_tensor(Wt)
        c = host(fq.gemm(qa["q"], qb["q"], fq.FP8Q_PERTENSOR, a_global=qa["s_dec"], b_global=qb["s_dec"]).float())
        oa, sa = Q.quantize_tensor(Ab)
        ob, sb = Q.quantize_tensor(workloads.bf16_bits(Wt))     # global scales over whole tensors
        for m0, n0 in _tiles(M, N, 20 + i):
            ref, t = G.reference(G.dequant_tensor(oa[m0:m0 + 128], sa), G.dequant_tensor(ob[n0:n0 + 128], sb))
            check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"per-tensor {i} tile {m0},{n0}")
        del qa, qb, c, Wt


def test_moe_grouped_fullsize_sampled(cuda_lib):
    """DeepSeek-V3 expert GEMMs: 32 experts, 16384 tokens x top-8, up and down projections."""
    fq = cuda_lib
    for proj in ("up", "down"):
        d = workloads.moe(device="cuda", proj=proj)
        A, W, offs = d["A"], d["W"], d["offsets"]
        Gn, K, N = W.shape
        qa = fq.quantize_1x128(A)
        B = torch.empty((Gn, N, K), dtype=torch.uint8, device="cuda")
        SB = torch.empty((Gn, N // 128, K // 128), dtype=torch.float32, device="cuda")
        for g in range(Gn):
            q = fq.quantize_128x128(W[g], plain=False)
            B[g].copy_(q["q_t"])
            SB[g].copy_(q["s"])
        c = host(fq.gemm(qa["q_row"], B, fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=qa["s_row"], b_scale=SB,
                         ld_sb=K // 128, m_offsets=offs.cuda()).float())
        tiles = G.sample_group_tiles(offs.numpy(), N, 64, seed=4)
        Ab = workloads.bf16_bits(A)
        for g, m0, m1, n0 in tiles:
            oa, sa = Q.quantize_1x128_rowwise(Ab[m0:m1])
            _, owt, sw = Q.quantize_128x128(workloads.bf16_bits(W[g][:, n0:n0 + 128]))
            ref, t = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
            check(c[m0:m1, n0:n0 + 128].astype(np.float64), ref, t, f"moe {proj} expert {g} tile {m0},{n0}")
        del qa, B, SB, d


def test_nvfp4_fprop_16x16_weights_fullsize_sampled(cuda_lib):
    """Llama-3.1-405B-shaped NVFP4 forward GEMM (8192, 16384, 53248): X rowwise 1x16 scales,
    W with 16x16 block scales (colwise output), 64 sampled output tiles."""
    fq = cuda_lib
    d = workloads.nvfp4(device="cuda", which=("X", "W"))
    X, W = d["X"], d["W"]
    qx = fq.rht16_quantize_sr(X, sf_layout=1)
    qw = fq.quantize_nvfp4_2d16(W, rowwise=False, colwise=True)
    c = host(fq.gemm(qx["q_row"], qw["q_col"], fq.FP8Q_NVFP4, a_scale=qx["sf_row"], b_scale=qw["sf_col"],
                     a_global=qx["g_row"], b_global=qw["g"], K=16384).float())
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    tiles = _tiles(8192, 53248, 7)
    rows_a = np.unique(np.concatenate([np.arange(m0, m0 + 128) for m0, _ in tiles]))
    oa, sa, ga = Q.quantize_nvfp4_rowwise(Xb, rows=rows_a)
    ia = {r: i for i, r in enumerate(rows_a)}
    G_w = amax_bf16(Wb)
    for m0, n0 in tiles:
        ra = [ia[r] for r in range(m0, m0 + 128)]
        _, _, ob, sb, gb = Q.quantize_nvfp4_2d(Wb[:, n0:n0 + 128], amax=G_w)
        ref, t = G.reference(G.dequant_nvfp4(oa[ra], sa[ra], ga), G.dequant_nvfp4(ob, sb, gb))
        check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"nvfp4 fprop tile {m0},{n0}")
    assert fq.device_status() == 0


def test_nvfp4_fullsize_sampled(cuda_lib):
    """Llama-3.1-405B-shaped NVFP4 dgrad (8192, 53248, 16384) and wgrad (16384, 8192, 53248).
    64 output tiles each: every pairing of 8 random 128-row bands with 8 random 128-column
    bands, so the oracle quantizes 8 bands of each operand (a stochastically rounded band of
    dY costs seconds in the oracle) while 64 tiles are compared."""
    fq = cuda_lib
    d = workloads.nvfp4(device="cuda")
    X, W, dY = d["X"], d["W"], d["dY"]
    Xb, Wb, dYb = workloads.bf16_bits(X), workloads.bf16_bits(W), workloads.bf16_bits(dY)
    qd = fq.rht16_quantize_sr(dY, rowwise=True, colwise=True, rht=fq.FP4Q_COL, rht_seed=5, sr=3, sr_seed=6,
                              sf_layout=1)
    qw = fq.rht16_quantize_sr(W, rowwise=True, sf_layout=1)
    c = host(fq.gemm(qd["q_row"], qw["q_row"], fq.FP8Q_NVFP4, a_scale=qd["sf_row"], b_scale=qw["sf_row"],
                     a_global=qd["g_row"], b_global=qw["g_row"], K=53248).float())
    tiles = G.sample_band_tiles(8192, 16384, 8, 8, seed=5)
    rows_a = np.unique(np.concatenate([np.arange(m0, m0 + 128) for m0, _ in tiles]))
    rows_b = np.unique(np.concatenate([np.arange(n0, n0 + 128) for _, n0 in tiles]))
    oa, sa, ga = Q.quantize_nvfp4_rowwise(dYb, sr=True, sr_seed=6, rows=rows_a)
    ob, sb, gb = Q.quantize_nvfp4_rowwise(Wb, rows=rows_b)
    ia = {r: i for i, r in enumerate(rows_a)}
    ib = {r: i for i, r in enumerate(rows_b)}
    for m0, n0 in tiles:
        ra = [ia[r] for r in range(m0, m0 + 128)]
        rb = [ib[r] for r in range(n0, n0 + 128)]
        ref, t = G.reference(G.dequant_nvfp4(oa[ra], sa[ra], ga), G.dequant_nvfp4(ob[rb], sb[rb], gb))
        check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"nvfp4 dgrad tile {m0},{n0}")
    del qw, c
    qx = fq.rht16_quantize_sr(X, rowwise=False, colwise=True, rht=fq.FP4Q_COL, rht_seed=5, sf_layout=1)
    c = host(fq.gemm(qx["q_col"], qd["q_col"], fq.FP8Q_NVFP4, a_scale=qx["sf_col"], b_scale=qd["sf_col"],
                     a_global=qx["g_col"], b_global=qd["g_col"], K=8192).float())
    tiles = G.sample_band_tiles(16384, 53248, 8, 8, seed=6)
    cols_a = np.unique(np.concatenate([np.arange(m0, m0 + 128) for m0, _ in tiles]))
    cols_b = np.unique(np.concatenate([np.arange(n0, n0 + 128) for _, n0 in tiles]))
    oa, sa, ga = Q.quantize_nvfp4_colwise(Xb, rht=True, rht_seed=5, rows=cols_a)
    ob, sb, gb = Q.quantize_nvfp4_colwise(dYb, rht=True, rht_seed=5, sr=True, sr_seed=6, rows=cols_b)
    ia = {r: i for i, r in enumerate(cols_a)}
    ib = {r: i for i, r in enumerate(cols_b)}
    for m0, n0 in tiles:
        ra = [ia[r] for r in range(m0, m0 + 128)]
        rb = [ib[r] for r in range(n0, n0 + 128)]
        ref, t = G.reference(G.dequant_nvfp4(oa[ra], sa[ra], ga), G.dequant_nvfp4(ob[rb], sb[rb], gb))
        check(c[m0:m0 + 128, n0:n0 + 128].astype(np.float64), ref, t, f"nvfp4 wgrad tile {m0},{n0}")
    assert fq.device_status() == 0
