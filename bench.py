"""Benchmark of the hot path: online fine-grained quantization + block-scaled GEMM on B200.

Default workload (one "step"), Llama-3-8B up-projection, blockwise recipe, forward and
backward with M = 8192 tokens, hidden K = 4096, FFN N = 14336:
  quantize X (1x128 rowwise + fused transposed colwise), quantize W (128x128, both
  layouts), quantize dY (1x128 rowwise + colwise), GEMM fprop, dgrad, wgrad.
Other workloads (--workload): tiny, mxfp8, moe, nvfp4, nvfp4_train, wgrad_acc, delayed,
fprop_quant (one JSON line each).

Metric: block-scaled GEMM TFLOP/s (the step's GEMM FLOPs over the whole step's device time,
quantization included) with per-kernel TFLOP/s and GB/s as fractions of the roofline.

Contract: python bench.py --gpus N --steps K --warmup W [--impl ours|reference]
  * N > 1: one rank per GPU under torch.distributed.run.  Launched without a WORLD_SIZE in
    the environment, bench.py starts torch.distributed.run itself with N ranks; launched
    by torch.distributed.run, it checks that WORLD_SIZE == N.  Every rank runs the step on
    its own tokens (weak scaling, no data-path collective); timing is the max over ranks
    (an all-reduce MAX over the NCCL group), and the line reports the group's size.
  * Inputs live in HBM before the timed region; the L2 is flushed between steps (a 256 MiB
    write, then a 256 MiB read so no dirty lines remain), outside the per-step events.
  * --impl reference times the CPU oracle (rank 0 only) on a bounded sample of the step.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "block-scaled FP8 GEMM TFLOPS & quantize GB/s on 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0   # nominal dense FP8 : BF16 tensor throughput ratio on B200
FP4_PER_BF16 = 4.0   # nominal dense FP4 : BF16


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ============================================================================ steps
class Launch:
    """One library call in a step: `fn()` enqueues its `kernels` launches on the current stream."""

    def __init__(self, name, fn, kernel, flop=0.0, bytes_=0.0, kernels=1):
        self.name, self.fn, self.kernel, self.flop, self.bytes = name, fn, kernel, flop, bytes_
        self.kernels = kernels


def b_1x128_fused(r, c):
    return r * c * (2 + 1 + 1) + 2 * r * c / 128 * 4


def b_1x128_row(r, c):
    return r * c * (2 + 1) + r * c / 128 * 4


def b_128(k, n):
    return k * n * (2 + 1 + 1) + (k // 128) * (n // 128) * 4


def b_mx(r, c):
    return r * c * (2 + 1) + r * c / 32


class LlamaStep:
    name = "llama8b"
    workload = "llama3-8b up-proj blockwise fwd+bwd: X 8192x4096, W 4096x14336, dY 8192x14336"

    def __init__(self, fq, rank, M=8192, K=4096, N=14336, separate_quant=False):
        self.fq, self.M, self.K, self.N = fq, M, K, N
        # the three tensors' quantizations as one multi-tensor launch (default) or three calls
        self.separate_quant = separate_quant
        self.workload = f"llama3-8b up-proj blockwise fwd+bwd: X {M}x{K}, W {K}x{N}, dY {M}x{N}"
        d = workloads.llama8b(device="cuda", M=M, K=K, N=N)
        if rank:   # other ranks: their own tokens, the same weights
            d["X"] = workloads.normal_bf16((M, K), 1.0, 10_000 + rank, 1e-3, 50.0, "cuda")
            d["dY"] = workloads.normal_bf16((M, N), 1e-3, 20_000 + rank, device="cuda")
        self.X, self.W, self.dY = d["X"], d["W"], d["dY"]
        dev = self.X.device
        u8, f32 = torch.uint8, torch.float32
        self.qx_r, self.qx_c = torch.empty((M, K), dtype=u8, device=dev), torch.empty((K, M), dtype=u8, device=dev)
        self.sx_r, self.sx_c = torch.empty((K // 128, M), dtype=f32, device=dev), torch.empty((M // 128, K), dtype=f32, device=dev)
        self.qw_t, self.qw = torch.empty((N, K), dtype=u8, device=dev), torch.empty((K, N), dtype=u8, device=dev)
        self.sw = torch.empty((N // 128, K // 128), dtype=f32, device=dev)
        self.qd_r, self.qd_c = torch.empty((M, N), dtype=u8, device=dev), torch.empty((N, M), dtype=u8, device=dev)
        self.sd_r, self.sd_c = torch.empty((N // 128, M), dtype=f32, device=dev), torch.empty((M // 128, N), dtype=f32, device=dev)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty((K, N), dtype=torch.bfloat16, device=dev)
        self.gemm_flop = 3 * 2.0 * M * N * K

    def inputs(self):
        return [self.X, self.W, self.dY]

    def outputs(self):
        return [self.Y, self.dX, self.dW]

    def launches(self):
        fq, M, K, N = self.fq, self.M, self.K, self.N
        P = lambda t: t.data_ptr()  # noqa: E731

        def q1x128(x, qr, sr, qc, sc, R, C):
            def f():
                st = fq.fp8q_quantize_1x128(P(x), R, C, C, P(qr), P(sr), sr.shape[1], P(qc), P(sc), sc.shape[1],
                                            fq._stream())
                assert st == 0, st
            return f

        # X (1x128, both outputs), W (128x128, both layouts) and dY (1x128, both outputs) in one
        # multi-tensor launch: one ramp and one partial last wave for the three tensors
        items = (fq.QuantItem * 3)()
        for it, x, (R, C) in zip(items, (self.X, self.W, self.dY), ((M, K), (K, N), (M, N))):
            it.x, it.rows, it.cols, it.ld_x = P(x), R, C, C
        items[0].kind = items[2].kind = fq.FP8Q_ITEM_1X128
        for it, (qr, sr, qc, sc) in ((items[0], (self.qx_r, self.sx_r, self.qx_c, self.sx_c)),
                                     (items[2], (self.qd_r, self.sd_r, self.qd_c, self.sd_c))):
            it.q_row, it.s_row, it.ld_s_row = P(qr), P(sr), sr.shape[1]
            it.q_col, it.s_col, it.ld_s_col = P(qc), P(sc), sc.shape[1]
        items[1].kind = fq.FP8Q_ITEM_128X128
        items[1].q_t, items[1].q, items[1].s = P(self.qw_t), P(self.qw), P(self.sw)

        def q128():
            st = fq.fp8q_quantize_128x128(P(self.W), K, N, N, P(self.qw_t), P(self.qw), P(self.sw), fq._stream())
            assert st == 0, st

        def qall():
            st = fq.fp8q_quantize_multi(items, 3, fq._stream())
            assert st == 0, st

        def gemm(a, b, layout, sa, sb, ld_sb, c):
            def f():
                fq.gemm(a, b, fq.FP8Q_BLOCKWISE, layout, a_scale=sa, b_scale=sb, ld_sb=ld_sb, out=c)
            return f

        def kernels(Mg, Ng, Kg, layout):
            # a GEMM whose last wave is split runs two kernels (the tiles and K ranges, the sum)
            return 2 if fq.gemm_workspace_bytes(Mg, Ng, Kg, fq.FP8Q_BLOCKWISE, layout) > 0 else 1

        if self.separate_quant:
            quant = [
                Launch("quantize_1x128 X (row+col)", q1x128(self.X, self.qx_r, self.sx_r, self.qx_c, self.sx_c, M, K),
                       "quantize", bytes_=b_1x128_fused(M, K)),
                Launch("quantize_128x128 W (both layouts)", q128, "quantize", bytes_=b_128(K, N)),
                Launch("quantize_1x128 dY (row+col)", q1x128(self.dY, self.qd_r, self.sd_r, self.qd_c, self.sd_c, M, N),
                       "quantize", bytes_=b_1x128_fused(M, N))]
        else:
            quant = [Launch("quantize X 1x128 (row+col), W 128x128 (both layouts), dY 1x128 (row+col): one launch",
                            qall, "quantize", bytes_=b_1x128_fused(M, K) + b_128(K, N) + b_1x128_fused(M, N))]
        return quant + [
            Launch("gemm blockwise fprop", gemm(self.qx_r, self.qw_t, fq.FP8Q_FPROP, self.sx_r, self.sw, K // 128, self.Y),
                   "gemm_blockwise", flop=2.0 * M * N * K, kernels=kernels(M, N, K, fq.FP8Q_FPROP)),
            Launch("gemm blockwise dgrad", gemm(self.qd_r, self.qw, fq.FP8Q_DGRAD, self.sd_r, self.sw, K // 128, self.dX),
                   "gemm_blockwise", flop=2.0 * M * N * K, kernels=kernels(M, K, N, fq.FP8Q_DGRAD)),
            Launch("gemm blockwise wgrad", gemm(self.qx_c, self.qd_c, fq.FP8Q_WGRAD, self.sx_c, self.sd_c, N, self.dW),
                   "gemm_blockwise", flop=2.0 * M * N * K, kernels=kernels(K, N, M, fq.FP8Q_WGRAD)),
        ]

    def cpu_sample(self, tiles=1):
        """Oracle on a bounded sample: the operands of `tiles` output tiles of each GEMM
        are quantized by the oracle from the BF16 inputs, then the FP64 reference tiles."""
        from oracle import gemm as G
        from oracle import quant as Q
        M, K, N = self.M, self.K, self.N
        if not hasattr(self, "_host_bits"):   # host copies, made once, outside the timed region
            self._host_bits = tuple(workloads.bf16_bits(t) for t in (self.X, self.W, self.dY))
        Xb, Wb, dYb = self._host_bits
        t0 = time.perf_counter()
        flop = 0.0
        for m0, n0 in G.sample_tiles(M, N, tiles, seed=2):
            oa, sa = Q.quantize_1x128_rowwise(Xb[m0:m0 + 128])
            _, owt, sw = Q.quantize_128x128(Wb[:, n0:n0 + 128])
            G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
            flop += 2.0 * 128 * 128 * K
        for m0, n0 in G.sample_tiles(M, K, tiles, seed=3):
            oa, sa = Q.quantize_1x128_rowwise(dYb[m0:m0 + 128])
            ow, _, sw = Q.quantize_128x128(Wb[n0:n0 + 128])
            G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(ow, sw, G.DGRAD))
            flop += 2.0 * 128 * 128 * N
        for m0, n0 in G.sample_tiles(K, N, tiles, seed=4):
            oa, sa = Q.quantize_1x128_colwise(Xb[:, m0:m0 + 128])
            ob, sb = Q.quantize_1x128_colwise(dYb[:, n0:n0 + 128])
            G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(ob, sb, G.WGRAD))
            flop += 2.0 * 128 * 128 * M
        dt = time.perf_counter() - t0
        return flop, dt, (f"{tiles} sampled 128x128 output tile(s) of each of fprop/dgrad/wgrad, operands "
                          "quantized by the oracle from the BF16 inputs, FP64 reference product")


def _llama_cpu_quant_sample(self):
    """Oracle quantizers on the step's full X (1x128 rowwise and colwise) and W (128x128,
    both layouts): algorithmic bytes, seconds, description (single-threaded NumPy)."""
    from oracle import quant as Q
    if not hasattr(self, "_host_bits"):
        self._host_bits = tuple(workloads.bf16_bits(t) for t in (self.X, self.W, self.dY))
    Xb, Wb, _ = self._host_bits
    M, K, N = self.M, self.K, self.N
    t0 = time.perf_counter()
    Q.quantize_1x128_rowwise(Xb)
    Q.quantize_1x128_colwise(Xb)
    Q.quantize_128x128(Wb)
    dt = time.perf_counter() - t0
    return (b_1x128_fused(M, K) + b_128(K, N), dt,
            f"1x128 rowwise+colwise of the full X ({M}x{K}) and 128x128 both layouts of the full W ({K}x{N})")


LlamaStep.cpu_quant_sample = _llama_cpu_quant_sample


class TinyStep(LlamaStep):
    name = "tiny"
    workload = "tiny blockwise fprop: A 256x512, B 512x256"

    def __init__(self, fq, rank, device="cuda"):
        self.fq = fq
        d = workloads.tiny(device=device)
        self.A, self.B = d["A"], d["B"]
        self.gemm_flop = 2.0 * 256 * 256 * 512
        if device == "cpu":          # host inputs only: the oracle's sample needs nothing else
            return
        dev = self.A.device
        self.qa = torch.empty((256, 512), dtype=torch.uint8, device=dev)
        self.sa = torch.empty((4, 256), dtype=torch.float32, device=dev)
        self.qbt = torch.empty((256, 512), dtype=torch.uint8, device=dev)
        self.sb = torch.empty((2, 4), dtype=torch.float32, device=dev)
        self.C = torch.empty((256, 256), dtype=torch.bfloat16, device=dev)

    def inputs(self):
        return [self.A, self.B]

    def outputs(self):
        return [self.C]

    def launches(self):
        fq = self.fq
        P = lambda t: t.data_ptr()  # noqa: E731

        def qa():
            assert fq.fp8q_quantize_1x128(P(self.A), 256, 512, 512, P(self.qa), P(self.sa), 256, None, None, 0,
                                          fq._stream()) == 0

        def qb():
            assert fq.fp8q_quantize_128x128(P(self.B), 512, 256, 256, P(self.qbt), None, P(self.sb), fq._stream()) == 0

        def g():
            fq.gemm(self.qa, self.qbt, fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=self.sa, b_scale=self.sb, out=self.C)

        return [Launch("quantize_1x128 A", qa, "quantize", bytes_=b_1x128_row(256, 512)),
                Launch("quantize_128x128 B", qb, "quantize", bytes_=256 * 512 * 3.0),
                Launch("gemm blockwise fprop", g, "gemm_blockwise", flop=self.gemm_flop)]

    def cpu_sample(self, tiles=1):
        from oracle import gemm as G
        from oracle import quant as Q
        t0 = time.perf_counter()
        oa, sa = Q.quantize_1x128_rowwise(workloads.bf16_bits(self.A))
        _, owt, sw = Q.quantize_128x128(workloads.bf16_bits(self.B))
        G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
        return self.gemm_flop, time.perf_counter() - t0, "the whole tiny step"


class FpropQuantStep:
    """Llama-3-8B up-projection forward with online quantization of its output for the next
    layer: X in 1x128 tiles, W in 128x128 blocks, then Y = X . W with the blockwise promotion,
    written as BF16 and, from the GEMM's epilogue, as 1x128 E4M3 codes and scales."""
    name = "fprop_quant"
    workload = "llama3-8b up-proj fprop with fused 1x128 quantization of Y: X 8192x4096, W 4096x14336"

    def __init__(self, fq, rank, M=8192, K=4096, N=14336):
        self.fq, self.M, self.K, self.N = fq, M, K, N
        d = workloads.llama8b(device="cuda", M=M, K=K, N=N)
        self.X, self.W = d["X"], d["W"]
        del d
        dev = self.X.device
        u8, f32 = torch.uint8, torch.float32
        self.qx_r, self.sx_r = torch.empty((M, K), dtype=u8, device=dev), torch.empty((K // 128, M), dtype=f32, device=dev)
        self.qw_t, self.qw = torch.empty((N, K), dtype=u8, device=dev), torch.empty((K, N), dtype=u8, device=dev)
        self.sw = torch.empty((N // 128, K // 128), dtype=f32, device=dev)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.qy, self.sy = torch.empty((M, N), dtype=u8, device=dev), torch.empty((N // 128, M), dtype=f32, device=dev)
        self.gemm_flop = 2.0 * M * N * K

    def inputs(self):
        return [self.X, self.W]

    def outputs(self):
        return [self.Y, self.qy, self.sy]

    def launches(self):
        fq, M, K, N = self.fq, self.M, self.K, self.N
        P = lambda t: t.data_ptr()  # noqa: E731

        def qx():
            assert fq.fp8q_quantize_1x128(P(self.X), M, K, K, P(self.qx_r), P(self.sx_r), M, None, None, 0,
                                          fq._stream()) == 0

        def qw():
            assert fq.fp8q_quantize_128x128(P(self.W), K, N, N, P(self.qw_t), P(self.qw), P(self.sw), fq._stream()) == 0

        def g():
            fq.gemm(self.qx_r, self.qw_t, fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=self.sx_r, b_scale=self.sw,
                    ld_sb=K // 128, out=self.Y, q_out=self.qy, s_out=self.sy)

        return [Launch("quantize_1x128 X (row)", qx, "quantize", bytes_=b_1x128_row(M, K)),
                Launch("quantize_128x128 W (both layouts)", qw, "quantize", bytes_=b_128(K, N)),
                Launch("gemm blockwise fprop + fused 1x128 quantization of Y", g, "gemm_blockwise",
                       flop=self.gemm_flop)]

    def cpu_sample(self, tiles=1):
        """Oracle on a bounded sample: `tiles` sampled 128x128 tiles of Y, operands quantized by
        the oracle, FP64 product, then the product's 1x128 quantization."""
        from oracle import gemm as G
        from oracle import quant as Q
        from oracle import formats as F
        M, K, N = self.M, self.K, self.N
        if not hasattr(self, "_host_bits"):
            self._host_bits = tuple(workloads.bf16_bits(t) for t in (self.X, self.W))
        Xb, Wb = self._host_bits
        t0 = time.perf_counter()
        flop = 0.0
        for m0, n0 in G.sample_tiles(M, N, tiles, seed=7):
            oa, sa = Q.quantize_1x128_rowwise(Xb[m0:m0 + 128])
            _, owt, sw = Q.quantize_128x128(Wb[:, n0:n0 + 128])
            ref, _ = G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
            Q.quantize_1x128_rowwise(F.f32_to_bf16_bits(ref.astype("float32")))
            flop += 2.0 * 128 * 128 * K
        return flop, time.perf_counter() - t0, f"{tiles} sampled 128x128 tile(s) of Y and their 1x128 quantization"


class WgradAccStep:
    """Llama-3-8B weight gradient with FP32 main-gradient accumulation: X and dY quantized
    in 1x128 tiles along the tokens (transposed outputs), then dW (FP32, 4096 x 14336) +=
    X^T . dY with the blockwise promotion."""
    name = "wgrad_acc"
    workload = "llama3-8b wgrad into FP32 main gradients: X 8192x4096, dY 8192x14336, dW 4096x14336 fp32 +="

    def __init__(self, fq, rank, M=8192, K=4096, N=14336):
        self.fq, self.M, self.K, self.N = fq, M, K, N
        d = workloads.llama8b(device="cuda", M=M, K=K, N=N)
        self.X, self.dY = d["X"], d["dY"]
        del d
        dev = self.X.device
        self.qx_c = torch.empty((K, M), dtype=torch.uint8, device=dev)
        self.sx_c = torch.empty((M // 128, K), dtype=torch.float32, device=dev)
        self.qd_c = torch.empty((N, M), dtype=torch.uint8, device=dev)
        self.sd_c = torch.empty((M // 128, N), dtype=torch.float32, device=dev)
        self.dW = torch.zeros((K, N), dtype=torch.float32, device=dev)
        self.gemm_flop = 2.0 * M * N * K

    def inputs(self):
        return [self.X, self.dY]

    def outputs(self):
        return [self.dW]

    def launches(self):
        fq, M, K, N = self.fq, self.M, self.K, self.N
        P = lambda t: t.data_ptr()  # noqa: E731

        def qcol(x, q, sc, C):
            def f():
                assert fq.fp8q_quantize_1x128(P(x), M, C, C, None, None, 0, P(q), P(sc), sc.shape[1],
                                              fq._stream()) == 0
            return f

        def g():
            fq.gemm(self.qx_c, self.qd_c, fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, a_scale=self.sx_c, b_scale=self.sd_c,
                    ld_sb=N, out=self.dW, accumulate_fp32=True)

        return [Launch("quantize_1x128 X colwise", qcol(self.X, self.qx_c, self.sx_c, K), "quantize",
                       bytes_=b_1x128_row(M, K)),
                Launch("quantize_1x128 dY colwise", qcol(self.dY, self.qd_c, self.sd_c, N), "quantize",
                       bytes_=b_1x128_row(M, N)),
                Launch("gemm blockwise wgrad FP32 accumulate", g, "gemm_blockwise_acc",
                       flop=self.gemm_flop,
                       kernels=2 if fq.gemm_workspace_bytes(K, N, M, fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD,
                                                            accumulate_fp32=True) > 0 else 1)]

    def cpu_sample(self, tiles=1):
        """Oracle on a bounded sample: `tiles` sampled 128x128 tiles of dW, operands quantized
        by the oracle, FP64 product added to the FP32 values the tiles held."""
        from oracle import gemm as G
        from oracle import quant as Q
        M, K, N = self.M, self.K, self.N
        if not hasattr(self, "_host_bits"):
            self._host_bits = tuple(workloads.bf16_bits(t) for t in (self.X, self.dY))
        Xb, dYb = self._host_bits
        t0 = time.perf_counter()
        flop = 0.0
        for m0, n0 in G.sample_tiles(K, N, tiles, seed=5):
            oa, sa = Q.quantize_1x128_colwise(Xb[:, m0:m0 + 128])
            ob, sb = Q.quantize_1x128_colwise(dYb[:, n0:n0 + 128])
            G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(ob, sb, G.WGRAD))
            flop += 2.0 * 128 * 128 * M
        dt = time.perf_counter() - t0
        return flop, dt, (f"{tiles} sampled 128x128 dW tile(s), operands quantized by the oracle from the BF16 "
                          "inputs, FP64 reference product")


class DelayedStep:
    """Per-tensor delayed scaling (amax history of 16 steps, rotated each step) on the
    Llama-3-8B up-projection: fprop X . W^T with E4M3 operands, dgrad dY . W with an E5M2
    gradient and E4M3 weights.  Each quantizer is one pass over its tensor."""
    name = "delayed"
    workload = ("llama3-8b up-proj, per-tensor delayed scaling (history 16): fprop X 8192x4096 e4m3 . W^T, "
                "dgrad dY 8192x14336 e5m2 . W e4m3")
    H = 16

    def __init__(self, fq, rank, M=8192, K=4096, N=14336):
        self.fq, self.M, self.K, self.N = fq, M, K, N
        d = workloads.llama8b(device="cuda", M=M, K=K, N=N)
        self.X, self.W, self.dY = d["X"], d["W"], d["dY"]
        self.Wt = self.W.t().contiguous()                     # N x K, the fprop B operand
        dev = self.X.device
        u8, f32 = torch.uint8, torch.float32
        self.hist = {k: torch.zeros(self.H, dtype=f32, device=dev) for k in ("x", "wt", "dy", "w")}
        self.q = {"x": torch.empty((M, K), dtype=u8, device=dev), "wt": torch.empty((N, K), dtype=u8, device=dev),
                  "dy": torch.empty((M, N), dtype=u8, device=dev), "w": torch.empty((K, N), dtype=u8, device=dev)}
        self.s = {k: torch.empty((1,), dtype=f32, device=dev) for k in self.q}
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.step = 0
        self.gemm_flop = 2 * 2.0 * M * N * K

    def inputs(self):
        return [self.X, self.W, self.dY]

    def outputs(self):
        return [self.Y, self.dX]

    def launches(self):
        fq = self.fq
        P = lambda t: t.data_ptr()  # noqa: E731
        src = {"x": self.X, "wt": self.Wt, "dy": self.dY, "w": self.W}
        fmt = {"x": fq.FP8Q_E4M3, "wt": fq.FP8Q_E4M3, "dy": fq.FP8Q_E5M2, "w": fq.FP8Q_E4M3}

        def quant(k):
            def f():
                x = src[k]
                pos = self.step % self.H
                if k == "w":
                    self.step += 1                            # last quantizer of the step
                assert fq.fp8q_quantize_tensor_delayed(P(x), x.shape[0], x.shape[1], x.stride(0), P(self.hist[k]),
                                                       self.H, pos, fmt[k], P(self.q[k]), P(self.s[k]),
                                                       fq._stream()) == 0
            return f

        def fprop():
            fq.gemm(self.q["x"], self.q["wt"], fq.FP8Q_PERTENSOR, a_global=self.s["x"], b_global=self.s["wt"],
                    out=self.Y)

        def dgrad():
            fq.gemm(self.q["dy"], self.q["w"], fq.FP8Q_PERTENSOR, a_global=self.s["dy"], b_global=self.s["w"],
                    out=self.dX, a_format=fq.FP8Q_E5M2)

        M, K, N = self.M, self.K, self.N
        return [Launch("quantize_tensor_delayed X e4m3", quant("x"), "quantize", bytes_=M * K * 3.0),
                Launch("quantize_tensor_delayed W^T e4m3", quant("wt"), "quantize", bytes_=N * K * 3.0),
                Launch("gemm per-tensor fprop e4m3", fprop, "gemm_pertensor", flop=2.0 * M * N * K),
                Launch("quantize_tensor_delayed dY e5m2", quant("dy"), "quantize", bytes_=M * N * 3.0),
                Launch("quantize_tensor_delayed W e4m3", quant("w"), "quantize", bytes_=K * N * 3.0),
                Launch("gemm per-tensor dgrad e5m2 x e4m3", dgrad, "gemm_pertensor", flop=2.0 * M * N * K)]

    def launch_count(self):
        return 4 * 2 + 2

    def cpu_sample(self, tiles=1):
        """Oracle on a bounded sample: the rows of `tiles` sampled 128x128 output tiles of each
        GEMM, quantized with the current histories (rows are independent under delayed
        scaling), then the FP64 reference tiles."""
        from oracle import gemm as G
        from oracle import quant as Q
        M, K, N = self.M, self.K, self.N
        if not hasattr(self, "_host_bits"):
            self._host_bits = tuple(workloads.bf16_bits(t) for t in (self.X, self.Wt, self.dY, self.W))
            self._host_hist = {k: v.cpu().numpy() for k, v in self.hist.items()}
        Xb, Wtb, dYb, Wb = self._host_bits
        h = self._host_hist
        t0 = time.perf_counter()
        flop = 0.0
        for m0, n0 in G.sample_tiles(M, N, tiles, seed=6):
            qa, sa, _ = Q.quantize_tensor_delayed(Xb[m0:m0 + 128], h["x"])
            qb, sb, _ = Q.quantize_tensor_delayed(Wtb[n0:n0 + 128], h["wt"])
            G.reference(G.dequant_tensor(qa, sa), G.dequant_tensor(qb, sb))
            flop += 2.0 * 128 * 128 * K
        for m0, n0 in G.sample_tiles(M, K, tiles, seed=7):
            qa, sa, _ = Q.quantize_tensor_delayed(dYb[m0:m0 + 128], h["dy"], fmt="e5m2")
            qb, sb, _ = Q.quantize_tensor_delayed(Wb[n0:n0 + 128], h["w"])
            G.reference(G.dequant_tensor(qa, sa, fmt="e5m2"), G.dequant_tensor(qb, sb))
            flop += 2.0 * 128 * 128 * N
        dt = time.perf_counter() - t0
        return flop, dt, (f"{tiles} sampled 128x128 output tile(s) of fprop and dgrad, rows quantized by the oracle "
                          "with the step's amax histories, FP64 reference product")


class MxStep:
    name = "mxfp8"
    workload = "MXFP8 (and per-tensor) GEMMs (M,K,N) = (8192,4096,4096), (8192,4096,14336), (8192,14336,4096)"

    def __init__(self, fq, rank, which=None):
        self.fq = fq
        d = workloads.mxfp8(device="cuda", which=which)
        self.items = []
        for i, (M, K, N) in enumerate(workloads.MXFP8_GEMMS):
            if which is not None and i not in which:
                continue
            A, W = d[f"A{i}"], d[f"W{i}"]
            dev = A.device
            it = {"M": M, "K": K, "N": N, "A": A, "W": W, "Wt": W.t().contiguous(),
                  "qa": torch.empty((M, K), dtype=torch.uint8, device=dev),
                  "ea": torch.empty(fq.fp8q_sf_bytes(fq.FP8Q_MXFP8, M, K, 1), dtype=torch.uint8, device=dev),
                  "qb": torch.empty((N, K), dtype=torch.uint8, device=dev),
                  "eb": torch.empty(fq.fp8q_sf_bytes(fq.FP8Q_MXFP8, N, K, 1), dtype=torch.uint8, device=dev),
                  "ta": torch.empty((M, K), dtype=torch.uint8, device=dev),
                  "tb": torch.empty((N, K), dtype=torch.uint8, device=dev),
                  "sa": torch.empty((1,), dtype=torch.float32, device=dev),
                  "sb": torch.empty((1,), dtype=torch.float32, device=dev),
                  "C": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                  "C2": torch.empty((M, N), dtype=torch.bfloat16, device=dev)}
            self.items.append(it)
        self.gemm_flop = sum(2.0 * 2 * it["M"] * it["N"] * it["K"] for it in self.items)

    def inputs(self):
        return [t for it in self.items for t in (it["A"], it["W"])]

    def outputs(self):
        return [t for it in self.items for t in (it["C"], it["C2"])]

    def launches(self):
        fq = self.fq
        P = lambda t: t.data_ptr()  # noqa: E731
        out = []
        for i, it in enumerate(self.items):
            M, K, N = it["M"], it["K"], it["N"]

            def qa(it=it, M=M, K=K):
                assert fq.fp8q_quantize_mx32(P(it["A"]), M, K, K, P(it["qa"]), P(it["ea"]), None, None, 1,
                                             fq._stream()) == 0

            def qb(it=it, K=K, N=N):
                assert fq.fp8q_quantize_mx32(P(it["W"]), K, N, N, None, None, P(it["qb"]), P(it["eb"]), 1,
                                             fq._stream()) == 0

            def g(it=it):
                fq.gemm(it["qa"], it["qb"], fq.FP8Q_MXFP8, a_scale=it["ea"], b_scale=it["eb"], out=it["C"])

            def ta(it=it, M=M, K=K):
                assert fq.fp8q_quantize_tensor(P(it["A"]), M, K, K, P(it["ta"]), P(it["sa"]), fq._stream()) == 0

            def tb(it=it, K=K, N=N):
                assert fq.fp8q_quantize_tensor(P(it["Wt"]), N, K, K, P(it["tb"]), P(it["sb"]), fq._stream()) == 0

            def g2(it=it):
                fq.gemm(it["ta"], it["tb"], fq.FP8Q_PERTENSOR, a_global=it["sa"], b_global=it["sb"], out=it["C2"])

            out += [Launch(f"quantize_mx32 A{i} rowwise", qa, "quantize", bytes_=b_mx(M, K)),
                    Launch(f"quantize_mx32 W{i} colwise", qb, "quantize", bytes_=b_mx(K, N)),
                    Launch(f"gemm mxfp8 {M}x{K}x{N}", g, "gemm_mxfp8", flop=2.0 * M * N * K),
                    Launch(f"quantize_tensor A{i}", ta, "quantize", bytes_=5.0 * M * K),
                    Launch(f"quantize_tensor W{i}^T", tb, "quantize", bytes_=5.0 * K * N),
                    Launch(f"gemm per-tensor {M}x{K}x{N}", g2, "gemm_pertensor", flop=2.0 * M * N * K)]
        return out

    def cpu_sample(self, tiles=1):
        from oracle import gemm as G
        from oracle import quant as Q
        t0 = time.perf_counter()
        flop = 0.0
        for i, it in enumerate(self.items):
            Ab, Wb = workloads.bf16_bits(it["A"]), workloads.bf16_bits(it["W"])
            for m0, n0 in G.sample_tiles(it["M"], it["N"], tiles, seed=10 + i):
                oa, ea = Q.quantize_mx_rowwise(Ab[m0:m0 + 128])
                ob, eb = Q.quantize_mx_colwise(Wb[:, n0:n0 + 128])
                G.reference(G.dequant_mx(oa, ea), G.dequant_mx(ob, eb))
                flop += 2.0 * 128 * 128 * it["K"]
        return flop, time.perf_counter() - t0, f"{tiles} sampled MXFP8 output tile(s) per GEMM, oracle-quantized"


class MoeStep:
    name = "moe"
    workload = "DeepSeek-V3 MoE grouped blockwise fprop: 32 experts, 16384 tokens x top-8, up 7168->2048, down 2048->7168"

    def __init__(self, fq, rank):
        self.fq = fq
        self.parts = []
        for proj in ("up", "down"):
            d = workloads.moe(device="cuda", proj=proj)
            A, W, offs = d["A"], d["W"], d["offsets"].cuda()
            Gn, K, N = W.shape
            M = A.shape[0]
            dev = A.device
            self.parts.append({"proj": proj, "A": A, "W": W, "offs": offs, "G": Gn, "K": K, "N": N, "M": M,
                               "qa": torch.empty((M, K), dtype=torch.uint8, device=dev),
                               "sa": torch.empty((K // 128, M), dtype=torch.float32, device=dev),
                               "B": torch.empty((Gn, N, K), dtype=torch.uint8, device=dev),
                               "SB": torch.empty((Gn, N // 128, K // 128), dtype=torch.float32, device=dev),
                               "C": torch.empty((M, N), dtype=torch.bfloat16, device=dev)})
        self.gemm_flop = sum(2.0 * p["M"] * p["N"] * p["K"] for p in self.parts)

    def inputs(self):
        return [t for p in self.parts for t in (p["A"], p["W"])]

    def outputs(self):
        return [p["C"] for p in self.parts]

    def launches(self):
        fq = self.fq
        P = lambda t: t.data_ptr()  # noqa: E731
        out = []
        for p in self.parts:
            M, K, N, Gn = p["M"], p["K"], p["N"], p["G"]

            def qa(p=p, M=M, K=K):
                assert fq.fp8q_quantize_1x128(P(p["A"]), M, K, K, P(p["qa"]), P(p["sa"]), M, None, None, 0,
                                              fq._stream()) == 0

            def qw(p=p, K=K, N=N, Gn=Gn):   # all experts' weights in one grouped call
                assert fq.fp8q_quantize_128x128_grouped(P(p["W"]), Gn, K, N, N, P(p["B"]), None, P(p["SB"]),
                                                        fq._stream()) == 0

            def g_(p=p, K=K):
                fq.gemm(p["qa"], p["B"], fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, a_scale=p["sa"], b_scale=p["SB"],
                        ld_sb=K // 128, m_offsets=p["offs"], out=p["C"])

            out += [Launch(f"quantize_1x128 A_{p['proj']}", qa, "quantize", bytes_=b_1x128_row(M, K)),
                    Launch(f"quantize_128x128 grouped W_{p['proj']} ({Gn} experts)", qw, "quantize",
                           bytes_=Gn * (K * N * 3.0 + (K // 128) * (N // 128) * 4)),
                    Launch(f"gemm grouped blockwise {p['proj']}", g_, "gemm_grouped", flop=2.0 * M * N * K)]
        return out

    def launch_count(self):
        return 3 * len(self.parts)

    def cpu_sample(self, tiles=1):
        from oracle import gemm as G
        from oracle import quant as Q
        t0 = time.perf_counter()
        flop = 0.0
        for p in self.parts:
            Ab = workloads.bf16_bits(p["A"])
            for g, m0, m1, n0 in G.sample_group_tiles(p["offs"].cpu().numpy(), p["N"], tiles, seed=4):
                oa, sa = Q.quantize_1x128_rowwise(Ab[m0:m1])
                _, owt, sw = Q.quantize_128x128(workloads.bf16_bits(p["W"][g][:, n0:n0 + 128]))
                G.reference(G.dequant_a_1x128(oa, sa), G.dequant_b_blockwise(owt, sw, G.FPROP))
                flop += 2.0 * (m1 - m0) * 128 * p["K"]
        return flop, time.perf_counter() - t0, f"{tiles} sampled grouped output tile(s) per projection"


class Nvfp4Step:
    name = "nvfp4"
    workload = "NVFP4 Llama-3.1-405B shapes: dgrad (8192,53248,16384), wgrad (16384,8192,53248)"

    def __init__(self, fq, rank, M=8192, H=16384, F=53248):
        self.fq, self.M, self.H, self.F = fq, M, H, F
        d = workloads.nvfp4(device="cuda", M=M, H=H, F=F)
        self.X, self.W, self.dY = d["X"], d["W"], d["dY"]
        dev = self.X.device
        u8 = torch.uint8
        sfb = lambda o, i: torch.empty(fq.fp8q_sf_bytes(fq.FP8Q_NVFP4, o, i, 1), dtype=u8, device=dev)  # noqa: E731
        self.qd_r, self.sd_r = torch.empty((M, F // 2), dtype=u8, device=dev), sfb(M, F)
        self.qd_c, self.sd_c = torch.empty((F, M // 2), dtype=u8, device=dev), sfb(F, M)
        self.qw, self.sw = torch.empty((H, F // 2), dtype=u8, device=dev), sfb(H, F)
        self.qx_c, self.sx_c = torch.empty((H, M // 2), dtype=u8, device=dev), sfb(H, M)
        self.g = torch.empty((4,), dtype=torch.float32, device=dev)
        self.dX = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty((H, F), dtype=torch.bfloat16, device=dev)
        self.gemm_flop = 2 * 2.0 * M * H * F

    def inputs(self):
        return [self.X, self.W, self.dY]

    def outputs(self):
        return [self.dX, self.dW]

    def launches(self):
        fq, M, H, F = self.fq, self.M, self.H, self.F
        P = lambda t: t.data_ptr()  # noqa: E731
        g = self.g

        def qd():
            assert fq.fp4q_rht16_quantize_sr(P(self.dY), M, F, F, fq.FP4Q_COL, 5, fq.FP4Q_ROW | fq.FP4Q_COL, 6,
                                             P(self.qd_r), P(self.sd_r), P(g[0:1]), P(self.qd_c), P(self.sd_c),
                                             P(g[1:2]), 1, fq._stream()) == 0

        def qw():
            assert fq.fp4q_rht16_quantize_sr(P(self.W), H, F, F, 0, 5, 0, 6, P(self.qw), P(self.sw), P(g[2:3]),
                                             None, None, None, 1, fq._stream()) == 0

        def qx():
            assert fq.fp4q_rht16_quantize_sr(P(self.X), M, H, H, fq.FP4Q_COL, 5, 0, 6, None, None, None,
                                             P(self.qx_c), P(self.sx_c), P(g[3:4]), 1, fq._stream()) == 0

        def dgrad():
            fq.gemm(self.qd_r, self.qw, fq.FP8Q_NVFP4, a_scale=self.sd_r, b_scale=self.sw, a_global=g[0:1],
                    b_global=g[2:3], K=F, out=self.dX)

        def wgrad():
            fq.gemm(self.qx_c, self.qd_c, fq.FP8Q_NVFP4, a_scale=self.sx_c, b_scale=self.sd_c, a_global=g[3:4],
                    b_global=g[1:2], K=M, out=self.dW)

        nv2 = lambda r, c: r * c * 4.0 + 2 * r * c * (0.5 + 1 / 16)  # noqa: E731  two outputs
        nv1 = lambda r, c: r * c * 4.0 + r * c * (0.5 + 1 / 16)      # noqa: E731  one output
        return [Launch("fp4q quantize dY (row SR + col RHT SR)", qd, "quantize_nvfp4", bytes_=nv2(M, F)),
                Launch("fp4q quantize W (row RNE)", qw, "quantize_nvfp4", bytes_=nv1(H, F)),
                Launch("fp4q quantize X (col RHT RNE)", qx, "quantize_nvfp4", bytes_=nv1(M, H)),
                Launch("gemm nvfp4 dgrad", dgrad, "gemm_nvfp4", flop=2.0 * M * H * F),
                Launch("gemm nvfp4 wgrad", wgrad, "gemm_nvfp4", flop=2.0 * M * H * F)]

    def cpu_sample(self, tiles=1):
        from oracle import gemm as G
        from oracle import quant as Q
        t0 = time.perf_counter()
        dYb = workloads.bf16_bits(self.dY[:1024])
        Wb = workloads.bf16_bits(self.W[:1024])
        # global amax over the sampled slabs stands in for the full tensors' (sample timing only)
        oa, sa, ga = Q.quantize_nvfp4_rowwise(dYb, sr=True, sr_seed=6, rows=list(range(128)))
        ob, sb, gb = Q.quantize_nvfp4_rowwise(Wb, rows=list(range(128)))
        G.reference(G.dequant_nvfp4(oa, sa, ga), G.dequant_nvfp4(ob, sb, gb))
        flop = 2.0 * 128 * 128 * self.F
        return flop, time.perf_counter() - t0, "1 dgrad output tile; amax over 1024-row slabs"


class Nvfp4TrainStep:
    """The NVFP4 training step of one Llama-3.1-405B MLP projection: fprop, dgrad and wgrad,
    with the weights quantized once in 16x16 blocks for both fprop and dgrad."""
    name = "nvfp4_train"
    workload = ("NVFP4 Llama-3.1-405B training step: fprop (8192,16384,53248) with 16x16-block weights, "
                "dgrad (8192,53248,16384), wgrad (16384,8192,53248)")

    def __init__(self, fq, rank, M=8192, H=16384, F=53248):
        self.fq, self.M, self.H, self.F = fq, M, H, F
        d = workloads.nvfp4(device="cuda", M=M, H=H, F=F)
        self.X, self.W, self.dY = d["X"], d["W"], d["dY"]
        dev = self.X.device
        u8 = torch.uint8
        sfb = lambda o, i: torch.empty(fq.fp8q_sf_bytes(fq.FP8Q_NVFP4, o, i, 1), dtype=u8, device=dev)  # noqa: E731
        self.qx_r, self.sx_r = torch.empty((M, H // 2), dtype=u8, device=dev), sfb(M, H)
        self.qx_c, self.sx_c = torch.empty((H, M // 2), dtype=u8, device=dev), sfb(H, M)
        self.qw_r, self.sw_r = torch.empty((H, F // 2), dtype=u8, device=dev), sfb(H, F)
        self.qw_c, self.sw_c = torch.empty((F, H // 2), dtype=u8, device=dev), sfb(F, H)
        self.qd_r, self.sd_r = torch.empty((M, F // 2), dtype=u8, device=dev), sfb(M, F)
        self.qd_c, self.sd_c = torch.empty((F, M // 2), dtype=u8, device=dev), sfb(F, M)
        self.g = torch.empty((5,), dtype=torch.float32, device=dev)
        self.Y = torch.empty((M, F), dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty((H, F), dtype=torch.bfloat16, device=dev)
        self.gemm_flop = 3 * 2.0 * M * H * F

    def inputs(self):
        return [self.X, self.W, self.dY]

    def outputs(self):
        return [self.Y, self.dX, self.dW]

    def launches(self):
        fq, M, H, F = self.fq, self.M, self.H, self.F
        P = lambda t: t.data_ptr()  # noqa: E731
        g = self.g

        def qx():   # rowwise RNE for fprop, colwise RHT RNE for wgrad
            assert fq.fp4q_rht16_quantize_sr(P(self.X), M, H, H, fq.FP4Q_COL, 5, 0, 6, P(self.qx_r), P(self.sx_r),
                                             P(g[0:1]), P(self.qx_c), P(self.sx_c), P(g[1:2]), 1, fq._stream()) == 0

        def qw():   # one 16x16-block quantization, both layouts
            assert fq.fp4q_quantize_2d16(P(self.W), H, F, F, P(self.qw_r), P(self.sw_r), P(self.qw_c), P(self.sw_c),
                                         P(g[2:3]), 1, fq._stream()) == 0

        def qd():   # rowwise SR for dgrad, colwise RHT SR for wgrad
            assert fq.fp4q_rht16_quantize_sr(P(self.dY), M, F, F, fq.FP4Q_COL, 5, fq.FP4Q_ROW | fq.FP4Q_COL, 6,
                                             P(self.qd_r), P(self.sd_r), P(g[3:4]), P(self.qd_c), P(self.sd_c),
                                             P(g[4:5]), 1, fq._stream()) == 0

        def fprop():
            fq.gemm(self.qx_r, self.qw_c, fq.FP8Q_NVFP4, a_scale=self.sx_r, b_scale=self.sw_c, a_global=g[0:1],
                    b_global=g[2:3], K=H, out=self.Y)

        def dgrad():
            fq.gemm(self.qd_r, self.qw_r, fq.FP8Q_NVFP4, a_scale=self.sd_r, b_scale=self.sw_r, a_global=g[3:4],
                    b_global=g[2:3], K=F, out=self.dX)

        def wgrad():
            fq.gemm(self.qx_c, self.qd_c, fq.FP8Q_NVFP4, a_scale=self.sx_c, b_scale=self.sd_c, a_global=g[1:2],
                    b_global=g[4:5], K=M, out=self.dW)

        nv2 = lambda r, c: r * c * 4.0 + 2 * r * c * (0.5 + 1 / 16)  # noqa: E731  two outputs
        return [Launch("fp4q quantize X (row RNE + col RHT RNE)", qx, "quantize_nvfp4", bytes_=nv2(M, H)),
                Launch("fp4q quantize W 16x16 blocks (both layouts)", qw, "quantize_nvfp4", bytes_=nv2(H, F)),
                Launch("gemm nvfp4 fprop (16x16 weights)", fprop, "gemm_nvfp4", flop=2.0 * M * H * F),
                Launch("fp4q quantize dY (row SR + col RHT SR)", qd, "quantize_nvfp4", bytes_=nv2(M, F)),
                Launch("gemm nvfp4 dgrad (16x16 weights)", dgrad, "gemm_nvfp4", flop=2.0 * M * H * F),
                Launch("gemm nvfp4 wgrad", wgrad, "gemm_nvfp4", flop=2.0 * M * H * F)]

    def cpu_sample(self, tiles=1):
        from oracle import gemm as G
        from oracle import quant as Q
        t0 = time.perf_counter()
        Xb = workloads.bf16_bits(self.X[:1024])
        Wb = workloads.bf16_bits(self.W[:, :128])
        # global amax over the sampled slabs stands in for the full tensors' (sample timing only)
        oa, sa, ga = Q.quantize_nvfp4_rowwise(Xb, rows=list(range(128)))
        _, _, ob, sb, gb = Q.quantize_nvfp4_2d(Wb)
        G.reference(G.dequant_nvfp4(oa, sa, ga), G.dequant_nvfp4(ob, sb, gb))
        flop = 2.0 * 128 * 128 * self.H
        return flop, time.perf_counter() - t0, "1 fprop output tile; amax over the sampled slabs"


STEPS = {"llama8b": LlamaStep, "tiny": TinyStep, "mxfp8": MxStep, "moe": MoeStep, "nvfp4": Nvfp4Step,
         "wgrad_acc": WgradAccStep, "delayed": DelayedStep, "nvfp4_train": Nvfp4TrainStep,
         "fprop_quant": FpropQuantStep}


# ============================================================================ measurement
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.summarize(lines)

    @staticmethod
    def summarize(lines):
        """nvidia-smi CSV lines (the fields of Q, no header, no units) -> median SM clock,
        maximum SM clock, throttle reasons seen Active in any sample, sample count.  Lines
        that do not parse (a partial last line when the sampler is stopped) are skipped."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[3:]))
                except ValueError:
                    pass
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": reasons, "samples": 0}
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def max_over_ranks(x, world):
    """The maximum of `x` over all ranks (the slowest rank's step time); a no-op at N = 1.
    Works on an NCCL group (CUDA tensor) and on a gloo group (CPU tensor)."""
    if world == 1:
        return float(x)
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flop_per_rank, world, ms):
    """Whole-job throughput: every rank runs its own step of `flop_per_rank` (weak scaling),
    timed by the slowest rank's `ms` per step."""
    return world * flop_per_rank / (ms * 1e-3) / 1e12


def step_kwargs(args):
    """Constructor arguments of the step for the smaller profiler cases (--tokens, --mx-shapes)."""
    kw = {}
    if args.tokens:
        kw["M"] = args.tokens
    if args.mx_shapes:
        kw["which"] = tuple(int(v) for v in args.mx_shapes.split(","))
    if args.separate_quant:
        kw["separate_quant"] = True
    return kw


def run_ours(args, rank, world, local_rank):
    import fp4_precision_gemm_b200 as fq
    torch.cuda.set_device(local_rank)
    fq.lib()
    step = STEPS[args.workload](fq, rank, **step_kwargs(args))
    launches = step.launches()
    n_launch = getattr(step, "launch_count", lambda: sum(L.kernels for L in launches))()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    clean = torch.zeros(64 << 20, dtype=torch.int32, device="cuda")   # 256 MiB, read after the flush
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        for L in launches:
            L.fn()
    torch.cuda.synchronize()
    assert fq.device_status() == 0
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in launches]
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.15)
    t_wall = time.perf_counter()
    for k in range(args.steps):
        # L2 flush outside the events: a 256 MiB write, then a 256 MiB read, so the step starts
        # from an L2 holding none of its data and no dirty lines (else the first kernel of
        # the step would pay the write-back of the flush buffer)
        flush.fill_(k & 0xFF)
        clean.max()
        for L, (a, b) in zip(launches, ev[k]):
            a.record(stream)
            L.fn()
            b.record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    clocks = sampler.stop()
    barrier()
    per = [[a.elapsed_time(b) for (a, b) in row] for row in ev]          # ms
    step_ms = [ev[k][0][0].elapsed_time(ev[k][-1][1]) for k in range(args.steps)]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world)
    status = fq.device_status()

    # per-kernel statistics (mean over the timed steps)
    peaks, src = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    kern = []
    for i, L in enumerate(launches):
        t_ms = statistics.mean(r[i] for r in per)
        d = {"name": L.name, "kernel": L.kernel, "ms": round(t_ms, 4)}
        if L.flop:
            tf = L.flop / (t_ms * 1e-3) / 1e12
            peak = fp4_peak if "nvfp4" in L.kernel else fp8_peak
            d.update({"tflops": round(tf, 1), "frac": round(tf / peak, 3)})
        if L.bytes:
            gbs = L.bytes / (t_ms * 1e-3) / 1e9
            d.update({"gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 3)})
        kern.append(d)
    # dominant kernel: the GEMM family with the largest share of the step
    fam = {}
    for d, L in zip(kern, launches):
        f = fam.setdefault(L.kernel, {"ms": 0.0, "flop": 0.0, "bytes": 0.0})
        f["ms"] += d["ms"]
        f["flop"] += L.flop
        f["bytes"] += L.bytes
    dom = max(fam, key=lambda k: fam[k]["ms"])
    f = fam[dom]
    if f["flop"]:
        peak = fp4_peak if "nvfp4" in dom else fp8_peak
        ach = f["flop"] / (f["ms"] * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 1), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / peak, 3), "traffic": None,
                "peak_source": f"{src}: bf16_tflops x {FP4_PER_BF16 if 'nvfp4' in dom else FP8_PER_BF16:g} "
                               "(nominal dense ratio), burst figure"}
    else:
        ach = f["bytes"] / (f["ms"] * 1e-3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 3), "traffic": None, "peak_source": f"{src}: hbm_gbs"}
    roof["traffic"] = traffic_for(dom, args.workload) if not (args.tokens or args.mx_shapes) else None

    make_step = lambda: STEPS[args.workload](fq, rank, **step_kwargs(args))  # noqa: E731
    e2e = measure_e2e(step, launches, stream, args, make_step, world) if (not args.no_e2e) else None
    value = job_tflops(step.gemm_flop, world, ms)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4_e2m1" if args.workload.startswith("nvfp4") else "fp8_e4m3",
        "data": "synthetic (seeded normal BF16 with outliers; see workloads.py)",
        "config": {"workload": step.workload, "l2": "flushed between steps (256 MiB write, then 256 MiB read)",
                   "gemm_tflop_per_step": round(step.gemm_flop / 1e12, 4),
                   "parallelism": f"dp{world} (independent replicas, no collective)",
                   **({"quantize_launch": "three calls" if step.separate_quant else "one multi-tensor launch"}
                      if hasattr(step, "separate_quant") else {})},
        "roofline": roof, "kernels": kern, "gpu_launches": n_launch * args.steps,
        "clocks": clocks, "e2e": e2e, "device_status": status, "wall_s_timed_region": round(t_wall, 3),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(step)
    return out


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, when one exists for this kernel
    and workload (null otherwise)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        return d.get(workload, {}).get(kernel)
    except (OSError, ValueError):
        return None


def measure_e2e(step, launches, stream, args, make_step, world):
    """Same step through the C ABI with the inputs in pinned HOST memory: every step's
    host->device copies, its kernels and the device->host copies of its results are inside
    the timed region.  Steps are pipelined over two device buffer sets on three streams: the
    inputs of step i+1 go up (one copy engine) and the results of step i-1 come down (the
    other) while step i's kernels run, as a training loop that streams its data would."""
    steps = [step, make_step()]
    launch_sets = [launches, steps[1].launches()]
    ins = [st.inputs() for st in steps]
    outs = [st.outputs() for st in steps]
    h_in = [t.cpu().pin_memory() for t in ins[0]]
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs[0]]
    bi = sum(t.numel() * t.element_size() for t in ins[0])
    bo = sum(t.numel() * t.element_size() for t in outs[0])
    reps = max(4, args.steps)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_o = [torch.cuda.Event() for _ in range(2)]
    with torch.cuda.stream(stream):
        for L in launch_sets[1]:        # the second buffer set's launches, once, untimed
            L.fn()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    s_out.wait_event(a)
    for i in range(reps):
        k = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_c[k])      # step i-2's kernels have read buffer set k
            for d, h in zip(ins[k], h_in):
                d.copy_(h, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_o[k])    # step i-2's results have left buffer set k
            for L in launch_sets[k]:
                L.fn()
            ev_c[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[k])
            for d, h in zip(outs[k], h_out):
                h.copy_(d, non_blocking=True)
            ev_o[k].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / reps, world)
    del steps, launch_sets
    return {"value": round(job_tflops(step.gemm_flop, world, ms), 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "pipelined": "2 buffer sets, H2D / kernels / D2H on 3 streams"}


def cpu_cores():
    """Threads the oracle's NumPy/BLAS calls use on this host."""
    try:
        import numpy as np  # noqa: F401
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info()] or [1]))
    except Exception:  # noqa: BLE001
        return int(torch.get_num_threads())


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(step):
    blas = cpu_cores()
    # a bounded sample of about 12 s of CPU work: time one sampled tile per GEMM, then size
    # the measured sample (more sampled tiles of the same workload) from it
    _, dt1, _ = step.cpu_sample(tiles=1)
    tiles = max(1, min(64, int(12.0 / max(dt1, 1e-3))))
    flop, dt, what = step.cpu_sample(tiles=tiles)
    out = {"value": round(flop / dt / 1e12, 6), "unit": "TFLOP/s", "cores": int(blas), "kind": "oracle",
           "sample": what, "seconds": round(dt, 2), "cpu_model": cpu_model(), "host_threads": os.cpu_count()}
    if hasattr(step, "cpu_quant_sample"):
        # the quantizers' oracle: elementwise NumPy, one thread whatever the BLAS thread count
        nbytes, qdt, qwhat = step.cpu_quant_sample()
        out["quantize"] = {"value": round(nbytes / qdt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                           "sample": qwhat, "seconds": round(qdt, 2)}
    return out


def run_reference(args, rank, world):
    """The CPU oracle as it stands, timed on the host cores on a bounded sample per step.
    Rank 0 alone runs it; the other ranks do no work."""
    if rank != 0:
        return None
    cuda = torch.cuda.is_available()
    if cuda:
        torch.cuda.set_device(0)
    import fp4_precision_gemm_b200 as fq
    if cuda:
        step = STEPS[args.workload](fq, 0)
    elif args.workload == "tiny":
        step = TinyStep(fq, 0, device="cpu")     # inputs drawn on the host (same recipe, CPU generator)
    else:
        return {"impl": "reference", "unavailable": "no CUDA device: the inputs of this workload are drawn on the GPU"}
    for _ in range(args.warmup):
        step.cpu_sample()
    flops, secs = 0.0, 0.0
    what = ""
    for _ in range(args.steps):
        f, dt, what = step.cpu_sample()
        flops += f
        secs += dt
    value = flops / secs / 1e12
    cb = {"cores": cpu_cores()}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded normal BF16 with outliers; see workloads.py)",
            "config": {"workload": step.workload, "sample": what},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cb["cores"], "kind": "oracle",
                             "sample": what},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(n, argv, timeout_s=None):
    """Runs this script as n ranks under torch.distributed.run on 127.0.0.1 (one node) and
    returns its exit code; each rank sees RANK / LOCAL_RANK / WORLD_SIZE in its environment."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd, timeout=timeout_s)


def init_ranks(n_expected, backend):
    """Reads the launcher's environment, checks that it started n_expected ranks, and joins
    the process group (short timeout, so ranks that wait for a lost peer end with an error).
    Returns (rank, world, local_rank)."""
    import datetime
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_expected:
        raise SystemExit(f"bench.py: --gpus {n_expected} but the launcher started WORLD_SIZE={world} ranks")
    if world > 1:
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
            kw["device_id"] = torch.device("cuda", local_rank)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=600 if backend == "gloo"
                                                                                  else 120), **kw)
    return rank, world, local_rank


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(STEPS) + ["all"], default="llama8b")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="llama8b / nvfp4: token count M (default 8192); smaller cases for profiler captures")
    ap.add_argument("--separate-quant", action="store_true",
                    help="llama8b only: quantize X, W and dY with three calls instead of one multi-tensor launch")
    ap.add_argument("--mx-shapes", default=None,
                    help="mxfp8 only: comma list of its GEMM shapes to run (0, 1, 2); smaller profiler cases")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.tokens and args.workload not in ("llama8b", "nvfp4", "nvfp4_train"):
        ap.error("--tokens applies to the llama8b and nvfp4 workloads only")
    if args.mx_shapes and args.workload != "mxfp8":
        ap.error("--mx-shapes applies to the mxfp8 workload only")
    if args.separate_quant and args.workload != "llama8b":
        ap.error("--separate-quant applies to the llama8b workload only")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))

    backend = "nccl" if (args.impl == "ours" and torch.cuda.is_available()) else "gloo"
    rank, world, local_rank = init_ranks(args.gpus, backend)
    comm = None
    if world > 1:
        comm = {"backend": torch.distributed.get_backend(), "world_size": torch.distributed.get_world_size()}
    names = sorted(STEPS) if args.workload == "all" else [args.workload]
    for name in names:
        args.workload = name
        if args.impl == "reference":
            out = run_reference(args, rank, world)
        else:
            out = run_ours(args, rank, world, local_rank)
        if rank == 0 and out is not None:
            if comm is not None and "unavailable" not in out:
                out["comm"] = comm
            print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
