"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no quantization or GEMM arithmetic: it only draws tensors.  It is the
one module that both the CPU oracle's tests and the CUDA path's tests and bench consume.

Recipe (every tensor):
  1. a torch.Generator on the requested device, seeded with base_seed * 100 + tensor_id;
  2. FP32 draw N(0, sigma) of the full shape (torch.randn, row-major);
  3. outliers: k = floor(frac * numel) positions drawn with torch.randint from the same
     generator, de-duplicated, and multiplied by the factor (in FP32);
  4. one cast to BF16 (round to nearest even).
MoE routing (DeepSeek-V3 shape): for each token, 8 distinct experts out of 32 drawn with
torch.multinomial without replacement, popularity p_e proportional to (e + 1)^-1.1.

Named workloads (sizes in elements; weights given K x N, row-major):
  tiny      A 256x512 N(0,1) 0.1% x100; B 512x256 N(0,0.02)                    seed 0
  llama8b   X 8192x4096 N(0,1) 0.1% x50; W 4096x14336 N(0,0.02);
            dY 8192x14336 N(0,1e-3)                                            seed 2
  mxfp8     A 8192x4096 (x2), 8192x14336 N(0,1); W 4096x4096, 4096x14336,
            14336x4096 N(0,0.02)                                               seed 3
  moe       16384 tokens x top-8 of 32 experts; A_up 131072x7168, A_down
            131072x2048 N(0,1); W_up 32x(7168x2048), W_down 32x(2048x7168)
            N(0,0.006)                                                         seed 4
  nvfp4     X 8192x16384 N(0,1); W 16384x53248 N(0,0.02); dY 8192x53248
            N(0,1e-3) 0.05% x100; rht_seed 5, sr_seed 6                       seed 5
"""
import math

import torch


def normal_bf16(shape, sigma, seed, outlier_frac=0.0, outlier_factor=1.0, device="cpu"):
    """BF16 tensor: N(0, sigma) in FP32, outliers multiplied in FP32, one cast to BF16."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    x.mul_(sigma)
    numel = x.numel()
    k = int(math.floor(outlier_frac * numel))
    if k > 0:
        idx = torch.randint(0, numel, (k,), generator=g, device=device)
        idx = torch.unique(idx)
        flat = x.view(-1)
        flat[idx] = flat[idx] * outlier_factor
    return x.to(torch.bfloat16)


def tensor_seed(base_seed, tensor_id):
    return base_seed * 100 + tensor_id


def moe_routing(tokens=16384, experts=32, topk=8, alpha=1.1, seed=400):
    """Per-expert token counts and row offsets (int32, length experts + 1)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    p = (torch.arange(experts, dtype=torch.float64) + 1.0) ** (-alpha)
    p = (p / p.sum()).to(torch.float32)
    choice = torch.multinomial(p.expand(tokens, experts), topk, replacement=False,
                               generator=g)
    counts = torch.bincount(choice.reshape(-1), minlength=experts)
    offsets = torch.zeros(experts + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(counts, 0)
    return counts.to(torch.int32), offsets.to(torch.int32)


# ----------------------------------------------------------------------------- configs
def tiny(device="cpu"):
    return {
        "A": normal_bf16((256, 512), 1.0, tensor_seed(0, 0), 1e-3, 100.0, device),
        "B": normal_bf16((512, 256), 0.02, tensor_seed(0, 1), device=device),
    }


def llama8b(device="cpu", M=8192, K=4096, N=14336):
    return {
        "X": normal_bf16((M, K), 1.0, tensor_seed(2, 0), 1e-3, 50.0, device),
        "W": normal_bf16((K, N), 0.02, tensor_seed(2, 1), device=device),
        "dY": normal_bf16((M, N), 1e-3, tensor_seed(2, 2), device=device),
    }


MXFP8_GEMMS = [(8192, 4096, 4096), (8192, 4096, 14336), (8192, 14336, 4096)]  # (M, K, N)


def mxfp8(device="cpu", which=None, outliers=False):
    out = {}
    for i, (M, K, N) in enumerate(MXFP8_GEMMS):
        if which is not None and i not in which:
            continue
        frac, fac = (1e-3, 50.0) if outliers else (0.0, 1.0)
        out[f"A{i}"] = normal_bf16((M, K), 1.0, tensor_seed(3, i), frac, fac, device)
        out[f"W{i}"] = normal_bf16((K, N), 0.02, tensor_seed(3, 3 + i), device=device)
    return out


def moe(device="cpu", proj="up", hidden=7168, inter=2048, experts=32):
    counts, offsets = moe_routing(seed=tensor_seed(4, 0), experts=experts)
    total = int(offsets[-1])
    if proj == "up":
        K, N, ida, idw = hidden, inter, 1, 2
    else:
        K, N, ida, idw = inter, hidden, 3, 4
    return {
        "A": normal_bf16((total, K), 1.0, tensor_seed(4, ida), device=device),
        "W": normal_bf16((experts, K, N), 0.006, tensor_seed(4, idw), device=device),
        "counts": counts, "offsets": offsets,
    }


def nvfp4(device="cpu", M=8192, H=16384, F=53248, which=("X", "W", "dY")):
    out = {"rht_seed": 5, "sr_seed": 6}
    if "X" in which:
        out["X"] = normal_bf16((M, H), 1.0, tensor_seed(5, 0), device=device)
    if "W" in which:
        out["W"] = normal_bf16((H, F), 0.02, tensor_seed(5, 1), device=device)
    if "dY" in which:
        out["dY"] = normal_bf16((M, F), 1e-3, tensor_seed(5, 2), 5e-4, 100.0, device)
    return out


def bf16_bits(t):
    """CPU numpy uint16 view of a BF16 tensor (for the oracle)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
