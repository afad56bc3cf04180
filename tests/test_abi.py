"""The C-ABI library loads on a machine without a GPU, exports every function include/fp8q.h
declares, and its host-side validation rejects bad arguments with the documented status
codes before touching the device (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

import fp4_precision_gemm_b200 as fq

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp8q.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(fq.library_path):
        from fp4_precision_gemm_b200 import build
        build.build()
    return fq.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp[48]q_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("fp8q_quantize_1x128", "fp8q_quantize_128x128", "fp8q_quantize_mx32",
                     "fp4q_rht16_quantize_sr", "fp8q_gemm_blockscaled"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fq.library_path], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)
    assert set(fq.EXPORTED_SYMBOLS) <= exported


def test_version_and_status_strings(L):
    assert fq.fp8q_version().startswith("fp8q ")
    assert "sm_100a" in fq.fp8q_version()
    for st in range(7):
        assert fq.fp8q_status_string(st)


def test_sf_bytes(L):
    assert fq.fp8q_sf_bytes(fq.FP8Q_MXFP8, 256, 512, fq.FP8Q_SF_ROWMAJOR) == 256 * 16
    assert fq.fp8q_sf_bytes(fq.FP8Q_MXFP8, 200, 96, fq.FP8Q_SF_MMA_TILED) == 256 * 4
    assert fq.fp8q_sf_bytes(fq.FP8Q_NVFP4, 300, 656, fq.FP8Q_SF_MMA_TILED) == 384 * 44
    assert fq.fp8q_sf_bytes(fq.FP8Q_BLOCKWISE, 300, 656, fq.FP8Q_SF_MMA_TILED) == 0


P = ctypes.c_void_p
ALIGNED = P(0x10000)          # never dereferenced: validation fails before any launch
MISALIGNED = P(0x10008)


def test_quantize_validation_codes(L):
    s = P(0)
    # no outputs at all
    assert fq.fp8q_quantize_1x128(ALIGNED, 128, 128, 128, None, None, 0, None, None, 0, s) == 1
    # rowwise needs cols % 128 == 0
    assert fq.fp8q_quantize_1x128(ALIGNED, 128, 100, 104, ALIGNED, ALIGNED, 128, None, None, 0, s) == 2
    # ld_x must be >= cols and a multiple of 8
    assert fq.fp8q_quantize_1x128(ALIGNED, 128, 128, 100, ALIGNED, ALIGNED, 128, None, None, 0, s) == 2
    # input must be 16-byte aligned
    assert fq.fp8q_quantize_1x128(MISALIGNED, 128, 128, 128, ALIGNED, ALIGNED, 128, None, None, 0, s) == 3
    # colwise needs rows % 128 == 0
    assert fq.fp8q_quantize_1x128(ALIGNED, 100, 128, 128, None, None, 0, ALIGNED, ALIGNED, 128, s) == 2
    # 128x128 needs both dims multiple of 128 and a scale pointer
    assert fq.fp8q_quantize_128x128(ALIGNED, 128, 200, 200, ALIGNED, None, ALIGNED, s) == 2
    assert fq.fp8q_quantize_128x128(ALIGNED, 128, 128, 128, ALIGNED, None, None, s) == 1
    # MX: bad layout enum, and colwise rows % 32
    assert fq.fp8q_quantize_mx32(ALIGNED, 64, 64, 64, ALIGNED, ALIGNED, None, None, 7, s) == 4
    assert fq.fp8q_quantize_mx32(ALIGNED, 48, 64, 64, None, None, ALIGNED, ALIGNED, 0, s) == 2
    # per-tensor: cols % 8
    assert fq.fp8q_quantize_tensor(ALIGNED, 4, 12, 16, ALIGNED, ALIGNED, s) == 2
    # NVFP4: unknown flag bits, cols % 16, partial output triple
    assert fq.fp4q_rht16_quantize_sr(ALIGNED, 16, 16, 16, 4, 0, 0, 0, ALIGNED, ALIGNED, ALIGNED,
                                     None, None, None, 0, s) == 4
    assert fq.fp4q_rht16_quantize_sr(ALIGNED, 16, 24, 24, 0, 0, 0, 0, ALIGNED, ALIGNED, ALIGNED,
                                     None, None, None, 0, s) == 2
    assert fq.fp4q_rht16_quantize_sr(ALIGNED, 16, 16, 16, 0, 0, 0, 0, ALIGNED, None, ALIGNED,
                                     None, None, None, 0, s) == 1


def test_quantize_empty_is_ok_without_launch(L):
    s = P(0)
    assert fq.fp8q_quantize_1x128(ALIGNED, 0, 128, 128, ALIGNED, ALIGNED, 0, None, None, 0, s) == 0
    assert fq.fp8q_quantize_128x128(ALIGNED, 0, 128, 128, ALIGNED, None, ALIGNED, s) == 0
    assert fq.fp8q_quantize_mx32(ALIGNED, 0, 64, 64, ALIGNED, ALIGNED, None, None, 0, s) == 0


def _args(**kw):
    a = fq.GemmArgs()
    a.recipe, a.layout = fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP
    a.M, a.N, a.K = 256, 256, 512
    a.a = a.b = a.c = a.a_scale = a.b_scale = 0x10000
    a.lda = a.ldb = 512
    a.ld_sa, a.ld_sb, a.ldc = 256, 4, 256
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_gemm_validation_codes(L):
    s = P(0)
    assert fq.fp8q_gemm_blockscaled(_args(K=500), s) == 2                    # K % 128
    assert fq.fp8q_gemm_blockscaled(_args(recipe=fq.FP8Q_NVFP4, K=384, lda=192, ldb=192), s) == 2
    assert fq.fp8q_gemm_blockscaled(_args(ldc=100), s) == 2                  # ldc < N
    assert fq.fp8q_gemm_blockscaled(_args(lda=520), s) == 2                  # lda % 16
    assert fq.fp8q_gemm_blockscaled(_args(a=0x10004), s) == 3                # alignment
    assert fq.fp8q_gemm_blockscaled(_args(a_scale=None), s) == 1
    assert fq.fp8q_gemm_blockscaled(_args(recipe=9), s) == 4
    assert fq.fp8q_gemm_blockscaled(_args(recipe=fq.FP8Q_PERTENSOR), s) == 1  # globals missing
    assert fq.fp8q_gemm_blockscaled(_args(layout=fq.FP8Q_DGRAD, ld_sb=1), s) == 2
    assert fq.fp8q_gemm_blockscaled(_args(layout=fq.FP8Q_WGRAD, ld_sb=100), s) == 2
    # grouped only for the blockwise FPROP layout
    assert fq.fp8q_gemm_blockscaled(_args(recipe=fq.FP8Q_MXFP8, m_offsets=0x10000, num_groups=2), s) == 4
    assert fq.fp8q_gemm_blockscaled(_args(num_groups=2, m_offsets=None), s) == 1
    assert L.fp8q_gemm_blockscaled(None, s) == 1
    # M == 0 or N == 0: nothing to do
    assert fq.fp8q_gemm_blockscaled(_args(M=0), s) == 0
    assert fq.fp8q_gemm_blockscaled(_args(N=0), s) == 0


@pytest.mark.parametrize("recipe,unit", [("FP8Q_BLOCKWISE", 128), ("FP8Q_MXFP8", 128), ("FP8Q_PERTENSOR", 128),
                                         ("FP8Q_NVFP4", 256)])
def test_gemm_k_rule_per_recipe(L, recipe, unit):
    """The header's K rule for each recipe: the smallest accepted K passes validation (on a
    machine without a GPU the call then fails at the first CUDA call, FP8Q_ERR_CUDA, never
    FP8Q_ERR_SHAPE); K one block smaller than the unit, or not a multiple of it, is
    FP8Q_ERR_SHAPE."""
    r = getattr(fq, recipe)
    fp4 = r == fq.FP8Q_NVFP4

    def call(K):
        kb = K // 2 if fp4 else K
        ld = max(16, (kb + 15) // 16 * 16)
        kw = dict(recipe=r, K=K, lda=ld, ldb=ld, ld_sb=max(1, K // 128))
        if r in (fq.FP8Q_PERTENSOR, fq.FP8Q_NVFP4):
            kw.update(a_global=0x10000, b_global=0x10000)
        return fq.fp8q_gemm_blockscaled(_args(**kw), P(0))

    import torch
    accepted = fq.FP8Q_OK if torch.cuda.is_available() else fq.FP8Q_ERR_CUDA
    if not torch.cuda.is_available():
        assert call(unit) == accepted
        assert call(3 * unit) == accepted
    assert call(unit // 2) == fq.FP8Q_ERR_SHAPE
    assert call(unit + unit // 4) == fq.FP8Q_ERR_SHAPE
    assert call(unit + 16) == fq.FP8Q_ERR_SHAPE


def test_product_path_has_no_cpu_fallback():
    """The binding must raise when the library is absent instead of computing on the host."""
    import importlib
    src = open(os.path.join(os.path.dirname(fq.__file__), "__init__.py")).read()
    assert "oracle" not in src and "numpy" not in src
    mod = importlib.import_module("fp4_precision_gemm_b200")
    saved_path, saved_lib = mod.library_path, mod._LIB
    try:
        mod.library_path, mod._LIB = "/nonexistent/libfp8q.so", None
        with pytest.raises(ImportError):
            mod.lib()
    finally:
        mod.library_path, mod._LIB = saved_path, saved_lib


def test_selftest_rejects_limits_out_of_range(L):
    assert L.fp8q_selftest_bounded_wait(10, None) == fq.FP8Q_ERR_SHAPE          # below 1 us
    assert L.fp8q_selftest_bounded_wait(5_000_000_000, None) == fq.FP8Q_ERR_SHAPE   # above 1 s


def test_grouped_weight_quantizer_validates_before_launching(L):
    s = None
    assert fq.fp8q_quantize_128x128_grouped(ALIGNED, -1, 128, 128, 128, ALIGNED, None, ALIGNED, s) == fq.FP8Q_ERR_SHAPE
    assert fq.fp8q_quantize_128x128_grouped(ALIGNED, 2, 128, 100, 128, ALIGNED, None, ALIGNED, s) == fq.FP8Q_ERR_SHAPE
    assert fq.fp8q_quantize_128x128_grouped(ALIGNED, 2, 128, 128, 128, ALIGNED, None, None, s) == fq.FP8Q_ERR_NULL
    assert fq.fp8q_quantize_128x128_grouped(ALIGNED, 0, 128, 128, 128, ALIGNED, None, ALIGNED, s) == fq.FP8Q_OK


def test_fp32_accumulate_is_blockwise_only_and_needs_ldc_multiple_of_4(L):
    s = None
    assert fq.fp8q_gemm_blockscaled(_args(recipe=fq.FP8Q_MXFP8, c_fp32_accumulate=1), s) == fq.FP8Q_ERR_UNSUPPORTED
    assert fq.fp8q_gemm_blockscaled(_args(c_fp32_accumulate=1, ldc=258), s) == fq.FP8Q_ERR_SHAPE


def test_delayed_quantizer_and_fp8_format_validation(L):
    s = None
    f = fq.fp8q_quantize_tensor_delayed
    assert f(ALIGNED, 8, 16, 16, ALIGNED, 0, 0, 0, ALIGNED, ALIGNED, s) == fq.FP8Q_ERR_SHAPE       # no history
    assert f(ALIGNED, 8, 16, 16, ALIGNED, 4, 4, 0, ALIGNED, ALIGNED, s) == fq.FP8Q_ERR_SHAPE       # pos out of range
    assert f(ALIGNED, 8, 16, 16, ALIGNED, 4, 0, 2, ALIGNED, ALIGNED, s) == fq.FP8Q_ERR_UNSUPPORTED # format
    assert f(ALIGNED, 8, 16, 16, None, 4, 0, 0, ALIGNED, ALIGNED, s) == fq.FP8Q_ERR_NULL
    g = fq.fp8q_gemm_blockscaled
    assert g(_args(a_format=1), s) == fq.FP8Q_ERR_UNSUPPORTED          # E5M2 is per-tensor only
    assert g(_args(recipe=fq.FP8Q_PERTENSOR, b_format=3), s) == fq.FP8Q_ERR_UNSUPPORTED


def test_nvfp4_2d16_validation(L):
    s = None
    f = fq.fp4q_quantize_2d16
    assert f(ALIGNED, 16, 24, 24, ALIGNED, ALIGNED, None, None, ALIGNED, 0, s) == fq.FP8Q_ERR_SHAPE      # cols % 16
    assert f(ALIGNED, 24, 16, 16, ALIGNED, ALIGNED, None, None, ALIGNED, 0, s) == fq.FP8Q_ERR_SHAPE      # rows % 16
    assert f(ALIGNED, 16, 16, 16, ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 0, s) == fq.FP8Q_ERR_NULL   # no g_dec
    assert f(ALIGNED, 16, 16, 16, None, None, None, None, ALIGNED, 0, s) == fq.FP8Q_ERR_NULL            # no output
    assert f(ALIGNED, 16, 16, 16, ALIGNED, None, None, None, ALIGNED, 0, s) == fq.FP8Q_ERR_NULL         # half a pair
    assert f(ALIGNED, 16, 16, 16, ALIGNED, ALIGNED, None, None, ALIGNED, 2, s) == fq.FP8Q_ERR_UNSUPPORTED
    assert f(ALIGNED, 16, 16, 16, P(0x10008), ALIGNED, None, None, ALIGNED, 0, s) == fq.FP8Q_ERR_ALIGN
    assert f(ALIGNED, 16, 16, 12, ALIGNED, ALIGNED, None, None, ALIGNED, 0, s) == fq.FP8Q_ERR_SHAPE      # ld_x < cols
    assert f(ALIGNED, 0, 16, 16, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 0, s) == fq.FP8Q_OK       # empty


def test_fused_output_quantization_validation(L):
    s = None
    base = dict(q_out=ALIGNED.value, s_out=ALIGNED.value, ld_q_out=256, ld_s_out=256, K=512, N=256, M=256, ldc=256)
    g = fq.fp8q_gemm_blockscaled
    assert g(_args(**{**base, "recipe": fq.FP8Q_MXFP8}), s) == fq.FP8Q_ERR_UNSUPPORTED      # blockwise only
    assert g(_args(**{**base, "c_fp32_accumulate": 1}), s) == fq.FP8Q_ERR_UNSUPPORTED       # not with FP32 C
    assert g(_args(**{**base, "s_out": None}), s) == fq.FP8Q_ERR_NULL
    assert g(_args(**{**base, "N": 200, "ldc": 200}), s) == fq.FP8Q_ERR_SHAPE               # N % 128
    assert g(_args(**{**base, "K": 256}), s) == fq.FP8Q_ERR_SHAPE                           # K >= 384
    assert g(_args(**{**base, "ld_q_out": 264}), s) == fq.FP8Q_ERR_SHAPE                    # % 16
    assert g(_args(**{**base, "ld_s_out": 100}), s) == fq.FP8Q_ERR_SHAPE                    # >= M
    assert g(_args(**{**base, "q_out": MISALIGNED.value}), s) == fq.FP8Q_ERR_ALIGN


def test_quantize_multi_validates_every_item_before_launching():
    """Bad items are rejected with their single-call status, before any launch (no GPU
    here, so a launch would fail with FP8Q_ERR_CUDA instead)."""
    S = 0x10000                   # never dereferenced: validation fails before any launch
    def item(kind, rows, cols, **kw):
        it = fq.QuantItem()
        it.kind, it.x, it.rows, it.cols, it.ld_x = kind, S, rows, cols, cols
        for k, v in kw.items():
            setattr(it, k, v)
        return it
    def call(*its):
        arr = (fq.QuantItem * max(len(its), 1))(*its)
        return fq.fp8q_quantize_multi(arr, len(its), None)
    one = dict(q_row=S, s_row=S, ld_s_row=128)
    w = dict(q_t=S, q=S, s=S)
    assert call() == fq.FP8Q_OK
    assert fq.fp8q_quantize_multi(None, 1, None) == fq.FP8Q_ERR_NULL
    arr = (fq.QuantItem * 9)(*[item(fq.FP8Q_ITEM_1X128, 0, 128, **one) for _ in range(9)])
    assert fq.fp8q_quantize_multi(arr, 9, None) == fq.FP8Q_ERR_SHAPE             # more than 8 items
    assert fq.fp8q_quantize_multi(arr, -1, None) == fq.FP8Q_ERR_SHAPE
    assert call(item(7, 128, 128, **one)) == fq.FP8Q_ERR_UNSUPPORTED              # unknown kind
    assert call(item(fq.FP8Q_ITEM_1X128, 128, 100, **one)) == fq.FP8Q_ERR_SHAPE  # cols % 128
    assert call(item(fq.FP8Q_ITEM_1X128, 128, 128)) == fq.FP8Q_ERR_NULL          # no output
    assert call(item(fq.FP8Q_ITEM_128X128, 128, 128, s=S)) == fq.FP8Q_ERR_NULL   # neither layout
    assert call(item(fq.FP8Q_ITEM_128X128, 128, 128, q=S)) == fq.FP8Q_ERR_NULL   # no scales
    assert call(item(fq.FP8Q_ITEM_128X128, 100, 128, **w)) == fq.FP8Q_ERR_SHAPE  # K % 128
    # a valid item first: the bad second item still stops the call before any launch
    assert call(item(fq.FP8Q_ITEM_1X128, 128, 128, **one),
                item(fq.FP8Q_ITEM_1X128, 128, 128, q_row=S + 1, s_row=S, ld_s_row=128)) == fq.FP8Q_ERR_ALIGN
    # empty items are skipped: nothing to launch
    assert call(item(fq.FP8Q_ITEM_1X128, 0, 128, **one), item(fq.FP8Q_ITEM_128X128, 128, 0, **w)) == fq.FP8Q_OK
    assert ctypes.sizeof(fq.QuantItem) == 112


@pytest.mark.skipif(subprocess.run(["which", "gcc"], capture_output=True).returncode != 0, reason="needs gcc")
def test_binding_structs_match_the_header_layout(tmp_path):
    """The ctypes mirrors have the size and field offsets that a C compiler gives the header's
    argument structs (compiled from include/fp8q.h on the host)."""
    exe = str(tmp_path / "abi_layout")
    here = os.path.dirname(os.path.abspath(__file__))
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), "-o", exe,
                    os.path.join(here, "host", "abi_layout.c")], check=True)
    got = dict(line.split() for line in subprocess.run([exe], check=True, capture_output=True,
                                                        text=True).stdout.splitlines())
    for cname, cls in (("fp8q_gemm_args", fq.GemmArgs), ("fp8q_quant_item", fq.QuantItem)):
        assert int(got[cname]) == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert int(got[f"{cname}.{field}"]) == getattr(cls, field).offset, (cname, field)
        assert sum(k.startswith(cname + ".") for k in got) == len(cls._fields_), cname


def test_gemm_workspace_bytes_is_zero_without_a_device_or_a_splittable_call(L):
    """The workspace query never fails: NULL arguments, non-blockwise recipes and, here with no
    GPU, every call report 0 (the GEMM then keeps its unsplit schedule)."""
    assert L.fp8q_gemm_workspace_bytes(None) == 0
    for recipe in (fq.FP8Q_BLOCKWISE, fq.FP8Q_MXFP8, fq.FP8Q_NVFP4):
        assert fq.gemm_workspace_bytes(8192, 14336, 4096, recipe, fq.FP8Q_FPROP) == 0
    assert fq.gemm_workspace_bytes(300, 19328, 6144, fq.FP8Q_BLOCKWISE, fq.FP8Q_WGRAD, accumulate_fp32=True) == 0
    assert fq.gemm_workspace_bytes(300, 19328, 6144, fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, fused_quant=True) == 0


def test_gemm_workspace_argument_checked_before_anything_runs(L):
    """A misaligned workspace given to a GEMM that could use one is an alignment error, found
    on the host before any launch."""
    a = fq.GemmArgs()
    a.recipe, a.layout, a.M, a.N, a.K = fq.FP8Q_BLOCKWISE, fq.FP8Q_FPROP, 256, 256, 512
    a.a = a.b = a.a_scale = a.b_scale = a.c = 1 << 20
    a.lda = a.ldb = 512
    a.ld_sa, a.ld_sb, a.ldc = 256, 4, 256
    a.workspace, a.workspace_bytes = (1 << 20) + 8, 1 << 20
    assert fq.fp8q_gemm_blockscaled(a, None) == fq.FP8Q_ERR_ALIGN
