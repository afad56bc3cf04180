"""Quantize kernels vs the CPU oracle, bit-exact (codes and scales), through the C ABI.

Small shapes span several 128x128 tiles with ragged tails; the edge cases cover all-zero
tiles, subnormal and maximal BF16 magnitudes and signed zeros; full-size workloads are
checked on sampled row and column bands (the oracle quantizes the same bands from the same
BF16 inputs)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import quant as Q

pytestmark = pytest.mark.gpu


def f32bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def host(t):
    return t.detach().cpu().numpy()


def crafted_bf16(R, C, seed):
    """Random data plus edge cases: a zero tile, subnormal magnitudes, BF16 max, -0.0."""
    x = workloads.normal_bf16((R, C), 1.0, seed, 1e-3, 100.0).float()
    x[:min(R, 128), :min(C, 128)] = 0.0
    if R > 130 and C > 256:
        x[130, 128:256] = torch.tensor(1e-40)                       # subnormal amax tile
        x[131, 128:256] = torch.tensor(3.3e38)                      # near BF16 max
        x[132, 128:192] = -0.0
    return x.to(torch.bfloat16)


# ----------------------------------------------------------------------------- 1x128
@pytest.mark.parametrize("R,C,row,col", [
    (300, 640, True, False), (384, 656, False, True), (384, 640, True, True),
    (1, 128, True, False), (128, 16, False, True), (256, 512, True, True)])
def test_1x128_parity(cuda_lib, R, C, row, col):
    fq = cuda_lib
    x = crafted_bf16(R, C, seed=R * 1000 + C)
    out = fq.quantize_1x128(x.cuda(), rowwise=row, colwise=col)
    bits = workloads.bf16_bits(x)
    if row:
        q, s = Q.quantize_1x128_rowwise(bits)
        assert np.array_equal(host(out["q_row"]), q)
        assert np.array_equal(f32bits(host(out["s_row"])[:, :R]), f32bits(s))
    if col:
        q, s = Q.quantize_1x128_colwise(bits)
        assert np.array_equal(host(out["q_col"]), q)
        assert np.array_equal(f32bits(host(out["s_col"])[:, :C]), f32bits(s))


def test_1x128_strided_input(cuda_lib):
    fq = cuda_lib
    big = workloads.normal_bf16((256, 1024), 1.0, 77).cuda()
    x = big[:, 128:640]                                   # row stride 1024 != cols
    out = fq.quantize_1x128(x, rowwise=True, colwise=True)
    bits = workloads.bf16_bits(x)
    q, s = Q.quantize_1x128_rowwise(bits)
    assert np.array_equal(host(out["q_row"]), q)
    qc, sc = Q.quantize_1x128_colwise(bits)
    assert np.array_equal(host(out["q_col"]), qc)


# ----------------------------------------------------------------------------- 128x128
@pytest.mark.parametrize("K,N", [(384, 640), (128, 128), (512, 256)])
def test_128x128_parity(cuda_lib, K, N):
    fq = cuda_lib
    w = crafted_bf16(K, N, seed=K + N)
    out = fq.quantize_128x128(w.cuda())
    q, qt, s = Q.quantize_128x128(workloads.bf16_bits(w))
    assert np.array_equal(host(out["q"]), q)
    assert np.array_equal(host(out["q_t"]), qt)
    assert np.array_equal(f32bits(host(out["s"])), f32bits(s))


# ----------------------------------------------------------------------------- multi-tensor
def _check_multi_item(spec, out, x):
    bits = workloads.bf16_bits(x)
    R, C = x.shape
    if spec[0] == "1x128":
        if spec[2]:
            q, s = Q.quantize_1x128_rowwise(bits)
            assert np.array_equal(host(out["q_row"]), q)
            assert np.array_equal(f32bits(host(out["s_row"])[:, :R]), f32bits(s))
        if spec[3]:
            q, s = Q.quantize_1x128_colwise(bits)
            assert np.array_equal(host(out["q_col"]), q)
            assert np.array_equal(f32bits(host(out["s_col"])[:, :C]), f32bits(s))
    else:
        q, qt, s = Q.quantize_128x128(bits)
        assert np.array_equal(f32bits(host(out["s"])), f32bits(s))
        if spec[2]:
            assert np.array_equal(host(out["q_t"]), qt)
        if spec[3]:
            assert np.array_equal(host(out["q"]), q)


@pytest.mark.parametrize("specs", [
    # the step's three tensors (activation, weight, gradient): both outputs each
    [("1x128", (384, 640), True, True), ("128x128", (384, 640), True, True), ("1x128", (256, 896), True, True)],
    # every item form, rowwise-only among them (the 3-CTA launch), an empty item skipped
    [("1x128", (300, 640), True, False), ("1x128", (384, 656), False, True), ("128x128", (512, 256), False, True),
     ("128x128", (256, 384), True, False), ("1x128", (0, 256), True, False), ("1x128", (1, 128), True, False)],
])
def test_quantize_multi_matches_the_oracle_per_item(cuda_lib, specs):
    """One multi-tensor launch gives every item exactly what its own quantizer gives
    (oracle), codes and scales bit for bit."""
    fq = cuda_lib
    xs = [crafted_bf16(max(R, 1), C, seed=31 * i + R + C)[:R] for i, (_, (R, C), _, _) in enumerate(specs)]
    outs = fq.quantize_multi([(k, x.cuda(), a, b) for (k, _, a, b), x in zip(specs, xs)])
    torch.cuda.synchronize()
    assert fq.device_status() == 0
    for spec, out, x in zip(specs, outs, xs):
        if x.shape[0] == 0:
            continue
        _check_multi_item(spec, out, x)


def test_quantize_multi_equals_separate_calls_on_the_llama8b_step(cuda_lib):
    """The Llama-3-8B step's X (1x128 both), W (128x128 both) and dY (1x128 both) in one
    launch equal the three separate calls byte for byte."""
    fq = cuda_lib
    W = workloads.llama8b(device="cuda")
    X, Wt, dY = W["X"], W["W"], W["dY"]
    outs = fq.quantize_multi([("1x128", X, True, True), ("128x128", Wt, True, True), ("1x128", dY, True, True)])
    ref = [fq.quantize_1x128(X, rowwise=True, colwise=True), fq.quantize_128x128(Wt),
           fq.quantize_1x128(dY, rowwise=True, colwise=True)]
    torch.cuda.synchronize()
    for a, b in zip(outs, ref):
        assert sorted(a) == sorted(b)
        for k in a:
            assert torch.equal(a[k], b[k]), k


# ----------------------------------------------------------------------------- MX
def test_128x128_grouped_matches_each_matrix(cuda_lib):
    """A stack of expert weight matrices quantized in one grouped call equals quantizing
    each matrix on its own (oracle), codes of both layouts and scales bit for bit."""
    fq = cuda_lib
    G, K, N = 3, 256, 384
    ws = [workloads.normal_bf16((K, N), 0.006, 40 + g, 1e-3, 30.0) for g in range(G)]
    w = torch.stack(ws).cuda()
    out = fq.quantize_128x128_grouped(w)
    assert fq.device_status() == 0
    for g in range(G):
        oq, oqt, os_ = Q.quantize_128x128(workloads.bf16_bits(ws[g]))
        assert np.array_equal(out["q"][g].cpu().numpy(), oq)
        assert np.array_equal(out["q_t"][g].cpu().numpy(), oqt)
        assert np.array_equal(out["s"][g].cpu().numpy().view(np.uint32), os_.astype(np.float32).view(np.uint32))


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("R,C,row,col", [(300, 672, True, False), (352, 656, False, True),
                                         (384, 640, True, True), (64, 32, True, True)])
def test_mx32_parity(cuda_lib, layout, R, C, row, col):
    fq = cuda_lib
    x = crafted_bf16(R, C, seed=5 * R + C)
    out = fq.quantize_mx32(x.cuda(), rowwise=row, colwise=col, sf_layout=layout)
    bits = workloads.bf16_bits(x)
    if row:
        q, e = Q.quantize_mx_rowwise(bits)
        assert np.array_equal(host(out["q_row"]), q)
        want = Q.sf_to_tiled(e) if layout == 1 else e.ravel()
        assert np.array_equal(host(out["e8m0_row"]), want)
    if col:
        q, e = Q.quantize_mx_colwise(bits)
        assert np.array_equal(host(out["q_col"]), q)
        want = Q.sf_to_tiled(e) if layout == 1 else e.ravel()
        assert np.array_equal(host(out["e8m0_col"]), want)


# ----------------------------------------------------------------------------- per tensor
@pytest.mark.parametrize("R,C", [(300, 648), (1, 8), (128, 4096)])
def test_per_tensor_parity(cuda_lib, R, C):
    fq = cuda_lib
    x = workloads.normal_bf16((R, C), 1.0, R + 3 * C, 1e-3, 50.0)
    out = fq.quantize_tensor(x.cuda())
    q, s = Q.quantize_tensor(workloads.bf16_bits(x))
    assert np.array_equal(host(out["q"]), q)
    assert f32bits(host(out["s_dec"]))[0] == f32bits(np.float32([s]))[0]


def test_per_tensor_empty_writes_unit_scale_on_the_stream(cuda_lib):
    """An empty tensor: amax 0 -> scale 1 -> decode scale 1.0, written by a kernel on the
    caller's stream (no host synchronization), for both per-tensor entry points."""
    import ctypes
    fq = cuda_lib
    L = fq.lib()
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((16,), dtype=torch.uint8, device="cuda")
    for fn in (L.fp8q_quantize_tensor, L.fp8q_quantize_tensor_noalloc):
        s = torch.full((1,), -3.0, dtype=torch.float32, device="cuda")
        side = torch.cuda.Stream()
        with torch.cuda.stream(side):
            assert fn(ctypes.c_void_p(x.data_ptr()), 0, 64, 64, ctypes.c_void_p(q.data_ptr()),
                      ctypes.c_void_p(s.data_ptr()), ctypes.c_void_p(side.cuda_stream)) == 0
        side.synchronize()
        assert float(s.item()) == 1.0


# ----------------------------------------------------------------------------- NVFP4
NV_CASES = [
    # R, C, row, col, rht, sr
    (300, 656, True, False, 0, 0),
    (300, 656, True, False, 1, 1),
    (368, 656, False, True, 0, 0),
    (368, 656, False, True, 2, 2),
    (384, 640, True, True, 2, 3),        # gradient recipe: rowwise SR, colwise RHT + SR
    (384, 640, True, True, 3, 0),
    (16, 16, True, True, 3, 3),
]


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("R,C,row,col,rht,sr", NV_CASES)
def test_nvfp4_parity(cuda_lib, layout, R, C, row, col, rht, sr):
    fq = cuda_lib
    x = workloads.normal_bf16((R, C), 1e-3, 11 * R + C, 5e-4, 100.0)
    out = fq.rht16_quantize_sr(x.cuda(), rowwise=row, colwise=col, rht=rht, rht_seed=5, sr=sr, sr_seed=6,
                               sf_layout=layout)
    bits = workloads.bf16_bits(x)
    if row:
        q, sf, g = Q.quantize_nvfp4_rowwise(bits, rht=bool(rht & 1), rht_seed=5, sr=bool(sr & 1), sr_seed=6)
        assert np.array_equal(host(out["q_row"]), q)
        want = Q.sf_to_tiled(sf) if layout == 1 else sf.ravel()
        assert np.array_equal(host(out["sf_row"]), want)
        assert f32bits(host(out["g_row"]))[0] == f32bits(np.float32([g]))[0]
    if col:
        q, sf, g = Q.quantize_nvfp4_colwise(bits, rht=bool(rht & 2), rht_seed=5, sr=bool(sr & 2), sr_seed=6)
        assert np.array_equal(host(out["q_col"]), q)
        want = Q.sf_to_tiled(sf) if layout == 1 else sf.ravel()
        assert np.array_equal(host(out["sf_col"]), want)
        assert f32bits(host(out["g_col"]))[0] == f32bits(np.float32([g]))[0]


def test_nvfp4_zero_tensor(cuda_lib):
    """All-zero input: G = 0 -> S_g = 1, every block scale 0, every magnitude 0.  The
    transform's sign flips turn some zeros into -0.0, whose code (0x8) the oracle gives too."""
    fq = cuda_lib
    x = torch.zeros((32, 32), dtype=torch.bfloat16)
    out = fq.rht16_quantize_sr(x.cuda(), rowwise=True, colwise=True, rht=3, sr=3, rht_seed=1, sr_seed=2)
    bits = workloads.bf16_bits(x)
    q, sf, g = Q.quantize_nvfp4_rowwise(bits, rht=True, rht_seed=1, sr=True, sr_seed=2)
    assert np.array_equal(host(out["q_row"]), q) and np.array_equal(host(out["sf_row"]), sf.ravel())
    q, sf, g = Q.quantize_nvfp4_colwise(bits, rht=True, rht_seed=1, sr=True, sr_seed=2)
    assert np.array_equal(host(out["q_col"]), q) and np.array_equal(host(out["sf_col"]), sf.ravel())
    assert int((host(out["q_row"]) & 0x77).max()) == 0 and int(host(out["sf_row"]).max()) == 0
    assert host(out["g_row"])[0] == 1.0 and host(out["g_col"])[0] == 1.0


# ----------------------------------------------------------------------------- full size, sampled
def _bands(n, size, rng, k=3):
    starts = sorted({0, (n // size - 1) * size, int(rng.integers(0, n // size)) * size})
    return np.concatenate([np.arange(s, s + size) for s in starts[:k]])


def test_llama8b_fused_1x128_sampled(cuda_lib):
    """X 8192x4096 (fused rowwise + transposed colwise, the bench's launch) and dY."""
    fq = cuda_lib
    d = workloads.llama8b()
    rng = np.random.default_rng(2)
    for name in ("X", "dY"):
        x = d[name]
        out = fq.quantize_1x128(x.cuda(), rowwise=True, colwise=True)
        bits = workloads.bf16_bits(x)
        rows = _bands(bits.shape[0], 128, rng)
        q, s = Q.quantize_1x128_rowwise(bits[rows])
        assert np.array_equal(host(out["q_row"][torch.from_numpy(rows).cuda()]), q)
        assert np.array_equal(f32bits(host(out["s_row"])[:, rows]), f32bits(s))
        cols = _bands(bits.shape[1], 128, rng)
        qc, sc = Q.quantize_1x128_colwise(bits[:, cols])
        assert np.array_equal(host(out["q_col"][torch.from_numpy(cols).cuda()]), qc)
        assert np.array_equal(f32bits(host(out["s_col"])[:, cols]), f32bits(sc))
        del out
    w = d["W"]
    out = fq.quantize_128x128(w.cuda())
    bits = workloads.bf16_bits(w)
    cols = _bands(bits.shape[1], 128, rng)
    q, qt, s = Q.quantize_128x128(bits[:, cols])
    assert np.array_equal(host(out["q"])[:, cols], q)
    assert np.array_equal(host(out["q_t"][torch.from_numpy(cols).cuda()]), qt)
    assert np.array_equal(f32bits(host(out["s"])[cols[::128] // 128]), f32bits(s))


def test_mxfp8_fullsize_sampled(cuda_lib):
    fq = cuda_lib
    d = workloads.mxfp8(which=[2])
    rng = np.random.default_rng(3)
    a, w = d["A2"], d["W2"]                           # A 8192x14336, W 14336x4096
    out = fq.quantize_mx32(a.cuda(), rowwise=True, sf_layout=1)
    bits = workloads.bf16_bits(a)
    rows = _bands(bits.shape[0], 128, rng)
    q, e = Q.quantize_mx_rowwise(bits[rows])
    assert np.array_equal(host(out["q_row"][torch.from_numpy(rows).cuda()]), q)
    tiled = host(out["e8m0_row"])
    ncols = bits.shape[1] // 32
    rr, cc = np.meshgrid(rows, np.arange(ncols), indexing="ij")
    assert np.array_equal(tiled[Q.sf_tiled_offset(rr, cc, ncols)], e)
    out = fq.quantize_mx32(w.cuda(), rowwise=False, colwise=True, sf_layout=1)
    bits = workloads.bf16_bits(w)
    cols = _bands(bits.shape[1], 128, rng)
    q, e = Q.quantize_mx_colwise(bits[:, cols])
    assert np.array_equal(host(out["q_col"][torch.from_numpy(cols).cuda()]), q)
    tiled = host(out["e8m0_col"])
    nsf = bits.shape[0] // 32
    rr, cc = np.meshgrid(cols, np.arange(nsf), indexing="ij")
    assert np.array_equal(tiled[Q.sf_tiled_offset(rr, cc, nsf)], e)


def test_nvfp4_gradient_fullsize_sampled(cuda_lib):
    """dY 8192x53248: rowwise SR (dgrad A) and colwise RHT + SR (wgrad B) in one call."""
    fq = cuda_lib
    d = workloads.nvfp4(which=("dY",), device="cuda")
    x = d["dY"]
    out = fq.rht16_quantize_sr(x, rowwise=True, colwise=True, rht=2, rht_seed=5, sr=3, sr_seed=6, sf_layout=1)
    bits = workloads.bf16_bits(x)
    rng = np.random.default_rng(5)
    rows = _bands(bits.shape[0], 128, rng, k=2)
    q, sf, g = Q.quantize_nvfp4_rowwise(bits, sr=True, sr_seed=6, rows=rows)
    assert np.array_equal(host(out["q_row"][torch.from_numpy(rows).cuda()]), q)
    assert f32bits(host(out["g_row"]))[0] == f32bits(np.float32([g]))[0]
    tiled = host(out["sf_row"])
    nsf = bits.shape[1] // 16
    rr, cc = np.meshgrid(rows, np.arange(nsf), indexing="ij")
    assert np.array_equal(tiled[Q.sf_tiled_offset(rr, cc, nsf)], sf)
    cols = _bands(bits.shape[1], 128, rng, k=2)
    q, sf, g = Q.quantize_nvfp4_colwise(bits, rht=True, rht_seed=5, sr=True, sr_seed=6, rows=cols)
    assert np.array_equal(host(out["q_col"][torch.from_numpy(cols).cuda()]), q)
    assert f32bits(host(out["g_col"]))[0] == f32bits(np.float32([g]))[0]
    tiled = host(out["sf_col"])
    nsf = bits.shape[0] // 16
    rr, cc = np.meshgrid(cols, np.arange(nsf), indexing="ij")
    assert np.array_equal(tiled[Q.sf_tiled_offset(rr, cc, nsf)], sf)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_tensor_delayed_parity_and_history(cuda_lib, fmt):
    """Delayed scaling over two iterations: codes and decode scale bit-exact with the oracle
    for the history given, and the tensor's amax recorded into the history slot."""
    fq = cuda_lib
    f = fq.FP8Q_E4M3 if fmt == "e4m3" else fq.FP8Q_E5M2
    x1 = workloads.normal_bf16((300, 648), 1.0, 71, 1e-3, 50.0)
    x2 = workloads.normal_bf16((300, 648), 3.0, 72, 1e-3, 50.0)     # wider than the history
    hist = torch.tensor([0.0, 20.0, 5.0, 0.0], dtype=torch.float32, device="cuda")
    h_host = hist.cpu().numpy().copy()
    for x, pos in ((x1, 1), (x2, 3)):
        out = fq.quantize_tensor_delayed(x.cuda(), hist, pos, f)
        assert fq.device_status() == 0
        xb = workloads.bf16_bits(x)
        oq, os_, oa = Q.quantize_tensor_delayed(xb, h_host, fmt)
        assert np.array_equal(out["q"].cpu().numpy(), oq)
        assert out["s_dec"].cpu().numpy().view(np.uint32)[0] == np.float32(os_).view(np.uint32)
        h_host[pos] = oa
        assert np.array_equal(hist.cpu().numpy().view(np.uint32), h_host.view(np.uint32))


# ----------------------------------------------------------------------------- NVFP4 16x16 weights
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("R,C,row,col", [
    (304, 656, True, True), (48, 400, True, False), (368, 96, False, True), (16, 16, True, True),
    (256, 512, True, True)])
def test_nvfp4_2d16_parity(cuda_lib, layout, R, C, row, col):
    """16x16-block weight quantizer: codes, scales (both layouts) and decode scale bit-exact."""
    fq = cuda_lib
    x = workloads.normal_bf16((R, C), 0.02, 7 * R + C, 1e-3, 50.0)
    if R >= 32 and C >= 32:
        x[16:32, 16:32] = 0.0                                    # an all-zero block: scale code 0
    out = fq.quantize_nvfp4_2d16(x.cuda(), rowwise=row, colwise=col, sf_layout=layout)
    q_row, sf_row, q_col, sf_col, g = Q.quantize_nvfp4_2d(workloads.bf16_bits(x))
    assert f32bits(host(out["g"]))[0] == f32bits(np.float32([g]))[0]
    if row:
        assert np.array_equal(host(out["q_row"]), q_row)
        assert np.array_equal(host(out["sf_row"]), Q.sf_to_tiled(sf_row) if layout == 1 else sf_row.ravel())
    if col:
        assert np.array_equal(host(out["q_col"]), q_col)
        assert np.array_equal(host(out["sf_col"]), Q.sf_to_tiled(sf_col) if layout == 1 else sf_col.ravel())
    assert "q_row" in out or not row
    assert "q_col" in out or not col


def test_nvfp4_2d16_zero_tensor(cuda_lib):
    fq = cuda_lib
    x = torch.zeros((32, 48), dtype=torch.bfloat16)
    out = fq.quantize_nvfp4_2d16(x.cuda(), sf_layout=0)
    q_row, sf_row, q_col, sf_col, g = Q.quantize_nvfp4_2d(workloads.bf16_bits(x))
    assert np.array_equal(host(out["q_row"]), q_row) and np.array_equal(host(out["q_col"]), q_col)
    assert int(host(out["sf_row"]).max()) == 0 and host(out["g"])[0] == 1.0


def test_nvfp4_2d16_weight_fullsize_sampled(cuda_lib):
    """Llama-3.1-405B weight (16384 x 53248): sampled 128-row bands of the rowwise output and
    128-column bands of the colwise output, against the oracle on the same bands with the
    whole tensor's amax."""
    fq = cuda_lib
    W = workloads.nvfp4(device="cuda", which=("W",))["W"]
    out = fq.quantize_nvfp4_2d16(W, sf_layout=0)
    bits = workloads.bf16_bits(W)
    G_amax = max(np.float32(np.abs(Q.as_f32(bits[r:r + 1024])).max()) for r in range(0, bits.shape[0], 1024))
    rng = np.random.default_rng(23)
    R, C = bits.shape
    q_row_d, q_col_d = host(out["q_row"]), host(out["q_col"])
    sf_row_d = host(out["sf_row"]).reshape(R, C // 16)
    sf_col_d = host(out["sf_col"]).reshape(C, R // 16)
    for r0 in sorted({0, R - 128, int(rng.integers(0, R // 128)) * 128}):
        q_row, sf_row, _, _, g = Q.quantize_nvfp4_2d(bits[r0:r0 + 128], amax=G_amax)
        assert np.array_equal(q_row_d[r0:r0 + 128], q_row) and np.array_equal(sf_row_d[r0:r0 + 128], sf_row)
    for c0 in sorted({0, C - 128, int(rng.integers(0, C // 128)) * 128}):
        _, _, q_col, sf_col, g = Q.quantize_nvfp4_2d(bits[:, c0:c0 + 128], amax=G_amax)
        assert np.array_equal(q_col_d[c0:c0 + 128], q_col) and np.array_equal(sf_col_d[c0:c0 + 128], sf_col)
    assert f32bits(host(out["g"]))[0] == f32bits(np.float32([g]))[0]
