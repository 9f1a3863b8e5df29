"""Parity of the CUDA path (through the C interface) with the CPU oracle.

Codes, scales, search choices, calibration exponents and pre-shifted
activations must be bit-identical; GEMM outputs must satisfy
max|Y - Y_ref| / max|Y_ref| <= 5e-3 (bf16 output, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

from w4a16_gemm_fp4_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 5e-3


@pytest.fixture(scope="module")
def fp4():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from w4a16_gemm_fp4_b200 import api, build
    build.build()
    api.lib()
    api.device_status(clear=True)
    return api


@pytest.fixture(autouse=True)
def _status_clean(request):
    yield
    if torch.cuda.is_available() and "fp4" in request.fixturenames:
        from w4a16_gemm_fp4_b200 import api
        st = api.device_status(clear=True)
        assert st == 0 or request.node.get_closest_marker("expect_status"), "device status %#x" % st


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def scales_bits(s):
    a = s.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.float16 else a.view(np.uint32)


def assert_quant_equal(res, ref):
    assert np.array_equal(res["packed"].cpu().numpy(), ref["packed"]), "packed codes differ"
    assert np.array_equal(scales_bits(res["scales"]), scales_bits(torch.from_numpy(ref["scales"]))), "scales differ"


def rel_err(Y, Yref):
    Y = Y.float().cpu().numpy().astype(np.float64) if isinstance(Y, torch.Tensor) else Y
    denom = np.max(np.abs(Yref))
    return float(np.max(np.abs(Y - Yref)) / (denom if denom > 0 else 1.0))


# ------------------------------------------------------------------- quantize

def test_quantize_tiny_fp32_scales(fp4, oracle_mod):
    case = synth.tiny()
    ref = oracle_mod.quantize(case["W"], 128, 1, False, None, "f32")
    res = fp4.quantize(dev_f32(case["W"]), 128, fp4.E2M1, False, None, "f32", want_sse=True)
    assert_quant_equal(res, ref)
    assert tuple(res["choice"].cpu().tolist()) == (1, 0)
    sse = res["sse"].cpu().numpy()
    assert sse[8] == pytest.approx(ref["sse"][8], rel=1e-12)


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("sdt", ["f16", "f32"])
def test_quantize_fixed_bitexact(fp4, oracle_mod, fmt, group, sdt):
    W, _ = synth.random_case(100 + fmt * 10 + group, 37, 384, 1, dist="t")
    ref = oracle_mod.quantize(W, group, fmt, False, None, sdt)
    res = fp4.quantize(dev_f32(W), group, fmt, False, None, sdt)
    assert_quant_equal(res, ref)


@pytest.mark.parametrize("j", [1, 4, 7])
def test_quantize_bias_candidates_bitexact(fp4, oracle_mod, j):
    """The SSE the GPU search reports for bias candidate j equals the oracle's
    SSE of quantizing with that j forced."""
    W, _ = synth.random_case(7 + j, 64, 256, 1, dist="t")
    ref_packed, ref_scales, ref_sse = oracle_mod.quantize_fixed(W, 128, 1, j, None, "f16")
    res = fp4.quantize(dev_f32(W), 128, fp4.E2M1, True, None, "f16", want_sse=True)
    sse = res["sse"].cpu().numpy()
    assert sse[8 + j] == pytest.approx(ref_sse, rel=1e-10)


def search_check(fp4, oracle_mod, W, group, fmt, bias, shift=None, sdt="f16"):
    ref = oracle_mod.quantize(W, group, fmt, bias, shift, sdt)
    res = fp4.quantize(dev_f32(W), group, fmt, bias, None if shift is None else
                       torch.from_numpy(shift).cuda(), sdt, want_sse=True)
    sse = res["sse"].cpu().numpy()
    ref_sse = ref["sse"]
    evaluated = ~np.isnan(ref_sse)
    assert np.array_equal(np.isnan(sse), ~evaluated)
    np.testing.assert_allclose(sse[evaluated], ref_sse[evaluated], rtol=1e-9, atol=0)
    gf, gj = res["choice"].cpu().tolist()
    of, oj = ref["choice"]
    if (gf, gj) != (of, oj):
        # only acceptable when the two candidates are within 1e-6 relative
        a, b = ref_sse[gf * 8 + gj], ref_sse[of * 8 + oj]
        assert abs(a - b) <= 1e-6 * max(a, b), ((gf, gj), (of, oj), a, b)
        ref = {"packed": None, "scales": None}
        p, s, _ = oracle_mod.quantize_fixed(W, group, gf, gj, shift, sdt)
        ref["packed"], ref["scales"] = p, s
    assert_quant_equal(res, ref)
    return (gf, gj)


@pytest.mark.parametrize("fmt,bias", [(-1, True), (-1, False), (1, True), (0, True), (2, True)])
def test_search_small(fp4, oracle_mod, fmt, bias):
    W, _ = synth.random_case(31, 96, 512, 1, dist="t")
    search_check(fp4, oracle_mod, W, 128, fmt, bias)


def test_search_tie_rule(fp4, oracle_mod):
    W = np.zeros((4, 128), np.float32)
    assert search_check(fp4, oracle_mod, W, 32, -1, True) == (0, 0)
    W[:, 0] = 168 * 2.0 ** -10
    W[:, 32] = -84 * 2.0 ** -10
    assert search_check(fp4, oracle_mod, W, 32, -1, True) == (0, 0)


def test_quantize_fold_bitexact(fp4, oracle_mod):
    rng = np.random.default_rng(41)
    X, _ = synth.outlier_activations(rng, 64, 512)
    shift, rho = oracle_mod.preshift_calibrate(X)
    W = synth.lognormal_row_weights(rng, 80, 512)
    search_check(fp4, oracle_mod, W, 128, 1, True, shift=shift)
    ref = oracle_mod.quantize(W, 128, 1, False, shift, "f16")
    res = fp4.quantize(dev_f32(W), 128, 1, False, torch.from_numpy(shift).cuda(), "f16")
    assert_quant_equal(res, ref)


def test_quantize_edge_values(fp4, oracle_mod):
    W = np.zeros((3, 128), np.float32)
    W[0, :8] = [6.0, -0.0, -0.2, 0.2, 3.5, 2.5, -5.0, 0.75]      # midpoints, -0, small negatives
    W[1, :4] = [1e-9, -1e-9, 5e-10, 0.0]                         # fp16 scale underflows to 0
    W[2, 64:] = -0.0
    for sdt in ("f16", "f32"):
        ref = oracle_mod.quantize(W, 32, 1, False, None, sdt)
        res = fp4.quantize(dev_f32(W), 32, 1, False, None, sdt)
        assert_quant_equal(res, ref)


@pytest.mark.expect_status
def test_quantize_nonfinite_sets_status(fp4):
    W = torch.zeros((4, 128), device="cuda")
    W[2, 7] = float("nan")
    fp4.quantize(W, 128, 1)
    assert fp4.device_status(clear=True) & fp4.DEV_NONFINITE_INPUT


@pytest.mark.expect_status
def test_quantize_fp16_overflow_sets_status(fp4):
    W = torch.zeros((2, 128), device="cuda")
    W[1, 3] = 1e6
    fp4.quantize(W, 128, 1, scale_dtype="f16")
    assert fp4.device_status(clear=True) & fp4.DEV_SCALE_OVERFLOW


def test_quantize_empty(fp4):
    W = torch.zeros((0, 128), device="cuda")
    res = fp4.quantize(W, 128, fp4.AUTO, True, want_sse=True)
    assert res["choice"].cpu().tolist() == [0, 0]
    assert res["packed"].numel() == 0


@pytest.mark.parametrize("fmt,sdt", [(1, "f16"), (0, "f32"), (2, "f16")])
def test_dequantize_bitexact(fp4, oracle_mod, fmt, sdt):
    W, _ = synth.random_case(51, 40, 256, 1)
    res = fp4.quantize(dev_f32(W), 64, fmt, False, None, sdt)
    got = fp4.dequantize(res["packed"], res["scales"], fmt, 64).cpu().numpy()
    ref = oracle_mod.dequantize(res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), fmt, 64)
    assert np.array_equal(got, ref.astype(np.float32))


# ------------------------------------------------------------------ pre-shift

@pytest.mark.parametrize("M,K", [(64, 512), (7, 136), (300, 1024)])
def test_preshift_bitexact(fp4, oracle_mod, M, K):
    rng = np.random.default_rng(M + K)
    X, _ = synth.outlier_activations(rng, M, K)
    X[:, 3] = 0            # an all-zero channel
    shift, rho = oracle_mod.preshift_calibrate(X)
    Xt = oracle_mod.preshift_apply(X, shift, rho)
    gshift, grho = fp4.preshift_calibrate(dev_bf16(X))
    assert np.array_equal(gshift.cpu().numpy(), shift)
    assert grho.cpu().numpy()[0] == rho
    gXt = fp4.preshift_apply(dev_bf16(X), gshift, grho)
    assert np.array_equal(host_bits(gXt), Xt)


def test_preshift_all_zero(fp4):
    shift, rho = fp4.preshift_calibrate(torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda"))
    assert rho.item() == 1.0 and int(shift.abs().sum()) == 0


# ----------------------------------------------------------------------- GEMM

def small_ws():
    """A workspace too small for the prepared activations: the GEMM then
    converts them inside the kernel."""
    return torch.empty(16, dtype=torch.uint8, device="cuda")


def gemm_case(fp4, oracle_mod, seed, N, K, M, group=128, fmt=1, sdt="f16", engine=0, splits=0, rho=None,
              workspace=None):
    W, X = synth.random_case(seed, N, K, M)
    ref_q = oracle_mod.quantize(W, group, fmt, False, None, sdt)
    res = fp4.quantize(dev_f32(W), group, fmt, False, None, sdt)
    assert_quant_equal(res, ref_q)
    xs = None if rho is None else torch.tensor([rho], dtype=torch.float32, device="cuda")
    Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], fmt, group, x_scale=xs, engine=engine, splits=splits,
                 workspace=workspace)
    Yref = oracle_mod.gemm(X, ref_q["packed"], ref_q["scales"], fmt, group, 1.0 if rho is None else rho)
    return rel_err(Y, Yref)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("N,K,group", [(256, 512, 128), (200, 384, 64), (37, 160, 32), (64, 1408, 128)])
def test_gemm_decode_engine(fp4, oracle_mod, M, N, K, group):
    assert gemm_case(fp4, oracle_mod, 7 * M + N, N, K, M, group=group, engine=fp4.ENGINE_DECODE) <= TOL


@pytest.mark.parametrize("M,splits", [(4, 0), (4, 148), (13, 0), (13, 148), (24, 0), (64, 0)])
@pytest.mark.parametrize("fmt,sdt", [(0, "f16"), (2, "f32"), (1, "f32"), (0, "f32"), (2, "f16"), (1, "f16")])
def test_gemm_decode_formats(fp4, oracle_mod, fmt, sdt, M, splits):
    """Every format and scale type through every decode kernel (M <= 16:
    row-block with splits = 0, streaming with a CTA count; M > 16: the
    tensor-memory kernel): E2M1 runs its codes through the hardware f16
    convert (activations scaled into the f16 range by a power of two),
    E1M2 and E3M0 by bit placement to bf16 (activations re-paired)."""
    assert gemm_case(fp4, oracle_mod, 3 + M, 96, 256, M, fmt=fmt, sdt=sdt, engine=fp4.ENGINE_DECODE, splits=splits,
                     rho=0.75) <= TOL


@pytest.mark.parametrize("act", [1, 2])
@pytest.mark.parametrize("M,N,K,group,engine,splits", [
    (4, 300, 1024, 128, 1, 0),      # row-block decode kernel
    (4, 300, 1024, 128, 1, 148),    # streaming decode kernel, whole tiles and split tiles
    (13, 300, 1024, 128, 1, 148),   # streaming, two token tiles
    (40, 300, 1024, 128, 1, 0),     # tensor-memory decode kernel
    (16, 300, 1024, 128, 2, 0),     # tensor engine, 16-token tile
    (64, 300, 2048, 128, 2, 0),     # tensor engine, 64-token tile, split K over a cluster
    (200, 300, 1024, 128, 2, 1),    # 128-token tile, f16 path (default workspace)
    (4, 300, 1024, 64, 1, 0),       # lookup-table decode kernel, group 64
    (40, 300, 1024, 32, 2, 0),      # tensor engine, group 32
])
def test_gemm_activation(fp4, oracle_mod, act, M, N, K, group, engine, splits):
    """The fused output activation (SiLU, GeLU) in every kernel's epilogue,
    after any split-K sum, against the oracle's activation of its fp64
    product; rho != 1 so that the activation sees the scaled value."""
    W, X = synth.random_case(60 + M + act, N, K, M)
    res = fp4.quantize(dev_f32(W), group, 1)
    xs = torch.tensor([0.75], dtype=torch.float32, device="cuda")
    Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, group, x_scale=xs, engine=engine, splits=splits,
                 act=act)
    Yref = oracle_mod.gemm_act(X, res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), 1, group, act, 0.75)
    assert rel_err(Y, Yref) <= TOL
    assert np.all(np.isfinite(Y.float().cpu().numpy()))


@pytest.mark.parametrize("M,N,K,engine,splits", [
    (4, 304, 1024, 1, 0),       # row-block decode kernel (pair in lane ^ 16)
    (4, 304, 1024, 1, 1),       # streaming kernel, one CTA: whole tiles, 128-byte rows (pair in lane ^ 8)
    (13, 304, 1024, 1, 148),    # streaming, two token tiles, every tile split (reducer quads)
    (5, 600, 384, 1, 2),        # streaming, one-group chunks of 256 rows (pair in lane ^ 4) and a split tile
    (40, 304, 1024, 1, 1),      # tensor-memory decode kernel, whole tiles (lane ^ 1)
    (40, 304, 1024, 1, 0),      # tensor-memory decode kernel, split tiles (reducer quads)
    (16, 304, 1024, 2, 0),      # tensor engine 16-token tile, split K over a cluster (quads)
    (64, 304, 1024, 2, 1),      # tensor engine 64-token tile, one CTA per tile (lane ^ 1)
    (200, 304, 1024, 2, 1),     # 128-token tile, f16 path, 16-byte output chunks
])
def test_gemm_silu_gate(fp4, oracle_mod, M, N, K, engine, splits):
    """Gate and up projections fused in one call: rows 2i / 2i+1 are the gate
    / up rows of output i, Y[m, i] = silu(y[m, 2i]) * y[m, 2i+1], in every
    group-128 kernel's epilogue."""
    W, X = synth.random_case(80 + M, N, K, M)
    res = fp4.quantize(dev_f32(W), 128, 1)
    xs = torch.tensor([1.25], dtype=torch.float32, device="cuda")
    Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, x_scale=xs, engine=engine, splits=splits,
                 act=fp4.ACT_SILU_GATE)
    assert tuple(Y.shape) == (M, N // 2)
    Yref = oracle_mod.gemm_act(X, res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), 1, 128,
                               oracle_mod.ACT_SILU_GATE, 1.25)
    assert rel_err(Y, Yref) <= TOL


def test_gemm_silu_gate_limits(fp4):
    """Gate/up pairs need an even row count and group 128."""
    W, X = synth.random_case(90, 63, 256, 2)
    res = fp4.quantize(dev_f32(W), 128, 1)
    with pytest.raises(fp4.Fp4Error) as err:
        fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, act=fp4.ACT_SILU_GATE,
                 out=torch.empty((2, 31), dtype=torch.bfloat16, device="cuda"))
    assert err.value.code == 2
    W, X = synth.random_case(91, 64, 256, 2)
    res = fp4.quantize(dev_f32(W), 64, 1)
    with pytest.raises(fp4.Fp4Error) as err:
        fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 64, act=fp4.ACT_SILU_GATE)
    assert err.value.code == 2


def test_gemm_activation_rejects_unknown(fp4):
    W, X = synth.random_case(70, 64, 256, 2)
    res = fp4.quantize(dev_f32(W), 128, 1)
    with pytest.raises(fp4.Fp4Error) as err:
        fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, act=4)
    assert err.value.code == 1


def test_gemm_decode_needs_workspace(fp4, oracle_mod):
    """The streaming decode kernels keep tile counters and partials in the
    workspace: forced without one (a CTA count selects them) the call
    refuses (FP4_ERR_WORKSPACE, nothing launched).  The row-block kernel
    needs none, and the automatic choice runs it."""
    W, X = synth.random_case(12, 200, 512, 8)
    res = fp4.quantize(dev_f32(W), 128, 1)
    with pytest.raises(fp4.Fp4Error) as err:
        fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, engine=fp4.ENGINE_DECODE, splits=148,
                 workspace=small_ws())
    assert err.value.code == 4
    Yref = oracle_mod.gemm(X, res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), 1, 128)
    Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, engine=fp4.ENGINE_DECODE, workspace=small_ws())
    assert rel_err(Y, Yref) <= TOL
    Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, workspace=small_ws())
    assert rel_err(Y, Yref) <= TOL


@pytest.mark.parametrize("N,K,M", [
    (10007, 256, 3),    # many row tiles, one chunk each, ragged last tile
    (40, 6272, 2),      # one row tile of 49 groups (odd: one-group chunks) over 49 CTAs
    (2400, 24576, 1),   # long K
    (5000, 11008, 8),
    (2500, 13824, 1),
    (64, 24704, 2),     # K of 193 groups
    (4101, 2048, 13),
    (600, 11008, 12),
    (128, 128, 5),      # a single chunk of one group
])
@pytest.mark.parametrize("splits", [0, 148])
def test_gemm_decode_block_schedule(fp4, oracle_mod, N, K, M, splits):
    """Decode engine, group 128.  splits = 148: the streaming kernel, whose
    code chunks of all row tiles split into one contiguous range per CTA
    (whole tiles stored directly, pieces reduced by the CTA that completes
    the tile), ragged row tiles, two- and one-group chunks.  splits = 0: the
    row-block kernel where the activations fit it (16-row blocks walked by
    persistent CTAs, ragged last block), the streaming kernel elsewhere."""
    assert gemm_case(fp4, oracle_mod, N + K, N, K, M, engine=fp4.ENGINE_DECODE, splits=splits, rho=1.5) <= TOL


@pytest.mark.parametrize("M", [9, 16, 17, 31, 32, 33, 48, 64])
@pytest.mark.parametrize("N,K", [(256, 512), (200, 1024), (1000, 4096)])
def test_gemm_decode_token_tiles(fp4, oracle_mod, N, K, M):
    """Decode engine token tiles of 16, 32 and 64 activation rows (MMA N),
    rows beyond M zero-filled by the activation copies."""
    assert gemm_case(fp4, oracle_mod, 3 * N + M, N, K, M, engine=fp4.ENGINE_DECODE, rho=0.5) <= TOL


@pytest.mark.parametrize("M", [1, 16, 40, 64])
@pytest.mark.parametrize("ctas", [1, 2, 3, 5, 8, 13, 24])
def test_gemm_decode_cta_counts(fp4, oracle_mod, ctas, M):
    """Decode engine with a forced number of CTAs (the split-K argument):
    3 row tiles x 8 chunks cut into 1..24 contiguous ranges, so tiles are
    whole, split in two, or shared by several CTAs."""
    assert gemm_case(fp4, oracle_mod, 17 + M, 300, 2048, M, engine=fp4.ENGINE_DECODE, splits=ctas,
                     rho=2.5) <= TOL


@pytest.mark.parametrize("ctas", [0, 7])
def test_gemm_decode_deterministic(fp4, ctas):
    """Pieces of a tile are added in CTA order by whichever CTA completes
    the tile: repeated calls agree bit for bit."""
    W, X = synth.random_case(79, 1000, 4096, 16)
    res = fp4.quantize(dev_f32(W), 128, 1)
    outs = [fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, engine=1, splits=ctas) for _ in range(4)]
    assert all(torch.equal(outs[0].view(torch.int16), o.view(torch.int16)) for o in outs[1:])


def test_gemm_decode_unaligned_scales(fp4, oracle_mod):
    """A scale pointer that is 4- but not 16-byte aligned: the scale rows are
    then read from global memory instead of travelling with the codes."""
    N, K, M = 700, 1024, 5
    W, X = synth.random_case(31, N, K, M)
    ref_q = oracle_mod.quantize(W, 128, 1, False, None, "f16")
    res = fp4.quantize(dev_f32(W), 128, fp4.E2M1, False, None, "f16")
    store = torch.empty(N * (K // 128) + 8, dtype=torch.float16, device="cuda")
    sc = store[2:2 + N * (K // 128)].view(N, K // 128)
    sc.copy_(res["scales"])
    assert sc.data_ptr() % 16 != 0
    Y = fp4.gemm(dev_bf16(X), res["packed"], sc, 1, 128, engine=fp4.ENGINE_DECODE)
    Yref = oracle_mod.gemm(X, ref_q["packed"], ref_q["scales"], 1, 128)
    assert rel_err(Y, Yref) <= TOL


@pytest.mark.parametrize("M", [1, 9, 16, 33, 64, 65, 128, 200, 256, 300])
@pytest.mark.parametrize("N,K,group", [(256, 512, 128), (200, 384, 64), (130, 96, 32)])
def test_gemm_tensor_engine(fp4, oracle_mod, M, N, K, group):
    assert gemm_case(fp4, oracle_mod, 11 * M + N, N, K, M, group=group, engine=fp4.ENGINE_TENSOR) <= TOL


@pytest.mark.parametrize("splits", [1, 2, 3, 5, 8])
def test_gemm_tensor_split_k(fp4, oracle_mod, splits):
    assert gemm_case(fp4, oracle_mod, 5, 256, 1024, 40, engine=fp4.ENGINE_TENSOR, splits=splits, rho=2.5) <= TOL


@pytest.mark.parametrize("M,N,fmt", [(65, 256, 1), (129, 200, 1), (300, 136, 1), (300, 130, 1), (200, 264, 0)])
def test_gemm_tensor_tile_store(fp4, oracle_mod, M, N, fmt):
    """Without split K the 128-token tile stores its output through shared
    memory in 16-byte chunks, bounded by M and N (N % 8 == 0); other N store
    element by element."""
    assert gemm_case(fp4, oracle_mod, M + 3 * N, N, 512, M, fmt=fmt, engine=fp4.ENGINE_TENSOR, splits=1,
                     rho=0.25) <= TOL


@pytest.mark.parametrize("fmt,sdt", [(0, "f16"), (2, "f32")])
def test_gemm_tensor_formats(fp4, oracle_mod, fmt, sdt):
    assert gemm_case(fp4, oracle_mod, 9, 128, 256, 100, fmt=fmt, sdt=sdt, engine=fp4.ENGINE_TENSOR) <= TOL


def test_gemm_split_k_deterministic(fp4):
    W, X = synth.random_case(77, 384, 2048, 48)
    res = fp4.quantize(dev_f32(W), 128, 1)
    outs = [fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, engine=2, splits=4) for _ in range(3)]
    assert all(torch.equal(outs[0], o) for o in outs[1:])


@pytest.mark.parametrize("N,K", [(11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("M", [1, 8, 16, 33, 64])
def test_gemm_repeat_bit_identical(fp4, N, K, M):
    """Both engines reduce in a fixed order, so repeated calls must agree bit
    for bit.  At these sizes there are hundreds of CTAs, two per SM, with
    long K ranges: a stage released before its readers were done shows up
    here as run-to-run differences."""
    W, X = synth.random_case(500 + M, N, K, M)
    res = fp4.quantize(dev_f32(W), 128, 1)
    Xd = dev_bf16(X)
    outs = [fp4.gemm(Xd, res["packed"], res["scales"], 1, 128) for _ in range(4)]
    for o in outs[1:]:
        assert torch.equal(outs[0].view(torch.int16), o.view(torch.int16))


def test_gemm_engines_agree(fp4, oracle_mod):
    """At M = 8 both engines apply; each meets the bound against the oracle,
    so they differ by at most twice the bound."""
    W, X = synth.random_case(78, 512, 1024, 8)
    res = fp4.quantize(dev_f32(W), 128, 1)
    a = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, engine=1).float()
    b = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, engine=2).float()
    Yref = oracle_mod.gemm(X, res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), 1, 128)
    assert rel_err(a, Yref) <= TOL and rel_err(b, Yref) <= TOL
    assert (a - b).abs().max().item() <= 2 * TOL * float(np.max(np.abs(Yref)))


def wide_range_rows(seed, M, K):
    """Activation rows at magnitudes 2^-60 .. 2^60 (far outside the f16
    range on both sides); a row alternating 2^20 and 2^-20 entries (row 1,
    or the only row); with three or more rows, a row of zeros (row 0)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    x *= np.exp2(rng.integers(-60, 61, M).astype(np.float32))[:, None]
    if M >= 3:
        x[0] = 0.0
    alt = 1 if M >= 2 else 0
    x[alt, 0::2] *= np.float32(2.0 ** 20)
    x[alt, 1::2] *= np.float32(2.0 ** -20)
    return synth.to_bf16_bits(x)


def row_rel_err(Y, Yref):
    """Largest per-row error relative to that row's max|Y_ref| (a zero row
    must come out zero)."""
    Y = Y.float().cpu().numpy().astype(np.float64)
    worst = 0.0
    for m in range(Yref.shape[0]):
        d = np.max(np.abs(Yref[m]))
        e = np.max(np.abs(Y[m] - Yref[m]))
        worst = max(worst, e / d if d > 0 else (0.0 if e == 0 else np.inf))
    return worst


@pytest.mark.parametrize("M,splits", [(65, 0), (200, 0), (300, 0), (300, 1), (130, 3), (9, 0), (16, 4), (33, 0),
                                      (64, 0), (64, 8)])
def test_gemm_f16_activation_rows(fp4, oracle_mod, M, splits):
    """The tensor engine runs E2M1 weights in f16 when given the workspace
    (every token tile but the 64-token one, which stays bf16): each activation row is rescaled by a power of two
    into the f16 range and the factor is undone in the epilogue (split-K:
    in the cluster reduction).  Rows 2^120 apart in magnitude must each meet
    the bound against their own magnitude, with and without the workspace
    (bf16 path)."""
    N, K = 256, 1024
    W, _ = synth.random_case(40 + M, N, K, 1)
    X = wide_range_rows(41 + M, M, K)
    res = fp4.quantize(dev_f32(W), 128, 1)
    Yref = oracle_mod.gemm(X, res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), 1, 128, 0.5)
    xs = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    need = fp4.gemm_workspace_size(M, N, K)
    assert need >= M * K * 2 + M * 4
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    eng = fp4.ENGINE_TENSOR
    a = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, x_scale=xs, splits=splits, workspace=ws,
                 engine=eng)
    b = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128, x_scale=xs, splits=splits, workspace=small,
                 engine=eng)
    assert row_rel_err(a, Yref) <= TOL
    assert row_rel_err(b, Yref) <= TOL


@pytest.mark.parametrize("K", [2176, 4224, 8320, 16512])
@pytest.mark.parametrize("M", [70, 1100])
def test_gemm_f16_row_lengths(fp4, oracle_mod, K, M):
    """Row lengths that take each form of the f16 activation pre-pass (the
    row held in 2, 4, 8 or 16 registers per thread, or read twice; 256
    threads per row, or 128 from 1024 rows)."""
    N = 128 if M < 1024 else 32
    W, _ = synth.random_case(K, N, K, 1)
    X = wide_range_rows(K + 1, M, K)
    res = fp4.quantize(dev_f32(W), 128, 1)
    Yref = oracle_mod.gemm(X, res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), 1, 128)
    Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128)
    assert row_rel_err(Y, Yref) <= TOL


@pytest.mark.parametrize("M", [1, 2, 8, 9, 12, 16, 33, 64])
@pytest.mark.parametrize("N,K,fmt", [(256, 1024, 1), (200, 2048, 1), (300, 512, 0), (136, 768, 2)])
def test_gemm_decode_wide_range(fp4, oracle_mod, M, N, K, fmt):
    """Decode engine on activation rows 2^120 apart in magnitude (far outside
    the f16 range on both sides), a zero row and a row alternating 2^20 and
    2^-20: each row meets the bound against its own magnitude.  E2M1 scales
    each activation row by a power of two into the f16 range (prepared once
    per call) and undoes it in fp32; the other formats multiply in bf16."""
    W, _ = synth.random_case(60 + M + N, N, K, 1)
    X = wide_range_rows(61 + M, M, K)
    res = fp4.quantize(dev_f32(W), 128, fmt)
    Yref = oracle_mod.gemm(X, res["packed"].cpu().numpy(), res["scales"].cpu().numpy(), fmt, 128, 0.5)
    xs = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    for ctas in (0, 1, 3):
        Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], fmt, 128, x_scale=xs, engine=fp4.ENGINE_DECODE,
                     splits=ctas)
        assert row_rel_err(Y, Yref) <= TOL, ctas


def test_gemm_empty_and_k0(fp4):
    packed = torch.zeros((16, 0), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((16, 0), dtype=torch.float16, device="cuda")
    X = torch.zeros((3, 0), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((3, 16), 7.0, dtype=torch.bfloat16, device="cuda")
    fp4.gemm(X, packed, scales, 1, 128, out=Y)
    assert torch.count_nonzero(Y).item() == 0
    Y0 = fp4.gemm(torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda"),
                  torch.zeros((16, 64), dtype=torch.uint8, device="cuda"),
                  torch.zeros((16, 1), dtype=torch.float16, device="cuda"), 1, 128)
    assert Y0.shape == (0, 16)


# ---------------------------------------------------------- full-size workloads

def sampled_check(fp4, oracle_mod, Xbits, packed, scales, fmt, group, Y, rho=1.0, rows=4, seed=0):
    """Whole rows of a full-size output against the oracle, element by
    element: rows 0 and M-1 and rows-2 random ones, every one of their N
    outputs.  The denominator is the oracle's own max|Y_ref| over those rows
    (at most the max over the whole output, so the check is never looser
    than the bound), and every output of Y must be finite."""
    M, N = Y.shape
    assert bool(torch.isfinite(Y.float()).all()), "non-finite GPU output"
    rng = np.random.default_rng(seed)
    sel = sorted({0, M - 1} | set(rng.integers(0, M, max(rows - 2, 0)).tolist()))
    ms = np.repeat(np.asarray(sel, np.int32), N)
    ns = np.tile(np.arange(N, dtype=np.int32), len(sel))
    ref = oracle_mod.gemm_sampled(Xbits, packed, scales, fmt, group, ms, ns, rho).reshape(len(sel), N)
    got = Y.float().cpu().numpy().astype(np.float64)[sel]
    denom = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref)) / (denom if denom > 0 else 1.0))


def test_llama7b_decode_full(fp4, oracle_mod):
    """11008x4096 weights of the LLaMA-7B decode workload: codes and scales
    bit-exact, decode GEMM at M in {1, 8, 16, 64} on sampled outputs."""
    case = synth.llama7b_decode(shapes=((11008, 4096),))[0]
    W = case["W"]
    ref = oracle_mod.quantize(W, 128, 1, False, None, "f16")
    res = fp4.quantize(dev_f32(W), 128, 1, False, None, "f16")
    assert_quant_equal(res, ref)
    for M, Xb in case["X"].items():
        Y = fp4.gemm(dev_bf16(Xb), res["packed"], res["scales"], 1, 128)
        assert sampled_check(fp4, oracle_mod, Xb, ref["packed"], ref["scales"], 1, 128, Y, seed=M) <= TOL, M


def test_llama7b_prefill_full(fp4, oracle_mod):
    """Outlier activations 2048x4096 with the pre-shift: calibration,
    activation prologue and folded quantization bit-exact; prefill GEMM on
    sampled outputs."""
    case = synth.llama7b_prefill(shapes=((4096, 4096),))
    X = case["X"]
    shift, rho = oracle_mod.preshift_calibrate(X)
    Xt = oracle_mod.preshift_apply(X, shift, rho)
    gshift, grho = fp4.preshift_calibrate(dev_bf16(X))
    assert np.array_equal(gshift.cpu().numpy(), shift) and grho.item() == rho
    gXt = fp4.preshift_apply(dev_bf16(X), gshift, grho)
    assert np.array_equal(host_bits(gXt), Xt)
    W = case["W"][0]
    ref = oracle_mod.quantize(W, 128, 1, False, shift, "f16")
    res = fp4.quantize(dev_f32(W), 128, 1, False, gshift, "f16")
    assert_quant_equal(res, ref)
    Y = fp4.gemm(gXt, res["packed"], res["scales"], 1, 128, x_scale=grho)
    assert sampled_check(fp4, oracle_mod, Xt, ref["packed"], ref["scales"], 1, 128, Y, rho=rho) <= TOL


def test_llama13b_search_full(fp4, oracle_mod):
    """Per-tensor search over 3 formats x 8 bias candidates on 5120x5120
    Student-t weights, then the M=512 GEMM on sampled outputs."""
    case = synth.llama13b_search(shapes=((5120, 5120),))
    W = case["W"][0]
    fj = search_check(fp4, oracle_mod, W, 128, -1, True)
    res = fp4.quantize(dev_f32(W), 128, -1, True)
    p, s, _ = oracle_mod.quantize_fixed(W, 128, fj[0], fj[1], None, "f16")
    Y = fp4.gemm(dev_bf16(case["X"]), res["packed"], res["scales"], fj[0], 128)
    assert sampled_check(fp4, oracle_mod, case["X"], p, s, fj[0], 128, Y) <= TOL


def test_llama13b_stack_layer_sample(fp4, oracle_mod):
    """One sampled layer of the 40-layer 13B-shaped stack (device-drawn
    weights): every matrix quantizes bit-exactly; the decode and prefill
    GEMMs match on sampled outputs."""
    rng = np.random.default_rng(4)
    for name, w in synth.stack_layer_weights(17):
        if name not in ("q", "down"):
            continue
        Wn = w.cpu().numpy()
        ref = oracle_mod.quantize(Wn, 128, 1, False, None, "f16")
        res = fp4.quantize(w.contiguous(), 128, 1, False, None, "f16")
        assert_quant_equal(res, ref)
        K = Wn.shape[1]
        for M in (1, 4, 16, 64, 2048):
            Xb = synth.activations(rng, M, K)
            Y = fp4.gemm(dev_bf16(Xb), res["packed"], res["scales"], 1, 128)
            assert sampled_check(fp4, oracle_mod, Xb, ref["packed"], ref["scales"], 1, 128, Y, rows=3) <= TOL


# -------------------------------------------------------- failure detection

@pytest.mark.expect_status
def test_bounded_wait_reports_timeout(fp4):
    """A wait nothing completes gives up after its bound and reports it;
    the context stays usable afterwards."""
    fp4.device_status(clear=True)
    fp4.selftest_bounded_wait(20000)
    st = fp4.device_status(clear=True)
    assert st & fp4.DEV_WAIT_TIMEOUT
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0
