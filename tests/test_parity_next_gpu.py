"""Parity of the scale-granularity quantizer, the 4-bit activation
quantizer and the W4A4 product (CUDA path through the C interface) with
the CPU oracle.

Codes, scales, bias-index maps and activation codes must be bit-identical
(a per-block bias search may differ from the oracle only where two
candidates' SSEs lie within 1e-9 of each other, and then the codes must
match the oracle re-run under the GPU's choice); W4A4 outputs must satisfy
max|Y - Y_ref| / max|Y_ref| <= 5e-3.
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


def scales_bits(a):
    a = a.cpu().numpy() if isinstance(a, torch.Tensor) else a
    return a.view(np.uint16) if a.dtype == np.float16 else a.view(np.uint32)


def rel_err(Y, Yref):
    Y = Y.float().cpu().numpy().astype(np.float64)
    denom = np.max(np.abs(Yref))
    return float(np.max(np.abs(Y - Yref)) / (denom if denom > 0 else 1.0))


def block_sse_per_j(oracle_mod, W, group, gran, heads, fmt, shift, sdt):
    """[8][blocks] SSE of every block under every fixed bias index (fp64,
    from the oracle's codes and scales)."""
    N, K = W.shape
    Wf = W.astype(np.float64) * (np.exp2(shift.astype(np.float64)) if shift is not None else 1.0)
    out = []
    for j in range(8):
        r = oracle_mod.quantize_blocks(W, group, gran, fmt, j, heads, shift, sdt)
        d2 = (Wf - oracle_mod.dequantize(r["packed"], r["scales"], fmt, group)) ** 2
        if gran == 0:
            out.append(d2.reshape(N, K // group, group).sum(axis=2).ravel())
        elif gran == 1:
            out.append(d2.sum(axis=1))
        else:
            out.append(d2.reshape(heads, -1).sum(axis=1))
    return np.array(out)


def check_blocks(fp4, oracle_mod, W, group, gran, heads, fmt, j, shift=None, sdt="f16"):
    dshift = None if shift is None else torch.from_numpy(shift).cuda()
    res = fp4.quantize_blocks(dev_f32(W), group, gran, heads, fmt, j, dshift, sdt)
    torch.cuda.synchronize()
    jm = res["jmap"].cpu().numpy()
    ref = oracle_mod.quantize_blocks(W, group, gran, fmt, None if j < 0 else j, heads, shift, sdt)
    if j < 0 and not np.array_equal(jm, ref["jmap"]):
        sse = block_sse_per_j(oracle_mod, W, group, gran, heads, fmt, shift, sdt)
        for b in np.nonzero(jm != ref["jmap"])[0]:
            assert sse[jm[b], b] <= sse[:, b].min() * (1 + 1e-9), (b, jm[b], ref["jmap"][b])
        ref = oracle_mod.quantize_blocks(W, group, gran, fmt, 0, heads, shift, sdt, jforce=jm)
    assert np.array_equal(jm, ref["jmap"]), "bias-index map differs"
    assert np.array_equal(res["packed"].cpu().numpy(), ref["packed"]), "packed codes differ"
    assert np.array_equal(scales_bits(res["scales"]), scales_bits(ref["scales"])), "scales differ"
    return res, ref


# ------------------------------------------------------------ granularity

@pytest.mark.parametrize("gran,heads,group", [(0, 0, 32), (0, 0, 128), (1, 0, 128), (1, 0, 64), (2, 4, 128),
                                              (2, 48, 32)])
@pytest.mark.parametrize("fmt,sdt", [(1, "f16"), (0, "f32"), (2, "f16")])
@pytest.mark.parametrize("j", [0, 5])
def test_quantize_blocks_fixed_bitexact(fp4, oracle_mod, gran, heads, group, fmt, sdt, j):
    rng = np.random.default_rng(60 + fmt)
    W = synth.lognormal_row_weights(rng, 48, 512)
    check_blocks(fp4, oracle_mod, W, group, gran, heads, fmt, j, None, sdt)


@pytest.mark.parametrize("gran,heads,group", [(0, 0, 32), (0, 0, 64), (0, 0, 128), (1, 0, 128), (2, 4, 128),
                                              (2, 12, 64)])
@pytest.mark.parametrize("fmt", [1, 0])
def test_quantize_blocks_search(fp4, oracle_mod, gran, heads, group, fmt):
    rng = np.random.default_rng(70 + gran)
    W = synth.student_t_weights(rng, 48, 1024)
    shift = rng.integers(-4, 1, 1024).astype(np.int8)
    check_blocks(fp4, oracle_mod, W, group, gran, heads, fmt, -1, shift)


def test_quantize_blocks_ragged_group_units(fp4, oracle_mod):
    """K = 96 at group 32: a 128-element unit spans rows (group blocks only)."""
    rng = np.random.default_rng(75)
    W = synth.normal_weights(rng, 7, 96)
    check_blocks(fp4, oracle_mod, W, 32, 0, 0, 1, -1)
    check_blocks(fp4, oracle_mod, W, 32, 0, 0, 1, 3)


def test_quantize_blocks_gemm_reads_them(fp4, oracle_mod):
    """The broadcast scales are an ordinary [N][K/group] layout: the GEMM
    on channel-granularity weights matches the oracle product."""
    rng = np.random.default_rng(76)
    W = synth.normal_weights(rng, 256, 1024)
    X = synth.activations(rng, 5, 1024)
    res, ref = check_blocks(fp4, oracle_mod, W, 128, 1, 0, 1, -1)
    Y = fp4.gemm(dev_bf16(X), res["packed"], res["scales"], 1, 128)
    assert rel_err(Y, oracle_mod.gemm(X, ref["packed"], ref["scales"], 1, 128)) <= TOL


def test_quantize_blocks_llama13b_full(fp4, oracle_mod):
    """Full-size 13B projections: the q projection 5120x5120 with one scale
    per attention head (40 heads of 128 rows) and a per-head bias search;
    the gate projection 13824x5120 per output channel."""
    case = synth.llama13b_search(shapes=((5120, 5120),))
    W = case["W"][0]
    check_blocks(fp4, oracle_mod, W, 128, 2, 40, 1, -1)
    rng = np.random.default_rng(77)
    W2 = synth.normal_weights(rng, 13824, 5120)
    check_blocks(fp4, oracle_mod, W2, 128, 1, 0, 1, 0)


@pytest.mark.expect_status
def test_quantize_blocks_nonfinite_sets_status(fp4):
    W = torch.zeros((8, 256), dtype=torch.float32, device="cuda")
    W[3, 7] = float("nan")
    fp4.quantize_blocks(W, 128, fp4.GRAN_CHANNEL, 0, fp4.E2M1, -1)
    assert fp4.device_status(clear=True) & fp4.DEV_NONFINITE_INPUT


# ------------------------------------------------------ 4-bit activations

@pytest.mark.parametrize("M,K", [(1, 4096), (7, 136), (64, 512), (300, 1024)])
@pytest.mark.parametrize("fmt,j", [(1, 0), (1, 3), (0, 0), (2, 7)])
def test_act_quantize_bitexact(fp4, oracle_mod, M, K, fmt, j):
    rng = np.random.default_rng(80 + M)
    X, _ = synth.outlier_activations(rng, M, K, frac=0.02, factor=50.0)
    cal, _ = synth.outlier_activations(rng, 16, K, frac=0.02, factor=40.0)   # separate calibration data
    shift, rho = oracle_mod.preshift_calibrate(cal)
    ref, s_ref = oracle_mod.act_quantize(X, rho, fmt, j, shift)
    gshift = torch.from_numpy(shift).cuda()
    grho = torch.tensor([rho], dtype=torch.float32, device="cuda")
    codes, s_a = fp4.act_quantize(dev_bf16(X), grho, fmt, j, gshift)
    assert s_a.item() == s_ref
    assert np.array_equal(codes.cpu().numpy(), ref)
    ref0, _ = oracle_mod.act_quantize(X, rho, fmt, j, None)
    codes0, _ = fp4.act_quantize(dev_bf16(X), grho, fmt, j, None)
    assert np.array_equal(codes0.cpu().numpy(), ref0)


def test_act_quantize_edges(fp4, oracle_mod):
    """Ties, both zeros, saturation and subnormal-sized values."""
    vals = np.array([0.5, -1.25, 2.5, 5.0, 7.0, -0.0, 0.24, 0.26, 1e-30, -1e-30, 6.0, 1e30, -1e30, 0.75, 1.75,
                     3.5], np.float32)
    X = synth.to_bf16_bits(np.tile(vals, (3, 1)))
    for rho in (6.0, 1.0, 3e-38):
        for fmt in (0, 1, 2):
            ref, s_ref = oracle_mod.act_quantize(X, rho, fmt, 0)
            codes, s_a = fp4.act_quantize(dev_bf16(X), torch.tensor([rho], device="cuda"), fmt, 0)
            assert s_a.item() == s_ref and np.array_equal(codes.cpu().numpy(), ref), (rho, fmt)


def test_act_quantize_empty_writes_the_scale(fp4, oracle_mod):
    X = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    codes, s_a = fp4.act_quantize(X, torch.tensor([6.0], device="cuda"), 1, 2)
    _, s_ref = oracle_mod.act_quantize(np.zeros((0, 64), np.uint16), 6.0, 1, 2)
    assert s_a.item() == s_ref and codes.numel() == 0


@pytest.mark.expect_status
def test_act_quantize_bad_rho_and_nonfinite(fp4):
    X = torch.ones((2, 64), dtype=torch.bfloat16, device="cuda")
    _, s_a = fp4.act_quantize(X, torch.tensor([0.0], device="cuda"), 1, 0)
    assert np.isnan(s_a.item()) and fp4.device_status(clear=True) & fp4.DEV_NONFINITE_INPUT
    X[1, 3] = float("inf")
    fp4.act_quantize(X, torch.tensor([2.0], device="cuda"), 1, 0)
    assert fp4.device_status(clear=True) & fp4.DEV_NONFINITE_INPUT


# ----------------------------------------------------------- W4A4 product

def w4a4_case(fp4, oracle_mod, seed, M, N, K, afmt=1, fmt=1, aj=0, sdt="f16"):
    rng = np.random.default_rng(seed)
    W = synth.normal_weights(rng, N, K)
    X, _ = synth.outlier_activations(rng, M, K)
    shift, rho = oracle_mod.preshift_calibrate(X)
    ap, s_a = oracle_mod.act_quantize(X, rho, afmt, aj, shift)
    wp, ws, _ = oracle_mod.quantize_fixed(W, 128, fmt, 0, shift, sdt)
    gap, gs = fp4.act_quantize(dev_bf16(X), torch.tensor([rho], device="cuda"), afmt, aj,
                               torch.from_numpy(shift).cuda())
    assert np.array_equal(gap.cpu().numpy(), ap) and gs.item() == s_a
    return ap, s_a, wp, ws, gap, gs


@pytest.mark.parametrize("M", [1, 5, 8, 16, 33, 64, 65, 300])
@pytest.mark.parametrize("N,K", [(256, 512), (200, 1024)])
def test_gemm_w4a4(fp4, oracle_mod, M, N, K):
    ap, s_a, wp, ws, gap, gs = w4a4_case(fp4, oracle_mod, 90 + M, M, N, K)
    Y = fp4.gemm_w4a4(gap, gs, torch.from_numpy(wp).cuda(), torch.from_numpy(ws).cuda(), 1, 1, 128)
    assert rel_err(Y, oracle_mod.gemm_w4a4(ap, 1, s_a, wp, ws, 1, 128)) <= TOL


@pytest.mark.parametrize("afmt,fmt,aj", [(0, 1, 2), (2, 0, 5), (1, 2, 7)])
def test_gemm_w4a4_formats(fp4, oracle_mod, afmt, fmt, aj):
    for M in (4, 130):
        ap, s_a, wp, ws, gap, gs = w4a4_case(fp4, oracle_mod, 95, M, 136, 768, afmt, fmt, aj, "f32")
        Y = fp4.gemm_w4a4(gap, gs, torch.from_numpy(wp).cuda(), torch.from_numpy(ws).cuda(), afmt, fmt, 128)
        assert rel_err(Y, oracle_mod.gemm_w4a4(ap, afmt, s_a, wp, ws, fmt, 128)) <= TOL, M


@pytest.mark.parametrize("act", [1, 3])
def test_gemm_w4a4_activation(fp4, oracle_mod, act):
    for M in (2, 96):
        ap, s_a, wp, ws, gap, gs = w4a4_case(fp4, oracle_mod, 97, M, 256, 512)
        Y = fp4.gemm_w4a4(gap, gs, torch.from_numpy(wp).cuda(), torch.from_numpy(ws).cuda(), 1, 1, 128, act=act)
        Yr = oracle_mod.gemm_w4a4(ap, 1, s_a, wp, ws, 1, 128)
        ref = oracle_mod.silu_gate(Yr) if act == 3 else oracle_mod.activation(Yr, act)
        assert rel_err(Y, ref) <= TOL, M


def test_w4a4_llama7b_prefill_full(fp4, oracle_mod):
    """The LLaMA-7B prefill workload in W4A4: calibration, activation codes
    and folded weights bit-exact at 2048x4096; the product on whole sampled
    rows of the 11008x4096 projection."""
    case = synth.llama7b_prefill(shapes=((11008, 4096),))
    X = case["X"]
    W = case["W"][0]
    shift, rho = oracle_mod.preshift_calibrate(X)
    gshift, grho = fp4.preshift_calibrate(dev_bf16(X))
    assert np.array_equal(gshift.cpu().numpy(), shift) and grho.item() == rho
    ap, s_a = oracle_mod.act_quantize(X, rho, 1, 0, shift)
    gap, gs = fp4.act_quantize(dev_bf16(X), grho, 1, 0, gshift)
    assert np.array_equal(gap.cpu().numpy(), ap) and gs.item() == s_a
    res = fp4.quantize(dev_f32(W), 128, 1, False, gshift, "f16")
    wp = res["packed"].cpu().numpy()
    ws = res["scales"].cpu().numpy()
    ref = oracle_mod.quantize(W, 128, 1, False, shift, "f16")
    assert np.array_equal(wp, ref["packed"]) and np.array_equal(ws.view(np.uint16), ref["scales"].view(np.uint16))
    Y = fp4.gemm_w4a4(gap, gs, res["packed"], res["scales"], 1, 1, 128)
    M, N = Y.shape
    assert bool(torch.isfinite(Y.float()).all())
    sel = [0, 777, 2047]
    ms = np.repeat(np.asarray(sel, np.int32), N)
    ns = np.tile(np.arange(N, dtype=np.int32), len(sel))
    yref = oracle_mod.gemm_w4a4_sampled(ap, 1, s_a, wp, ws, 1, 128, ms, ns).reshape(len(sel), N)
    got = Y.float().cpu().numpy().astype(np.float64)[sel]
    assert float(np.max(np.abs(got - yref)) / np.max(np.abs(yref))) <= TOL


@pytest.mark.parametrize("M,N,K", [(65, 256, 512), (128, 384, 1024), (300, 200, 768), (2048, 256, 4096)])
def test_gemm_w4a4_native_matches_expand(fp4, oracle_mod, M, N, K):
    """E2M1 x E2M1 from M = 65 runs on kind::f8f6f4 MMAs with no
    dequantization; codes at a 16- (not 32-) byte offset take the expanding
    16-bit path.  Both meet the bound against the oracle."""
    ap, s_a, wp, ws, gap, gs = w4a4_case(fp4, oracle_mod, 98 + M, M, N, K)
    gw, gsc = torch.from_numpy(wp).cuda(), torch.from_numpy(ws).cuda()
    ref = oracle_mod.gemm_w4a4(ap, 1, s_a, wp, ws, 1, 128)
    Yn = fp4.gemm_w4a4(gap, gs, gw, gsc, 1, 1, 128)
    buf = torch.empty(gap.numel() + 16, dtype=torch.uint8, device="cuda")
    shifted = buf[16:].view(gap.shape)
    shifted.copy_(gap)
    assert shifted.data_ptr() % 32 == 16
    Ye = fp4.gemm_w4a4(shifted, gs, gw, gsc, 1, 1, 128)
    assert rel_err(Yn, ref) <= TOL and rel_err(Ye, ref) <= TOL


@pytest.mark.parametrize("M", [65, 200])
def test_gemm_w4a4_native_ragged_and_formats(fp4, oracle_mod, M):
    """Ragged N and M tails on the native path, fp32 weight scales, a
    shifted activation bias index."""
    ap, s_a, wp, ws, gap, gs = w4a4_case(fp4, oracle_mod, 99, M, 130, 384, 1, 1, 5, "f32")
    Y = fp4.gemm_w4a4(gap, gs, torch.from_numpy(wp).cuda(), torch.from_numpy(ws).cuda(), 1, 1, 128)
    assert rel_err(Y, oracle_mod.gemm_w4a4(ap, 1, s_a, wp, ws, 1, 128)) <= TOL
