"""Host-side checks of the C interface that need no GPU: the library loads,
exports every entry point the header declares, and rejects bad arguments
before touching the device."""
import ctypes
import os
import re

import pytest

from w4a16_gemm_fp4_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4w4a16.h")


@pytest.fixture(scope="module")
def L():
    from w4a16_gemm_fp4_b200 import build
    build.build()
    return api.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^FP4_API\s+[\w\s\*]*?\b(fp4_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_interface():
    names = declared_functions()
    assert "fp4_quantize" in names and "fp4_gemm" in names and "fp4_preshift_calibrate" in names
    assert set(names) == set(api.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # and they are real dynamic exports, not just resolvable names
    out = os.popen("nm -D --defined-only %s" % api.LIB_PATH).read()
    for name in declared_functions():
        assert re.search(r" T %s$" % name, out, flags=re.M), name


def test_version_and_strings(L):
    assert L.fp4_abi_version() == 100
    assert L.fp4_status_string(0) == b"ok"
    assert b"workspace" in L.fp4_status_string(4)


FAKE = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced
MIS = ctypes.c_void_p((1 << 20) + 8)     # misaligned


def q(L, W=FAKE, N=4, K=128, group=128, fmt=1, bias=0, shift=None, sdt=1, packed=FAKE, scales=FAKE,
      choice=FAKE, sse=None, ws=None, wsb=0):
    return L.fp4_quantize(W, N, K, group, fmt, bias, shift, sdt, packed, scales, choice, sse, ws, wsb, None)


def test_quantize_argument_errors(L):
    assert q(L, group=48) == 2
    assert q(L, K=96, group=64) == 2
    assert q(L, N=-1) == 1
    assert q(L, fmt=3) == 1
    assert q(L, fmt=-2) == 1
    assert q(L, sdt=2) == 1
    assert q(L, choice=None) == 1
    assert q(L, W=None) == 1
    assert q(L, W=MIS) == 3
    assert q(L, packed=MIS) == 3
    assert q(L, shift=MIS) == 3
    # search needs a workspace
    assert q(L, fmt=-1, bias=1) == 4
    need = L.fp4_quantize_workspace_size(4, 128, 128, -1, 1)
    assert need > 0
    assert q(L, fmt=-1, bias=1, ws=FAKE, wsb=need - 8) == 4


def test_gemm_argument_errors(L):
    Xp, Pp, Sp, Yp = (ctypes.c_void_p(a << 20) for a in (1, 2, 3, 4))

    def g(X=Xp, packed=Pp, scales=Sp, sdt=1, fmt=1, M=4, N=64, K=256, group=128, Y=Yp, engine=0,
          splits=0):
        return L.fp4_gemm_ex(X, packed, scales, sdt, fmt, M, N, K, group, None, Y, None, 0, engine, splits, None)
    assert g(group=256) == 2
    assert g(K=192) == 2
    assert g(fmt=-1) == 1
    assert g(M=-1) == 1
    assert g(Y=None) == 1
    assert g(X=MIS) == 3
    assert g(Y=MIS) == 3
    assert g(engine=7) == 1
    assert g(splits=-1) == 1
    assert g(M=65, engine=1) == 2         # decode engine: M <= 64 at group 128 ...
    assert g(M=9, group=64, engine=1) == 2  # ... and M <= 8 otherwise
    assert g(Y=Xp) == 1                   # output aliases the input
    # empty problems succeed without touching the device
    assert g(M=0) == 0
    assert g(N=0) == 0


def rowblk_two_buffers(M, K):
    """The group-128 row-block kernel's shared-memory plan (activations staged
    once per CTA; 16-row block buffers of codes and f32 scale rows; the
    cross-warp reduction area): True when it runs with two block buffers."""
    if K > 24576 or M > 16:
        return False
    def smem(nw, nbuf):
        return nbuf * (16 * (K // 2) + 16 * (K // 128) * 4) + M * (2 * K + 64) + \
            2 * nw * 32 * 4 * 4 * (2 if M > 8 else 1) + 128
    for nbuf in (2, 1):
        if 2 * (smem(8, nbuf) + 1024 + 128) <= 228 * 1024 or smem(16, nbuf) <= 226 * 1024:
            return nbuf == 2
    return False


def test_gemm_engine_choice(L):
    """Automatic engine: the decode engine for M <= 8 (group 128 at any K;
    groups 32 and 64: the lookup-table kernel), and for 9 <= M <= 16 at
    group 128 where the row-block kernel runs with two block buffers; the
    tensor engine otherwise (it measures faster there)."""
    e = L.fp4_gemm_engine_for
    for K in (128, 4096, 11008, 24576, 40960):
        for M in (1, 4, 8):
            assert e(M, 4096, K, 128) == 1
        for M in (9, 16):
            assert e(M, 4096, K, 128) == (1 if rowblk_two_buffers(M, K) else 2), (M, K)
        for M in (17, 64, 65):
            assert e(M, 4096, K, 128) == 2
        assert e(2048, 11008, K, 128) == 2
    assert rowblk_two_buffers(12, 2048) and not rowblk_two_buffers(16, 4096)
    assert e(8, 64, 4096, 32) == 1 and e(8, 4096, 4096, 64) == 1
    assert e(9, 4096, 4096, 64) == 2 and e(9, 4096, 4096, 32) == 2
    assert e(0, 4096, 4096, 128) == 0 and e(4, 4096, 4096, 96) == 0
    assert api.gemm_engine_for(8, 4096, 4096) == api.ENGINE_DECODE
    assert api.gemm_engine_for(16, 11008, 11008) == api.ENGINE_TENSOR


def test_preshift_argument_errors(L):
    assert L.fp4_preshift_calibrate(FAKE, 4, 12, FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert L.fp4_preshift_calibrate(FAKE, 4, 64, FAKE, None, FAKE, 1 << 20, None) == 1
    assert L.fp4_preshift_calibrate(FAKE, 4, 64, FAKE, FAKE, None, 0, None) == 4
    assert L.fp4_preshift_apply(FAKE, 4, 64, FAKE, FAKE, FAKE, None) == 1   # in place
    assert L.fp4_preshift_apply(FAKE, 4, 64, FAKE, FAKE, MIS, None) == 3
    assert L.fp4_preshift_apply(FAKE, 0, 64, FAKE, FAKE, FAKE, None) == 0


def test_workspace_sizes(L):
    # decode engine (M <= 64): the activations prepared once per call (M x K
    # halves, then one fp32 factor per row, each rounded up to 256 bytes),
    # two fp32 partial tiles [token tile][128] per CTA (one CTA per SM: 148
    # without a device) and one counter per 128-row tile
    def up(b):
        return (b + 255) // 256 * 256

    def dec(M, N, K, bt):
        tiles = (N + 127) // 128
        chunks = tiles * ((K // 128) // (2 if (K // 128) % 2 == 0 else 1))
        ctas = min(148, chunks)
        return up(M * K * 2) + up(M * 4) + 2 * ctas * bt * 128 * 4 + up(tiles * 4)
    def skinny(M, N, K):  # counter block + two M x TR partial tiles per CTA
        G = K // 128
        tr = 128 if G % 2 == 0 else 256     # tile rows: 2-group or 1-group chunks of 16 KB
        tiles = (N + tr - 1) // tr
        chunks = tiles * (G // (2 if G % 2 == 0 else 1))
        ctas = min(148, chunks)
        return 65536 + up(2 * ctas * M * tr * 4)
    assert L.fp4_gemm_workspace_size(1, 4096, 4096) == skinny(1, 4096, 4096)
    assert L.fp4_gemm_workspace_size(9, 200, 384) == skinny(9, 200, 384)
    assert L.fp4_gemm_workspace_size(16, 11008, 4096) == skinny(16, 11008, 4096)
    assert L.fp4_gemm_workspace_size(17, 4096, 4096) == 65536 + dec(17, 4096, 4096, 32)
    assert L.fp4_gemm_workspace_size(33, 11008, 4096) == 65536 + dec(33, 11008, 4096, 64)
    assert L.fp4_gemm_workspace_size(64, 200, 384) == 65536 + dec(64, 200, 384, 64)   # 2 tiles x 3 one-group chunks
    assert L.fp4_gemm_workspace_size(65, 4096, 4096) == 65536 + ((65 * 4096 * 2 + 255) // 256) * 256 + 65 * 4
    assert L.fp4_gemm_workspace_size(2048, 4096, 4096) == 65536 + 2048 * 4096 * 2 + 2048 * 4
    assert L.fp4_quantize_workspace_size(4096, 4096, 128, 1, 0) >= 8
    assert L.fp4_preshift_workspace_size(2048, 4096) >= 4096 * 4


def test_quantize_blocks_argument_errors(L):
    def qb(N=8, K=256, group=128, gran=1, heads=0, fmt=1, j=0, shift=None, sdt=1, packed=FAKE, scales=FAKE,
           jmap=None, ws=None, wsb=0):
        return L.fp4_quantize_blocks(FAKE, N, K, group, gran, heads, fmt, j, shift, sdt, packed, scales, jmap, ws,
                                     wsb, None)
    assert qb(fmt=-1) == 1                     # the format is fixed
    assert qb(j=8) == 1 and qb(j=-2) == 1
    assert qb(gran=3) == 1
    assert qb(gran=2, heads=0) == 1
    assert qb(gran=2, heads=3) == 2            # N % heads
    assert qb(K=96, group=32) == 2             # channel blocks need K % 128 == 0
    assert qb(group=48) == 2
    assert qb(packed=MIS) == 3
    assert qb(N=0) == 0
    # workspace: channel/head blocks keep their absmax (and, searched, 64 B
    # per 128 weights + one byte per block); group blocks need none
    def up(b):
        return (b + 255) // 256 * 256
    assert L.fp4_quantize_blocks_workspace_size(8, 256, 128, 0, 0, -1) == 0
    assert L.fp4_quantize_blocks_workspace_size(8, 256, 128, 1, 0, 0) == up(8 * 4)
    assert L.fp4_quantize_blocks_workspace_size(8, 256, 128, 2, 4, -1) == up(4 * 4) + up(8 * 256 // 128 * 64) + up(4)
    assert qb(j=-1, ws=None) == 4
    need = L.fp4_quantize_blocks_workspace_size(8, 256, 128, 1, 0, -1)
    assert qb(j=-1, ws=FAKE, wsb=need - 1) == 4


def test_act_quantize_and_w4a4_argument_errors(L):
    aq = L.fp4_act_quantize
    assert aq(FAKE, 4, 60, None, FAKE, 1, 0, FAKE, FAKE, None) == 2      # K % 8
    assert aq(FAKE, 4, 64, None, None, 1, 0, FAKE, FAKE, None) == 1      # rho required
    assert aq(FAKE, 4, 64, None, FAKE, 1, 8, FAKE, FAKE, None) == 1      # j
    assert aq(FAKE, 4, 64, None, FAKE, -1, 0, FAKE, FAKE, None) == 1     # fixed format
    assert aq(MIS, 4, 64, None, FAKE, 1, 0, FAKE, FAKE, None) == 3
    assert aq(FAKE, 4, 64, MIS, FAKE, 1, 0, FAKE, FAKE, None) == 3
    g = L.fp4_gemm_w4a4
    need = L.fp4_gemm_w4a4_workspace_size(4, 256, 512)
    assert need == (L.fp4_gemm_workspace_size(4, 256, 512) + 255) // 256 * 256 + 4 * 512 * 2
    assert g(FAKE, 1, FAKE, FAKE, FAKE, 1, 1, 4, 256, 512, 128, 0, FAKE, None, 0, None) == 4
    assert g(FAKE, 1, FAKE, FAKE, FAKE, 1, 1, 4, 256, 512, 128, 0, FAKE, FAKE, need - 16, None) == 4
    assert g(FAKE, 5, FAKE, FAKE, FAKE, 1, 1, 4, 256, 512, 128, 0, FAKE, FAKE, need, None) == 1
    assert g(FAKE, 1, None, FAKE, FAKE, 1, 1, 4, 256, 512, 128, 0, FAKE, FAKE, need, None) == 1
    assert g(MIS, 1, FAKE, FAKE, FAKE, 1, 1, 4, 256, 512, 128, 0, FAKE, FAKE, need, None) == 3
    assert g(FAKE, 1, FAKE, FAKE, FAKE, 1, 1, 4, 256, 512, 128, 4, FAKE, FAKE, need, None) == 1   # act
    assert g(FAKE, 1, FAKE, FAKE, FAKE, 1, 1, 0, 256, 512, 128, 0, FAKE, None, 0, None) == 0      # M == 0
