"""The C ABI library: it builds, loads, exports every declared symbol, and its
host-side checks reject bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a4.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in {"if", "defined"}))


@pytest.fixture(scope="module")
def so():
    from bit_diffusion_transformer_nvfp4_b200 import build
    build.build()
    import bit_diffusion_transformer_nvfp4_b200 as w
    return w.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["nvfp4_quantize_act", "nvfp4_pack_weight", "w4a4_gemm", "w4a4_linear", "nvfp4_sf_bytes",
              "nvfp4_quant_workspace_bytes", "w4a4_workspace_bytes", "w4a4_device_status",
              "w4a4_status_string", "nvfp4_sf_to_rowmajor"]:
        assert n in names


def test_every_declared_symbol_is_exported(so):
    for n in declared_functions():
        assert hasattr(so, n), n
        assert isinstance(getattr(so, n), ctypes._CFuncPtr)


def test_sizes(so):
    assert so.nvfp4_sf_bytes(300, 512) == 384 * 32
    assert so.nvfp4_sf_bytes(128, 3072) == 128 * 192
    assert so.nvfp4_sf_bytes(0, 256) == 0
    assert so.nvfp4_sf_bytes(10, 100) == 0
    assert so.nvfp4_quant_workspace_bytes(4608, 3072, 32) > 4608 * 32 * 4
    assert so.nvfp4_quant_workspace_bytes(4608, 3000, 32) == 0
    assert so.nvfp4_quant_workspace_bytes(4608, 3072, 16) > 0
    assert so.nvfp4_quant_workspace_bytes(4608, 3072, 24) == 0
    ws = so.w4a4_workspace_bytes(4608, 9216, 3072, 32)
    assert ws >= 4608 * 1536 + 4608 * 192 + 4608 * 128
    assert so.w4a4_workspace_bytes(4608, 9210, 3072, 32) == 0


def test_status_strings(so):
    for st in range(-8, 1):
        assert so.w4a4_status_string(st)
    assert so.w4a4_status_string(-7) == b"a device-side pipeline wait exceeded its bound"


def test_host_validation_before_any_launch(so):
    import bit_diffusion_transformer_nvfp4_b200 as w
    P = 1 << 20  # aligned fake device address, never dereferenced
    big = 1 << 30
    q = w.lib().nvfp4_quantize_act
    assert q(None, 128, 512, 512, None, None, 0, None, P, P, P, None, P, big, None) == -1     # NULL X
    assert q(P, 128, 500, 512, None, None, 0, None, P, P, P, None, P, big, None) == -2        # K % 64
    assert q(P, 128, 512, 500, None, None, 0, None, P, P, P, None, P, big, None) == -2        # ldx < K
    assert q(P, 128, 512, 512, None, None, 24, None, P, P, P, None, P, big, None) == -2       # rank
    assert q(P, 128, 512, 512, None, None, 16, None, P, P, P, None, P, big, None) == -1       # rank 16, no L1t
    assert q(P, 128, 512, 512, None, None, 32, None, P, P, P, None, P, big, None) == -1       # no L1t
    assert q(P + 2, 128, 512, 512, None, None, 0, None, P, P, P, None, P, big, None) == -3    # alignment
    assert q(P, 128, 512, 512, None, None, 0, None, P, P, P, None, P, 16, None) == -5         # workspace
    g = w.lib().w4a4_gemm
    assert g(P, P, P, None, 128, 100, 512, P, P, P, None, 0, None, 0, P, 100, None) == -2     # N % 8
    assert g(P, P, P, None, 128, 128, 512, P, P, P, None, 0, None, 7, P, 128, None) == -8     # epilogue
    assert g(P, P, P, None, 128, 128, 512, P, P, P, None, 0, None, 0, P, 120, None) == -2     # ldy < N
    assert g(P, P, P, None, 128, 128, 512, P, P, P, None, 32, None, 0, P, 128, None) == -1    # no U/L2t
    h = w.lib().nvfp4_sf_to_rowmajor
    assert h(P, 128, 500, P, None) == -2                                                      # K % 64
    assert h(None, 128, 512, P, None) == -1                                                   # NULL
    assert h(P, 128, 512, P + 4, None) == -3                                                  # alignment
    pw = w.lib().nvfp4_pack_weight
    assert pw(P, 5, 128, 512, 512, P, P, P, P, big, None) == -8                               # dtype



def test_k_and_fp8_column_bounds(so):
    """K up to 2^20 (the widest row the tensor-amax pass covers with its 1024
    partial maxima of 256 segments) and FP8 columns up to 2^21 are accepted;
    one step past either bound is a size error before any launch."""
    import bit_diffusion_transformer_nvfp4_b200 as w
    P = 1 << 20
    big = 1 << 30
    kmax = 1 << 20
    hdr = open(HEADER).read()
    assert re.search(r"#define W4A4_MAX_K \(\(int64_t\)1 << 20\)", hdr) and w.MAX_K == kmax
    assert so.nvfp4_quant_workspace_bytes(128, kmax, 32) > 0
    assert so.nvfp4_quant_workspace_bytes(128, kmax + 64, 32) == 0
    assert so.w4a4_workspace_bytes(128, 256, kmax, 32) > 0
    assert so.w4a4_workspace_bytes(128, 256, kmax + 64, 32) == 0
    assert so.nvfp4_quantize_act(P, 128, kmax + 64, kmax + 64, None, None, 0, None, P, P, P, None, P, big,
                                 None) == -2
    assert so.nvfp4_pack_weight(P, 1, 128, kmax + 64, kmax + 64, P, P, P, P, big, None) == -2
    assert so.w4a4_gemm(P, P, P, None, 128, 128, kmax + 64, P, P, P, None, 0, None, 0, P, 128, None) == -2
    assert so.w4a4_linear(P, 128, 128, kmax + 64, P, P, P, None, P, P, 32, None, 0, P, P, big, None) == -2
    assert so.fp8_quant_workspace_bytes(128, 1 << 21) > 0
    assert so.fp8_quant_workspace_bytes(128, (1 << 21) + 8) == 0
    assert so.fp8_quantize(P, 128, (1 << 21) + 8, (1 << 21) + 8, 0, P, (1 << 21) + 8, P, P, big, None) == -2


def test_host_validation_linear_and_amax_entries(so):
    """The whole-path and given/next-amax entry points reject bad arguments on
    the host, in the documented order, before touching a GPU."""
    P = 1 << 20  # aligned fake device address, never dereferenced
    big = 1 << 30
    lin = so.w4a4_linear
    #        X  M    N    K    Wq Wsf t_w inv_s L1t L2t r   bias  epi Y  ws  ws_bytes stream
    assert lin(P, 128, 100, 512, P, P, P, None, P, P, 32, None, 0, P, P, big, None) == -2   # N % 8
    assert lin(P, 128, 128, 500, P, P, P, None, P, P, 32, None, 0, P, P, big, None) == -2   # K % 64
    assert lin(P, 128, 128, 512, P, P, P, None, P, P, 24, None, 0, P, P, big, None) == -2   # rank
    assert lin(P, 128, 128, 512, P, P, P, None, P, P, 32, None, 7, P, P, big, None) == -8   # epilogue
    assert lin(None, 128, 128, 512, P, P, P, None, P, P, 32, None, 0, P, P, big, None) == -1  # NULL X
    assert lin(P, 128, 128, 512, P, P, P, None, None, P, 32, None, 0, P, P, big, None) == -1  # rank 32, no L1t
    assert lin(P, 128, 128, 512, P, P, P, None, P, P, 32, None, 0, P, P, 16, None) == -5    # workspace size
    assert lin(P, 128, 128, 512, P, P, P, None, P, P, 32, None, 0, P, P + 2, big, None) == -3  # workspace align
    qa = so.nvfp4_quantize_act_with_amax
    #        X  M    K    ldx inv_s L1t r  t_w  amax   Xq Xsf t_x U     ws  ws_bytes stream
    assert qa(P, 128, 512, 512, None, None, 0, None, None, P, P, P, None, P, big, None) == -1  # no amax
    assert qa(P, 128, 512, 512, None, None, 0, None, P + 2, P, P, P, None, P, big, None) == -3  # amax align
    assert qa(P, 128, 500, 512, None, None, 0, None, P, P, P, P, None, P, big, None) == -2      # K % 64
    gn = so.w4a4_gemm_next_amax
    #       Xq Xsf t_x U     M    N    K    Wq Wsf t_w L2t  r  bias  epi Y  ldy  inv_s  amax   stream
    assert gn(P, P, P, None, 128, 128, 512, P, P, P, None, 0, None, 0, P, 128, None, None, None) == -1
    assert gn(P, P, P, None, 128, 128, 512, P, P, P, None, 0, None, 0, P, 128, P + 4, P, None) == -3
    assert gn(P, P, P, None, 128, 128, 512, P, P, P, None, 0, None, 0, P, 128, None, P + 2, None) == -3
    assert gn(P, P, P, None, 128, 100, 512, P, P, P, None, 0, None, 0, P, 100, None, P, None) == -2

def test_empty_problems_are_noops(so):
    """M == 0 (N == 0 for packing) with valid sizes: W4A4_OK at once, with
    NULL buffers, no device needed; invalid sizes still fail."""
    assert so.nvfp4_quantize_act(None, 0, 512, 512, None, None, 32, None, None, None, None, None, None, 0,
                                 None) == 0
    assert so.nvfp4_quantize_act_with_amax(None, 0, 512, 512, None, None, 0, None, None, None, None, None, None,
                                           None, 0, None) == 0
    assert so.nvfp4_quantize_act_noalloc(None, 0, 512, 512, None, None, 16, None, None, None, None, None,
                                         None) == 0
    assert so.w4a4_gemm(None, None, None, None, 0, 128, 512, None, None, None, None, 32, None, 0, None, 128,
                        None) == 0
    assert so.w4a4_gemm_next_amax(None, None, None, None, 0, 128, 512, None, None, None, None, 0, None, 1,
                                  None, 128, None, None, None) == 0
    assert so.w4a4_linear(None, 0, 128, 512, None, None, None, None, None, None, 16, None, 0, None, None, 0,
                          None) == 0
    assert so.nvfp4_pack_weight(None, 1, 0, 512, 512, None, None, None, None, 0, None) == 0
    assert so.nvfp4_sf_to_rowmajor(None, 0, 512, None, None) == 0
    assert so.nvfp4_quantize_act(None, 0, 500, 512, None, None, 0, None, None, None, None, None, None, 0,
                                 None) == -2
    assert so.w4a4_gemm(None, None, None, None, 0, 100, 512, None, None, None, None, 0, None, 0, None, 100,
                        None) == -2


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU path")
def test_no_gpu_reports_arch_error(so):
    P = 1 << 20
    st = so.nvfp4_quantize_act(P, 128, 512, 512, None, None, 0, None, P, P, P, None, P, 1 << 30, None)
    assert st == -4


def _header_define(name):
    src = open(HEADER).read()
    m = re.search(r"#define " + name + r" \((.*)\)\s*$", src, flags=re.M)
    assert m, name
    return m.group(1)


def test_k_multiple_of_64_is_accepted(so):
    """One FP4 MMA K-step (64 elements, four scale blocks) is the unit: K =
    3136 = 49 x 64 passes every size check (and reaches the device check)."""
    assert so.nvfp4_quant_workspace_bytes(4608, 3136, 32) > 0
    assert so.nvfp4_quant_workspace_bytes(4608, 64, 0) > 0
    assert so.nvfp4_quant_workspace_bytes(4608, 3100, 32) == 0
    assert so.w4a4_workspace_bytes(4608, 9216, 3136, 32) > 0
    assert so.nvfp4_sf_bytes(128, 3136) == 128 * 196
    if not __import__("torch").cuda.is_available():
        P = 1 << 20
        st = so.nvfp4_quantize_act(P, 128, 3136, 3136, None, None, 0, None, P, P, P, None, P, 1 << 30, None)
        assert st == -4


def test_workspace_layout_does_not_depend_on_the_sizes(so):
    """The synchronisation words sit at fixed offsets (documented in the
    header); only the low-rank partial sums at the end grow with M."""
    bar = int(_header_define("W4A4_WS_BARRIER_OFFSET").split(")")[-1])
    tick = int(_header_define("W4A4_WS_TICKETS_OFFSET").split(")")[-1])
    assert (bar, tick) == (4096, 5120)
    max_rows = 1 << 22
    upart = tick + 4 * (max_rows // 128)
    for M, K in [(1, 64), (128, 3072), (4608, 3072), (9216, 3072), (18432, 12288), (16896, 24576)]:
        b0 = so.nvfp4_quant_workspace_bytes(M, K, 0)
        b32 = so.nvfp4_quant_workspace_bytes(M, K, 32)
        assert b0 == upart, (M, K)
        assert b32 > upart and (b32 - upart) % (128 * 32 * 4) == 0, (M, K)
    # with a low-rank branch the counters cover at most 2^22 rows
    assert so.nvfp4_quant_workspace_bytes(max_rows, 64, 32) > 0
    assert so.nvfp4_quant_workspace_bytes(max_rows + 1, 64, 32) == 0
    assert so.nvfp4_quant_workspace_bytes(max_rows + 1, 64, 0) > 0
    P = 1 << 20
    assert so.nvfp4_quantize_act(P, max_rows + 1, 64, 64, None, P, 32, P, P, P, P, P, P, 1 << 40, None) == -2


def test_wait_bound_argument_check(so):
    assert so.w4a4_set_wait_bound(5) == -8
    if not __import__("torch").cuda.is_available():
        assert so.w4a4_set_wait_bound(0) == -4


def test_swiglu_argument_checks(so):
    """w4a4_gemm_swiglu rejects bad splits, strides and pointers on the host."""
    P = 1 << 20
    f = so.w4a4_gemm_swiglu
    #        Xq Xsf t_x U     M    N     K    Wq Wsf t_w L2t  r  bias n_plain Y  ldy H  ldh  s     amax  stream
    assert f(P, P, P, None, 128, 1024, 512, P, P, P, None, 0, None, 128, P, 128, P, 448, None, None, None) == -2
    assert f(P, P, P, None, 128, 1024, 512, P, P, P, None, 0, None, 256, P, 256, P, 368, None, None, None) == -2
    assert f(P, P, P, None, 128, 1040, 512, P, P, P, None, 0, None, 256, P, 256, P, 392, None, None, None) == -2
    assert f(P, P, P, None, 128, 1024, 512, P, P, P, None, 0, None, 1024, P, 1024, P, 8, None, None, None) == -2
    assert f(P, P, P, None, 128, 1024, 512, P, P, P, None, 0, None, 256, P, 256, None, 384, None, None, None) == -1
    assert f(P, P, P, None, 128, 1024, 512, P, P, P, None, 0, None, 256, P, 256, P + 2, 384, None, None, None) == -3
    assert f(None, None, None, None, 0, 1024, 512, None, None, None, None, 0, None, 256, None, 256, None, 384,
             None, None, None) == 0


def test_rope_argument_checks(so):
    """w4a4_gemm_rope rejects bad head sizes, table strides and pointers on the host."""
    P = 1 << 20

    def call(n_rope=256, d_head=128, rope=P, ld_rope=128, n_plain=512, N=768, H=P, ldh=128, M=128):
        #                Xq Xsf t_x U  M  N  K    Wq Wsf t_w L2t  r  bias
        return so.w4a4_gemm_rope(P, P, P, None, M, N, 512, P, P, P, None, 0, None,
                                 n_rope, d_head, rope, ld_rope, n_plain, P, n_plain, H, ldh, None, None, None)
    if not __import__("torch").cuda.is_available():
        assert call() == -4                                  # valid: reaches the device check
        assert call(N=512, H=None, ldh=0) == -4              # no SwiGLU features
        assert call(d_head=32, ld_rope=36) == -4             # padded table rows
    assert call(d_head=48, n_rope=240, ld_rope=48) == -2     # head size not a multiple of 32
    assert call(n_rope=192) == -2                            # not a whole number of heads
    assert call(n_rope=0) == -2                              # nothing to turn: use w4a4_gemm_swiglu
    assert call(n_rope=768, n_plain=512) == -2               # beyond the plain features
    assert call(ld_rope=96) == -2                            # table row shorter than a head
    assert call(ld_rope=130) == -2                           # table rows not 16-byte aligned
    assert call(n_plain=384) == -2                           # SwiGLU split not a multiple of 256
    assert call(rope=None) == -1
    assert call(rope=P + 4) == -3
    assert call(H=None) == -1                                # SwiGLU features need H
    assert call(M=0, rope=None) == 0                         # empty problem


def test_fp8_argument_checks(so):
    """fp8_quantize and attention_fp8 reject bad sizes, strides and pointers on the host."""
    P = 1 << 20
    q = so.fp8_quantize
    ws = so.fp8_quant_workspace_bytes(256, 256)
    assert ws >= 4096 and so.fp8_quant_workspace_bytes(256, 250) == 0
    #        X  rows cols ldx tr out ldo  scale ws  bytes stream
    assert q(P, 256, 250, 256, 0, P, 256, P, P, ws, None) == -2          # cols % 8
    assert q(P, 250, 256, 256, 1, P, 256, P, P, ws, None) == -2          # transposed rows % 16
    assert q(P, 256, 256, 256, 1, P, 248, P, P, ws, None) == -2          # transposed row shorter than rows
    assert q(P, 256, 256, 256, 2, P, 256, P, P, ws, None) == -8          # transpose flag
    assert q(P, 256, 256, 256, 0, P, 256, P, P, 16, None) == -5          # workspace too small
    assert q(P, 256, 256, 256, 0, None, 256, P, P, ws, None) == -1
    assert q(P + 8, 256, 256, 256, 0, P, 256, P, P, ws, None) == -3
    assert q(None, 0, 256, 256, 0, None, 256, None, None, 0, None) == 0   # empty tensor
    a = so.attention_fp8
    c = __import__("ctypes").c_float(0.0884)
    #        Q  K  Vt B  S    H  ldq  ldk  ldvt sq sk sv scale O  ldo  stream
    assert a(P, P, P, 1, 200, 2, 256, 256, 256, P, P, P, c, P, 256, None) == -2     # S % 128
    assert a(P, P, P, 1 << 8, 1 << 23, 1, 128, 128, 1 << 31, P, P, P, c, P, 128, None) == -2   # tokens beyond 2^30
    assert a(P, P, P, 1, 256, 2, 128, 256, 256, P, P, P, c, P, 256, None) == -2     # ldq < heads * 128
    assert a(P, P, P, 2, 256, 2, 256, 256, 256, P, P, P, c, P, 256, None) == -2     # ldvt < batch * S
    assert a(P, P, P, 1, 256, 2, 256, 256, 256, P, P, P, __import__("ctypes").c_float(0.0), P, 256, None) == -8
    assert a(P, P, P, 1, 256, 2, 256, 256, 256, None, P, P, c, P, 256, None) == -1
    assert a(P, P, P + 4, 1, 256, 2, 256, 256, 256, P, P, P, c, P, 256, None) == -3
    assert a(None, None, None, 0, 256, 2, 256, 256, 0, None, None, None, c, None, 256, None) == 0
    if not __import__("torch").cuda.is_available():
        assert a(P, P, P, 1, 256, 2, 256, 256, 256, P, P, P, c, P, 256, None) == -4   # valid: reaches the device check


def test_fp4_mma_rate_argument_checks(so):
    """w4a4_fp4_mma_rate rejects bad counts, modes and pointers on the host."""
    P = 1 << 20
    f = so.w4a4_fp4_mma_rate
    assert f(0, 1, P, None) == -2
    assert f((1 << 20) + 1, 1, P, None) == -2
    assert f(100, 2, P, None) == -8
    assert f(100, 1, None, None) == -1
    assert f(100, 0, P + 4, None) == -3
    if not __import__("torch").cuda.is_available():
        assert f(100, 1, P, None) == -4        # valid: reaches the device check


def test_quantize_next_argument_checks(so):
    """w4a4_gemm_quantize_next rejects bad column ranges, strides and pointers on the host."""
    P = 1 << 20
    f = so.w4a4_gemm_quantize_next
    #          Xq Xsf t_x U  M    N    K    Wq Wsf t_w L2t  r  bias epi n_plain Y  ldy H  ldh s  t  q  ldq sf nK   col  amax stream
    ok = dict(n_plain=384, next_K=384, col=0, ldq=192)
    def call(n_plain=384, next_K=384, col=0, ldq=192, t=P, sf=P, q=P, epi=0, N=384):
        return f(P, P, P, None, 128, N, 512, P, P, P, None, 0, None, epi, n_plain, P, N, None, 0, None, t, q, ldq,
                 sf, next_K, col, None, None)
    if not __import__("torch").cuda.is_available():
        assert call() == -4                                    # valid: reaches the device check
    assert call(next_K=320) == -2                              # columns beyond next_K
    assert call(next_K=448, col=64) == -2                      # 448 % 64 ok, but col + 384 > 448
    assert call(next_K=512, col=32) == -2                      # column offset not a multiple of 64
    assert call(ldq=176) == -2                                 # codes row shorter than next_K / 2
    assert call(t=None) == -1                                  # no tensor scale
    assert call(q=None) == -1
    assert call(sf=P + 4) == -3
    assert call(n_plain=200) == -2                             # SwiGLU split not a multiple of 256
    assert call(n_plain=0, N=416, next_K=256) == -2            # SwiGLU outputs 208 not a multiple of 32
    assert call(epi=7) == -8


def test_sizes_of_empty_problems(so):
    """Size queries for M == 0 (an empty batch) return the fixed layout, not a crash."""
    upart = 5120 + 4 * ((1 << 22) // 128)
    for r in (0, 16, 32):
        assert so.nvfp4_quant_workspace_bytes(0, 512, r) == upart
        assert so.w4a4_workspace_bytes(0, 384, 512, r) >= upart
