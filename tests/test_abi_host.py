"""Host-only checks of the C ABI: the library loads, exports what the header
declares, and rejects bad arguments before touching the GPU (no device needed)."""
import ctypes
import subprocess

import pytest

import mxfp4_block_rotation_b200 as mxq
from mxfp4_block_rotation_b200 import build as mxq_build

INVALID = 1


@pytest.fixture(scope="module")
def L():
    mxq_build.build()
    return mxq.lib()


def test_exports_every_declared_symbol(L):
    names = mxq.declared_symbols()
    assert {"mxq_smooth_rotate_quantize", "mxq_dequantize", "mxq_smooth_rotate_f32", "mxq_sync_check",
            "mxq_status_string", "mxq_last_cuda_error", "mxq_version"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", mxq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)


def test_status_strings_and_version(L):
    for s in range(5):
        assert mxq.status_string(s).startswith(("MXQ_OK", "MXQ_ERR"))
    assert mxq.status_string(99) == "unknown mxq_status"
    assert mxq.version() >= 10000


P = ctypes.c_void_p


def _q(L, x, rows, cols, r, lam, c, s):
    return L.mxq_smooth_rotate_quantize(P(x), rows, cols, P(r), P(lam), P(c), P(s), None)


def test_rejects_bad_shapes_before_launch(L):
    good = 0x100000
    assert _q(L, good, -1, 32, good, None, good * 2, good * 3) == INVALID
    assert _q(L, good, 4, 33, good, None, good * 2, good * 3) == INVALID
    assert _q(L, good, 4, -32, good, None, good * 2, good * 3) == INVALID
    assert _q(L, good, 1 << 31, 32, good, None, good * 2, good * 3) == INVALID
    assert L.mxq_last_cuda_error().startswith(b"invalid argument")


def test_rejects_null_and_misaligned(L):
    a = 0x100000
    assert _q(L, None, 4, 64, a, None, a * 2, a * 3) == INVALID
    assert _q(L, a, 4, 64, None, None, a * 2, a * 3) == INVALID
    assert _q(L, a, 4, 64, a * 5, None, None, a * 3) == INVALID
    assert _q(L, a + 8, 4, 64, a * 5, None, a * 2, a * 3) == INVALID        # X not 16-B aligned
    assert _q(L, a, 4, 64, a * 5 + 1, None, a * 2, a * 3) == INVALID        # R^ odd address
    assert _q(L, a, 4, 64, a * 5, a * 7 + 2, a * 2, a * 3) == INVALID       # Lambda not 4-B aligned
    assert _q(L, a, 4, 64, a * 5, None, a * 2 + 4, a * 3) == INVALID        # codes not 16-B aligned
    assert L.mxq_smooth_rotate_f32(P(a), 4, 64, P(a * 5), None, P(a * 2 + 8), None) == INVALID
    # scales in the MMA layout: a null or not 16-byte-aligned buffer
    assert L.mxq_smooth_rotate_quantize_mma(P(a), 4, 64, P(a * 5), None, P(a * 2), None, None) == INVALID
    assert L.mxq_smooth_rotate_quantize_mma(P(a), 4, 64, P(a * 5), None, P(a * 2), P(a * 3 + 4), None) == INVALID
    assert L.mxq_smooth_rotate_quantize_nvfp4_mma(P(a), 4, 64, P(a * 5), None, P(a * 6), P(a * 2), P(a * 3 + 2),
                                                  None) == INVALID
    assert L.mxq_smooth_rotate_quantize_nvfp4_mma(P(a), 4, 64, P(a * 5), None, None, P(a * 2), P(a * 3),
                                                  None) == INVALID   # no tensor scale
    # dequantize: Lambda without R^, misaligned output
    assert L.mxq_dequantize(P(a), P(a * 2), 4, 64, None, P(a * 3), P(a * 4), None) == INVALID
    assert L.mxq_dequantize(P(a), P(a * 2), 4, 64, None, None, P(a * 4 + 2), None) == INVALID


def test_rejects_overlapping_outputs(L):
    a = 0x100000
    # codes overlap X
    assert _q(L, a, 4, 64, a * 5, None, a + 16, a * 3) == INVALID
    # scales overlap codes
    assert _q(L, a, 4, 64, a * 5, None, a * 2, a * 2 + 16) == INVALID
    # dequant output overlaps the codes
    assert L.mxq_dequantize(P(a), P(a * 2), 4, 64, None, None, P(a), None) == INVALID


def test_empty_is_a_noop(L):
    a = 0x100000
    assert _q(L, a, 0, 64, a * 5, None, a * 2, a * 3) == 0
    assert _q(L, a, 4, 0, a * 5, None, a * 2, a * 3) == 0
    assert L.mxq_dequantize(P(a), P(a * 2), 0, 64, None, None, P(a * 4), None) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    r = torch.eye(32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mxq.smooth_rotate_quantize(x, r)


def _search(L, x, rows, cols, lam, K, n, R, rhat=None, trace=None, linf=None, steps=None, group=None, ws=None,
            wsb=1 << 30):
    return L.mxq_rotation_search(P(x), rows, cols, P(lam), K, n, P(R), P(rhat), P(trace), P(linf), P(steps),
                                 P(group), P(ws), wsb, None)


def test_rotation_search_rejects_bad_arguments(L):
    a = 0x100000
    ws = 0x40000000
    assert L.mxq_rotation_search_workspace_bytes(4, 64, 32) >= 512 + 32 * 64 * 8 + 4 * 32 * 8
    assert L.mxq_rotation_search_workspace_bytes(0, 64, 32) == 0
    assert L.mxq_rotation_search_workspace_bytes(4, 64, 0) == 0
    assert _search(L, a, 0, 64, None, 8, 32, a * 3, ws=ws) == INVALID          # no rows
    assert _search(L, a, 4, 0, None, 8, 32, a * 3, ws=ws) == INVALID           # no groups
    assert _search(L, a, 4, 48, None, 8, 32, a * 3, ws=ws) == INVALID          # cols not a multiple of 32
    assert _search(L, a, 4, 64, None, -1, 32, a * 3, ws=ws) == INVALID         # negative K
    assert _search(L, a, 4, 64, None, 65537, 32, a * 3, ws=ws) == INVALID      # K too large
    assert _search(L, a, 4, 64, None, 8, 0, a * 3, ws=ws) == INVALID           # empty angle grid
    assert _search(L, a, 4, 64, None, 8, 129, a * 3, ws=ws) == INVALID
    assert _search(L, None, 4, 64, None, 8, 32, a * 3, ws=ws) == INVALID       # null X
    assert _search(L, a, 4, 64, None, 8, 32, None, ws=ws) == INVALID           # null R
    assert _search(L, a + 8, 4, 64, None, 8, 32, a * 3, ws=ws) == INVALID      # X not 16-B aligned
    assert _search(L, a, 4, 64, None, 8, 32, a * 3 + 4, ws=ws) == INVALID      # R not 8-B aligned
    assert _search(L, a, 4, 64, None, 8, 32, a * 3, ws=ws + 128) == INVALID    # workspace not 256-B aligned
    assert _search(L, a, 4, 64, None, 8, 32, a * 3, ws=ws, wsb=64) == INVALID  # workspace too small
    assert _search(L, a, 4, 64, None, 8, 32, a * 3, ws=None) == INVALID        # no workspace
    assert _search(L, a, 4, 64, None, 8, 32, a + 64, ws=ws) == INVALID         # R overlaps X
    assert _search(L, a, 4, 64, None, 8, 32, a * 3, linf=a * 3 + 8192 - 8, ws=ws) == INVALID  # linf overlaps R
    assert L.mxq_last_cuda_error().startswith(b"invalid argument")


def test_block_variant_rejects_bad_arguments(L):
    a = 0x100000

    def q(rows, cols, blk, lam=None, codes=a * 2, x=a):
        return L.mxq_rotate_quantize_block(P(x), rows, cols, blk, P(a * 5), P(lam), P(codes), P(a * 3), None)

    assert q(4, 128, 48) == INVALID                     # not a supported block width
    assert q(4, 128, 256) == INVALID
    assert q(4, 96, 64) == INVALID                      # cols not a multiple of the block
    assert q(4, 192, 128) == INVALID
    assert q(4, 128, 64, lam=a * 7) == INVALID          # Λ with a block wider than a group
    assert q(4, 128, 128, lam=a * 7) == INVALID
    assert q(4, 128, 64, x=a + 8) == INVALID            # X not 16-B aligned
    assert q(4, 128, 64, codes=a + 16) == INVALID       # codes overlap X
    assert L.mxq_last_cuda_error().startswith(b"invalid argument")
    assert q(0, 128, 128) == 0 and q(4, 0, 64) == 0     # empty: nothing to do
    assert L.mxq_rotate_block_f32(P(a), 4, 96, 64, P(a * 5), None, P(a * 2), None) == INVALID


def test_nvfp4_rejects_bad_arguments(L):
    a = 0x100000

    def nv(x, rows, cols, r, lam, st, codes, scales):
        return L.mxq_smooth_rotate_quantize_nvfp4(P(x), rows, cols, P(r), P(lam), P(st), P(codes), P(scales), None)

    assert nv(a, 0, 64, a * 5, None, None, None, None) == 0                      # nothing to do
    assert nv(a, 4, 48, a * 5, None, a * 7, a * 2, a * 3) == INVALID            # cols not a multiple of 32
    assert nv(a, 4, 64, a * 5, None, None, a * 2, a * 3) == INVALID             # no tensor scale
    assert nv(a, 4, 64, a * 5, None, a * 7 + 2, a * 2, a * 3) == INVALID        # tensor scale not 4-B aligned
    assert nv(a, 4, 64, a * 5, None, a * 7, a * 2, a * 3 + 1) == INVALID        # scales at an odd address
    assert nv(a, 4, 64, a * 5, None, a * 7, a * 2, None) == INVALID             # no scales
    assert nv(a, 4, 64, a * 5, None, a * 2 + 4, a * 2, a * 3) == INVALID        # tensor scale inside the codes
    assert L.mxq_last_cuda_error().startswith(b"invalid argument")


def test_gemm_and_scale_layout_reject_bad_arguments(L):
    """The consumer GEMMs and the scale-atom layouts: sizes, nulls, alignment and overlaps
    are refused on the host (nothing here reaches a device query)."""
    a = 0x100000
    M, N, K = 256, 256, 512
    nca = M * K // 2
    # atom arrays: one 512-byte atom per 128 rows x 4 scale columns
    assert L.mxq_scales_mma_bytes(256, 512) == 2 * 4 * 512
    assert L.mxq_scales_mma_bytes(129, 160) == 2 * 2 * 512
    assert L.mxq_nvfp4_scales_mma_bytes(256, 512) == 2 * 8 * 512
    assert L.mxq_nvfp4_scales_mma_bytes(1, 32) == 512
    for f in (L.mxq_scales_mma_bytes, L.mxq_nvfp4_scales_mma_bytes):
        assert f(0, 64) == 0 and f(4, 0) == 0 and f(4, 48) == 0 and f(-1, 64) == 0

    def mx(ac, asf, bc, bsf, m, n, k, y, bf16=0):
        return L.mxq_mxfp4_gemm(P(ac), P(asf), P(bc), P(bsf), m, n, k, P(y), bf16, None)

    def nv(ac, asf, ta, bc, bsf, tb, m, n, k, y, bf16=0):
        return L.mxq_nvfp4_gemm(P(ac), P(asf), P(ta), P(bc), P(bsf), P(tb), m, n, k, P(y), bf16, None)

    ok = (a, a * 2, a * 3, a * 4)
    y = a * 64
    assert mx(*ok, -1, N, K, y) == INVALID                       # negative size
    assert mx(*ok, M, N, 48, y) == INVALID                       # K not a multiple of 32
    assert mx(*ok, 1 << 31, N, K, y) == INVALID                  # past the 32-bit tile indices
    assert mx(*ok, M, N, K, y, bf16=2) == INVALID                # output type flag
    assert mx(*ok, 0, N, K, None) == 0 and mx(*ok, M, 0, K, None) == 0   # nothing to compute
    assert mx(*ok, M, N, K, None) == INVALID                     # no output
    assert mx(*ok, M, N, K, y + 8) == INVALID                    # output not 16-byte aligned
    assert mx(None, a * 2, a * 3, a * 4, M, N, K, y) == INVALID  # no A codes
    assert mx(a, a * 2, a * 3, None, M, N, K, y) == INVALID      # no B scales
    assert mx(a + 8, a * 2, a * 3, a * 4, M, N, K, y) == INVALID # codes not 16-byte aligned
    assert mx(a, a * 2 + 4, a * 3, a * 4, M, N, K, y) == INVALID # scale atoms not 16-byte aligned
    assert mx(*ok, M, N, K, a + nca - 16) == INVALID             # output overlaps A's codes
    assert L.mxq_last_cuda_error().startswith(b"invalid argument")

    okn = (a, a * 2, a * 5, a * 3, a * 4, a * 6)
    assert nv(*okn, M, N, 40, y) == INVALID                      # K not a multiple of 32
    assert nv(a, a * 2, None, a * 3, a * 4, a * 6, M, N, K, y) == INVALID       # no A tensor scale
    assert nv(a, a * 2, a * 5, a * 3, a * 4, a * 6 + 2, M, N, K, y) == INVALID  # tensor scale not 4-byte aligned
    assert nv(*okn, M, N, K, a * 5) == INVALID                   # output overlaps a tensor scale
    assert nv(*okn, 0, N, K, None) == 0

    for lay in (L.mxq_scales_to_mma_layout, L.mxq_nvfp4_scales_to_mma_layout):
        assert lay(P(a), -1, 64, P(a * 2), None) == INVALID     # negative rows
        assert lay(P(a), 4, 48, P(a * 2), None) == INVALID      # K not a multiple of 32
        assert lay(P(a), 0, 64, None, None) == 0                 # nothing to lay out
        assert lay(None, 4, 64, P(a * 2), None) == INVALID      # no input
        assert lay(P(a), 4, 64, P(a * 2 + 8), None) == INVALID  # output not 16-byte aligned
        assert lay(P(a), 4, 64, P(a - 16), None) == INVALID     # output overlaps the scales
        assert L.mxq_last_cuda_error().startswith(b"invalid argument")


def test_quant_error_and_weight_side_reject_bad_arguments(L):
    """The error metric and the weights' quantiser: the host-side checks, and the
    workspace size the error metric asks for (one double per partial sum)."""
    a = 0x100000
    # one partial sum per 512 groups and lane quarter without Lambda; per 128 x 64 tile and
    # lane quarter with it
    assert L.mxq_quant_error_workspace_bytes(4, 64, 0) == 4 * 8
    assert L.mxq_quant_error_workspace_bytes(300, 4096, 0) == 75 * 4 * 8
    assert L.mxq_quant_error_workspace_bytes(300, 4096, 1) == 3 * 64 * 4 * 8
    assert L.mxq_quant_error_workspace_bytes(0, 64, 0) == 0 and L.mxq_quant_error_workspace_bytes(4, 48, 1) == 0

    def qe(x, rows, cols, r, lam, err, mean, ws, wsb):
        return L.mxq_quant_error(P(x), rows, cols, P(r), P(lam), P(err), P(mean), P(ws), wsb, None)

    ws, wsb = a * 9, 1 << 20
    assert qe(a, 4, 48, a * 5, None, None, a * 3, ws, wsb) == INVALID           # cols not a multiple of 32
    assert qe(a, 4, 64, a * 5, None, None, None, ws, wsb) == INVALID            # no mean
    assert qe(a, 4, 64, a * 5, None, None, a * 3 + 4, ws, wsb) == INVALID       # mean not 8-byte aligned
    assert qe(a, 0, 64, a * 5, None, None, a * 3, ws, wsb) == INVALID           # the mean of nothing
    assert qe(None, 4, 64, a * 5, None, None, a * 3, ws, wsb) == INVALID        # no X
    assert qe(a + 8, 4, 64, a * 5, None, None, a * 3, ws, wsb) == INVALID       # X not 16-byte aligned
    assert qe(a, 4, 64, a * 5, None, a * 2 + 2, a * 3, ws, wsb) == INVALID      # errors not 4-byte aligned
    assert qe(a, 4, 64, a * 5, None, None, a * 3, None, wsb) == INVALID         # no workspace
    assert qe(a, 4, 64, a * 5, None, None, a * 3, ws, 31) == INVALID            # workspace too small
    assert qe(a, 4, 64, a * 5, None, None, a * 3, ws + 4, wsb) == INVALID       # workspace not 8-byte aligned
    assert qe(a, 4, 64, a * 5, None, None, a + 64, ws, wsb) == INVALID          # mean inside X
    assert qe(a, 4, 64, a * 5, None, None, a * 3, a * 3, wsb) == INVALID        # workspace holds the mean
    assert L.mxq_last_cuda_error().startswith(b"invalid argument")

    def wq(w, rows, cols, r, lam, codes, scales):
        return L.mxq_weight_rotate_quantize(P(w), rows, cols, P(r), P(lam), P(codes), P(scales), None)

    assert wq(a, 4, 48, a * 5, None, a * 2, a * 3) == INVALID                   # cols not a multiple of 32
    assert wq(a, 4, 64, a * 5, a * 7 + 2, a * 2, a * 3) == INVALID              # Lambda not 4-byte aligned
    assert wq(a, 4, 64, a * 5, None, a + 16, a * 3) == INVALID                  # codes overlap W
    assert wq(a, 0, 64, a * 5, None, a * 2, a * 3) == 0                         # nothing to do


def test_noalloc_refuses_one_past_either_limit_before_any_cuda_call(L):
    """mxq_quant_error_noalloc's fixed array holds 131072 partial sums.  Without Lambda one sum
    covers 128 groups (four per 512-group stage), so 16,777,217 groups is one group too many.
    With Lambda one sum covers a warp's 32 rows of a 128 x 64 tile, four per tile, so 32,769
    tiles is one too many, even when the elements would fit: 129 rows round up to two row
    tiles.  Both are refused from the sizes alone, so no device is needed."""
    a = 0x100000
    assert L.mxq_quant_error_workspace_bytes(1, 16777216 * 32, 0) == 131072 * 8
    assert L.mxq_quant_error_workspace_bytes(1, 16777217 * 32, 0) > 131072 * 8
    st = L.mxq_quant_error_noalloc(P(a), 1, 16777217 * 32, P(a), None, None, P(a), None)
    assert st == INVALID and b"scratch" in L.mxq_last_cuda_error()
    cols = 16385 * 64 - 32   # rounds up to 16385 column tiles; 2 row tiles -> 32,770 tiles
    assert 129 * cols < 16777216 * 16   # fewer elements than the with-Lambda bound
    assert L.mxq_quant_error_workspace_bytes(129, cols, 1) > 131072 * 8
    st = L.mxq_quant_error_noalloc(P(a), 129, cols, P(a), P(a), None, P(a), None)
    assert st == INVALID and b"scratch" in L.mxq_last_cuda_error()
