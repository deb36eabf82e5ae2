"""Host-side checks of the C-ABI library (no GPU needed, no kernel launched).

The library must load, export every entry point that include/*.h declares,
and reject bad arguments synchronously, before touching the device.  Only
argument checks that return before any CUDA call are exercised here.
"""
import glob
import os
import re

import pytest

from xlstm_mlstm_matrix_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(path).read()
        names.update(re.findall(r"XLSTM_API\s+[\w\s\*]*?\b(xlstm_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(capi.LIB_PATH):
        from xlstm_mlstm_matrix_b200 import build
        build.build()
    return capi.load()


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 7, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(capi.EXPORTED) <= set(names)


def test_version_and_status_strings(lib):
    assert "sm_100a" in capi.xlstm_mlstm_version()
    assert capi.xlstm_status_string(capi.XLSTM_OK) == "ok"
    assert "timed out" in capi.xlstm_status_string(capi.XLSTM_ERR_TIMEOUT)


def test_workspace_size(lib):
    d = capi.make_desc(8, 8, 4096, 256, 512)
    assert capi.xlstm_mlstm_workspace_size(d) >= 256


def _seg_bytes(BH, G, dqk, dv):
    """Scratch of G segments: (G-1) summaries per sequence, each region 256-aligned."""
    a = lambda x: (x + 255) // 256 * 256
    n = (G - 1) * BH
    off_m = a(n * 16)
    off_n = a(off_m + n * 4)
    off_c = a(off_n + n * dqk * 4)
    return a(off_c + n * dv * dqk * 4)


def test_parallel_workspace_size(lib):
    base = capi.xlstm_mlstm_workspace_size
    par = capi.xlstm_mlstm_workspace_size_parallel
    # long-context layer: 8 sequences of 1024 chunks on 148 SMs -> 18 segments of 57 chunks
    d = capi.make_desc(1, 8, 65536, 128, 128, capi.XLSTM_BF16, 128 ** -0.5, 64)
    assert par(d) == base(d) + _seg_bytes(8, 18, 128, 128)
    # 2 heads x 4 value slices, 18 chunks: 2 segments of 9 chunks
    d = capi.make_desc(1, 2, 1100, 256, 512, capi.XLSTM_BF16, 1.0, 64)
    assert par(d) == base(d) + _seg_bytes(2, 2, 256, 512)
    # no segments: enough heads to fill the GPU, too short, fp32, another chunk length
    for B, H, T, dqk, dv, dt, L in [(8, 8, 4096, 256, 512, capi.XLSTM_BF16, 64),
                                    (256, 4, 512, 64, 64, capi.XLSTM_BF16, 64),
                                    (1, 1, 64 * 15, 128, 128, capi.XLSTM_BF16, 64),
                                    (1, 8, 65536, 128, 128, capi.XLSTM_F32, 64),
                                    (1, 8, 65536, 128, 128, capi.XLSTM_BF16, 32),
                                    (1, 8, 65536, 96, 128, capi.XLSTM_BF16, 64)]:
        d = capi.make_desc(B, H, T, dqk, dv, dt, 1.0, L)
        assert par(d) == base(d), (B, H, T, dqk, dv, dt, L)
    assert lib.xlstm_mlstm_workspace_size_parallel(None) == 0
    # 74 sequences on 148 SMs allow two segments each, of 2000 chunks: the 1024-chunk
    # cap on a segment makes it four segments of 1000
    d = capi.make_desc(1, 74, 64 * 4000, 64, 128, capi.XLSTM_BF16, 1.0, 64)
    assert par(d) == base(d) + _seg_bytes(74, 4, 64, 128)


FAKE = dict(q=0x10000, k=0x20000, v=0x30000, i=0x40000, f=0x50000, h=0x60000, ws=0x100000)


def call(desc, **over):
    a = dict(FAKE, **over)
    return capi.xlstm_mlstm_fwd_chunkwise(desc, a["q"], a["k"], a["v"], a["i"], a["f"],
                                          a.get("C0"), a.get("n0"), a.get("m0"), a["h"],
                                          a.get("C1"), a.get("n1"), a.get("m1"), a["ws"],
                                          a.get("wsb", 256))


@pytest.mark.parametrize("field,value", [("B", 0), ("H", -1), ("T", -1), ("d_qk", 8), ("d_qk", 520),
                                         ("d_v", 24), ("d_v", 0), ("qkv_dtype", 7)])
def test_bad_dims_rejected(lib, field, value):
    d = capi.make_desc(1, 1, 4, 32, 32)
    setattr(d, field, value)
    assert call(d) == capi.XLSTM_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected(lib):
    d = capi.make_desc(1, 1, 4, 32, 32)
    assert call(d, q=None) == capi.XLSTM_ERR_INVALID_ARG
    assert call(d, h=None) == capi.XLSTM_ERR_INVALID_ARG
    assert call(d, k=FAKE["k"] + 4) == capi.XLSTM_ERR_INVALID_ARG
    assert call(d, ws=FAKE["ws"] + 16) == capi.XLSTM_ERR_INVALID_ARG
    # partial state: all three or none
    assert call(d, C0=0x70000) == capi.XLSTM_ERR_INVALID_ARG


def test_overlaps_rejected(lib):
    d = capi.make_desc(1, 1, 4, 32, 32)
    assert call(d, h=FAKE["q"]) == capi.XLSTM_ERR_INVALID_ARG          # out over an input
    assert call(d, C1=FAKE["h"] + 64) == capi.XLSTM_ERR_INVALID_ARG    # two outputs overlap


def test_workspace_and_chunk_rules(lib):
    d = capi.make_desc(1, 1, 4, 32, 32)
    assert call(d, ws=None) == capi.XLSTM_ERR_WORKSPACE
    assert call(d, wsb=8) == capi.XLSTM_ERR_WORKSPACE
    d.chunk = 48
    assert call(d) == capi.XLSTM_ERR_UNSUPPORTED
    # bf16 inputs run on the tensor-core kernel, whose chunk is 64, or 128 at d_qk <= 128:
    # other lengths are refused (before any device call), never sent to another kernel
    for dqk, L in ((64, 16), (64, 32), (64, 256), (128, 256), (256, 128), (256, 32)):
        d = capi.make_desc(1, 1, 4, dqk, 64, capi.XLSTM_BF16, 1.0, L)
        assert call(d) == capi.XLSTM_ERR_UNSUPPORTED, (dqk, L)
        assert capi.xlstm_mlstm_chunkwise_kernel(d) == "none", (dqk, L)
    # L = 128 needs a shape the tensor-core kernel takes (d_v a multiple of 64)
    assert capi.xlstm_mlstm_chunkwise_kernel(capi.make_desc(1, 1, 4, 64, 32, capi.XLSTM_BF16, 1.0, 128)) == "none"
    for dqk, L in ((64, 0), (64, 64), (256, 64), (64, 128), (128, 128)):
        # "tcgen05" on a GPU (the driver's tensor-map encoder); not "none" anywhere
        d = capi.make_desc(1, 1, 4, dqk, 64, capi.XLSTM_BF16, 1.0, L)
        assert capi.xlstm_mlstm_chunkwise_kernel(d) != "none", (dqk, L)
    # fp32 inputs: the CUDA-core kernel takes 16, 32, 64 and 128
    for L in (16, 32, 64, 128):
        assert capi.xlstm_mlstm_chunkwise_kernel(capi.make_desc(1, 1, 4, 64, 64, capi.XLSTM_F32, 1.0, L)) == "simt"
    for L in (48, 256):
        d = capi.make_desc(1, 1, 4, 64, 64, capi.XLSTM_F32, 1.0, L)
        assert call(d) == capi.XLSTM_ERR_UNSUPPORTED, L


def test_output_stage_arguments_checked(lib):
    """xlstm_mlstm_fwd_chunkwise_out: bad dtypes, a misaligned o_pre and an o_pre
    that overlaps h are refused before any device work; NULL out is the plain call."""
    d = capi.make_desc(2, 2, 64, 64, 64, capi.XLSTM_BF16, 1.0, 64)
    a = dict(FAKE)
    h_bytes16 = 2 * 2 * 64 * 64 * 2

    def call_out(o, odt, hdt, h=a["h"]):
        out = capi.xlstm_mlstm_output_t(o, odt, hdt)
        return capi.xlstm_mlstm_fwd_chunkwise_out(d, out, a["q"], a["k"], a["v"], a["i"], a["f"], None, None, None,
                                                  h, None, None, None, a["ws"], 256)
    assert call_out(0x70000, capi.XLSTM_BF16, 7) == capi.XLSTM_ERR_INVALID_ARG
    assert call_out(0x70000, 9, capi.XLSTM_F32) == capi.XLSTM_ERR_INVALID_ARG
    assert call_out(0x70002, capi.XLSTM_BF16, capi.XLSTM_F32) == capi.XLSTM_ERR_INVALID_ARG
    # o_pre inside h (bf16 h: h_bytes16 bytes from 0x60000)
    assert call_out(0x60000 + h_bytes16 - 16, capi.XLSTM_BF16, capi.XLSTM_BF16) == capi.XLSTM_ERR_INVALID_ARG
    # the same o_pre just past a bf16 h is fine as far as overlap goes; it fails later only on the
    # (fake) workspace, which the argument checks do not reach: use a too-small workspace instead
    out = capi.xlstm_mlstm_output_t(0x60000 + h_bytes16, capi.XLSTM_BF16, capi.XLSTM_BF16)
    assert capi.xlstm_mlstm_fwd_chunkwise_out(d, out, a["q"], a["k"], a["v"], a["i"], a["f"], None, None, None,
                                              a["h"], None, None, None, a["ws"], 16) == capi.XLSTM_ERR_WORKSPACE
    # NULL out: the plain call's checks
    assert capi.xlstm_mlstm_fwd_chunkwise_out(d, None, a["q"], a["k"], a["v"], a["i"], a["f"], None, None, None,
                                              None, None, None, None, a["ws"], 256) == capi.XLSTM_ERR_INVALID_ARG


def test_step_rejects_partial_in_place(lib):
    d = capi.make_desc(2, 2, 1, 32, 32)
    C, n, m = 0x70000, 0x80000, 0x90000
    # C_new overlapping C without being identical
    st = capi.xlstm_mlstm_step(d, FAKE["q"], FAKE["k"], FAKE["v"], FAKE["i"], FAKE["f"],
                               C, n, m, FAKE["h"], C + 256, 0xA0000, 0xB0000)
    assert st == capi.XLSTM_ERR_INVALID_ARG
    st = capi.xlstm_mlstm_step(d, FAKE["q"], FAKE["k"], FAKE["v"], FAKE["i"], FAKE["f"],
                               C, n, m, None, C, n, m)
    assert st == capi.XLSTM_ERR_INVALID_ARG
