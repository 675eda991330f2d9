"""The C-ABI library loads, exports every entry point that include/mxq.h declares, and
rejects bad arguments on the host with the documented status -- before any launch, so
these checks need no GPU (no call here reaches a kernel)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxq.h")


@pytest.fixture(scope="module")
def mxq():
    from block_scaled_weight_b200.build import build
    build()
    from block_scaled_weight_b200 import mxq as m
    return m


def declared_symbols():
    return re.findall(r"^MXQ_API [^(]*?\b(mxq_\w+)\(", open(HEADER).read(), re.M)


def test_library_exports_every_declared_symbol(mxq):
    decl = declared_symbols()
    assert len(decl) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", mxq.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (mxq_\w+)", out))
    assert set(decl) <= exported, set(decl) - exported
    assert set(decl) == set(mxq.EXPORTS)
    lib = ctypes.CDLL(mxq.lib_path())
    for name in decl:
        assert getattr(lib, name) is not None


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "mxq.h"\nint main(void){mxq_params p={0};(void)p;'
                   'return (int)mxq_status_string(MXQ_OK)[0] == 0;}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I",
                    os.path.join(ROOT, "include"), str(src)], check=True)


def test_status_strings_and_metrics(mxq):
    lib = mxq._lib
    for code in range(8):
        assert lib.mxq_status_string(code)
    m = mxq.mxq_metrics_from_sums([4.0, 16.0, 1.0, 4.0])
    assert m["weight_rel"] == 0.5 and m["h_rel"] == 0.5 and m["sse"] == 4.0


def test_workspace_queries(mxq):
    assert mxq.mxq_act_sqmean_workspace(0, 100) == 0
    assert mxq.mxq_act_sqmean_workspace(244449, 9728) % (9728 * 8) == 0
    assert mxq.mxq_act_sqmean_workspace(244449, 9728) > 0
    assert mxq.mxq_error_workspace(2560, 9728) > 0


FAKE = 0x10000          # 16-byte aligned, never dereferenced: every call below is rejected
ODD = 0x10004           # 4-byte but not 16-byte aligned


def q(mxq, W=FAKE, dt=1, n=64, k=256, ld=256, h=FAKE, codes=FAKE, scales=FAKE, **pk):
    p = mxq.params(**pk) if pk else mxq.params("nvfp4", "sse", 16)
    return mxq._lib.mxq_quantize(W, dt, n, k, ld, h, ctypes.byref(p), codes, scales, None)


def test_quantize_rejections(mxq):
    S = {v: k for k, v in mxq.STATUS.items()}
    assert q(mxq, W=None) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, dt=7) == S["MXQ_ERR_DTYPE"]
    assert q(mxq, n=-1) == S["MXQ_ERR_SHAPE"]
    assert q(mxq, k=250, ld=256) == S["MXQ_ERR_SHAPE"]            # k % 16
    assert q(mxq, ld=200) == S["MXQ_ERR_SHAPE"]                   # ld < k
    assert q(mxq, W=ODD) == S["MXQ_ERR_ALIGN"]
    assert q(mxq, ld=260) == S["MXQ_ERR_ALIGN"]                   # 520 bytes
    assert q(mxq, codes=ODD) == S["MXQ_ERR_ALIGN"]
    assert q(mxq, codes=None) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, fmt="nvfp4", mode="hopt", block=16, h=None) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, fmt="nvfp4", mode="hopt", block=16, h=ODD) == S["MXQ_ERR_ALIGN"]
    assert q(mxq, fmt="nvfp4", mode="sse", block=64) == S["MXQ_ERR_UNSUPPORTED"]
    assert q(mxq, fmt="int8", mode="sse", block=16) == S["MXQ_ERR_UNSUPPORTED"]
    assert q(mxq, fmt="e4m3", mode="hopt", block=32) == S["MXQ_ERR_UNSUPPORTED"]
    assert q(mxq, fmt="e4m3", mode="hopt", block=64, n=96) == S["MXQ_ERR_SHAPE"]
    assert q(mxq, fmt="e4m3", mode="hopt", block=64, log_points=1) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, fmt="e4m3", mode="hopt", block=64, log_lo_exp2=3.0) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, fmt="nvfp4", mode="sse", block=16, window=-2) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, fmt="nvfp4", mode="sse", block=16, ctas_per_sm=-1) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, fmt="int4", mode="sse", block=64) == S["MXQ_ERR_UNSUPPORTED"]
    assert q(mxq, fmt="int4", mode="sse", block=16, scale_fmt="ue8m0") == S["MXQ_ERR_UNSUPPORTED"]
    assert q(mxq, fmt="nvfp4", mode="sse", block=16, scale_fmt=7) == S["MXQ_ERR_INVALID_ARG"]
    assert q(mxq, fmt="int8", mode="sse", block=32, scale_fmt="ue4m4") == S["MXQ_ERR_UNSUPPORTED"]
    assert q(mxq, fmt="e4m3", mode="sse", block=64, scale_fmt="ue5m3") == S["MXQ_ERR_UNSUPPORTED"]
    p = mxq.params("nvfp4", "sse", 16)
    p.mode = 9
    assert mxq._lib.mxq_quantize(FAKE, 1, 64, 256, 256, FAKE, ctypes.byref(p), FAKE, FAKE,
                                 None) == S["MXQ_ERR_INVALID_ARG"]
    assert mxq._lib.mxq_quantize(FAKE, 1, 64, 256, 256, FAKE, None, FAKE, FAKE,
                                 None) == S["MXQ_ERR_INVALID_ARG"]
    assert b"params" in mxq._lib.mxq_last_error()


def test_empty_problems_are_no_ops(mxq):
    p = mxq.params("nvfp4", "hopt", 16)
    assert mxq._lib.mxq_quantize(None, 1, 0, 256, 256, None, ctypes.byref(p), None, None,
                                 None) == 0
    assert mxq._lib.mxq_quantize(None, 1, 64, 0, 0, None, ctypes.byref(p), None, None,
                                 None) == 0
    assert mxq._lib.mxq_dequant(None, None, ctypes.byref(p), 0, 256, None, None) == 0


def test_act_sqmean_rejections(mxq):
    S = {v: k for k, v in mxq.STATUS.items()}
    f = mxq._lib.mxq_act_sqmean
    need = mxq.mxq_act_sqmean_workspace(1000, 256)
    assert f(None, 1, 1000, 256, 256, FAKE, FAKE, need, None) == S["MXQ_ERR_INVALID_ARG"]
    assert f(FAKE, 1, 1000, 252, 256, FAKE, FAKE, need, None) == S["MXQ_ERR_SHAPE"]  # cols % 8
    assert f(FAKE, 0, 1000, 254, 256, FAKE, FAKE, need, None) == S["MXQ_ERR_SHAPE"]  # cols % 4
    assert f(FAKE, 1, 1000, 256, 256, FAKE, FAKE, need - 8, None) == S["MXQ_ERR_WORKSPACE"]
    assert f(FAKE, 1, 1000, 256, 256, FAKE, None, need, None) == S["MXQ_ERR_WORKSPACE"]
    assert f(FAKE, 1, 1000, 256, 256, None, FAKE, need, None) == S["MXQ_ERR_INVALID_ARG"]
    assert f(FAKE, 3, 1000, 256, 256, FAKE, FAKE, need, None) == S["MXQ_ERR_DTYPE"]
    assert f(FAKE + 8, 1, 1000, 256, 256, FAKE, FAKE, need, None) == S["MXQ_ERR_ALIGN"]
    assert f(FAKE, 1, 1000, 256, 256, FAKE, FAKE + 4, need, None) == S["MXQ_ERR_ALIGN"]
    assert f(FAKE, 1, 0, 0, 0, None, None, 0, None) == 0                # empty
    g = mxq._lib.mxq_act_sqmean_finalize
    assert g(FAKE, -1, 8, 8, FAKE, None) == S["MXQ_ERR_SHAPE"]
    assert g(None, 2, 8, 8, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]


def test_project_and_error_rejections(mxq):
    S = {v: k for k, v in mxq.STATUS.items()}
    pr = mxq._lib.mxq_project
    assert pr(FAKE, 16, 0, 0, 0.3, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]  # not an E4M3 value
    assert pr(FAKE, 16, 0, 0, 500.0, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert pr(FAKE, 16, 2, 0, -1.0, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert pr(FAKE, 16, 5, 0, 1.0, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert pr(FAKE + 2, 16, 0, 0, 1.0, FAKE, None) == S["MXQ_ERR_ALIGN"]
    assert pr(FAKE, 16, 0, 3, 3.0, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]  # not a power of 2
    assert pr(FAKE, 16, 0, 1, 0.1, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]  # not a UE4M4 value
    assert pr(FAKE, 16, 0, 2, 122880.0 * 2, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert pr(FAKE, 16, 3, 9, 1.0, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]  # unknown grid
    assert pr(FAKE, 16, 1, 1, 1.0, FAKE, None) == S["MXQ_ERR_UNSUPPORTED"]  # INT8 on UE4M4
    assert pr(FAKE, 0, 0, 3, 2.0 ** -127, FAKE, None) == 0               # empty: no launch
    p = mxq.params("nvfp4", "sse", 16)
    e = mxq._lib.mxq_error
    need = mxq.mxq_error_workspace(64, 256)
    assert e(FAKE, 1, 64, 256, 256, FAKE, FAKE, None, ctypes.byref(p), None, FAKE, need,
             None) == S["MXQ_ERR_INVALID_ARG"]
    assert e(FAKE, 1, 64, 256, 256, FAKE, FAKE, None, ctypes.byref(p), FAKE, FAKE, need - 1,
             None) == S["MXQ_ERR_WORKSPACE"]
    assert e(FAKE, 1, 64, 256, 256, ODD, FAKE, None, ctypes.byref(p), FAKE, FAKE, need,
             None) == S["MXQ_ERR_ALIGN"]


def test_gptq_rejections(mxq):
    S = {v: k for k, v in mxq.STATUS.items()}
    L = mxq._lib
    # 64 x 64 E4M3 tiles
    tiles = L.mxq_gptq_tiles
    assert tiles(FAKE, 1, 64, 96, 96, FAKE, FAKE, FAKE, None) == S["MXQ_ERR_SHAPE"]     # k % 64
    assert tiles(FAKE, 1, 100, 128, 128, FAKE, FAKE, FAKE, None) == S["MXQ_ERR_SHAPE"]  # n % 64
    assert tiles(FAKE, 5, 64, 128, 128, FAKE, FAKE, FAKE, None) == S["MXQ_ERR_DTYPE"]
    assert tiles(FAKE, 1, 64, 128, 128, None, FAKE, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert tiles(FAKE, 1, 64, 128, 128, ODD, FAKE, FAKE, None) == S["MXQ_ERR_ALIGN"]
    assert tiles(FAKE, 1, 64, 128, 128, FAKE, FAKE + 2, FAKE, None) == S["MXQ_ERR_ALIGN"]
    prep = L.mxq_gptq_prepare
    assert prep(FAKE, -1, 0.01, FAKE, None) == S["MXQ_ERR_SHAPE"]
    assert prep(FAKE, 2, float("nan"), FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert prep(FAKE, 2, -0.1, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert prep(None, 2, 0.01, FAKE, None) == S["MXQ_ERR_INVALID_ARG"]
    assert prep(FAKE, 2, 0.01, ODD, None) == S["MXQ_ERR_ALIGN"]
    assert prep(None, 0, 0.01, None, None) == 0                                        # empty
    # Hessian, factor, order, sweep
    gram = L.mxq_act_gram
    gws = mxq.mxq_act_gram_workspace(100, 64)
    assert gws >= 256 and mxq.mxq_act_gram_workspace(0, 64) == 0
    assert gram(FAKE, 0, 100, 64, 64, FAKE, FAKE, gws, None) == S["MXQ_ERR_DTYPE"]      # float32 X
    assert gram(FAKE, 1, 100, 64, 64, None, FAKE, gws, None) == S["MXQ_ERR_INVALID_ARG"]
    assert gram(FAKE, 1, 100, 64, 64, ODD, FAKE, gws, None) == S["MXQ_ERR_ALIGN"]
    assert gram(FAKE, 1, 100, 64, 64, FAKE, None, gws, None) == S["MXQ_ERR_WORKSPACE"]
    assert gram(FAKE, 1, 100, 64, 64, FAKE, FAKE, gws - 8, None) == S["MXQ_ERR_WORKSPACE"]
    assert gram(FAKE, 1, 100, 64, 64, FAKE, FAKE + 8, gws, None) == S["MXQ_ERR_ALIGN"]
    assert gram(None, 1, 100, 0, 0, None, None, 0, None) == 0                          # no columns
    mm = L.mxq_nvfp4_gemm
    mws = mxq.mxq_nvfp4_gemm_workspace() if hasattr(mxq, "mxq_nvfp4_gemm_workspace") else \
        L.mxq_nvfp4_gemm_workspace()
    assert mm(FAKE, FAKE, FAKE, FAKE, 128, 128, 96, FAKE, FAKE, mws, None) == S["MXQ_ERR_SHAPE"]
    assert mm(FAKE, FAKE, FAKE, FAKE, -1, 128, 64, FAKE, FAKE, mws, None) == S["MXQ_ERR_SHAPE"]
    assert mm(FAKE, FAKE, FAKE, FAKE, 128, 128, 64, None, FAKE, mws, None) == S["MXQ_ERR_INVALID_ARG"]
    assert mm(None, FAKE, FAKE, FAKE, 128, 128, 64, FAKE, FAKE, mws, None) == S["MXQ_ERR_INVALID_ARG"]
    assert mm(FAKE + 8, FAKE, FAKE, FAKE, 128, 128, 64, FAKE, FAKE, mws, None) == S["MXQ_ERR_ALIGN"]
    assert mm(FAKE, FAKE, FAKE, FAKE + 4, 128, 128, 64, FAKE, FAKE, mws, None) == S["MXQ_ERR_ALIGN"]
    assert mm(FAKE, FAKE, FAKE, FAKE, 128, 128, 64, FAKE, None, mws, None) == S["MXQ_ERR_WORKSPACE"]
    assert mm(FAKE, FAKE, FAKE, FAKE, 128, 128, 64, FAKE, FAKE, mws - 8, None) == S["MXQ_ERR_WORKSPACE"]
    assert mm(None, None, None, None, 0, 128, 64, None, None, 0, None) == 0            # empty
    fac = L.mxq_gptq_factor
    need = mxq.mxq_gptq_factor_workspace(256)
    assert need == 256 + 2 * 256 * 256 * 8
    assert fac(FAKE, 256, 64, None, 0.01, FAKE, FAKE, need, None) == S["MXQ_ERR_UNSUPPORTED"]
    assert fac(FAKE, 250, 16, None, 0.01, FAKE, FAKE, need, None) == S["MXQ_ERR_SHAPE"]
    assert fac(FAKE, 256, 16, None, float("inf"), FAKE, FAKE, need, None) == S["MXQ_ERR_INVALID_ARG"]
    assert fac(FAKE, 256, 16, None, 0.01, FAKE, None, need, None) == S["MXQ_ERR_WORKSPACE"]
    assert fac(FAKE, 256, 16, None, 0.01, FAKE, FAKE, need - 8, None) == S["MXQ_ERR_WORKSPACE"]
    assert fac(ODD, 256, 16, None, 0.01, FAKE, FAKE, need, None) == S["MXQ_ERR_ALIGN"]
    assert fac(FAKE, 256, 16, FAKE + 2, 0.01, FAKE, FAKE, need, None) == S["MXQ_ERR_ALIGN"]
    assert fac(FAKE, 65552, 16, None, 0.01, FAKE, FAKE, need, None) == S["MXQ_ERR_SHAPE"]
    assert fac(None, 0, 16, None, 0.01, None, None, 0, None) == 0                       # empty
    p4 = mxq.params("nvfp4", "hopt", 16)
    p8 = mxq.params("int8", "hopt", 32)
    order = L.mxq_gptq_order
    ows = mxq.mxq_gptq_order_workspace(64, 256, p4)
    assert order(FAKE, 1, 64, 256, 256, FAKE, ctypes.byref(p8), FAKE, FAKE, ows,
                 None) == S["MXQ_ERR_UNSUPPORTED"]
    assert order(FAKE, 1, 64, 256, 256, None, ctypes.byref(p4), FAKE, FAKE, ows,
                 None) == S["MXQ_ERR_INVALID_ARG"]
    assert order(FAKE, 1, 64, 256, 256, FAKE, ctypes.byref(p4), None, FAKE, ows,
                 None) == S["MXQ_ERR_INVALID_ARG"]
    assert order(FAKE, 1, 64, 16 * 2049, 16 * 2049, FAKE, ctypes.byref(p4), FAKE, FAKE, ows,
                 None) == S["MXQ_ERR_SHAPE"]                                            # > 2048 blocks
    assert order(FAKE, 1, 64, 256, 256, FAKE, ctypes.byref(p4), FAKE, FAKE, ows - 8,
                 None) == S["MXQ_ERR_WORKSPACE"]
    sweep = L.mxq_gptq
    sws = mxq.mxq_gptq_workspace(64, 256)
    assert sws == 64 * 256 * 4 + 2 * 64 * 64 * 4 + 256
    pe = mxq.params("e4m3", "hopt", 64)
    assert sweep(FAKE, 1, 64, 256, 256, FAKE, FAKE, None, ctypes.byref(pe), FAKE, FAKE, FAKE,
                 sws, None) == S["MXQ_ERR_UNSUPPORTED"]
    assert sweep(FAKE, 1, 64, 256, 256, FAKE, None, None, ctypes.byref(p4), FAKE, FAKE, FAKE,
                 sws, None) == S["MXQ_ERR_INVALID_ARG"]
    assert sweep(FAKE, 1, 64, 256, 256, None, FAKE, None, ctypes.byref(p4), FAKE, FAKE, FAKE,
                 sws, None) == S["MXQ_ERR_INVALID_ARG"]                                 # hopt, no h
    assert sweep(FAKE, 1, 64, 256, 256, FAKE, FAKE, None, ctypes.byref(p4), FAKE, FAKE, FAKE,
                 sws - 8, None) == S["MXQ_ERR_WORKSPACE"]
    assert sweep(FAKE, 1, 65535 * 64 + 64, 256, 256, FAKE, FAKE, None, ctypes.byref(p4), FAKE,
                 FAKE, FAKE, sws, None) == S["MXQ_ERR_SHAPE"]
    assert sweep(None, 1, 0, 256, 256, None, None, None, ctypes.byref(p4), None, None, None, 0,
                 None) == 0                                                              # empty
