"""The GEMM schedules the library picks for the workloads' shapes, queried on
the host through frt_gemm_plan_info (148 SMs when no device is visible, the
B200's count).  These pin the choices the kernel notes describe: small-M
shapes swap operands and split K over a thread-block cluster; large shapes
run on CTA pairs with the widest tile that keeps the SMs busy; a long-K
shape with few tiles takes K in halves over two pairs; the gated epilogues
stay in the token-row orientation."""

import ctypes as C

import pytest


@pytest.fixture(scope="module")
def frt():
    from fp8_transformer_block_b200 import frt as f
    return f


@pytest.mark.parametrize("shape,want", [
    # action-expert q/k/v (50 tokens, N 2560, K 2048): 40 weight tiles x 3 splits
    ((50, 2560, 2048, 0), dict(swap=1, cluster=1, tile_rows=64, tile_cols=64, splits=3,
                               units=120, k_blocks=16)),
    # tiny / stack layer (K 512): 10 tiles x 2 splits of 2 K-blocks
    ((64, 640, 512, 0), dict(swap=1, cluster=1, tile_rows=64, splits=2, units=20)),
    ((1, 640, 512, 0), dict(swap=1, cluster=1, splits=2, units=20)),
    # more than 64 tokens: the token tile widens to 128
    ((128, 2560, 2048, 0), dict(swap=1, tile_cols=128, splits=3)),
    # video-DiT q/k/v: 256-wide pair tiles, 32 x 36 tiles over 148 CTAs
    ((8192, 9216, 3072, 0), dict(swap=0, pair=1, split2=0, tile_cols=256, units=1152,
                                 grid=148)),
    # gate/up with the GEGLU epilogue: pairs, 256-wide (gate and up together)
    ((1024, 32768, 2048, 1), dict(swap=0, pair=1, tile_cols=256, units=512)),
    # long K: the wide (256 x 512) pair tiles, whose single-buffered
    # accumulator exposes the epilogue, pay off
    ((2048, 4096, 8192, 0), dict(pair=1, split2=0, tile_cols=512, units=64)),
    ((2048, 8192, 8192, 1), dict(pair=1, tile_cols=512, units=128)),
    # less than a wave of wide tiles: 256-wide pairs keep more SMs busy
    ((1100, 2048, 512, 1), dict(pair=1, tile_cols=256, units=40)),
    ((256, 9216, 3072, 0), dict(pair=1, tile_cols=128, units=72)),
    # MLP down projection (K 16384, 32 tiles): K in halves over two pairs
    ((1024, 2048, 16384, 0), dict(pair=1, split2=1, tile_cols=256, units=32, grid=128,
                                  k_blocks=128)),
    # DiT FFN with the GELU epilogue, and its down projection (K 12288: wide)
    ((8192, 12288, 3072, 2), dict(pair=1, tile_cols=256, units=1536)),
    ((8192, 3072, 12288, 0), dict(pair=1, split2=0, tile_cols=512, units=192)),
    # 4096-row stack layer (N 640): 160-wide pair tiles, 16 x 4 tiles
    ((4096, 640, 512, 0), dict(pair=1, tile_cols=160, units=64)),
    # the gated epilogues never swap, even at 50 tokens
    ((50, 4096, 512, 1), dict(swap=0, pair=0, cluster=0)),
])
def test_plan(frt, shape, want):
    got = frt.frt_gemm_plan_info(*shape)
    for k, v in want.items():
        assert got[k] == v, f"{shape}: {k} = {got[k]}, expected {v}"
    # invariants of every plan: no more CTAs than the units need (a unit is
    # one CTA, one split of a cluster tile, a pair's tile on 2 CTAs, or a
    # K-halves tile on 4), at most one wave of pairs, one orientation
    per_unit = 4 if got["split2"] else 2 if got["pair"] else 1
    assert 1 <= got["grid"] <= per_unit * got["units"]
    if got["pair"]:
        assert got["grid"] <= 148 and got["grid"] % 2 == 0
    assert not (got["swap"] and got["pair"])
    assert got["splits"] >= 1 and (got["cluster"] or not got["swap"] or got["splits"] == 1)


def test_plan_info_argument_checks(frt):
    buf = (C.c_int * 4)()
    assert frt.raw_call("frt_gemm_plan_info", 50, 2560, 2048, 0, buf, 4) == frt.FRT_EINVAL
    buf = (C.c_int * frt.FRT_PLAN_INFO_LEN)()
    assert frt.raw_call("frt_gemm_plan_info", 50, 0, 2048, 0, buf,
                        frt.FRT_PLAN_INFO_LEN) == frt.FRT_ESHAPE
    assert frt.raw_call("frt_gemm_plan_info", 50, 2560, 2048, 7, buf,
                        frt.FRT_PLAN_INFO_LEN) == frt.FRT_EINVAL
    assert frt.raw_call("frt_gemm_plan_info", 0, 2560, 2048, 0, buf,
                        frt.FRT_PLAN_INFO_LEN) == frt.FRT_OK
    assert list(buf) == [0] * frt.FRT_PLAN_INFO_LEN  # no rows: nothing launched
