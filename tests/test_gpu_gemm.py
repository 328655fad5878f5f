"""GPU parity of the tcgen05 int8 GEMM against the CPU oracle.

* w8a8_gemm_i32: raw int32 accumulators, bit-exact to the oracle's exact
  int64 dot products (the paper's "bit-exact int32 accumulation", abstract);
* w8a8_gemm: fused dequant + bias epilogue, bf16 within 1 ulp of the
  oracle's binary32 epilogue rounded to bf16, no NaN.

Shapes cover ragged M / N / K tails, every tile configuration, few CTAs
(many tiles per persistent CTA), and the long-K workload with all-+-127
rows (|acc| = 12288 * 127^2)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.util import bf16_bits_to_torch, bf16_ulp_diff, is_nan_bits, row_chunks, torch_bf16_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w8():
    import w8a8_int8_gemm_b200 as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _codes(rng, rows, K):
    return rng.integers(-127, 128, (rows, K), dtype=np.int8)


def _i32(w8, xq, wq, config=None):
    acc = w8.w8a8_gemm_i32(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), config=config)
    torch.cuda.synchronize()
    return acc.cpu().numpy().astype(np.int64)


SHAPES = [(1, 8, 16), (63, 136, 48), (129, 264, 272), (64, 128, 256), (200, 520, 400), (257, 256, 1040),
          (384, 392, 144), (520, 776, 2064)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_i32_ragged_shapes(w8, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 13 + K)
    xq, wq = _codes(rng, M, K), _codes(rng, N, K)
    assert np.array_equal(_i32(w8, xq, wq), oracle.gemm_i64(xq, wq))


CONFIGS = [dict(block_m=bm, block_n=bn, stages=st, grid=g, raster_group=rg)
           for bm, bn, st in [(128, 256, 4), (128, 256, 2), (128, 128, 6), (128, 128, 3),
                              (256, 256, 6), (256, 256, 2), (256, 128, 8), (256, 128, 3)]
           for g, rg in [(148, 16), (4, 1), (2, 5)]]


def _cid(c):
    return f"m{c['block_m']}_n{c['block_n']}_st{c['stages']}_g{c['grid']}_r{c['raster_group']}"


@pytest.mark.parametrize("cfg", CONFIGS, ids=_cid)
def test_i32_every_config(w8, cfg):
    rng = np.random.default_rng(cfg["block_n"] + cfg["stages"] * 10 + cfg["grid"])
    M, N, K = 300, 776, 656
    xq, wq = _codes(rng, M, K), _codes(rng, N, K)
    assert np.array_equal(_i32(w8, xq, wq, config=cfg), oracle.gemm_i64(xq, wq))


# CTA pairs with K a multiple of 128 and at least 4 chunks of ring depth load
# boxes spanning two K-chunks; K = 128 (mod 256) leaves the second chunk of
# the last stage outside the tensor (filled with zeros).
PAIR_CHUNK_CASES = [((300, 776, 128), 6), ((300, 776, 384), 6), ((257, 520, 1024), 4), ((129, 264, 3072), 5),
                    ((520, 1032, 640), 8)]


@pytest.mark.parametrize("shape,stages", PAIR_CHUNK_CASES, ids=lambda v: str(v))
@pytest.mark.parametrize("bn", [256, 128])
def test_pair_double_chunk_stages(w8, shape, stages, bn):
    M, N, K = shape
    if stages > (6 if bn == 256 else 8):
        pytest.skip("ring deeper than shared memory holds for this tile")
    rng = np.random.default_rng(M + K + bn)
    xq, wq = _codes(rng, M, K), _codes(rng, N, K)
    for grid, rg in ((148, 8), (4, 1)):
        cfg = dict(block_m=256, block_n=bn, stages=stages, grid=grid, raster_group=rg)
        assert np.array_equal(_i32(w8, xq, wq, config=cfg), oracle.gemm_i64(xq, wq)), cfg
    got, want = _bf16_gemm_case(w8, M, N, K, M * 5 + K, True,
                                dict(block_m=256, block_n=bn, stages=stages, grid=148, raster_group=8))
    assert bf16_ulp_diff(got, want).max() <= 1


# CTA-pair grids with a short last round (256 x 256 tiles; its tiles run as
# 256 x 128 items): 8 tiles on 6 pairs, 15 tiles on 12 pairs, with single-
# (K % 128 != 0) and double-chunk stages.
PAIR_TAIL_CASES = [((300, 776, 656), 12, 6), ((300, 776, 1024), 12, 6), ((520, 1032, 640), 24, 6),
                   ((520, 1032, 640), 24, 4), ((520, 1032, 3072), 24, 5)]


@pytest.mark.parametrize("shape,grid,stages", PAIR_TAIL_CASES, ids=lambda v: str(v))
def test_pair_tail_halves(w8, shape, grid, stages):
    M, N, K = shape
    cfg = dict(block_m=256, block_n=256, stages=stages, grid=grid, raster_group=1)
    rng = np.random.default_rng(M + grid + K)
    xq, wq = _codes(rng, M, K), _codes(rng, N, K)
    assert np.array_equal(_i32(w8, xq, wq, config=cfg), oracle.gemm_i64(xq, wq))
    got, want = _bf16_gemm_case(w8, M, N, K, M * 7 + grid + K, True, cfg)
    assert bf16_ulp_diff(got, want).max() <= 1


# Grids that leave a short last round: its tiles are split into two half-width
# items (e.g. 12 tiles on 5 CTAs: 10 whole tiles, then 2 tiles as 4 halves).
TAIL_CASES = [((300, 776, 656), 5), ((300, 776, 656), 9), ((129, 520, 1040), 4), ((260, 1032, 272), 13)]


@pytest.mark.parametrize("shape,grid", TAIL_CASES, ids=lambda v: str(v))
def test_tail_halves_i32_and_bf16(w8, shape, grid):
    M, N, K = shape
    cfg = dict(block_m=128, block_n=256, stages=4, grid=grid, raster_group=1)
    rng = np.random.default_rng(M + grid)
    xq, wq = _codes(rng, M, K), _codes(rng, N, K)
    assert np.array_equal(_i32(w8, xq, wq, config=cfg), oracle.gemm_i64(xq, wq))
    got, want = _bf16_gemm_case(w8, M, N, K, M * 3 + grid, True, cfg)
    assert bf16_ulp_diff(got, want).max() <= 1


def test_i32_identity_and_extremes(w8):
    """Closed forms: identity weight gives 127 * xq; all +-127 rows at K = 12288."""
    rng = np.random.default_rng(1)
    K = 256
    xq = _codes(rng, 130, K)
    eye = (np.eye(K, dtype=np.int64) * 127).astype(np.int8)
    assert np.array_equal(_i32(w8, xq, eye), 127 * xq.astype(np.int64))
    K = 12288
    x = np.stack([np.full(K, 127, np.int8), np.full(K, -127, np.int8)])
    acc = _i32(w8, x, np.concatenate([x, x, x, x]))
    big = K * 127 * 127
    assert acc[0, 0] == big and acc[0, 1] == -big and acc[1, 0] == -big and acc[1, 1] == big


def test_long_k_workload_every_row(w8):
    """MLP down-projection 4096 x 3072 x 12288 with the all-+-127 rows, in
    the launch configuration the benchmark selects: the int32 accumulators
    of w8a8_gemm_i32 and the bf16 outputs of w8a8_gemm (dequantization +
    bias epilogue) against the oracle on every row (its exact GEMM in row
    chunks); the closed form K * 127^2 on the extreme rows."""
    wl = workloads.WORKLOADS["mlp_down_1024"]
    d = workloads.make(wl)
    dev = torch.device("cuda")
    xq, wq = torch.from_numpy(d["xq"]).to(dev), torch.from_numpy(d["wq"]).to(dev)
    acc = w8.w8a8_gemm_i32(xq, wq)
    out = w8.w8a8_gemm(xq, wq, torch.from_numpy(d["scale_a"]).to(dev), torch.from_numpy(d["scale_w"]).to(dev),
                       bf16_bits_to_torch(d["bias"], dev))
    torch.cuda.synchronize()
    assert w8.w8a8_read_device_error() == 0
    acc = acc.cpu().numpy()
    got = torch_bf16_to_bits(out)
    assert not is_nan_bits(got).any()
    big = wl.K * 127 * 127
    assert acc[0, 0] == big and acc[1, 0] == -big and acc[0, 1] == -big and acc[1, 1] == big
    for rows in row_chunks(wl.M):
        want = oracle.gemm_i64(d["xq"][rows], d["wq"])
        assert np.array_equal(acc[rows], want), f"accumulators differ in rows {rows}"
        bf = oracle.epilogue(want, d["scale_a"][rows], d["scale_w"], d["bias"])
        assert bf16_ulp_diff(got[rows], bf).max() <= 1, f"outputs differ in rows {rows}"


def test_i32_matches_torch_int_mm(w8):
    """The paper checks its accumulator against torch._int_mm; do the same
    where torch supports it on this device."""
    rng = np.random.default_rng(2)
    M, N, K = 256, 512, 768
    xq, wq = _codes(rng, M, K), _codes(rng, N, K)
    a = torch.from_numpy(xq).cuda()
    b = torch.from_numpy(wq).cuda()
    try:
        ref = torch._int_mm(a, b.t())
    except RuntimeError as e:  # not supported for this device / layout
        pytest.skip(f"torch._int_mm unavailable: {e}")
    torch.cuda.synchronize()
    assert torch.equal(w8.w8a8_gemm_i32(a, b), ref)


def _bf16_gemm_case(w8, M, N, K, seed, bias=True, config=None):
    rng = np.random.default_rng(seed)
    xq, wq = _codes(rng, M, K), _codes(rng, N, K)
    sa = np.exp(rng.uniform(np.log(1e-4), np.log(1e-1), M)).astype(np.float32)
    sw = np.exp(rng.uniform(np.log(1e-4), np.log(1e-1), N)).astype(np.float32)
    bias_bits = workloads.gen_bias(N, seed) if bias else None
    dev = torch.device("cuda")
    out = w8.w8a8_gemm_ex(torch.from_numpy(xq).to(dev), torch.from_numpy(wq).to(dev),
                          torch.from_numpy(sa).to(dev), torch.from_numpy(sw).to(dev),
                          bf16_bits_to_torch(bias_bits, dev) if bias else None, config=config)
    torch.cuda.synchronize()
    got = torch_bf16_to_bits(out)
    want = oracle.epilogue(oracle.gemm_i64(xq, wq), sa, sw, bias_bits)
    return got, want


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("bias", [True, False])
def test_bf16_epilogue(w8, M, N, K, bias):
    got, want = _bf16_gemm_case(w8, M, N, K, M + N + K, bias)
    assert not is_nan_bits(got).any()
    assert bf16_ulp_diff(got, want).max() <= 1


@pytest.mark.parametrize("cfg", CONFIGS[::3], ids=_cid)
def test_bf16_epilogue_configs(w8, cfg):
    got, want = _bf16_gemm_case(w8, 300, 776, 656, cfg["block_n"] + cfg["stages"], True, cfg)
    assert bf16_ulp_diff(got, want).max() <= 1


def test_empty_problem(w8):
    xq = torch.empty((0, 64), dtype=torch.int8, device="cuda")
    wq = torch.zeros((16, 64), dtype=torch.int8, device="cuda")
    out = w8.w8a8_gemm(xq, wq, torch.empty(0, device="cuda"), torch.ones(16, device="cuda"))
    assert out.shape == (0, 16)


def test_selected_configs_valid(w8):
    for name, wl in workloads.WORKLOADS.items():
        c = w8.w8a8_select_config(wl.M, wl.N, wl.K)
        assert c["block_m"] in (128, 256) and c["block_n"] in (128, 256), (name, c)
        assert 1 <= c["grid"] <= torch.cuda.get_device_properties(0).multi_processor_count
