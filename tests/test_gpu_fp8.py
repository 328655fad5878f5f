"""GPU parity of the FP8 (OCP E4M3) variant against the CPU oracle.

* quantizers: E4M3 codes and fp32 scales bit-exact (ties, subnormal codes,
  signed zeros, zero rows, subnormal fp32 scales included);
* GEMM accumulators (tcgen05 kind::f8f6f4, fp32): bit-exact to the exact
  sum whenever every partial sum is an fp32 value (codes whose values are
  multiples of 1/8 with |v| <= 8, so that any summation order is exact),
  for every tile configuration; for arbitrary finite codes, within the
  bound of any fp32 summation order, |acc - exact| <= (K-1) 2^-23 sum|p|
  (the classical bound for n terms summed in any order with unit roundoff
  2^-23, which also covers truncating adders);
* bf16 epilogue: bit-exact to the oracle where the accumulator is exact;
  otherwise within 1 bf16 ulp plus the accumulator bound scaled by
  scale_a * scale_w;
* the linear layer, on small shapes and on the 1024px MLP up-projection
  (4096 x 12288 x 3072) with sampled rows.

The paper ("Realizing Native INT8 Compute for Diffusion Transformers on
Consumer GPUs", abstract) uses FP8 as its comparison baseline; the
per-token x per-channel E4M3 scheme is the reading stated in
include/w8a8.h."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.oracle_pins import edge_rows
from tests.util import bf16_bits_to_torch, bf16_ulp_diff, is_nan_bits, row_chunks, torch_bf16_to_bits

pytestmark = pytest.mark.gpu

U23 = 2.0 ** -23


@pytest.fixture(scope="module")
def w8():
    import w8a8_int8_gemm_b200 as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 values through torch's float8_e4m3fn (independent of both sides)."""
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


ALL_CODES = np.arange(256, dtype=np.uint8)
FINITE = ALL_CODES[~np.isnan(_decode(ALL_CODES))]
_vals = _decode(FINITE)
# Codes whose values are multiples of 1/8 with |v| <= 8: products are
# multiples of 2^-6 with |p| <= 64, so for K < 4096 every partial sum, in any
# order, is a multiple of 2^-6 below 2^18 in magnitude -- an fp32 value.
EXACT = FINITE[(np.abs(_vals) <= 8) & (np.mod(_vals * 8, 1) == 0)]


def _exact_codes(rng, rows, K):
    assert K * 64 < 2 ** 18, "partial sums must stay below 2^24 units of 1/64"
    return rng.choice(EXACT, (rows, K))


def _any_codes(rng, rows, K):
    return rng.choice(FINITE, (rows, K))


def _acc(w8, xq, wq, config=None):
    acc = w8.w8a8_gemm_fp8_f32(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), config=config)
    torch.cuda.synchronize()
    return acc.cpu().numpy().astype(np.float64)


def _abs_sum(xq, wq):
    """sum_k |x_k w_k| in binary64 (sign bits cleared)."""
    return oracle.gemm_fp8(xq & 0x7F, wq & 0x7F)


def _bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (normal range; 2^-133 below it)."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return 2.0 ** (e - 7)


# --------------------------------------------------------------- quantizers


def _fp8_tie_rows(K: int) -> np.ndarray:
    """Rows with absmax 448 (scale exactly 1) whose other elements are the
    midpoints between adjacent E4M3 values (ties) and the values themselves,
    both signs; and one row scaled by 2^-20 (scale 2^-20 exactly)."""
    pos = np.sort(_decode(FINITE[(FINITE < 0x7F)]))
    mids = 0.5 * (pos[:-1] + pos[1:])
    vals = np.concatenate([[448.0], mids, -mids, pos, -pos, [-0.0]])
    rows = []
    for start in range(0, len(vals), K - 1):
        r = np.zeros(K)
        chunk = vals[start:start + K - 1]
        r[0] = 448.0
        r[1:1 + len(chunk)] = chunk
        rows.append(r)
    rows.append(rows[0] * 2.0 ** -20)
    return np.stack(rows).astype(np.float32)


def _bits(x: np.ndarray) -> np.ndarray:
    return oracle.f32_to_bf16_bits(x.astype(np.float32))


@pytest.mark.parametrize("M,K", [(1, 16), (37, 272), (130, 1024), (64, 3072), (33, 4096), (17, 8192), (5, 12288)])
def test_quantize_act_fp8(w8, M, K):
    rng = np.random.default_rng(M * 31 + K)
    x = workloads.gen_activations(M, K, seed=M + K, outliers=True)
    x = np.concatenate([x, _bits(edge_rows(K, rng)), _bits(_fp8_tie_rows(K))])
    q, s = w8.w8a8_quantize_act_fp8(bf16_bits_to_torch(x, "cuda"))
    torch.cuda.synchronize()
    q_want, s_want = oracle.quantize_act_fp8(x)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_want.view(np.uint32))
    got = q.cpu().numpy()
    assert np.array_equal(got, q_want), np.argwhere(got != q_want)[:8]


@pytest.mark.parametrize("N,K", [(8, 16), (40, 784), (136, 3072), (24, 8208)])
def test_quantize_weight_fp8(w8, N, K):
    rng = np.random.default_rng(N + K)
    w = workloads.gen_weight(N, K, seed=N * K)
    tiny = (rng.standard_normal((4, K)) * 1e-41).astype(np.float32)   # subnormal scales
    w = np.concatenate([w, tiny, np.zeros((1, K), np.float32), _fp8_tie_rows(K), edge_rows(K, rng)])
    q, s = w8.w8a8_quantize_weight_fp8(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    q_want, s_want = oracle.quantize_weight_fp8(w)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_want.view(np.uint32))
    got = q.cpu().numpy()
    assert np.array_equal(got, q_want), np.argwhere(got != q_want)[:8]


def test_quantize_strided_fp8(w8):
    """Row strides larger than K on both sides (a slice of a wider buffer)."""
    x = workloads.gen_activations(50, 512, seed=9)
    xt = bf16_bits_to_torch(x, "cuda")
    wide = torch.zeros((50, 640), dtype=torch.bfloat16, device="cuda")
    wide[:, :512] = xt
    qbuf = torch.full((50, 528), 0x55, dtype=torch.uint8, device="cuda")
    q, s = w8.w8a8_quantize_act_fp8(wide[:, :512], xq=qbuf[:, :512])
    torch.cuda.synchronize()
    q_want, s_want = oracle.quantize_act_fp8(x)
    assert np.array_equal(qbuf[:, :512].cpu().numpy(), q_want)
    assert (qbuf[:, 512:].cpu().numpy() == 0x55).all(), "wrote past the row"
    assert np.array_equal(s.cpu().numpy(), s_want)


# -------------------------------------------------------------------- GEMM


SHAPES = [(1, 8, 16), (63, 136, 48), (129, 264, 272), (200, 520, 400), (257, 256, 1040), (520, 776, 2064)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_acc_exact_sums(w8, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 13 + K)
    xq, wq = _exact_codes(rng, M, K), _exact_codes(rng, N, K)
    assert np.array_equal(_acc(w8, xq, wq), oracle.gemm_fp8(xq, wq))


CONFIGS = [dict(block_m=bm, block_n=bn, stages=st, grid=g, raster_group=rg)
           for bm, bn, st in [(128, 256, 4), (128, 256, 2), (128, 128, 6), (256, 256, 6), (256, 128, 8),
                              (256, 128, 3)]
           for g, rg in [(148, 16), (4, 1), (2, 5)]]


def _cid(c):
    return f"m{c['block_m']}_n{c['block_n']}_st{c['stages']}_g{c['grid']}_r{c['raster_group']}"


@pytest.mark.parametrize("cfg", CONFIGS, ids=_cid)
def test_acc_every_config(w8, cfg):
    rng = np.random.default_rng(cfg["block_n"] + cfg["stages"] * 10 + cfg["grid"])
    M, N, K = 300, 776, 656
    xq, wq = _exact_codes(rng, M, K), _exact_codes(rng, N, K)
    assert np.array_equal(_acc(w8, xq, wq, config=cfg), oracle.gemm_fp8(xq, wq))


@pytest.mark.parametrize("K,stages", [(384, 6), (1024, 4), (2048, 5)])
def test_acc_pair_double_chunk_stages(w8, K, stages):
    """CTA pairs loading two K-chunks per box (K % 128 == 0, ring >= 4 chunks)."""
    rng = np.random.default_rng(K + stages)
    M, N = 300, 520
    xq, wq = _exact_codes(rng, M, K), _exact_codes(rng, N, K)
    for bn in (256, 128):
        cfg = dict(block_m=256, block_n=bn, stages=stages, grid=148, raster_group=8)
        assert np.array_equal(_acc(w8, xq, wq, config=cfg), oracle.gemm_fp8(xq, wq)), cfg


@pytest.mark.parametrize("shape,grid,bm,stages", [((300, 776, 656), 5, 128, 4), ((129, 520, 1040), 4, 128, 4),
                                                  ((300, 776, 1024), 12, 256, 6), ((520, 1032, 640), 24, 256, 5)],
                         ids=lambda v: str(v))
def test_acc_tail_halves(w8, shape, grid, bm, stages):
    M, N, K = shape
    cfg = dict(block_m=bm, block_n=256, stages=stages, grid=grid, raster_group=1)
    rng = np.random.default_rng(M + grid)
    xq, wq = _exact_codes(rng, M, K), _exact_codes(rng, N, K)
    assert np.array_equal(_acc(w8, xq, wq, config=cfg), oracle.gemm_fp8(xq, wq))


def test_acc_identity_and_closed_forms(w8):
    """1.0 on the diagonal selects the activations; rows of 448 * 448 sum to
    K * 448^2 exactly (an fp32 value for K = 1024)."""
    rng = np.random.default_rng(3)
    K = 256
    xq = _any_codes(rng, 130, K)
    eye = np.zeros((K, K), np.uint8)
    eye[np.arange(K), np.arange(K)] = 0x38  # 1.0
    assert np.array_equal(_acc(w8, xq, eye), _decode(xq))
    K = 1024
    x = np.stack([np.full(K, 0x7E, np.uint8), np.full(K, 0xFE, np.uint8)])
    acc = _acc(w8, x, np.concatenate([x] * 4))
    big = K * 448.0 * 448.0
    assert acc[0, 0] == big and acc[0, 1] == -big and acc[1, 0] == -big and acc[1, 1] == big


@pytest.mark.parametrize("M,N,K", [(129, 264, 272), (257, 520, 3072), (130, 256, 12288)])
def test_acc_any_codes_within_fp32_bound(w8, M, N, K):
    """Arbitrary finite codes (subnormals, both signs, the whole range):
    within the bound of fp32 summation in any order."""
    rng = np.random.default_rng(M + N + K)
    xq, wq = _any_codes(rng, M, K), _any_codes(rng, N, K)
    got = _acc(w8, xq, wq)
    exact = oracle.gemm_fp8(xq, wq)
    bound = (K - 1) * U23 * _abs_sum(xq, wq)
    err = np.abs(got - exact)
    assert (err <= bound).all(), float((err / np.maximum(bound, 1e-300)).max())


def _bf16_case(w8, M, N, K, seed, exact_codes, bias=True, config=None):
    rng = np.random.default_rng(seed)
    gen = _exact_codes if exact_codes else _any_codes
    xq, wq = gen(rng, M, K), gen(rng, N, K)
    sa = workloads.gen_log_uniform(M, rng)
    sw = workloads.gen_log_uniform(N, rng)
    bias_bits = workloads.gen_bias(N, seed) if bias else None
    dev = torch.device("cuda")
    out = w8.w8a8_gemm_fp8_ex(torch.from_numpy(xq).to(dev), torch.from_numpy(wq).to(dev),
                              torch.from_numpy(sa).to(dev), torch.from_numpy(sw).to(dev),
                              bf16_bits_to_torch(bias_bits, dev) if bias else None, config=config)
    torch.cuda.synchronize()
    got = torch_bf16_to_bits(out)
    exact = oracle.gemm_fp8(xq, wq)
    want = oracle.epilogue_fp8(exact, sa, sw, bias_bits)
    acc_bound = (K - 1) * U23 * _abs_sum(xq, wq)
    return got, want, acc_bound * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)


def _within(got_bits, want_bits, value_bound):
    """|got - want| <= 1 bf16 ulp (of the larger) + the propagated accumulator bound."""
    g = oracle.bf16_bits_to_f32(got_bits).astype(np.float64)
    w = oracle.bf16_bits_to_f32(want_bits).astype(np.float64)
    ulp = _bf16_ulp(np.maximum(np.abs(g), np.abs(w)))
    return np.abs(g - w) <= ulp + value_bound * (1 + 1e-6)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("bias", [True, False])
def test_bf16_epilogue_exact_acc(w8, M, N, K, bias):
    got, want, _ = _bf16_case(w8, M, N, K, M + N + K, True, bias)
    assert not is_nan_bits(got).any()
    assert bf16_ulp_diff(got, want).max() <= 1


@pytest.mark.parametrize("cfg", CONFIGS[::3], ids=_cid)
def test_bf16_epilogue_configs(w8, cfg):
    got, want, _ = _bf16_case(w8, 300, 776, 656, cfg["block_n"] + cfg["stages"], True, True, cfg)
    assert bf16_ulp_diff(got, want).max() <= 1


@pytest.mark.parametrize("M,N,K", [(129, 264, 272), (257, 520, 3072)])
def test_bf16_epilogue_any_codes(w8, M, N, K):
    got, want, vb = _bf16_case(w8, M, N, K, M * N, False, True)
    assert not is_nan_bits(got).any()
    assert _within(got, want, vb).all()


# ------------------------------------------------------------ linear layer


def _linear_case(w8, M, N, K, seed, outliers=False):
    x = workloads.gen_activations(M, K, seed=seed, outliers=outliers)
    w = workloads.gen_weight(N, K, seed=seed + 1)
    bias_bits = workloads.gen_bias(N, seed + 2)
    dev = torch.device("cuda")
    wq, sw = w8.w8a8_quantize_weight_fp8(torch.from_numpy(w).to(dev))
    xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
    sa = torch.empty((M,), dtype=torch.float32, device=dev)
    out = w8.w8a8_linear_fp8(bf16_bits_to_torch(x, dev), wq, sw, bf16_bits_to_torch(bias_bits, dev),
                             ws_xq=xq, ws_scale_a=sa)
    torch.cuda.synchronize()
    return x, w, bias_bits, out, xq, sa, wq, sw


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (77, 200, 336), (300, 776, 1024), (520, 264, 3072)])
def test_linear_fp8(w8, M, N, K):
    x, w, bias_bits, out, xq, sa, wq, sw = _linear_case(w8, M, N, K, M + N + K, outliers=True)
    xq_want, sa_want = oracle.quantize_act_fp8(x)
    wq_want, sw_want = oracle.quantize_weight_fp8(w)
    assert np.array_equal(xq.cpu().numpy(), xq_want) and np.array_equal(sa.cpu().numpy(), sa_want)
    assert np.array_equal(wq.cpu().numpy(), wq_want) and np.array_equal(sw.cpu().numpy(), sw_want)
    exact = oracle.gemm_fp8(xq_want, wq_want)
    want = oracle.epilogue_fp8(exact, sa_want, sw_want, bias_bits)
    vb = (K - 1) * U23 * _abs_sum(xq_want, wq_want) * sa_want[:, None].astype(np.float64) * sw_want[None, :]
    got = torch_bf16_to_bits(out)
    assert not is_nan_bits(got).any()
    assert _within(got, want, vb).all()


def test_linear_fp8_mlp_up_1024_every_row(w8):
    """1024px MLP up-projection, 4096 x 12288 x 3072, in the launch
    configuration the benchmark uses: the weight codes and scales, every
    token's codes and scale bit-exact; every output row within one bf16 ulp
    plus the propagated fp32-summation bound of the oracle's exact sum (its
    GEMM in row chunks)."""
    wl = workloads.WORKLOADS["mlp_up_1024"]
    d = workloads.make(wl)
    dev = torch.device("cuda")
    wq, sw = w8.w8a8_quantize_weight_fp8(torch.from_numpy(d["w"]).to(dev))
    xq = torch.empty((wl.M, wl.K), dtype=torch.uint8, device=dev)
    sa = torch.empty((wl.M,), dtype=torch.float32, device=dev)
    out = w8.w8a8_linear_fp8(bf16_bits_to_torch(d["x"], dev), wq, sw, bf16_bits_to_torch(d["bias"], dev),
                             ws_xq=xq, ws_scale_a=sa)
    torch.cuda.synchronize()
    wq_want, sw_want = oracle.quantize_weight_fp8(d["w"])
    assert np.array_equal(wq.cpu().numpy(), wq_want) and np.array_equal(sw.cpu().numpy(), sw_want)
    xq_want, sa_want = oracle.quantize_act_fp8(d["x"])
    assert np.array_equal(xq.cpu().numpy(), xq_want) and np.array_equal(sa.cpu().numpy(), sa_want)
    got_all = torch_bf16_to_bits(out)
    assert not is_nan_bits(got_all).any()
    for rows in row_chunks(wl.M):
        exact = oracle.gemm_fp8(xq_want[rows], wq_want)
        want = oracle.epilogue_fp8(exact, sa_want[rows], sw_want, d["bias"])
        vb = (wl.K - 1) * U23 * _abs_sum(xq_want[rows], wq_want) * sa_want[rows, None].astype(np.float64) * \
            sw_want[None, :]
        ok = _within(got_all[rows], want, vb)
        assert ok.all(), (rows, int((~ok).sum()), int(bf16_ulp_diff(got_all[rows], want).max()))


def test_fp8_empty_and_errors(w8):
    dev = torch.device("cuda")
    xq = torch.empty((0, 64), dtype=torch.uint8, device=dev)
    wq = torch.zeros((16, 64), dtype=torch.uint8, device=dev)
    out = w8.w8a8_gemm_fp8(xq, wq, torch.empty(0, device=dev), torch.ones(16, device=dev))
    assert out.shape == (0, 16)
    lib = w8.raw_lib()
    a = torch.zeros((4, 48), dtype=torch.uint8, device=dev)
    b = torch.zeros((12, 48), dtype=torch.uint8, device=dev)
    acc = torch.zeros((4, 12), dtype=torch.float32, device=dev)
    assert lib.w8a8_gemm_fp8_f32(a.data_ptr(), b.data_ptr(), acc.data_ptr(), 4, 12, 48, None) == 1  # N % 8
    assert lib.w8a8_gemm_fp8_f32(a.data_ptr() + 8, b.data_ptr(), acc.data_ptr(), 4, 8, 48, None) == 2
    code = w8.w8a8_read_device_error(clear=True)
    assert code == 0
