"""GPU parity of the row quantizers (w8a8_quantize_act, w8a8_quantize_weight)
against the CPU oracle: int8 codes and fp32 scales must be bit-exact.

Paper: "Realizing Native INT8 Compute for Diffusion Transformers on Consumer
GPUs" (arXiv 2606.14598), abstract -- per-token activation quantization and
per-channel weight quantization of W8A8."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import oracle_pins as P
from tests.util import bf16_bits_to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w8():
    import w8a8_int8_gemm_b200 as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _run_act(w8, bits, ldx_pad=0, ldq_pad=0):
    M, K = bits.shape
    dev = torch.device("cuda")
    xfull = torch.zeros((M, K + ldx_pad), dtype=torch.bfloat16, device=dev)
    xfull[:, :K] = bf16_bits_to_torch(bits, dev)
    x = xfull[:, :K]
    qfull = torch.full((M, K + ldq_pad), 99, dtype=torch.int8, device=dev)
    q = qfull[:, :K]
    q, s = w8.w8a8_quantize_act(x, xq=q)
    torch.cuda.synchronize()
    if ldq_pad:
        assert (qfull[:, K:] == 99).all(), "quantizer wrote past K in the padded output rows"
    return q.cpu().numpy(), s.cpu().numpy()


def _assert_same(q, s, bits):
    qo, so = oracle.quantize_act(bits)
    assert np.array_equal(s.view(np.uint32), so.view(np.uint32)), "scale_a differs from the oracle"
    bad = np.argwhere(q != qo)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"


# Every launch path: one-row warps (K <= 4096; 4, 8, 12 and 16 vectors per
# lane, with M past one wave of resident warps: 4200 x 1024 ... 3000 x 4096);
# one block per row up to K = 32768 (8, 12 and 16 vectors per thread); the
# two-pass kernel beyond.
@pytest.mark.parametrize("M,K", [(1, 16), (7, 48), (9, 272), (63, 1024), (64, 2048), (33, 3072),
                                 (17, 4096), (5, 4112), (3, 12288), (2, 20000 // 16 * 16), (2369, 1024),
                                 (4200, 1024), (4500, 2048), (5000, 3072), (3000, 4096), (2, 24576),
                                 (3, 24592), (2, 40000)])
def test_act_random_shapes(w8, M, K):
    rng = np.random.default_rng(M * 100003 + K)
    x = rng.standard_normal((M, K)).astype(np.float32) * np.float32(3.0)
    bits = P.to_bits(x)
    q, s = _run_act(w8, bits)
    _assert_same(q, s, bits)


def test_act_edge_rows(w8):
    """Zero rows, -0, a single non-zero, bf16 subnormals, exact ties, huge values."""
    rng = np.random.default_rng(3)
    K = 512
    x = P.edge_rows(K, rng)
    bits = P.to_bits(x)
    # rows from the hand-worked fixture, padded with zeros to K
    for xs, _, _ in P.read_rows("quant_act_rows.txt"):
        r = np.zeros(K, np.float32)
        vals = np.array([float(v) for v in xs], np.float32)
        r[:len(vals)] = vals
        bits = np.concatenate([bits, P.bf16_bits(r)[None, :]])
    q, s = _run_act(w8, bits)
    _assert_same(q, s, bits)


def _bf16_pattern(v):
    return int(np.array([v], np.float32).view(np.uint32)[0] >> 16)


# Row maxima whose significands have few bits (127 x / amax is then an exact
# half-integer for many x), an all-ones significand, and the scales next to
# 2^-100, below which rows are quantized by IEEE division.
TIE_AMAX = [1.0, 3.0, 0.75, 5.0, 7.0, 127.0, 254.0, 1.9921875, 0.1875, 96.0, 127.0 * 2.0 ** -100]


def _tie_rows(K):
    """Rows [amax, then every bf16 value with |x| <= amax, both signs]."""
    rows = []
    pats = [_bf16_pattern(a) for a in TIE_AMAX]
    p100 = _bf16_pattern(127.0 * 2.0 ** -100)
    pats += [p100 - 1, p100 + 1]
    for a in pats:
        pos = np.arange(0, a + 1, dtype=np.uint32).astype(np.uint16)
        vals = np.concatenate([pos, pos | np.uint16(0x8000)])
        for c in range(0, len(vals), K - 1):
            seg = vals[c:c + K - 1]
            row = np.zeros(K, np.uint16)
            row[0] = a
            row[1:1 + len(seg)] = seg
            rows.append(row)
    return np.stack(rows)


@pytest.mark.parametrize("K", [3072, 12288, 40000])
def test_act_dense_ties(w8, K):
    """Every bf16 value below each of several row maxima, many of them exact
    half-integer quotients, on the warp, block and two-pass paths."""
    bits = _tie_rows(K)
    q, s = _run_act(w8, bits)
    _assert_same(q, s, bits)


def test_weight_dense_ties(w8):
    """fp32 rows with values planted at (and a few ulps around) every
    half-integer multiple of the row's scale, for scales from 2^-100 up."""
    rng = np.random.default_rng(11)
    K = 1296
    h = np.arange(-254, 255, dtype=np.float32) * np.float32(0.5)
    rows = []
    amaxes = list(np.float32(2.0) ** rng.uniform(-93, 100, 60).astype(np.float32) * rng.uniform(1, 2, 60))
    edge = np.float32(127.0 * 2.0 ** -100)
    amaxes += [edge, np.nextafter(edge, np.float32(0)), np.nextafter(edge, np.float32(1))]
    for a in amaxes:
        a = np.float32(a)
        s = np.float32(a / np.float32(127.0))
        x = (h * s).astype(np.float32)
        d = rng.integers(-2, 3, x.shape).astype(np.int32)
        x = (x.view(np.int32) + d * (x != 0)).view(np.float32)
        x = np.clip(x, -a, a)
        row = np.zeros(K, np.float32)
        row[0] = a
        row[1:1 + len(x)] = x
        rows.append(row)
    w = np.stack(rows)
    wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    wq_o, sw_o = oracle.quantize_weight(w)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), sw_o.view(np.uint32))
    bad = np.argwhere(wq.cpu().numpy() != wq_o)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"


def test_act_strided(w8):
    rng = np.random.default_rng(4)
    bits = P.to_bits(rng.standard_normal((37, 320)).astype(np.float32))
    q, s = _run_act(w8, bits, ldx_pad=24, ldq_pad=48)
    _assert_same(q, s, bits)


@pytest.mark.parametrize("name", ["tiny", "qkv_768", "mlp_up_1024"])
def test_act_workloads_full(w8, name):
    """Every row of the workload's activations, bit-exact."""
    wl = workloads.WORKLOADS[name]
    bits = workloads.gen_activations(wl.M, wl.K, wl.seed, wl.outliers)
    q, s = _run_act(w8, bits)
    _assert_same(q, s, bits)


def test_act_long_k_workload_full(w8):
    """The 9216 x 12288 input of the MLP down-projection sweep (24 KB rows)."""
    wl = workloads.WORKLOADS["sweep_down"]
    bits = workloads.gen_activations(wl.M, wl.K, wl.seed, wl.outliers)
    q, s = _run_act(w8, bits)
    _assert_same(q, s, bits)


def test_act_empty(w8):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, s = w8.w8a8_quantize_act(x)
    assert q.shape == (0, 64) and s.shape == (0,)


@pytest.mark.parametrize("N,K", [(128, 256), (136, 48), (12288, 3072), (3072, 12288), (8, 12304)])
def test_weight_quant(w8, N, K):
    rng = np.random.default_rng(N + K)
    w = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    wq_o, sw_o = oracle.quantize_weight(w)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), sw_o.view(np.uint32))
    assert np.array_equal(wq.cpu().numpy(), wq_o)


def test_weight_quant_golden_and_subnormal(w8):
    """Hand-worked weight rows, including an fp32 subnormal row that clamps
    and one whose scale underflows to zero."""
    K = 64
    rows = []
    for ws, _, _ in P.read_rows("quant_weight_rows.txt"):
        r = np.zeros(K, np.float32)
        vals = np.array([P.parse_num(v) for v in ws], np.float32)
        r[:len(vals)] = vals
        rows.append(r)
    w = np.stack(rows)
    wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    wq_o, sw_o = oracle.quantize_weight(w)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), sw_o.view(np.uint32))
    assert np.array_equal(wq.cpu().numpy(), wq_o)
