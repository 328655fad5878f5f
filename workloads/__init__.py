"""Seeded synthetic DiT linear-layer workloads.

This module draws random inputs and nothing else: it holds none of the
W8A8 method's arithmetic (no quantization, no GEMM, no epilogue), so both
the CUDA path's tests and the CPU oracle can take their inputs from it.

The shapes are the linear layers of a diffusion transformer with hidden
size 3072, as in the paper "Realizing Native INT8 Compute for Diffusion
Transformers on Consumer GPUs" (abstract: the kernel replaces the DiT's
linear layers; results at 768px and 1024px).  The paper's model weights and
activations are not available, so seeded Gaussians stand in for them:

* activations X ~ N(0, 1), rounded once to bf16 (round to nearest even, by
  torch's CPU conversion);
* weights W ~ N(0, 0.02^2) in fp32, to be quantized per output channel;
* bias ~ N(0, 0.1^2), rounded once to bf16 (sigma 0.1; the description of
  the workload gives "N(0,0.1)" and we read 0.1 as the standard deviation);
* the MLP up-projection at 1024px scales a fixed seeded 1% of the K
  channels (31 of 3072) by 20 before rounding, as activation outliers;
* the long-K MLP down-projection gives int8 codes and fp32 scales directly:
  codes uniform in [-127, 127] with rows 0/1 of X and of W all +127 / all
  -127 (the worst-case |acc| = K * 127^2), scales log-uniform in
  [1e-4, 1e-1].

Generator: numpy PCG64 (``numpy.random.default_rng``), seed 20260612 plus
the workload's index.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SEED_BASE = 20260612


@dataclass(frozen=True)
class Workload:
    name: str
    index: int            # seed offset
    M: int
    N: int
    K: int
    kind: str             # "linear" (bf16 X, fp32 W) or "gemm_int8" (int8 codes given)
    outliers: bool = False
    note: str = ""
    tags: tuple = field(default_factory=tuple)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def ops(self) -> int:
        """Integer ops of the GEMM (one multiply + one add per MAC)."""
        return 2 * self.M * self.N * self.K


WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("tiny", 1, 64, 128, 256, "linear", note="oracle-sized check, 64 tokens"),
    Workload("qkv_768", 2, 2304, 9216, 3072, "linear",
             note="768px attention QKV projection, 48x48 image tokens"),
    Workload("mlp_up_1024", 3, 4096, 12288, 3072, "linear", outliers=True,
             note="1024px MLP up-projection, 64x64 tokens, 1% outlier channels x20"),
    Workload("mlp_down_1024", 4, 4096, 3072, 12288, "gemm_int8",
             note="1024px MLP down-projection, long K, int8 codes given"),
    Workload("sweep_qkv", 5, 9216, 9216, 3072, "linear",
             note="batch 2 at 1024px + 512 text tokens: QKV"),
    Workload("sweep_out", 5, 9216, 3072, 3072, "linear",
             note="batch 2 at 1024px + 512 text tokens: attention out"),
    Workload("sweep_up", 5, 9216, 12288, 3072, "linear",
             note="batch 2 at 1024px + 512 text tokens: MLP up"),
    Workload("sweep_down", 5, 9216, 3072, 12288, "linear",
             note="batch 2 at 1024px + 512 text tokens: MLP down"),
]}

HEADLINE = "mlp_up_1024"


@dataclass(frozen=True)
class BlockLayer:
    name: str
    N: int
    K: int
    source: str           # "x" / "a": a block input; otherwise the name of the layer whose output feeds it
    act: str = ""         # "gelu": the layer reads GELU(source), the GELU fused into its quantizer


@dataclass(frozen=True)
class Block:
    """The linear layers of one DiT block over M tokens, in execution order.
    Inputs "x" (the block input) and "a" (the attention result feeding the
    attention output projection) are seeded bf16 N(0, 1); the norm and the
    attention are not part of the method, so MLP up reads the attention
    output projection's result directly.  MLP down reads GELU of MLP up's
    output, the GELU computed inside its quantizer."""
    name: str
    index: int
    M: int
    layers: tuple
    note: str = ""

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def ops(self) -> int:
        return sum(2 * self.M * l.N * l.K for l in self.layers)

    def inputs(self, rows: slice | None = None) -> dict:
        """Seeded host inputs: x, a (bf16 bits, rows of the token stream),
        per layer w (fp32) and bias (bf16 bits)."""
        r0 = 0 if rows is None else rows.start
        m = self.M if rows is None else rows.stop - rows.start
        d = {"x": gen_activations(m, self.layers[0].K, self.seed, row_offset=r0),
             "a": gen_activations(m, 3072, self.seed + 100, row_offset=r0)}
        for i, l in enumerate(self.layers):
            d["w_" + l.name] = gen_weight(l.N, l.K, self.seed + 10 + i)
            d["bias_" + l.name] = gen_bias(l.N, self.seed + 20 + i)
        return d


BLOCKS: dict[str, Block] = {b.name: b for b in [
    Block("dit_block_1024", 6, 9216,
          (BlockLayer("qkv", 9216, 3072, "x"), BlockLayer("attn_out", 3072, 3072, "a"),
           BlockLayer("mlp_up", 12288, 3072, "attn_out"), BlockLayer("mlp_down", 3072, 12288, "mlp_up", act="gelu")),
          note="the four linears of one DiT block, batch 2 at 1024px + 512 text tokens (M = 9216)"),
]}


def _to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), by torch's CPU rounding."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def outlier_channels(K: int, seed: int) -> np.ndarray:
    """The fixed seeded set of round(1% of K) activation-outlier channels."""
    rng = np.random.default_rng(seed + 7919)
    n = int(round(0.01 * K))
    return np.sort(rng.choice(K, size=n, replace=False))


def gen_activations(M: int, K: int, seed: int, outliers: bool = False,
                    row_offset: int = 0) -> np.ndarray:
    """bf16 bit patterns [M, K] of X ~ N(0,1) (plus x20 outlier channels).

    Rows are drawn in blocks keyed by (seed, block index), so a row subset
    ``row_offset .. row_offset+M`` is the same whatever M is asked for."""
    block = 256
    out = np.empty((M, K), np.uint16)
    chans = outlier_channels(K, seed) if outliers else None
    r = 0
    while r < M:
        g = row_offset + r
        b = g // block
        lo = g - b * block
        n = min(block - lo, M - r)
        rng = np.random.default_rng([seed, 1, b])
        x = rng.standard_normal((block, K), dtype=np.float32)[lo:lo + n]
        if chans is not None:
            x[:, chans] *= np.float32(20.0)
        out[r:r + n] = _to_bf16_bits(x)
        r += n
    return out


def gen_weight(N: int, K: int, seed: int) -> np.ndarray:
    """fp32 W [N, K] ~ N(0, 0.02^2), to be quantized per output channel."""
    rng = np.random.default_rng([seed, 2])
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(0.02)
    return w


def gen_bias(N: int, seed: int) -> np.ndarray:
    """bf16 bit patterns [N] of bias ~ N(0, 0.1^2)."""
    rng = np.random.default_rng([seed, 3])
    return _to_bf16_bits(rng.standard_normal(N, dtype=np.float32) * np.float32(0.1))


def gen_int8_codes(rows: int, K: int, rng: np.random.Generator, extreme_rows: bool) -> np.ndarray:
    q = rng.integers(-127, 128, size=(rows, K), dtype=np.int8)
    if extreme_rows and rows >= 2:
        q[0, :] = 127
        q[1, :] = -127
    return q


def gen_log_uniform(n: int, rng: np.random.Generator, lo: float = 1e-4, hi: float = 1e-1) -> np.ndarray:
    return np.exp(rng.uniform(np.log(lo), np.log(hi), size=n)).astype(np.float32)


def gen_gemm_int8(M: int, N: int, K: int, seed: int):
    """Inputs of the int8-given GEMM workload: (xq, wq, scale_a, scale_w, bias_bits)."""
    rng = np.random.default_rng([seed, 4])
    xq = gen_int8_codes(M, K, rng, True)
    wq = gen_int8_codes(N, K, rng, True)
    sa = gen_log_uniform(M, rng)
    sw = gen_log_uniform(N, rng)
    return xq, wq, sa, sw, gen_bias(N, seed)


def make(name_or_wl, rows: slice | None = None) -> dict:
    """All host inputs of a workload as numpy arrays.

    "linear" workloads give x (bf16 bits [M,K]), w (fp32 [N,K]), bias (bf16
    bits [N]); "gemm_int8" ones give xq, wq, scale_a, scale_w, bias."""
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    if wl.kind == "linear":
        r0 = 0 if rows is None else rows.start
        m = wl.M if rows is None else rows.stop - rows.start
        return {"x": gen_activations(m, wl.K, wl.seed, wl.outliers, row_offset=r0),
                "w": gen_weight(wl.N, wl.K, wl.seed),
                "bias": gen_bias(wl.N, wl.seed)}
    xq, wq, sa, sw, bias = gen_gemm_int8(wl.M, wl.N, wl.K, wl.seed)
    if rows is not None:
        xq, sa = xq[rows], sa[rows]
    return {"xq": xq, "wq": wq, "scale_a": sa, "scale_w": sw, "bias": bias}


def shard_rows(M: int, world: int, rank: int) -> slice:
    """Contiguous token range of ``rank`` when M tokens are split over ``world``
    ranks (tokens are independent, so no exchange is needed)."""
    per, extra = divmod(M, world)
    lo = rank * per + min(rank, extra)
    return slice(lo, lo + per + (1 if rank < extra else 0))
