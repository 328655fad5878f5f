"""GPU parity of chains of W8A8 linear layers recorded as one CUDA graph
(w8a8_chain_*), against the CPU oracle run layer by layer.

Each layer is the w8a8_linear path, whose codes, scales and accumulators are
bit-exact and whose epilogue performs the oracle's binary32 operations in
the oracle's order; a later layer's input is then exactly the oracle's
input for it, so whole chains are compared for equality, output by output
(no ulp allowance accumulates along the chain).

* a small chain whose layers feed one another, with an independent layer,
  an empty layer and ragged shapes, on every row;
* the DiT block of the full-block sweep at batch 2, 1024px + 512 text tokens
  (M = 9216): QKV 3072->9216 on the block input; attention output
  3072->3072 on a second input (the attention result, which is not part of
  this method); MLP up 3072->12288 on the attention output's result; MLP
  down 12288->3072 on GELU of MLP up's result, the GELU fused into MLP
  down's quantizer (the norm is not part of this method).  Weights quantized on the GPU are
  checked against the oracle's; the chain is checked on every row."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.util import bf16_bits_to_torch, row_chunks, torch_bf16_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w8():
    import w8a8_int8_gemm_b200 as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _weights(w8, N, K, seed):
    w = workloads.gen_weight(N, K, seed)
    wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    wq_o, sw_o = oracle.quantize_weight(w)
    assert np.array_equal(wq.cpu().numpy(), wq_o) and np.array_equal(sw.cpu().numpy(), sw_o)
    return wq, sw, wq_o, sw_o


def _oracle_layer(x_bits, wq_o, sw_o, bias_bits):
    out, xq, sa, _ = oracle.linear(x_bits, wq_o, sw_o, bias_bits)
    return out, xq, sa


def test_small_chain_all_rows(w8):
    M = 300
    x = workloads.gen_activations(M, 256, seed=41)
    shapes = [(512, 256), (272, 512), (256, 272)]   # (N, K): each layer feeds the next
    xt = bf16_bits_to_torch(x, "cuda")
    layers, ref = [], []
    cur_t, cur_o = xt, x
    for i, (N, K) in enumerate(shapes):
        wq, sw, wq_o, sw_o = _weights(w8, N, K, 50 + i)
        b = workloads.gen_bias(N, 60 + i)
        l = w8.linear_layer(cur_t, wq, sw, bf16_bits_to_torch(b, "cuda"))
        layers.append(l)
        out_o, xq_o, sa_o = _oracle_layer(cur_o, wq_o, sw_o, b)
        ref.append((out_o, xq_o, sa_o))
        cur_t, cur_o = l["out"], out_o
    # an independent layer on the block input, and an empty one
    wq, sw, wq_o, sw_o = _weights(w8, 1024, 256, 70)
    layers.append(w8.linear_layer(xt, wq, sw, None))
    ref.append(_oracle_layer(x, wq_o, sw_o, None))
    empty = w8.linear_layer(torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"), wq, sw, None)
    chain = w8.w8a8_chain_create(layers + [empty])
    assert w8.w8a8_chain_layers(chain) == 5
    for rep in range(2):   # replays give the same result
        for l in layers:
            l["out"].fill_(float("nan"))
        chain.launch()
        torch.cuda.synchronize()
        assert w8.w8a8_read_device_error() == 0
        for l, (out_o, xq_o, sa_o) in zip(layers, ref):
            assert np.array_equal(l["ws_xq"].cpu().numpy(), xq_o)
            assert np.array_equal(l["ws_scale_a"].cpu().numpy().view(np.uint32), sa_o.view(np.uint32))
            assert np.array_equal(torch_bf16_to_bits(l["out"]), out_o), f"layer {l['N']}x{l['K']} replay {rep}"
    chain.close()


def test_dit_block_1024_batch2(w8):
    """The four linears of one DiT block at M = 9216 as one graph, every
    row: the oracle runs the block layer by layer on chunks of rows (rows are
    independent through every layer), each layer fed the oracle's own output
    of the layer before (GELU'd for MLP down)."""
    blk = workloads.BLOCKS["dit_block_1024"]
    M = blk.M
    d = blk.inputs()
    dev = torch.device("cuda")
    src_t = {"x": bf16_bits_to_torch(d["x"], dev), "a": bf16_bits_to_torch(d["a"], dev)}
    L, wo = {}, {}
    for l in blk.layers:
        w = d["w_" + l.name]
        wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).to(dev))
        torch.cuda.synchronize()
        wq_o, sw_o = oracle.quantize_weight(w)
        assert np.array_equal(wq.cpu().numpy(), wq_o) and np.array_equal(sw.cpu().numpy(), sw_o)
        wo[l.name] = (wq_o, sw_o)
        act = w8.ACT_GELU if l.act == "gelu" else w8.ACT_NONE
        L[l.name] = w8.linear_layer(src_t[l.source], wq, sw, bf16_bits_to_torch(d["bias_" + l.name], dev),
                                    input_act=act)
        src_t[l.name] = L[l.name]["out"]
    chain = w8.w8a8_chain_create([L[l.name] for l in blk.layers])
    chain.launch()
    torch.cuda.synchronize()
    assert w8.w8a8_read_device_error() == 0
    got = {l.name: (torch_bf16_to_bits(L[l.name]["out"]), L[l.name]["ws_xq"].cpu().numpy(),
                    L[l.name]["ws_scale_a"].cpu().numpy()) for l in blk.layers}
    chain.close()
    for rows in row_chunks(M):
        src_o = {"x": d["x"][rows], "a": d["a"][rows]}
        for l in blk.layers:
            x_rows = oracle.gelu(src_o[l.source]) if l.act == "gelu" else src_o[l.source]
            out_o, xq_o, sa_o = _oracle_layer(x_rows, *wo[l.name], d["bias_" + l.name])
            src_o[l.name] = out_o
            out_g, xq_g, sa_g = got[l.name]
            assert np.array_equal(xq_g[rows], xq_o), (l.name, rows)
            assert np.array_equal(sa_g[rows].view(np.uint32), sa_o.view(np.uint32)), (l.name, rows)
            assert np.array_equal(out_g[rows], out_o), (l.name, rows)


def test_chain_errors(w8):
    wq = torch.zeros((16, 64), dtype=torch.int8, device="cuda")
    sw = torch.ones(16, device="cuda")
    x = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    good = w8.linear_layer(x, wq, sw)
    bad = dict(good, N=12)     # N % 8 != 0
    with pytest.raises(w8.W8A8Error):
        w8.w8a8_chain_create([good, bad])
    with pytest.raises(w8.W8A8Error):
        w8.w8a8_chain_create([])
    c = w8.w8a8_chain_create([good])
    c.close()
    with pytest.raises(ValueError):
        c.launch()
