"""int8 expert weights and the weight-streaming (swap-AB) kernel, against the oracle.

The oracle quantises the same bf16 weights itself (fp32 decisions); the GPU's
codes and scales must match bit for bit.  Parity of the layer is then taken
against the weight-only definition: the oracle's plain layer with exact
(fp64) activations and the dequantised weights q * scale in place of the
bf16 ones, under the usual bf16 output bar.  The kernel's 15-bit activation
row codes are its own route onto the int8 tensor cores, not part of the
method; they are checked separately, as kernel internals, against the
oracle's row coder and its 8-bit layer.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_07_b200 as moe
from synth import configs

from parity_util import LayerInputs, check_dispatch, check_layer_out, check_routing, run_steps_w8, to_np64

pytestmark = pytest.mark.gpu
W = configs.WORKLOADS


@pytest.mark.parametrize("shape", [(8, 256, 384), (8, 384, 256), (8, 640, 128)])
def test_quantizer_bit_exact(shape):
    E, K, N = shape
    w = configs.normal(configs.SEED, 77, shape, std=1.0 / np.sqrt(K), dtype="bf16")
    w[2, :, 7] = 0  # a zero channel
    cfg = moe.Config(64, 256, 384, dtype="bf16")
    q, s = moe.quantize_int8(cfg, torch.from_numpy(w).view(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_int8(w)
    np.testing.assert_array_equal(q.cpu().numpy(), qr)
    np.testing.assert_array_equal(s.cpu().numpy(), sr)


CASES = {
    "w8_decode": dict(T=32, d=256, f=384, capacity_factor=4.0),
    "w8_token_chunks": dict(T=700, d=256, f=384),           # up to ~220 rows per expert: 2 token blocks
    "w8_skew_drop": dict(T=512, d=512, f=256, logit_bias=(1.5, 0.5, 0, 0, 0, 0, 0, 0)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_int8_layer_matches_oracle(name):
    w = configs.scaled(W["mid_bf16"], name=name, **CASES[name])
    L = LayerInputs(w)
    qw = moe.QuantizedExperts(L.cfg, L.dev["wg"], L.dev["wu"], L.dev["wd"])
    g = run_steps_w8(L, qw)
    check_routing(L, g, oracle.router_logits(L.x, L.wr, L.bias))
    check_dispatch(L, g)
    n = int(g["offsets"][-1])
    # the row codes of x_perm are an encoding: bit-exact against the oracle's
    x_hi, x_lo, x_sc = oracle.quantize_rows(L.x[g["perm"][:n]])
    np.testing.assert_array_equal(g["ws"]["x_hi"][:n].cpu().numpy(), x_hi)
    np.testing.assert_array_equal(g["ws"]["x_lo"][:n].cpu().numpy(), x_lo)
    np.testing.assert_array_equal(g["ws"]["x_scale"][:n].cpu().numpy(), x_sc)
    q = [oracle.quantize_int8(m) for m in (L.wg, L.wu, L.wd)]
    # parity: the weight-only definition (exact activations, dequantised weights)
    ref = oracle.layer_forward(L.x, L.wr, *(oracle.DequantizedExperts(qq, ss) for qq, ss in q),
                               w.capacity_factor, logit_bias=L.bias)
    same = (np.sort(g["idx"], 1) == np.sort(ref["idx"], 1)).all(1)
    keep = ((g["slot_of"] >= 0) == (ref["slot_of"] >= 0)).all(1)
    rows = np.nonzero(same & keep)[0]
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"][rows], rows)
    # kernel internals: the same layer with the kernel's activation row coding replayed
    ref8 = oracle.layer_forward_w8(L.x, L.wr, q[0][0], q[0][1], q[1][0], q[1][1], q[2][0], q[2][1],
                                   w.capacity_factor, logit_bias=L.bias)
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref8["out"][rows], rows)
    # the one-call layer entry point gives the same bits
    out = moe.layer_forward_w8(L.cfg, L.dev["x"], L.dev["wr"], qw, logit_bias=L.dev["bias"])
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])
    assert moe.get_device_error() == 0


def test_int8_is_close_to_bf16_layer():
    # the quantised layer approximates the bf16 layer to within the int8 step (loose sanity bar)
    w = configs.scaled(W["mid_bf16"], name="w8_vs_bf16", T=64, d=512, f=1024, capacity_factor=4.0)
    L = LayerInputs(w)
    qw = moe.QuantizedExperts(L.cfg, L.dev["wg"], L.dev["wu"], L.dev["wd"])
    a = to_np64(moe.layer_forward_w8(L.cfg, L.dev["x"], L.dev["wr"], qw))
    b = to_np64(moe.layer_forward(L.cfg, L.dev["x"], L.dev["wr"], L.dev["wg"], L.dev["wu"], L.dev["wd"]))
    rel = np.sqrt(np.mean((a - b) ** 2)) / np.sqrt(np.mean(b ** 2))
    assert rel < 0.03, rel
