"""Deployable codes on the GPU against the oracle: packing bit for bit at every width, decoding equal
to GPTQ's W_hat bit for bit, and the dequantized layer product."""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import rel_fro, to64
from post_quantization_expert_b200 import clha as L

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_pack_bit_exact(ctx, bits):
    g = np.random.default_rng(bits)
    rows, d_in = 37, 384
    codes = g.integers(0, 2 ** bits, size=(rows, d_in), dtype=np.uint8)
    packed = torch.full((rows, d_in * bits // 32), 0xFFFFFFFF, dtype=torch.int64, device=DEV).to(torch.int32)
    L.clha_pack_codes(ctx, torch.from_numpy(codes).to(DEV), rows, d_in, bits, packed)
    got = packed.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(got, O.pack_codes(codes, bits))


def test_decode_is_gptq_w_hat_and_layer_product(ctx):
    g = torch.Generator().manual_seed(5)
    d_out, d_in, bits = 256, 512, 3
    A = torch.randn((d_in, d_in // 2), generator=g).double()
    H = (A @ A.T / (d_in // 2) + 0.05 * torch.eye(d_in, dtype=torch.float64)).float()
    U = torch.empty((1, d_in, d_in), device=DEV)
    L.clha_factor(ctx, H[None].to(DEV).contiguous(), 1, d_in, U)
    W = (0.02 * torch.randn((1, d_out, d_in), generator=g)).to(torch.bfloat16).to(DEV)
    codes = torch.empty((1, d_out, d_in), dtype=torch.uint8, device=DEV)
    sc = torch.empty((1, d_out, d_in // 128), device=DEV)
    zs = torch.empty((1, d_out, d_in // 128), dtype=torch.uint8, device=DEV)
    Wh = torch.empty((1, d_out, d_in), device=DEV)
    L.clha_quantize(ctx, U, 1, W, 1, d_out, d_in, bits, codes, sc, zs, Wh)
    packed = torch.empty((d_out, d_in * bits // 32), dtype=torch.int32, device=DEV)
    L.clha_pack_codes(ctx, codes[0], d_out, d_in, bits, packed)
    dec = torch.empty((d_out, d_in), device=DEV)
    L.clha_dequantize(ctx, packed, sc[0], zs[0], d_out, d_in, bits, dec)
    assert torch.equal(dec, Wh[0])                                  # bit for bit
    for n, xdt in ((100, torch.bfloat16), (64, torch.float32), (1, torch.bfloat16)):
        X = torch.randn((n, d_in), generator=g).to(xdt).to(DEV)
        Y = torch.empty((n, d_out), device=DEV)
        L.clha_dequant_matmul(ctx, X, n, packed, sc[0], zs[0], d_out, d_in, bits, Y)
        torch.cuda.synchronize()
        want = O.dequant_matmul(to64(X), packed.cpu().numpy().view(np.uint32), sc[0].cpu().numpy(),
                                zs[0].cpu().numpy(), bits)
        assert rel_fro(Y.double().cpu().numpy(), want) < 1e-5      # fp32 FMA over d_in terms
