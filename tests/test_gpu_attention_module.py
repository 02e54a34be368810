"""The autograd function and the self-attention module around the kernels.

Gradients come from the library's backward through torch.autograd; outputs
and gradients are compared with the fp64 oracle on the selection the GPU
made (read back from the layer), and the full-attention switch with the
oracle's dense attention.
"""
import math

import numpy as np
import pytest

import oracle as O
import synth
from synth.video_latents import round_to

from .gpu_util import TOL, from_device, out_err, to_device, unpack_bits

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_attention_layer_b200 import LayerShape  # noqa: E402
from block_sparse_attention_layer_b200.attention import (VMoBAFunction,  # noqa: E402
                                                         VMoBASelfAttention)
from block_sparse_attention_layer_b200.layer import VMoBALayer  # noqa: E402

T, H, W, NH, D = 8, 16, 16, 2, 128
BOXES = ((1, 16, 16), (8, 4, 4), (2, 4, 4))


@pytest.mark.parametrize("mode,full", [(0, False), (1, False), (2, False), (2, True)])
def test_autograd_function_matches_oracle(mode, full):
    q, k, v = synth.make_qkv(140 + mode, 0, T, H, W, NH, D)
    dout = synth.make_dout(140 + mode, 0, T * H * W, NH, D)
    q, k, v, dout = (round_to(x, "bf16") for x in (q, k, v, dout))
    layer = VMoBALayer(LayerShape(T, H, W, NH, D, mode, *BOXES[mode], "bf16"))
    qt, kt, vt = (to_device(x, "bf16").requires_grad_(True) for x in (q, k, v))
    scale = 1 / math.sqrt(D)
    out = VMoBAFunction.apply(qt, kt, vt, layer, 0.4, full, scale)
    out.backward(to_device(dout, "bf16"))
    torch.cuda.synchronize()
    g = unpack_bits(layer.sel.cpu().numpy(), layer.n_blocks)
    if full:
        assert g.all()
    box = O.mode_box(mode, T, H, W, *BOXES[mode])
    blk = O.block_of_token(T, H, W, box)
    o_ref, _ = O.attention_fwd(q, k, v, g, blk, scale)
    dq_ref, dk_ref, dv_ref = O.attention_bwd(q, k, v, g, blk, scale, dout)
    assert out_err(from_device(out.detach()), o_ref, "bf16") <= TOL["bf16"]
    assert out_err(from_device(qt.grad), dq_ref, "bf16") <= TOL["bf16"]
    assert out_err(from_device(kt.grad), dk_ref, "bf16") <= TOL["bf16"]
    assert out_err(from_device(vt.grad), dv_ref, "bf16") <= TOL["bf16"]


def test_self_attention_module_layers_and_switch():
    dim = NH * D
    torch.manual_seed(0)
    for layer_idx in (0, 1, 2, 3):
        m = VMoBASelfAttention(dim, NH, T, H, W, layer_idx, BOXES, tau=0.3)
        assert m.mode == layer_idx % 3
        x = (torch.randn(T * H * W, dim, device="cuda") * 0.5).to(torch.bfloat16)
        x.requires_grad_(True)
        for full in (False, True):
            y = m(x, full_attention=full)
            y.float().square().mean().backward()
            torch.cuda.synchronize()
            assert y.shape == x.shape and torch.isfinite(y).all()
            assert torch.isfinite(m.qkv.weight.grad).all() and torch.isfinite(x.grad).all()
            # the module's output: projections of the oracle's attention on
            # the selection the kernels used
            with torch.no_grad():      # the exact bf16 q, k, v the kernels were given
                qkv = m.qkv(x.detach()).view(-1, 3, NH, D).double().cpu().numpy()
            q, k, v = (qkv[:, i].copy() for i in range(3))
            g = unpack_bits(m.layer.sel.cpu().numpy(), m.layer.n_blocks)
            if full:
                assert g.all()
            box = O.mode_box(m.mode, T, H, W, *BOXES[m.mode])
            o_ref, _ = O.attention_fwd(q, k, v, g, O.block_of_token(T, H, W, box), m.scale)
            o_ref = torch.from_numpy(round_to(o_ref.reshape(-1, dim), "bf16"))
            y_ref = o_ref @ m.proj.weight.double().cpu().T + m.proj.bias.double().cpu()
            assert (y.double().cpu() - y_ref).abs().max().item() <= 0.05
            m.zero_grad()
            x.grad = None


def test_two_forwards_before_the_backwards():
    """Two micro-batches through one layer object: forward A, forward B,
    backward B, backward A.  Each backward must see its own forward's
    selection and state, so every gradient equals the one a fresh layer gives
    for that input alone (the kernels are deterministic: bit-identical)."""
    mode = 2
    shape = LayerShape(T, H, W, NH, D, mode, *BOXES[mode], "bf16")
    scale = 1 / math.sqrt(D)
    inputs = []
    for seed in (150, 151):
        q, k, v = synth.make_qkv(seed, 0, T, H, W, NH, D)
        dout = synth.make_dout(seed, 0, T * H * W, NH, D)
        inputs.append([to_device(round_to(x, "bf16"), "bf16") for x in (q, k, v, dout)])

    def grads(layer, q, k, v, dout, full=False):
        qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
        out = VMoBAFunction.apply(qt, kt, vt, layer, 0.4, full, scale)
        return out, (qt, kt, vt), dout

    ref = []
    for q, k, v, dout in inputs:
        out, leaves, d = grads(VMoBALayer(shape), q, k, v, dout)
        out.backward(d)
        ref.append([out.detach().clone()] + [x.grad.clone() for x in leaves])

    shared = VMoBALayer(shape)
    runs = [grads(shared, *inp) for inp in inputs]       # forward A, forward B
    for idx in (1, 0):                                    # backward B, backward A
        out, leaves, d = runs[idx]
        out.backward(d)
    torch.cuda.synchronize()
    for idx, (out, leaves, _) in enumerate(runs):
        assert torch.equal(out.detach(), ref[idx][0])
        for x, r in zip(leaves, ref[idx][1:]):
            assert torch.equal(x.grad, r)
