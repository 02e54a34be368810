"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and validates arguments synchronously (no GPU needed: every
call here is rejected before anything is launched)."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_layer_b200 as V
from block_sparse_attention_layer_b200 import _lib
from synth import WORKLOADS

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "vmoba.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vmoba_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 10
    L = V.lib()
    for n in names:
        assert hasattr(L, n), f"libvmoba.so does not export {n}"


def test_mode_cycle():
    assert [V.mode_for_layer(l) for l in range(6)] == [0, 1, 2, 0, 1, 2]
    assert V.mode_for_layer(-1) == -1


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_block_count_and_workspace(wid, mode):
    w = WORKLOADS[wid]
    bt, bh, bw = w.boxes[mode]
    sh = V.LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, mode, bt, bh, bw, w.dtype)
    nb = V.num_blocks(sh)
    assert nb == (w.T // bt) * (w.H // bh) * (w.W // bw)
    ws = V.workspace_size(sh)
    # the fp32 score pool dominates the workspace
    assert ws >= 4 * w.n_heads * w.s * nb
    assert ws % 256 == 0
    assert V.bwd_workspace_size(sh) >= 4 * w.n_heads * w.s


def test_mode_selects_which_box_axes_apply():
    # 1D ignores bh, bw; 2D ignores bt; 3D uses all three
    assert V.num_blocks(V.LayerShape(4, 6, 8, 1, 64, 0, 2, 5, 7)) == 2
    assert V.num_blocks(V.LayerShape(4, 6, 8, 1, 64, 1, 3, 3, 4)) == 4
    assert V.num_blocks(V.LayerShape(4, 6, 8, 1, 64, 2, 2, 3, 4)) == 8


BAD = ctypes.c_void_p(0x100000)   # aligned, never dereferenced: calls below fail validation


def _shape(**kw):
    base = dict(T=4, H=8, W=8, n_heads=2, head_dim=64, mode=2, bt=2, bh=4, bw=4, dtype="f32")
    base.update(kw)
    return V.LayerShape(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(bt=3), -2),                 # box does not divide T
    (dict(head_dim=96), -2),          # unsupported head_dim
    (dict(n_heads=0), -2),
    (dict(T=0), -2),
    (dict(mode=3), -1),
])
def test_invalid_shapes_rejected(kw, code):
    sh = _shape(**kw)
    L = V.lib()
    assert L.vmoba_num_blocks(ctypes.byref(sh.c())) == code
    assert L.vmoba_workspace_size(ctypes.byref(sh.c())) == 0
    rc = L.vmoba_partition(ctypes.byref(sh.c()), BAD, BAD, BAD, BAD, BAD, None)
    assert rc == code


def test_invalid_dtype_rejected():
    c = _shape().c()
    c.dtype = 7
    assert V.lib().vmoba_num_blocks(ctypes.byref(c)) == -3


def test_null_and_misaligned_pointers_rejected():
    sh = _shape().c()
    L = V.lib()
    assert L.vmoba_partition(ctypes.byref(sh), None, BAD, BAD, BAD, BAD, None) == -1
    odd = ctypes.c_void_p(0x100004)
    assert L.vmoba_partition(ctypes.byref(sh), odd, BAD, BAD, BAD, BAD, None) == -1
    assert L.vmoba_attn_fwd(ctypes.byref(sh), BAD, BAD, BAD, BAD, BAD, 1 << 30, 0.0, None,
                            BAD, None) == -1


def test_selection_calls_reject_misaligned_q_and_blocks():
    """The selection kernels read q and the block means in 16-byte vectors: an
    element-offset view must come back as VMOBA_ERR_ARG, with nothing launched."""
    sh = _shape().c()
    L = V.lib()
    odd = ctypes.c_void_p(0x100004)
    ws = 1 << 30
    for q, b in ((odd, BAD), (BAD, odd)):
        assert L.vmoba_score_select(ctypes.byref(sh), q, b, 0.5, 0.0, BAD, BAD, BAD, ws,
                                    None) == -1
        assert L.vmoba_score_select_variant(ctypes.byref(sh), q, b, 0, 0.5, 0.0, BAD, BAD,
                                            BAD, ws, None) == -1
        assert L.vmoba_score_select_static(ctypes.byref(sh), q, b, 0.5, 0.0, BAD, BAD,
                                           None) == -1


@pytest.mark.parametrize("tau", [0.0, -0.5, float("nan")])
def test_tau_out_of_range_rejected(tau):
    sh = _shape().c()
    rc = V.lib().vmoba_score_select(ctypes.byref(sh), BAD, BAD, tau, 0.0, BAD, BAD, BAD,
                                    1 << 30, None)
    assert rc == -1


@pytest.mark.parametrize("variant,param", [
    (1, 0.0), (1, 2.5), (1, -3.0), (3, 0.0), (3, 1.5), (0, 0.0), (2, -0.1),
    (2, float("nan")), (3, float("nan")), (4, 0.0), (4, float("nan")), (5, 1.0), (-1, 1.0)])
def test_selection_variant_arguments_rejected(variant, param):
    sh = _shape().c()
    rc = V.lib().vmoba_score_select_variant(ctypes.byref(sh), BAD, BAD, variant, param, 0.0,
                                            BAD, BAD, BAD, 1 << 30, None)
    assert rc == -1


def test_small_workspace_rejected():
    # below the smallest layout (one pair slot per head) every call refuses;
    # between that and the every-pair size the calls derive a smaller pair
    # capacity from ws_bytes instead
    sh = _shape()
    assert 0 < V.workspace_size(sh, 1e-300) < V.workspace_size(sh)
    tiny = 4096                           # holds not even the fixed part of the layout
    L = V.lib()
    rc = L.vmoba_score_select(ctypes.byref(sh.c()), BAD, BAD, 0.5, 0.0, BAD, BAD, BAD,
                              tiny, None)
    assert rc == -4
    rc = L.vmoba_build_plan(ctypes.byref(sh.c()), BAD, None, V.workspace_size(sh), None)
    assert rc == -4                       # no workspace pointer
    rc = L.vmoba_attn_bwd(ctypes.byref(sh.c()), BAD, BAD, BAD, BAD, BAD, V.workspace_size(sh),
                          0.0, BAD, BAD, BAD, BAD, BAD, BAD, 0, None)
    assert rc == -4                       # backward workspace missing


def test_status_strings():
    L = V.lib()
    for code in range(-8, 1):
        assert L.vmoba_status_string(code)
    assert L.vmoba_status_string(0) == b"ok"
    assert b"unknown" in L.vmoba_status_string(12345)


def test_binding_rejects_wrong_tensors_before_the_call():
    torch = pytest.importorskip("torch")
    sh = _shape()
    k = torch.zeros((sh.s, 2, 64), dtype=torch.float32)
    with pytest.raises(ValueError):
        _lib.partition(sh, k, k, k, k, k)   # wrong shapes for k_perm / blocks


def test_full_attention_steps_of_the_training_strategy():
    from block_sparse_attention_layer_b200.attention import full_attention_steps
    assert full_attention_steps(50) == 13 and full_attention_steps(40) == 10
    assert full_attention_steps(1) == 1 and full_attention_steps(8, 0.0) == 0


@pytest.mark.parametrize("wid", [3, 4, 5])
def test_bounded_workspace_sizes(wid):
    """A workspace sized for the method's selection at tau holds a quarter of
    the pairs: much smaller than the every-pair size, monotone in the
    fraction, equal to it at the whole pool, invalid fractions give 0."""
    w = WORKLOADS[wid]
    sh = V.LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, 2, *w.boxes[2], w.dtype)
    full = V.workspace_size(sh)
    sizes = [V.workspace_size(sh, f) for f in (0.05, 0.1, 0.25, 0.5, 1.0, 3.0)]
    assert sizes == sorted(sizes)
    assert sizes[-2] == sizes[-1] == full
    assert sizes[2] < 0.5 * full
    L = V.lib()
    for bad in (0.0, -1.0, float("nan")):
        assert L.vmoba_workspace_size_bounded(ctypes.byref(sh.c()), bad) == 0
