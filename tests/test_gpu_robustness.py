"""Failure handling and out-of-bounds checks on the GPU, without faulting it.

* Bounded waits: with a short host-set spin budget and the forward's K/V
  producer told to issue nothing, every consumer wait of the tensor-core
  forward runs out with no copy or MMA in flight; the kernel unwinds, frees
  its TMEM and latches VMOBA_ERR_TIMEOUT in the workspace status word, and a
  following normal call on the same context matches the oracle.
* Guard bands: every output buffer and the workspace are placed inside a
  larger allocation whose margins hold a byte pattern; after selection,
  plan, forward and backward the margins must be untouched (no kernel wrote
  outside its buffer).
"""
import math

import numpy as np
import pytest

import oracle as O
import synth
from synth.video_latents import round_to

from .gpu_util import TOL, from_device, out_err, pack_bits, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_attention_layer_b200 import LayerShape, _lib  # noqa: E402
from block_sparse_attention_layer_b200.layer import VMoBALayer  # noqa: E402

T, H, W, NH, D = 8, 16, 16, 2, 128
VMOBA_ERR_TIMEOUT = -6


def _inputs(seed):
    q, k, v = synth.make_qkv(seed, 0, T, H, W, NH, D)
    dout = synth.make_dout(seed, 0, T * H * W, NH, D)
    return [round_to(x, "bf16") for x in (q, k, v, dout)]


def test_bounded_wait_times_out_and_the_context_stays_usable():
    mode, box = 0, (1, 16, 16)
    q, k, v, _ = _inputs(160)
    sh = LayerShape(T, H, W, NH, D, mode, *box, "bf16")
    L = VMoBALayer(sh)
    qd = to_device(q, "bf16")
    L.select(qd, to_device(k, "bf16"), to_device(v, "bf16"), 0.4)
    torch.cuda.synchronize()
    assert _lib.get_status(L.ws) == 0
    try:
        _lib.debug_set_wait(wait_cycles=200_000, skip_forward_loads=True)
        L.forward(qd)
        torch.cuda.synchronize()
    finally:
        _lib.debug_set_wait(0, False)
    assert _lib.get_status(L.ws) == VMOBA_ERR_TIMEOUT
    assert _lib.get_status(L.ws) == 0            # reading clears the word
    # the same context and workspace, a normal call: correct results
    out, _ = L.forward(qd)
    torch.cuda.synchronize()
    assert _lib.get_status(L.ws) == 0
    from tests.gpu_util import unpack_bits
    g = unpack_bits(L.sel.cpu().numpy(), L.n_blocks)
    blk = O.block_of_token(T, H, W, O.mode_box(mode, T, H, W, *box))
    o_ref, _ = O.attention_fwd(q, k, v, g, blk, 1 / math.sqrt(D))
    assert out_err(from_device(out), o_ref, "bf16") <= TOL["bf16"]


def test_debug_wait_arguments_validated():
    L = _lib.lib()
    assert L.vmoba_debug_set_wait(-1, 0) == -1
    assert L.vmoba_debug_set_wait(0, 2) == -1
    assert L.vmoba_debug_set_wait(0, 0) == 0


GUARD = 4096          # bytes of margin on each side (a multiple of 256: keeps alignment)
PATTERN = 0xA5


class Guarded:
    """A device buffer of ``nbytes`` inside an allocation with GUARD-byte
    margins filled with PATTERN; ``view`` is the usable part."""

    def __init__(self, nbytes, dtype, shape):
        self.nbytes = nbytes
        self.raw = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.view = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def margins_intact(self):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.nbytes:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


@pytest.mark.parametrize("mode,box,d", [(0, (1, 16, 16), 128), (2, (2, 4, 4), 128),
                                        (1, (8, 4, 4), 64)])
def test_guard_bands_around_outputs_and_workspace(mode, box, d):
    q, k, v = synth.make_qkv(170 + mode, 0, T, H, W, NH, d)
    dout = synth.make_dout(170 + mode, 0, T * H * W, NH, d)
    q, k, v, dout = (round_to(x, "bf16") for x in (q, k, v, dout))
    sh = LayerShape(T, H, W, NH, d, mode, *box, "bf16")
    s = sh.s
    nb = _lib.num_blocks(sh)
    wb = (nb + 31) // 32
    bf = torch.bfloat16
    bufs = {
        "k_perm": Guarded(NH * s * d * 2, bf, (NH, s, d)),
        "v_perm": Guarded(NH * s * d * 2, bf, (NH, s, d)),
        "blocks": Guarded(NH * nb * d * 4, torch.float32, (NH, nb, d)),
        "sel": Guarded(NH * s * wb * 4, torch.int32, (NH, s, wb)),
        "stats": Guarded(NH * _lib.HEAD_STATS_DTYPE.itemsize, torch.uint8,
                         (NH * _lib.HEAD_STATS_DTYPE.itemsize,)),
        "ws": Guarded(_lib.workspace_size(sh), torch.uint8, (_lib.workspace_size(sh),)),
        "ws_bwd": Guarded(_lib.bwd_workspace_size(sh), torch.uint8,
                          (_lib.bwd_workspace_size(sh),)),
        "out": Guarded(s * NH * d * 2, bf, (s, NH, d)),
        "lse": Guarded(NH * s * 4, torch.float32, (NH, s)),
        "dq": Guarded(s * NH * d * 2, bf, (s, NH, d)),
        "dk": Guarded(s * NH * d * 2, bf, (s, NH, d)),
        "dv": Guarded(s * NH * d * 2, bf, (s, NH, d)),
    }
    b = {n: g.view for n, g in bufs.items()}
    qd, kd, vd, dod = (to_device(x, "bf16") for x in (q, k, v, dout))
    _lib.partition(sh, kd, vd, b["k_perm"], b["v_perm"], b["blocks"])
    _lib.score_select(sh, qd, b["blocks"], 0.4, 0.0, b["sel"], b["stats"], b["ws"])
    _lib.build_plan(sh, b["sel"], b["ws"])
    _lib.attn_fwd(sh, qd, b["k_perm"], b["v_perm"], b["sel"], b["ws"], 0.0, b["out"], b["lse"])
    _lib.attn_bwd(sh, qd, b["k_perm"], b["v_perm"], b["sel"], b["ws"], 0.0, b["lse"], dod,
                  b["dq"], b["dk"], b["dv"], b["ws_bwd"])
    torch.cuda.synchronize()
    for name, g in bufs.items():
        assert g.margins_intact(), f"a kernel wrote outside {name}"
    # and the results are right (the guarded buffers were really used)
    box3 = O.mode_box(mode, T, H, W, *box)
    blk = O.block_of_token(T, H, W, box3)
    from tests.gpu_util import unpack_bits
    g = unpack_bits(b["sel"].cpu().numpy(), nb)
    o_ref, _ = O.attention_fwd(q, k, v, g, blk, 1 / math.sqrt(d))
    assert out_err(from_device(b["out"]), o_ref, "bf16") <= TOL["bf16"]
    dq_ref, dk_ref, dv_ref = O.attention_bwd(q, k, v, g, blk, 1 / math.sqrt(d), dout)
    assert out_err(from_device(b["dq"]), dq_ref, "bf16") <= TOL["bf16"]
    assert out_err(from_device(b["dk"]), dk_ref, "bf16") <= TOL["bf16"]
    assert out_err(from_device(b["dv"]), dv_ref, "bf16") <= TOL["bf16"]


def _layer_run(sh, q, k, v, dout, tau, frac):
    L = VMoBALayer(sh, max_pair_fraction=frac)
    qd = to_device(q, "bf16")
    L.step(qd, to_device(k, "bf16"), to_device(v, "bf16"), tau, dout=to_device(dout, "bf16"))
    torch.cuda.synchronize()
    return L


@pytest.mark.parametrize("mode,box", [(0, (1, 16, 16)), (2, (2, 4, 4))])
def test_workspace_sized_for_tau_gives_the_same_results(mode, box):
    """A workspace sized for the method's selection at tau (a quarter of the
    pairs) derives a smaller pair capacity from its size; every output equals
    the every-pair workspace's bit for bit."""
    q, k, v, dout = _inputs(190 + mode)
    sh = LayerShape(T, H, W, NH, D, mode, *box, "bf16")
    tau = 0.25
    assert _lib.workspace_size(sh, tau) < _lib.workspace_size(sh)
    a = _layer_run(sh, q, k, v, dout, tau, None)
    b = _layer_run(sh, q, k, v, dout, tau, tau)
    assert _lib.get_status(b.ws) == 0
    for name in ("sel", "out", "lse", "dq", "dk", "dv"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_selection_beyond_the_workspace_is_refused_on_the_device():
    """A workspace sized for 1 % of the pairs given a selection that keeps
    ~40 %: the plan leaves every head empty and latches VMOBA_ERR_WORKSPACE;
    nothing is written past the buffers (outputs zero, LSE -inf) and the
    context stays usable for a correct call."""
    q, k, v, dout = _inputs(195)
    sh = LayerShape(T, H, W, NH, D, 0, 1, 16, 16, "bf16")
    L = _layer_run(sh, q, k, v, dout, 0.4, 0.01)
    assert _lib.get_status(L.ws) == -4           # VMOBA_ERR_WORKSPACE
    assert not L.out.any() and not L.dq.any() and not L.dk.any() and not L.dv.any()
    assert torch.isneginf(L.lse).all()
    good = _layer_run(sh, q, k, v, dout, 0.4, 0.5)
    assert _lib.get_status(good.ws) == 0
    from tests.gpu_util import unpack_bits
    g = unpack_bits(good.sel.cpu().numpy(), good.n_blocks)
    blk = O.block_of_token(T, H, W, O.mode_box(0, T, H, W, 1, 16, 16))
    o_ref, _ = O.attention_fwd(q, k, v, g, blk, 1 / math.sqrt(D))
    assert out_err(from_device(good.out), o_ref, "bf16") <= TOL["bf16"]
