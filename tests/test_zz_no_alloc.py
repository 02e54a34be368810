"""The allocation-free selection entry point (vmoba_score_select_static).

It exists for callers that cannot call cudaMalloc when they select, for
example an engine that pooled all device memory at start-up and forbids
later allocations, or a plugin that is given no allocator: it keeps its
scratch in a fixed device array owned by the library.  Its results must be
the ones the workspace entry point produces on the same inputs, call after
call (the shared array keeps the previous call's contents, so a stale
histogram or search state would show up on the second call).

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

from synth import WORKLOADS

from .gpu_util import to_device, workload_arrays

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_attention_layer_b200 import LayerShape, _lib  # noqa: E402
from block_sparse_attention_layer_b200.layer import VMoBALayer  # noqa: E402


def _shape(w, mode):
    return LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, mode, *w.boxes[mode], w.dtype)


@pytest.mark.parametrize("wid,mode,tau", [(2, 2, 0.5), (2, 0, 0.25), (1, 1, 0.5)])
def test_static_scratch_selection_matches_workspace_selection(wid, mode, tau):
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    sh = _shape(w, mode)
    L = VMoBALayer(sh)
    qd = to_device(q, w.dtype)
    L.partition_only(to_device(k, w.dtype), to_device(v, w.dtype))
    _lib.score_select(sh, qd, L.blocks, tau, 0.0, L.sel, L.stats, L.ws)
    torch.cuda.synchronize()
    ref_bits = L.sel.clone()
    ref_stats = _lib.decode_stats(L.stats)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        bits = torch.full_like(L.sel, -1)
        stats = torch.zeros_like(L.stats)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        reserved0 = torch.cuda.memory_reserved()
        rc = _lib.lib().vmoba_score_select_static(
            ctypes.byref(sh.c()), ctypes.c_void_p(qd.data_ptr()),
            ctypes.c_void_p(L.blocks.data_ptr()), tau, 0.0, ctypes.c_void_p(bits.data_ptr()),
            ctypes.c_void_p(stats.data_ptr()), stream)
        assert rc == 0
        torch.cuda.synchronize()
        if call == 1:
            # after the first call (which may load the module holding the array),
            # a call takes no device memory from the driver or from torch's pool
            free1, _ = torch.cuda.mem_get_info()
            assert free1 == free0
            assert torch.cuda.memory_reserved() == reserved0
        # the pair set is an integer result: bit-exact
        assert torch.equal(bits, ref_bits)
        st = _lib.decode_stats(stats)
        assert np.array_equal(st["n_selected"], ref_stats["n_selected"])
        assert np.array_equal(st["cut_score"], ref_stats["cut_score"])
        assert np.array_equal(st["all_selected"], ref_stats["all_selected"])
        # the mass is summed with atomics (order varies): same bar as the oracle tests
        assert np.abs(st["mass"] - ref_stats["mass"]).max() < 1e-4


def test_static_scratch_rejects_problems_beyond_its_size():
    BAD = ctypes.c_void_p(0x100000)
    w = WORKLOADS[4]
    for dtype in ("bf16", "f32"):
        # 12 x 55296 x 24 fp32 scores = 64 MB > 16 MiB
        sh = LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, 0, *w.boxes[0], dtype)
        assert 4 * w.n_heads * w.s * 24 > _lib.STATIC_SELECT_SCRATCH_BYTES
        rc = _lib.lib().vmoba_score_select_static(ctypes.byref(sh.c()), BAD, BAD, 0.25, 0.0,
                                                  BAD, BAD, None)
        assert rc == -4             # VMOBA_ERR_WORKSPACE, nothing launched
