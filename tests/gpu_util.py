"""Helpers shared by the GPU parity tests: seeded inputs on both sides,
bitmap packing, and the pair-set comparison rule."""
from __future__ import annotations

import math

import numpy as np

import synth
from synth.video_latents import round_to

BAND_REL = 1e-4          # pairs whose score is within 1e-4 relative of the cut are not compared
TOL = {"f32": 1e-4, "bf16": 2e-2}   # max-abs error of O, dQ, dK, dV against fp64


def out_err(got: np.ndarray, exact: np.ndarray, dtype: str) -> float:
    """Max-abs error of a stored output against the exact fp64 result, beyond the
    half-ulp rounding that storing the exact value in ``dtype`` costs by itself."""
    import oracle as O
    return O.io_excess_error(got, exact, dtype)


def workload_arrays(w, layer: int, with_dout: bool = False):
    """fp64 arrays of the workload's inputs, already rounded to the I/O dtype."""
    q, k, v = synth.make_qkv(w.wid, layer, w.T, w.H, w.W, w.n_heads, w.head_dim,
                             kind=w.kind, head_gain=w.head_gain)
    out = [round_to(x, w.dtype) for x in (q, k, v)]
    if with_dout:
        out.append(round_to(synth.make_dout(w.wid, layer, w.s, w.n_heads, w.head_dim), w.dtype))
    return out


def to_device(x: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def from_device(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def pack_bits(mask: np.ndarray) -> np.ndarray:
    """[..., N_b] bool -> [..., ceil(N_b/32)] int32, bit j%32 of word j//32."""
    nb = mask.shape[-1]
    wb = (nb + 31) // 32
    pad = np.zeros(mask.shape[:-1] + (wb * 32,), dtype=bool)
    pad[..., :nb] = mask
    bytes_ = np.packbits(pad, axis=-1, bitorder="little")
    return np.ascontiguousarray(bytes_).view("<u4").astype(np.uint32).view(np.int32)


def unpack_bits(words: np.ndarray, nb: int) -> np.ndarray:
    w = np.ascontiguousarray(words).view(np.uint32).astype("<u4")
    bits = np.unpackbits(w.view(np.uint8), axis=-1, bitorder="little")
    return bits[..., :nb].astype(bool)


def pair_set_mismatch(gpu_mask_h, S_h, oracle_mask_h, cut: float) -> int:
    """Pairs that differ and lie outside the 1e-4 relative band around the cut."""
    band = np.abs(S_h - cut) <= BAND_REL * abs(cut)
    return int(((gpu_mask_h != oracle_mask_h) & ~band).sum())


def sample_rows(s: int, n: int, seed: int, must=()) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in rng.choice(s, size=min(n, s), replace=False))
    rows.update(int(r) for r in must)
    rows.update((0, s - 1))
    return np.array(sorted(rows))


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
