"""The video-latent input recipe of ``video_latents`` evaluated with torch on a
device, for benchmarks whose inputs are too large to draw on the host in
reasonable time (the 30-layer, 75600-token stack draws 30 x 4 tensors of
11.6 M values).

Same counter-based splitmix64 stream, same seeds, same Box-Muller, blur,
projection and gains as the numpy generator: the 64-bit stream and the
uniforms are bit-identical, and the normals agree with numpy's to a few ulp
of fp64 (log and cos may round differently), which the bf16 rounding of the
stored inputs almost always absorbs.  The parity tests use the numpy
generator; only bench.py draws from this one.  It holds no step of the
attention method.
"""
from __future__ import annotations

import math

import torch

from .video_latents import (_PART_EPS, _PART_FIELDS, _PART_GAIN, _PART_W, _PART_W_DELTA,
                            _gauss_kernel, seed_for)

_MASK64 = (1 << 64) - 1


def _s64(x: int) -> int:
    """An unsigned 64-bit constant as the signed int64 with the same bits."""
    x &= _MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_M1 = _s64(0xBF58476D1CE4E5B9)
_M2 = _s64(0x94D049BB133111EB)


def _lshr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns (torch's >> is arithmetic)."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def splitmix64_stream(seed: int, n: int, offset: int = 0, device="cuda") -> torch.Tensor:
    """Element i is mix64(seed + (offset + i + 1) * golden), as int64 bit patterns
    (two's-complement wrap-around is the mod 2^64 arithmetic of the stream)."""
    z = torch.arange(offset + 1, offset + n + 1, dtype=torch.int64, device=device)
    z = z * _GOLDEN + _s64(seed)
    z = (z ^ _lshr(z, 30)) * _M1
    z = (z ^ _lshr(z, 27)) * _M2
    return z ^ _lshr(z, 31)


def uniform01(seed: int, n: int, device="cuda") -> torch.Tensor:
    """n uniforms in (0, 1] as float64: ((z >> 11) + 1) * 2^-53."""
    z = _lshr(splitmix64_stream(seed, n, device=device), 11)
    return (z.to(torch.float64) + 1.0) * (2.0 ** -53)


def standard_normal(seed: int, n: int, device="cuda") -> torch.Tensor:
    """n N(0,1) float64 draws by Box-Muller on consecutive uniform pairs."""
    u = uniform01(seed, 2 * n, device).view(n, 2)
    return torch.sqrt(-2.0 * torch.log(u[:, 0])) * torch.cos(u[:, 1] * (2.0 * math.pi))


def _blur_axis(a: torch.Tensor, axis: int, sigma: float) -> torch.Tensor:
    k = torch.tensor(_gauss_kernel(sigma), dtype=a.dtype, device=a.device)
    r = (k.numel() - 1) // 2
    n = a.shape[axis]
    idx = torch.clamp(torch.arange(-r, n + r, device=a.device), 0, n - 1)   # clamp-to-edge
    padded = torch.index_select(a, axis, idx)
    out = torch.zeros_like(a)
    for t in range(k.numel()):
        out += k[t] * padded.narrow(axis, t, n)
    return out


def smooth_fields(T, H, W, r, seed, sigma=(1.0, 2.0, 2.0), device="cuda") -> torch.Tensor:
    """r blurred unit-variance fields on the grid, [s][r] float64."""
    g = standard_normal(seed, r * T * H * W, device).view(r, T, H, W)
    for ax, sg in zip((1, 2, 3), sigma):
        g = _blur_axis(g, ax, sg)
    g = g.reshape(r, -1)
    g = (g - g.mean(dim=1, keepdim=True)) / g.std(dim=1, unbiased=False, keepdim=True)
    return g.T.contiguous()


def _iid(seed, s, n_heads, d, device):
    return standard_normal(seed, s * n_heads * d, device).view(s, n_heads, d)


def make_qkv(workload_id, layer, T, H, W, n_heads, head_dim, kind="smooth", head_gain=False,
             rank=8, coherence=0.4, device="cuda", dtype=torch.bfloat16):
    """Q, K, V [s][n_heads][head_dim] on ``device``, rounded to ``dtype`` (the
    numpy generator's recipe; see its module doc)."""
    s, d = T * H * W, head_dim
    if kind == "iid":
        return tuple(_iid(seed_for(workload_id, layer, x, _PART_EPS), s, n_heads, d, device)
                     .to(dtype) for x in ("q", "k", "v"))
    if kind != "smooth":
        raise ValueError(f"unknown input kind {kind!r}")
    sd = math.sqrt(1.0 / rank)
    F = smooth_fields(T, H, W, rank, seed_for(workload_id, layer, "q", _PART_FIELDS),
                      device=device)
    Wq = standard_normal(seed_for(workload_id, layer, "q", _PART_W), n_heads * rank * d,
                         device).view(n_heads, rank, d) * sd
    Wk = Wq + 0.5 * sd * standard_normal(seed_for(workload_id, layer, "k", _PART_W_DELTA),
                                         n_heads * rank * d, device).view(n_heads, rank, d)
    Fv = smooth_fields(T, H, W, rank, seed_for(workload_id, layer, "v", _PART_FIELDS),
                       device=device)
    Wv = standard_normal(seed_for(workload_id, layer, "v", _PART_W), n_heads * rank * d,
                         device).view(n_heads, rank, d) * sd
    a = float(coherence)
    norm = 1.0 / math.sqrt(a * a + 1.0)
    proj = lambda F_, W_: torch.matmul(F_[None], W_).permute(1, 0, 2)   # noqa: E731
    out = []
    for name, F_, W_ in (("q", F, Wq), ("k", F, Wk), ("v", Fv, Wv)):
        x = (a * proj(F_, W_) + _iid(seed_for(workload_id, layer, name, _PART_EPS), s, n_heads,
                                     d, device)) * norm
        if head_gain and name != "v":
            c = 0.5 + 1.5 * uniform01(seed_for(workload_id, layer, "q", _PART_GAIN), n_heads,
                                      device)
            x = x * c[None, :, None]
        out.append(x.to(torch.float32).to(dtype).contiguous())
    return tuple(out)


def make_dout(workload_id, layer, s, n_heads, head_dim, device="cuda", dtype=torch.bfloat16):
    """dO ~ N(0, 1) [s][n_heads][head_dim] on ``device``."""
    return _iid(seed_for(workload_id, layer, "dout", _PART_EPS), s, n_heads, head_dim,
                device).to(torch.float32).to(dtype).contiguous()
