"""Counter-based generator for the synthetic layers the solver is measured on.

Definition (the same on every device; torch integer ops are exact, the float64
transcendental functions are the device's own):

* ``h(seed, stream, i) = splitmix64((seed << 48) ^ (stream << 40) ^ i)``; the
  splitmix64 finaliser is Steele, Lea and Flood's (OOPSLA 2014) as published by
  Vigna.
* Standard normal number ``i`` of a stream is the Box-Muller transform of
  ``u1 = ((h(2i) >> 11) + 0.5) / 2**53`` and ``u2 = (h(2i+1) >> 11) / 2**53``:
  ``z = sqrt(-2 ln u1) * cos(2 pi u2)``.
* Weights ``W[r, c] = float32(z_W[r*d_in + c] / sqrt(d_in))``.
* Channel scales ``s_c = exp(sigma * g_c)`` with ``g`` a normal stream; then
  ``m = floor(p*d_in + 0.5)`` outlier channels, picked by a partial Fisher-Yates
  shuffle driven by ``h``, get ``s_c *= f``.
* Activations ``X[t, c] = bf16(float32(z_X[t*d_in + c] * s_c))``, both
  roundings to nearest even.

The shapes and distributions follow the layers the SparseGPT review
(devpress.csdn.net, "SparseGPT: Massive Language Models Can Be Accurately
Pruned in One-Shot") prunes: OPT-, Llama- and Qwen-class linear layers whose
input channels have very uneven activation scales (section 五) with a few
outlier channels.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

_M64 = (1 << 64) - 1


def _s64(c: int) -> int:
    """Two's-complement int64 value of an unsigned 64-bit constant."""
    c &= _M64
    return c - (1 << 64) if c >= (1 << 63) else c


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_MIX1 = _s64(0xBF58476D1CE4E5B9)
_MIX2 = _s64(0x94D049BB133111EB)


def _lsr(x: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return torch.bitwise_and(torch.bitwise_right_shift(x, k), (1 << (64 - k)) - 1)


def _splitmix64(x: torch.Tensor) -> torch.Tensor:
    z = x + _GOLDEN
    z = torch.bitwise_xor(z, _lsr(z, 30)) * _MIX1
    z = torch.bitwise_xor(z, _lsr(z, 27)) * _MIX2
    return torch.bitwise_xor(z, _lsr(z, 31))


def _counter(seed: int, stream: int, idx: torch.Tensor) -> torch.Tensor:
    if not (0 <= seed < (1 << 15) and 0 <= stream < 256):
        raise ValueError("seed must be in [0, 2**15) and stream in [0, 256)")
    return torch.bitwise_xor(idx, (seed << 48) | (stream << 40))


def hash64(seed: int, stream: int, idx: torch.Tensor) -> torch.Tensor:
    return _splitmix64(_counter(seed, stream, idx))


def normals(seed: int, stream: int, start: int, count: int,
            device="cpu") -> torch.Tensor:
    """``count`` standard normals (float64) of a stream, from index ``start``."""
    if start < 0 or start + count > (1 << 39):
        raise ValueError("normal index out of the counter's range")
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    a = _lsr(hash64(seed, stream, 2 * i), 11).to(torch.float64)
    b = _lsr(hash64(seed, stream, 2 * i + 1), 11).to(torch.float64)
    u1 = (a + 0.5) * (2.0 ** -53)
    u2 = b * (2.0 ** -53)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def bf16_bits_to_f64(x: torch.Tensor) -> torch.Tensor:
    """Exact widening of a bf16 tensor to float64 (on the CPU)."""
    return x.to(torch.float32).to(torch.float64)


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer to prune: W is [d_out, d_in], X is [n_tok, d_in]."""
    name: str
    d_in: int
    d_out: int
    n_tok: int
    sigma: float = 1.0      # lognormal spread of the per-channel scales
    p_out: float = 0.01     # fraction of outlier channels
    f_out: float = 20.0     # outlier scale multiplier
    w_key: int = 0          # stream offset (x10) of this layer's weights
    x_key: int = 0          # stream offset (x10) of this layer's input
    runs: tuple = ("2:4",)  # "2:4" or "unstructured:<sparsity>"
    seed: int = 0

    @property
    def weights(self) -> int:
        return self.d_in * self.d_out

    def with_(self, **kw) -> "LayerSpec":
        d = dict(self.__dict__)
        d.update(kw)
        return LayerSpec(**d)


def channel_scales(spec: LayerSpec, device="cpu") -> torch.Tensor:
    """Per-input-channel scale s_c (float64, length d_in)."""
    d = spec.d_in
    g = normals(spec.seed, 3 + 10 * spec.x_key, 0, d, device="cpu")
    s = torch.exp(spec.sigma * g)
    m = int(math.floor(spec.p_out * d + 0.5))
    perm = list(range(d))
    if m:
        h = _lsr(hash64(spec.seed, 4 + 10 * spec.x_key,
                        torch.arange(m, dtype=torch.int64)), 11).tolist()
        for i in range(m):
            j = i + h[i] % (d - i)
            perm[i], perm[j] = perm[j], perm[i]
        s[torch.tensor(perm[:m])] *= spec.f_out
    return s.to(device)


_CHUNK = 1 << 24   # elements drawn per step (bounds the int64 temporaries)


def gen_weights(spec: LayerSpec, device="cpu", rows=None) -> torch.Tensor:
    """W [d_out, d_in] float32, or only the listed rows (a LongTensor/list)."""
    d, r = spec.d_in, spec.d_out
    stream = 1 + 10 * spec.w_key
    scale = 1.0 / math.sqrt(d)
    if rows is not None:
        rows = [int(x) for x in rows]
        out = torch.empty((len(rows), d), dtype=torch.float32, device=device)
        for k, rr in enumerate(rows):
            out[k] = (normals(spec.seed, stream, rr * d, d, device) * scale).to(torch.float32)
        return out
    out = torch.empty((r, d), dtype=torch.float32, device=device)
    step = max(1, _CHUNK // d)
    for r0 in range(0, r, step):
        r1 = min(r, r0 + step)
        z = normals(spec.seed, stream, r0 * d, (r1 - r0) * d, device)
        out[r0:r1] = (z * scale).to(torch.float32).view(r1 - r0, d)
    return out


def gen_activations(spec: LayerSpec, device="cpu", t0: int = 0,
                    count: int | None = None, scales=None) -> torch.Tensor:
    """Rows [t0, t0+count) of X as a bf16 tensor [count, d_in]."""
    d = spec.d_in
    if count is None:
        count = spec.n_tok - t0
    s = channel_scales(spec, device) if scales is None else scales.to(device)
    out = torch.empty((count, d), dtype=torch.bfloat16, device=device)
    stream = 2 + 10 * spec.x_key
    step = max(1, _CHUNK // d)
    for a in range(0, count, step):
        b = min(count, a + step)
        z = normals(spec.seed, stream, (t0 + a) * d, (b - a) * d, device).view(b - a, d)
        out[a:b] = (z * s).to(torch.float32).to(torch.bfloat16)
    return out


def _qwen_block(n_tok: int = 131072) -> list:
    """The seven linear layers of one Qwen3-32B-shaped decoder block.

    hidden 5120, 64 query heads and 8 key/value heads of width 128, MLP width
    25600. q/k/v share one input (attention input), gate/up share another.
    Each distinct input gets its own channel-scale draw (x_key).
    """
    base = dict(n_tok=n_tok, sigma=1.0, p_out=0.01, f_out=20.0, runs=("2:4",))
    return [
        LayerSpec("q_proj", 5120, 8192, w_key=0, x_key=0, **base),
        LayerSpec("k_proj", 5120, 1024, w_key=1, x_key=0, **base),
        LayerSpec("v_proj", 5120, 1024, w_key=2, x_key=0, **base),
        LayerSpec("o_proj", 8192, 5120, w_key=3, x_key=1, **base),
        LayerSpec("gate_proj", 5120, 25600, w_key=4, x_key=2, **base),
        LayerSpec("up_proj", 5120, 25600, w_key=5, x_key=2, **base),
        LayerSpec("down_proj", 25600, 5120, w_key=6, x_key=3, **base),
    ]


CONFIGS = {
    # small layer the oracle finishes in seconds
    "layer256": [LayerSpec("layer256", 256, 256, 2048)],
    # OPT-125M-shaped layer, 128 sequences x 2048 tokens
    "opt125m_768": [LayerSpec("opt125m_768", 768, 768, 128 * 2048,
                              runs=("2:4", "unstructured:0.5"))],
    # Llama-7B MLP down-projection
    "llama7b_down": [LayerSpec("llama7b_down", 11008, 4096, 131072,
                               sigma=1.5, p_out=0.005, f_out=50.0)],
    # Llama-7B q_proj, unstructured at three sparsities
    "llama7b_q": [LayerSpec("llama7b_q", 4096, 4096, 262144,
                            runs=("unstructured:0.5", "unstructured:0.7",
                                  "unstructured:0.8"))],
    # Qwen3-32B-shaped decoder block
    "qwen3_32b_block": _qwen_block(),
    # a Llama-7B-wide layer with a short calibration set, sized for profiler
    # captures of the factorisation and sweep kernels (X 268 MB > L2)
    "profile_4096": [LayerSpec("profile_4096", 4096, 4096, 32768, runs=("2:4",))],
}
