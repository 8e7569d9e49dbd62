"""Seeded synthetic inputs (no codec arithmetic lives here).

One counter-based generator serves every test, the benchmark and the CPU
baseline, on CPU or GPU, so the oracle and the CUDA path always read the same
host bytes.  Definition:

* stream key: ``key = splitmix64(seed * 2**32 + tensor_id)``
* element i of the stream: ``u64_i = splitmix64(key + (i + 1) * 0x9E3779B97F4A7C15)``
  (splitmix64 = Steele, Lea & Flood's SplitMix64 output function)
* uniform: ``(u64 >> 11) * 2**-53`` in [0, 1)
* normal: Box-Muller on pairs (u1, u2) = (uniform_{2p}, uniform_{2p+1}):
  ``r = sqrt(-2 ln(1 - u1))``, ``z_{2p} = r cos(2 pi u2)``, ``z_{2p+1} = r sin(2 pi u2)``
* Student-t(4): ``T = Z / sqrt(chi2_4 / 4)``, ``chi2_4 = -2 ln((1 - u_a)(1 - u_b))``

All integer arithmetic is done on int64 tensors with wrap-around (two's
complement), logical shifts emulated by masking.  Transcendentals run in fp64
on the tensor's device, so CPU and GPU streams can differ in the last bit;
every consumer therefore generates once and hands the same bytes to both sides.

Workloads (shapes and value distributions of the pages' Llama/Qwen-class
layers; the pages' own checkpoints and wikitext-2 are not used):
  * ``single_matrix``: 2048x2048 fp32 ~N(0, 0.02^2), x fp32 ~N(0,1)
  * ``llama3_8b_layer``: q,o 4096x4096; k,v 1024x4096; gate,up 14336x4096;
    down 4096x14336; bf16 ~N(0, 0.02^2) with 1% of input columns replaced by
    0.02*10*T, T ~ Student-t(4); x bf16 ~N(0,1)
  * ``ffn_70b``: gate,up 28672x8192; down 8192x28672; bf16 ~N(0, 0.015^2)
  * ``prefill``: W 8192x8192 bf16 ~N(0, 0.02^2); X 2048x8192 bf16 ~N(0,1)
"""
from __future__ import annotations

import math

import torch

_MASK64 = (1 << 64) - 1


def _s64(v: int) -> int:
    """Reinterpret an unsigned 64-bit constant as int64."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_M1 = _s64(0xBF58476D1CE4E5B9)
_M2 = _s64(0x94D049BB133111EB)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _M1
    z = (z ^ _srl(z, 27)) * _M2
    return z ^ _srl(z, 31)


def _mix_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return _s64(_mix_int(((seed << 32) + tensor_id + 0x9E3779B97F4A7C15) & _MASK64))


def uniform(seed: int, tensor_id: int, count: int, device="cpu", offset: int = 0) -> torch.Tensor:
    """fp64 uniforms in [0, 1): elements offset .. offset+count-1 of the stream."""
    key = stream_key(seed, tensor_id)
    i = torch.arange(offset + 1, offset + count + 1, dtype=torch.int64, device=device)
    z = _mix(key + i * _GOLDEN)
    return _srl(z, 11).to(torch.float64) * (2.0 ** -53)


def normal(seed: int, tensor_id: int, count: int, device="cpu") -> torch.Tensor:
    """fp64 standard normals, Box-Muller on consecutive uniform pairs."""
    pairs = (count + 1) // 2
    u = uniform(seed, tensor_id, 2 * pairs, device).view(pairs, 2)
    r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))
    th = (2.0 * math.pi) * u[:, 1]
    z = torch.stack((r * torch.cos(th), r * torch.sin(th)), dim=1).reshape(-1)
    return z[:count]


def student_t4(seed: int, tensor_id: int, count: int, device="cpu") -> torch.Tensor:
    z = normal(seed, tensor_id, count, device)
    u = uniform(seed, tensor_id + (1 << 20), 2 * count, device).view(count, 2)
    chi2 = -2.0 * (torch.log1p(-u[:, 0]) + torch.log1p(-u[:, 1]))
    return z / torch.sqrt(chi2 / 4.0)


def gaussian_matrix(seed: int, tensor_id: int, rows: int, cols: int, std: float,
                    dtype=torch.bfloat16, device="cpu", chunk_rows: int | None = None) -> torch.Tensor:
    """rows x cols matrix ~N(0, std^2) rounded (nearest-even) to ``dtype``.

    Generated in row chunks (the stream index is the row-major element index)
    to bound temporary memory on large matrices."""
    out = torch.empty((rows, cols), dtype=dtype, device=device)
    if chunk_rows is None:
        chunk_rows = max(1, (1 << 24) // max(cols, 1))
    # Box-Muller pairs must not straddle chunks: keep chunk sizes even
    if (chunk_rows * cols) % 2:
        chunk_rows += 1
    key_rows = 0
    while key_rows < rows:
        r = min(chunk_rows, rows - key_rows)
        start = key_rows * cols
        pairs = (r * cols + 1) // 2
        u = uniform(seed, tensor_id, 2 * pairs, device, offset=start).view(pairs, 2)
        rad = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))
        th = (2.0 * math.pi) * u[:, 1]
        z = torch.stack((rad * torch.cos(th), rad * torch.sin(th)), dim=1).reshape(-1)[: r * cols]
        out[key_rows:key_rows + r] = (z * std).view(r, cols).to(dtype)
        key_rows += r
    return out


def outlier_columns(seed: int, tensor_id: int, cols: int, frac: float = 0.01, device="cpu") -> torch.Tensor:
    """ceil(frac * cols) distinct column indices drawn uniformly without replacement."""
    cnt = math.ceil(frac * cols)
    u = uniform(seed, tensor_id + (2 << 20), cols, device)
    return torch.argsort(u)[:cnt].sort().values


def llama_weight(seed: int, tensor_id: int, rows: int, cols: int, std: float = 0.02,
                 outlier_frac: float = 0.01, device="cpu") -> torch.Tensor:
    """bf16 ~N(0, std^2) with a seeded 1% of input columns replaced by std*10*T, T~t(4)."""
    W = gaussian_matrix(seed, tensor_id, rows, cols, std, torch.bfloat16, device)
    if outlier_frac > 0:
        cols_idx = outlier_columns(seed, tensor_id, cols, outlier_frac, device)
        t = student_t4(seed, tensor_id + (3 << 20), rows * cols_idx.numel(), device)
        W[:, cols_idx] = (std * 10.0 * t).view(rows, cols_idx.numel()).to(torch.bfloat16)
    return W


# Llama-3-8B decoder layer shapes: name -> (out_features N, in_features K)
LLAMA3_8B_LAYER = {
    "q": (4096, 4096), "k": (1024, 4096), "v": (1024, 4096), "o": (4096, 4096),
    "gate": (14336, 4096), "up": (14336, 4096), "down": (4096, 14336),
}
# which activation vector feeds each matrix (q/k/v share one input, gate/up another)
LLAMA3_8B_INPUTS = {"q": "attn", "k": "attn", "v": "attn", "o": "attn_out",
                    "gate": "ffn", "up": "ffn", "down": "ffn_mid"}

FFN_70B = {"gate": (28672, 8192), "up": (28672, 8192), "down": (8192, 28672)}


def llama3_8b_layer(seed: int = 0, device="cpu", names=None):
    """(weights {name: bf16 [N, K]}, activations {input: bf16 [K]}) for one layer."""
    names = list(LLAMA3_8B_LAYER) if names is None else names
    weights = {}
    for tid, name in enumerate(LLAMA3_8B_LAYER):
        if name in names:
            n, k = LLAMA3_8B_LAYER[name]
            weights[name] = llama_weight(seed + tid, 0, n, k, device=device)
    acts = {}
    for aid, act in enumerate(("attn", "attn_out", "ffn", "ffn_mid")):
        k = 14336 if act == "ffn_mid" else 4096
        acts[act] = gaussian_matrix(1, aid, 1, k, 1.0, torch.bfloat16, device).view(k)
    return weights, acts


def single_matrix(device="cpu"):
    """2048x2048 fp32 ~N(0, 0.02^2) (seed 0) and x fp32 ~N(0,1) (seed 1)."""
    W = gaussian_matrix(0, 0, 2048, 2048, 0.02, torch.float32, device)
    x = gaussian_matrix(1, 0, 1, 2048, 1.0, torch.float32, device).view(2048)
    return W, x
