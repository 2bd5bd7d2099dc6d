"""Seeded synthetic inputs for the Kimi Delta Attention (KDA) layer.

This module is the one place that draws random inputs. Tests, ``bench.py`` and
``__graft_entry__.smoke()`` take inputs from here, and the same arrays go to the
CUDA library and to the CPU oracle. It holds none of the method's arithmetic:
only a counter-based generator and the input distributions of the workloads.

Generator: splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used counter-style. Element ``i`` of stream
``(seed, tag)`` is ``mix(key(seed, tag) + (i + 1) * 0x9E3779B97F4A7C15)``, so any
slice of a stream can be drawn on its own (a 1M-token sequence is drawn one
segment at a time). Uniforms are the top 53 bits plus one half, in (0, 1).
Normals use Box-Muller (cosine branch): z_j = sqrt(-2 ln u_2j) cos(2 pi u_2j+1).

Workload distributions (Kimi K3 technical FAQ, "What is KDA": queries and keys
are L2-normalised before the recurrence; the shapes and laws are those of the
KDA workloads named in the module docstring of ``bench.py``):
  q, k ~ N(0, 1), then L2-normalised per (token, head) in fp64;
  v ~ N(0, 1);
  beta = sigmoid(N(0, 1));
  g = log alpha = -softplus(N(0, 1)) * 0.1, per key channel;
  decode/verify states ~ N(0, 0.1^2).
The q, k, v arrays are rounded once to the I/O type (bf16 or fp32, round to
nearest even); g, beta and states are stored as fp32.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream tags, one per drawn quantity
TAG = {"q": 1, "k": 2, "v": 3, "g": 4, "beta": 5, "state": 6, "lens": 7,
       "draft": 8, "resume": 9, "perm": 10, "slots": 11, "misc": 12, "conv": 13,
       "convstate": 14}

_BLOCK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function applied elementwise to a uint64 array."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tag: int) -> np.uint64:
    with np.errstate(over="ignore"):
        a = _mix(np.array([np.uint64(seed & 0xFFFFFFFFFFFFFFFF)], dtype=np.uint64))
        b = _mix(np.array([np.uint64(tag) * GAMMA], dtype=np.uint64))
    return np.uint64(a[0] ^ b[0])


def _bits(key: np.uint64, start: int, n: int) -> np.ndarray:
    idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + idx * GAMMA)


def _uniform_block(key, start, n):
    b = _bits(key, start, n)
    return ((b >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def _normal_block(key, start, n):
    u = _uniform_block(key, 2 * start, 2 * n)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _blocked(fn, key, start, n, out_dtype=np.float64, transform=None):
    out = np.empty(n, dtype=out_dtype)

    def work(off):
        m = min(_BLOCK, n - off)
        x = fn(key, start + off, m)
        if transform is not None:
            x = transform(x)
        out[off:off + m] = x

    offs = list(range(0, n, _BLOCK))
    if len(offs) <= 1:
        for o in offs:
            work(o)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, offs))
    return out


def uniform(seed: int, tag: str, n: int, start: int = 0) -> np.ndarray:
    return _blocked(_uniform_block, stream_key(seed, TAG[tag]), start, n)


def normal(seed: int, tag: str, n: int, start: int = 0, out_dtype=np.float64,
           transform=None) -> np.ndarray:
    return _blocked(_normal_block, stream_key(seed, TAG[tag]), start, n, out_dtype, transform)


def _to_io(x64: np.ndarray, io: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x64, dtype=np.float32))
    if io == "bf16":
        return t.to(torch.bfloat16)
    if io == "fp32":
        return t
    raise ValueError(io)


def _normalised_rows(seed, tag, t0, T, H, d, io):
    """[T, H, d] standard normals from token t0 on, L2-normalised per row (fp64)."""
    out = torch.empty((T, H, d), dtype=torch.bfloat16 if io == "bf16" else torch.float32)
    rows_per_block = max(1, _BLOCK // (H * d))
    key = stream_key(seed, TAG[tag])

    def work(r0):
        r1 = min(T, r0 + rows_per_block)
        x = _normal_block(key, (t0 + r0) * H * d, (r1 - r0) * H * d).reshape(r1 - r0, H, d)
        x /= np.sqrt((x * x).sum(axis=-1, keepdims=True))
        out[r0:r1] = _to_io(x, io)

    starts = list(range(0, T, rows_per_block))
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, starts))
    return out


def _plain_rows(seed, tag, t0, T, H, d, io):
    out = torch.empty((T, H, d), dtype=torch.bfloat16 if io == "bf16" else torch.float32)
    rows_per_block = max(1, _BLOCK // (H * d))
    key = stream_key(seed, TAG[tag])

    def work(r0):
        r1 = min(T, r0 + rows_per_block)
        x = _normal_block(key, (t0 + r0) * H * d, (r1 - r0) * H * d).reshape(r1 - r0, H, d)
        out[r0:r1] = _to_io(x, io)

    starts = list(range(0, T, rows_per_block))
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, starts))
    return out


def _gate(x):
    # g = log alpha = -softplus(z) * 0.1, evaluated stably in fp64
    return -(np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))) * 0.1


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def token_inputs(seed: int, T: int, H: int, dk: int, dv: int, io: str = "bf16",
                 t0: int = 0) -> dict:
    """Per-token inputs for tokens [t0, t0+T) of one seeded token stream.

    Returns CPU tensors q, k [T,H,dk] and v [T,H,dv] in the I/O type, g [T,H,dk]
    fp32 and beta [T,H] fp32. A packed ragged batch is simply consecutive tokens
    of the stream; a long sequence can be drawn segment by segment via t0.
    """
    q = _normalised_rows(seed, "q", t0, T, H, dk, io)
    k = _normalised_rows(seed, "k", t0, T, H, dk, io)
    v = _plain_rows(seed, "v", t0, T, H, dv, io)
    g = torch.from_numpy(normal(seed, "g", T * H * dk, start=t0 * H * dk, out_dtype=np.float32,
                                transform=_gate).reshape(T, H, dk))
    beta = torch.from_numpy(normal(seed, "beta", T * H, start=t0 * H, out_dtype=np.float32,
                                   transform=_sigmoid).reshape(T, H))
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta}


def raw_qk(seed: int, T: int, H: int, dk: int, io: str = "bf16", t0: int = 0) -> dict:
    """Raw (pre-front-end) q and k of tokens [t0, t0+T): N(0, 1) per element, rounded
    to the I/O type (tags q and k of the same streams as token_inputs, unnormalised)."""
    return {"q": _plain_rows(seed, "q", t0, T, H, dk, io),
            "k": _plain_rows(seed, "k", t0, T, H, dk, io)}


def conv_weights(seed: int, H: int, dk: int, taps: int) -> tuple:
    """Short-conv weights for q and k, [H, dk, taps] fp32 each: N(0, 1) / sqrt(taps)."""
    x = normal(seed, "conv", 2 * H * dk * taps, out_dtype=np.float32,
               transform=lambda z: z / math.sqrt(taps)).reshape(2, H, dk, taps)
    return torch.from_numpy(x[0].copy()), torch.from_numpy(x[1].copy())


def conv_states(seed: int, n: int, H: int, dk: int, taps: int, io: str = "bf16") -> torch.Tensor:
    """n conv states [n, 2, H, dk, taps-1] fp32 holding earlier raw inputs: N(0, 1)
    values rounded to the I/O type (what a carried conv state contains)."""
    x = normal(seed, "convstate", n * 2 * H * dk * (taps - 1)).reshape(n, 2, H, dk, taps - 1)
    return _to_io(x, io).float()


def states(seed: int, n: int, H: int, dk: int, dv: int, std: float = 0.1, tag: str = "state",
           start: int = 0) -> torch.Tensor:
    """n fp32 states [n, H, dk, dv] with entries N(0, std^2)."""
    x = normal(seed, tag, n * H * dk * dv, start=start * H * dk * dv, out_dtype=np.float32,
               transform=lambda z: z * std)
    return torch.from_numpy(x.reshape(n, H, dk, dv))


def draft_lengths(seed: int, n: int, lo: int = 1, hi: int = 8, start: int = 0) -> list[int]:
    """n integers uniform in {lo..hi} (speculative draft lengths), elements start..
    start+n-1 of the stream."""
    u = uniform(seed, "draft", n, start=start)
    return [lo + int(x * (hi - lo + 1)) for x in u]


def lognormal_lengths(seed: int, n: int, mu: float, sigma: float, lo: int, hi: int) -> list[int]:
    """n lengths round(exp(mu + sigma z)) clipped to [lo, hi]."""
    z = normal(seed, "lens", n)
    return [int(min(hi, max(lo, round(math.exp(mu + sigma * x))))) for x in z]


def permutation(seed: int, n: int, tag: str = "perm") -> list[int]:
    """A seeded permutation of range(n) (sort by uniform keys)."""
    u = uniform(seed, tag, n)
    return [int(i) for i in np.argsort(u, kind="stable")]


def randint(seed: int, tag: str, n: int, lo: int, hi: int) -> list[int]:
    """n integers uniform in {lo..hi}."""
    u = uniform(seed, tag, n)
    return [lo + int(x * (hi - lo + 1)) for x in u]


# ---------------------------------------------------------------------------
# The same streams drawn on a CUDA device (torch, int64 with wrapping arithmetic
# standing in for uint64), for benchmark inputs of tens of GB that the host would
# take minutes to draw. The bits of every stream are identical to the host's; the
# fp64 log/cos/sqrt/exp of the device library can differ from the host's in the
# last bit, so an element can differ by one rounding step after the cast to the I/O
# type. Parity tests use the host generator above.
# ---------------------------------------------------------------------------
def _s64(x: int) -> int:
    return x - (1 << 64) if x >= (1 << 63) else x


_GAMMA_S, _M1_S, _M2_S = _s64(int(GAMMA)), _s64(int(_M1)), _s64(int(_M2))


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_dev(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _M1_S
    z = (z ^ _srl(z, 27)) * _M2_S
    return z ^ _srl(z, 31)


def _normal_dev(key: np.uint64, start: int, n: int, device) -> torch.Tensor:
    """float64 normals of elements start .. start+n-1 of a stream, on `device`."""
    k = _s64(int(key))
    idx = torch.arange(2 * start + 1, 2 * start + 2 * n + 1, dtype=torch.int64, device=device)
    b = _mix_dev(k + idx * _GAMMA_S)
    u = (_srl(b, 11).to(torch.float64) + 0.5) * (1.0 / 9007199254740992.0)
    u1, u2 = u[0::2], u[1::2]
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)


def _rows_dev(seed, tag, t0, T, H, d, io, device, normalise):
    out = torch.empty((T, H, d), dtype=torch.bfloat16 if io == "bf16" else torch.float32,
                      device=device)
    key = stream_key(seed, TAG[tag])
    rows = max(1, (1 << 24) // (H * d))
    for r0 in range(0, T, rows):
        r1 = min(T, r0 + rows)
        x = _normal_dev(key, (t0 + r0) * H * d, (r1 - r0) * H * d, device).view(r1 - r0, H, d)
        if normalise:
            x = x / torch.sqrt((x * x).sum(dim=-1, keepdim=True))
        out[r0:r1] = x.float().to(out.dtype)
    return out


def _flat_dev(seed, tag, start, n, device, transform):
    out = torch.empty(n, dtype=torch.float32, device=device)
    key = stream_key(seed, TAG[tag])
    blk = 1 << 24
    for o in range(0, n, blk):
        m = min(blk, n - o)
        out[o:o + m] = transform(_normal_dev(key, start + o, m, device)).float()
    return out


def token_inputs_device(seed: int, T: int, H: int, dk: int, dv: int, io: str = "bf16",
                        t0: int = 0, device="cuda") -> dict:
    """token_inputs drawn on a CUDA device (see the note above)."""
    gate = lambda x: -(torch.clamp(x, min=0.0) + torch.log1p(torch.exp(-x.abs()))) * 0.1  # noqa: E731
    return {"q": _rows_dev(seed, "q", t0, T, H, dk, io, device, True),
            "k": _rows_dev(seed, "k", t0, T, H, dk, io, device, True),
            "v": _rows_dev(seed, "v", t0, T, H, dv, io, device, False),
            "g": _flat_dev(seed, "g", t0 * H * dk, T * H * dk, device, gate).view(T, H, dk),
            "beta": _flat_dev(seed, "beta", t0 * H, T * H, device, torch.sigmoid).view(T, H)}


def states_device(seed: int, n: int, H: int, dk: int, dv: int, std: float = 0.1,
                  tag: str = "state", device="cuda") -> torch.Tensor:
    """states drawn on a CUDA device (see the note above)."""
    return _flat_dev(seed, tag, 0, n * H * dk * dv, device, lambda z: z * std).view(n, H, dk, dv)


# ---------------------------------------------------------------------------
# The five KDA workloads. Shapes and laws follow the workload table of the
# KDA hot path; seeds are 1000 + workload index.
# ---------------------------------------------------------------------------
WORKLOADS = {
    "tiny_fp32": dict(seed=1000, H=2, T=64, d=32, chunk=16, io="fp32"),
    "prefill_8k": dict(seed=1001, H=64, T=8192, d=128, chunk=64, io="bf16", snap=256),
    "decode_verify_512": dict(seed=1002, n_seq=512, H=64, d=128, io="bf16", state_std=0.1,
                              draft_lo=1, draft_hi=8),
    "ragged_prefix_32": dict(seed=1003, n_seq=32, H=64, d=128, chunk=64, io="bf16", snap=256,
                             mu=math.log(4096), sigma=1.0, lo=512, hi=65536,
                             prefix=16384, n_resume=16),
    "long_1m": dict(seed=1004, H=64, T=1 << 20, d=128, chunk=64, io="bf16", snap=4096,
                    segment=1 << 16),
}


def ragged_plan(seed: int, n_seq: int, mu: float, sigma: float, lo: int, hi: int,
                prefix: int, n_resume: int, snap: int) -> dict:
    """Sequence lengths and resume points of the ragged packed-prefill workload.

    Each sequence's lognormal length counts its new tokens. ``n_resume`` of the
    sequences (a seeded choice) resume from the state after m*snap tokens of a
    shared prefix of ``prefix`` tokens, m uniform in {1..prefix/snap}; their
    start_pos is m*snap. The others start from the zero state at position 0.
    """
    lens = lognormal_lengths(seed, n_seq, mu, sigma, lo, hi)
    perm = permutation(seed, n_seq)
    resumers = sorted(perm[:n_resume])
    ms = randint(seed, "resume", n_resume, 1, prefix // snap)
    start = [0] * n_seq
    for s, m in zip(resumers, ms):
        start[s] = m * snap
    return {"lens": lens, "start_pos": start, "resumers": resumers,
            "resume_block": dict(zip(resumers, ms))}
