"""Seeded model parameters for the oracle.

Parameter list.  The parameters are enumerated in a fixed order; parameter
number p (0, 1, 2, ...) is the p-th entry of ``param_specs(cfg)``.  Matrices
are stored as [out, in] (row-major, the input dimension contiguous), so a
linear map is ``y = x @ W.T + b``.

Distribution.  Weight matrices, biases, the per-block modulation tables and
the LoRA factors are N(0, 0.02) -- the synthetic configs state N(0, 0.02)
weights; biases and LoRA B are drawn rather than zeroed so every term is
exercised.  RMSNorm / QK-norm gains are 1 (standard initialisation).

Counter-based generator (one published construction, written out here; the
CUDA library implements the same rule independently):

* ``key_p = seed XOR (p * G mod 2^64)`` with G = 0x9E3779B97F4A7C15,
* element e (row-major index) uses counters ``c_k = key_p + 2e + k`` (mod 2^64),
  k = 0, 1,
* ``r_k = splitmix64(c_k)``: the output of Steele, Lea & Flood's SplitMix64
  step taken from state ``c_k`` (add G, then the two xor-shift-multiply
  rounds with 0xBF58476D1CE4E5B9 and 0x94D049BB133111EB, then a final
  xor-shift by 31),
* ``u_k = ((r_k >> 11) + 1) * 2^-53`` in (0, 1],
* Box-Muller ``z = sqrt(-2 ln u_0) * cos(2 pi u_1)`` in float64, then
  ``float32(std * z)`` with round-to-nearest-even,
* for bf16 models every parameter is then rounded to bf16 (RNE) and the model
  is defined by those rounded values.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .config import WamConfig

G = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)
STD = 0.02
_CHUNK = 1 << 20


def _expert_specs(cfg: WamConfig, expert: str):
    v = expert == "video"
    d = cfg.d_video if v else cfg.d_action
    F = cfg.ffn_video if v else cfg.ffn_action
    A = cfg.attn_dim
    s = []
    p = expert + "."
    s += [(p + "t1.w", (d, 256), STD), (p + "t1.b", (d,), STD),
          (p + "t2.w", (d, d), STD), (p + "t2.b", (d,), STD),
          (p + "mod.w", (6 * d, d), STD), (p + "mod.b", (6 * d,), STD)]
    if v and cfg.video_patch_dim > 0:
        s += [(p + "in.w", (d, cfg.video_patch_dim), STD), (p + "in.b", (d,), STD)]
    if not v:
        s += [(p + "in.w", (d, cfg.action_dim), STD), (p + "in.b", (d,), STD)]
    lora = (not v) and cfg.lora_rank > 0
    r = cfg.lora_rank
    for i in range(cfg.n_blocks):
        b = f"{p}blk{i}."
        s += [(b + "T", (6, d), STD),
              (b + "qkv.w", (3 * A, d), STD), (b + "qkv.b", (3 * A,), STD),
              (b + "qn.g", (A,), None), (b + "kn.g", (A,), None),
              (b + "o.w", (d, A), STD), (b + "o.b", (d,), STD),
              (b + "ffn1.w", (F, d), STD), (b + "ffn1.b", (F,), STD),
              (b + "ffn2.w", (d, F), STD), (b + "ffn2.b", (d,), STD)]
        if lora:
            s += [(b + "qkv.la", (r, d), STD), (b + "qkv.lb", (3 * A, r), STD),
                  (b + "o.la", (r, A), STD), (b + "o.lb", (d, r), STD),
                  (b + "ffn1.la", (r, d), STD), (b + "ffn1.lb", (F, r), STD),
                  (b + "ffn2.la", (r, F), STD), (b + "ffn2.lb", (d, r), STD)]
    if v and cfg.video_has_output:
        s += [(p + "fn.g", (d,), None), (p + "out.w", (cfg.video_patch_dim, d), STD),
              (p + "out.b", (cfg.video_patch_dim,), STD)]
    if not v:
        s += [(p + "fn.g", (d,), None), (p + "out.w", (cfg.action_dim, d), STD),
              (p + "out.b", (cfg.action_dim,), STD)]
    return s


def param_specs(cfg: WamConfig):
    """[(name, shape, std or None for unit gains)] in generation order."""
    return _expert_specs(cfg, "video") + _expert_specs(cfg, "action")


def splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 output for state ``x`` (uint64 array, wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = x + G
        z = (z ^ (z >> np.uint64(30))) * _C1
        z = (z ^ (z >> np.uint64(27))) * _C2
        return z ^ (z >> np.uint64(31))


def normal_block(seed: int, pid: int, start: int, count: int) -> np.ndarray:
    """Standard normals (float64) for elements [start, start+count) of parameter pid."""
    with np.errstate(over="ignore"):
        key = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) ^ (np.uint64(pid) * G)
        e2 = np.arange(start, start + count, dtype=np.uint64) * np.uint64(2)
        c0 = key + e2
        c1 = c0 + np.uint64(1)
    u0 = ((splitmix64(c0) >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
    u1 = ((splitmix64(c1) >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
    return np.sqrt(-2.0 * np.log(u0)) * np.cos(2.0 * np.pi * u1)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 (ties to even), returned as float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1))
    return _POOL


_POOL = None


def generate_param(cfg: WamConfig, seed: int, pid: int, shape, std) -> np.ndarray:
    n = int(np.prod(shape))
    if std is None:
        out = np.ones(n, np.float32)
    else:
        out = np.empty(n, np.float32)

        def fill(s):
            c = min(_CHUNK, n - s)
            out[s:s + c] = (std * normal_block(seed, pid, s, c)).astype(np.float32)
        starts = range(0, n, _CHUNK)
        if n > _CHUNK:   # chunks are independent (counter-based); numpy releases the GIL
            list(_pool().map(fill, starts))
        else:
            fill(0)
    if cfg.dtype == "bf16":
        out = round_bf16(out)
    return out.reshape(shape)


def generate_params(cfg: WamConfig, seed: int, only=None) -> dict:
    """All parameters as float32 arrays (exact values of the model).

    ``only``: optional predicate on the name, to generate a subset (the
    generator is random access, so a subset has the same values).
    """
    out = {}
    for pid, (name, shape, std) in enumerate(param_specs(cfg)):
        if only is not None and not only(name):
            continue
        out[name] = generate_param(cfg, seed, pid, shape, std)
    return out
