"""Seeded synthetic inputs for CommVQ decode attention.

This module holds no arithmetic of the method: it only draws random tensors in the
layouts the library and the oracle both take, so that the two sides can be compared
on identical inputs.  Both the tests and the benchmark use it.

Layouts (8-scalar groups; the 64-scalar-group workloads in brackets):
  q          [B, Hq, 128]            float32 values (bf16 workloads: the exact
                                      float32 value of each bf16, plus the raw bits)
  key_cb     [Hkv, 16, R, 256, 4, 2]  float32 (re, im) of each complex codeword
                                     [Hkv, 2, R, 64, 32, 2]
  val_cb     [Hkv, 16, R, 256, 8]     float32  [Hkv, 2, R, 64, 64]
  key_codes  [B, Hkv, T_cap, R, 16]   uint8    [B, Hkv, 2, R, T_cap] (planar)
  val_codes  [B, Hkv, T_cap, R, 16]   uint8    [B, Hkv, 2, R, T_cap]
  seq_lens   [B]                      int32
  new keys / values [B, Hkv, 128]     float32 (new_tokens: one decode step's append)

Every tensor and every layer draws from its own stream of
numpy.random.SeedSequence(seed).spawn(...), so workloads are reproducible bit for bit.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

N_CODES = 256
ROPE_BASE = 500000.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    t_cap: int
    R: int
    q_dtype: str                 # "f32" | "bf16"
    cb_std: float                # std of every codebook entry
    codes: str = "uniform"       # "uniform" | "zipf1.1"
    lens: str = "full"           # "full" | "uniform1024-8192"
    layers: int = 1
    rope_base: float = ROPE_BASE
    seed: int = 0
    group_dim: int = 8           # scalars per quantization group: 8 or 64

    @property
    def n_groups(self) -> int:
        return 128 // self.group_dim

    @property
    def n_codes(self) -> int:
        return N_CODES if self.group_dim == 8 else 64

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


# The five workloads.  Readings of points the descriptions leave open: variance 1/2
# ("~N(0,1/2)") for every 2-bit workload, fp32 queries where the dtype is not given,
# RoPE base 500000 and seed 0 throughout, one codebook per KV head everywhere.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("single_head_T4096_R1", 1, 1, 1, 4096, 1, "f32", 1.0),
        Workload("llama8b_layer_T32768_R2", 1, 32, 8, 32768, 2, "bf16", math.sqrt(0.5)),
        Workload("llama8b_layer_T131072_R1", 1, 32, 8, 131072, 1, "f32", 1.0),
        Workload("llama8b_batch16_ragged_R2_zipf", 16, 32, 8, 8192, 2, "f32", math.sqrt(0.5),
                 codes="zipf1.1", lens="uniform1024-8192"),
        Workload("llama8b_32layers_B4_T65536_R2", 4, 32, 8, 65536, 2, "bf16", math.sqrt(0.5),
                 layers=32),
        # the paper's own parameterization: 64-entry codebooks over groups of 64 scalars
        # (32 RoPE pairs), R = 11 ("1-bit", 1.03 bits) and R = 21 ("2-bit", 1.97 bits);
        # codebook std sqrt(1/R) so a key or value has unit variance per scalar
        Workload("llama8b_layer_T131072_R11_g64", 1, 32, 8, 131072, 11, "f32",
                 math.sqrt(1.0 / 11), group_dim=64),
        Workload("llama8b_layer_T32768_R21_g64", 1, 32, 8, 32768, 21, "bf16",
                 math.sqrt(1.0 / 21), group_dim=64),
    ]
}
WORKLOAD_ORDER = list(WORKLOADS)


def bf16_round(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 to bfloat16 (nearest, ties to even).  Returns (bits uint16,
    exact float32 value of those bits)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    back = (r.astype(np.uint32) << 16).view(np.float32)
    return r, back


def zipf_codes(rng: np.random.Generator, shape, s: float = 1.1) -> np.ndarray:
    """Codes with P(code = k - 1) proportional to k^-s, k = 1..256 (code 0 most frequent)."""
    k = np.arange(1, N_CODES + 1, dtype=np.float64)
    p = k ** (-s)
    cdf = np.cumsum(p / p.sum())
    cdf[-1] = 1.0
    u = rng.random(size=shape)
    return np.searchsorted(cdf, u, side="right").astype(np.uint8)


def _codes(rng, shape, kind, n_codes=N_CODES):
    if kind == "uniform":
        n = int(np.prod(shape))
        c = np.frombuffer(rng.bytes(n), dtype=np.uint8).reshape(shape).copy()
        return c if n_codes == N_CODES else c % np.uint8(n_codes)   # 256 % n_codes == 0
    if kind == "zipf1.1":
        return zipf_codes(rng, shape, 1.1)
    raise ValueError(kind)


def make_seq_lens(w: Workload, batch: int | None = None) -> np.ndarray:
    B = batch if batch is not None else w.batch
    if w.lens == "full":
        return np.full(B, w.t_cap, dtype=np.int32)
    if w.lens == "uniform1024-8192":
        rng = np.random.default_rng(np.random.SeedSequence([w.seed, 7919]))
        return rng.integers(1024, 8192, size=B, endpoint=True).astype(np.int32)
    raise ValueError(w.lens)


def generate(w: Workload, layer: int = 0, t_cap: int | None = None,
             batch: int | None = None, seq_lens: np.ndarray | None = None) -> dict:
    """All inputs of one layer of workload `w`.  `t_cap` / `batch` shrink the
    workload (the draws for the first entries stay those of a smaller call only
    through the same seed, not element for element)."""
    B = batch if batch is not None else w.batch
    T = t_cap if t_cap is not None else w.t_cap
    ss = np.random.SeedSequence([w.seed, layer])
    s_q, s_kc, s_vc, s_kcode, s_vcode = ss.spawn(5)
    R, Hq, Hkv = w.R, w.n_q_heads, w.n_kv_heads

    q32 = np.random.default_rng(s_q).standard_normal((B, Hq, 128), dtype=np.float32)
    if w.q_dtype == "bf16":
        q_bits, q_val = bf16_round(q32)
    else:
        q_bits, q_val = None, q32
    NG, NC, gd = w.n_groups, w.n_codes, w.group_dim
    key_cb = (np.random.default_rng(s_kc).standard_normal((Hkv, NG, R, NC, gd // 2, 2),
                                                          dtype=np.float32)
              * np.float32(w.cb_std)).astype(np.float32)
    val_cb = (np.random.default_rng(s_vc).standard_normal((Hkv, NG, R, NC, gd),
                                                          dtype=np.float32)
              * np.float32(w.cb_std)).astype(np.float32)
    # 8-scalar groups: token-major [B, Hkv, T, R, 16]; 64-scalar groups: planar
    # [B, Hkv, 2, R, T] (each (group, round) row of codes contiguous over tokens)
    code_shape = (B, Hkv, T, R, NG) if gd == 8 else (B, Hkv, NG, R, T)
    key_codes = _codes(np.random.default_rng(s_kcode), code_shape, w.codes, NC)
    val_codes = _codes(np.random.default_rng(s_vcode), code_shape, w.codes, NC)
    if seq_lens is None:
        seq_lens = make_seq_lens(w, B)
        seq_lens = np.minimum(seq_lens, T).astype(np.int32)
    return dict(q=q_val, q_bits=q_bits, q_dtype=w.q_dtype, key_cb=key_cb, val_cb=val_cb,
                key_codes=key_codes, val_codes=val_codes,
                seq_lens=np.asarray(seq_lens, dtype=np.int32),
                n_q_heads=Hq, n_kv_heads=Hkv, R=R, t_cap=T, batch=B,
                rope_base=w.rope_base, group_dim=gd,
                codes_layout="token" if gd == 8 else "planar")


def new_tokens(w: Workload, layer: int = 0, batch: int | None = None):
    """One decode step's new keys and values [B, Hkv, 128] (float32, unit Gaussian: the
    variance of a sum of R codewords of std sqrt(1/R)), as written to the cache by the
    append call; pre-RoPE keys.  Their own seed stream, separate from generate()'s."""
    B = batch if batch is not None else w.batch
    s_k, s_v = np.random.SeedSequence([w.seed, layer, 1]).spawn(2)
    shape = (B, w.n_kv_heads, 128)
    return (np.random.default_rng(s_k).standard_normal(shape, dtype=np.float32),
            np.random.default_rng(s_v).standard_normal(shape, dtype=np.float32))


def small(batch=1, n_q_heads=4, n_kv_heads=1, t_cap=64, R=1, q_dtype="f32", cb_std=1.0,
          codes="uniform", seq_lens=None, seed=0, rope_base=ROPE_BASE, group_dim=8) -> dict:
    """A small custom case with the same generators (for parity and edge-case tests)."""
    w = Workload("custom", batch, n_q_heads, n_kv_heads, t_cap, R, q_dtype, cb_std,
                 codes=codes, seed=seed, rope_base=rope_base, group_dim=group_dim)
    if seq_lens is None:
        seq_lens = np.full(batch, t_cap, dtype=np.int32)
    return generate(w, seq_lens=np.asarray(seq_lens, dtype=np.int32))
