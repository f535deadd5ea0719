"""CommVQ decode attention on B200: Python binding of libcvq.

The calls of the library, one-to-one with include/cvq.h:

  qtable(shape, q, key_cb)                       -> P table      (cvq_qtable)
  decode_attn(shape, ptable, codes..., n_splits) -> partials     (cvq_decode_attn)
  decode_attn_gqa(shape, q, key_cb, codes...)    -> partials     (cvq_decode_attn_gqa)
  combine(shape, partials)                       -> (out, lse)   (cvq_combine)
  attend_fused(shape, q, key_cb, codes...)       -> (out, lse)   (cvq_attend)
  naive_dequant / naive_decode                   -> the comparison path
  encode_append(shape, keys, values, ...)        -> codes written (cvq_encode_append)
  fault_status(clear)                            -> device fault bits (cvq_fault_status)

plus attend(), which allocates the intermediate buffers with torch and runs the calls in
order.  Tensors are torch CUDA tensors in the layouts documented in cvq.h; work is
enqueued on torch's current CUDA stream.  torch provides device memory and streams
only: every arithmetic step runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import _binding as _b
from ._binding import CVQ_BF16, CVQ_F32, CvqError, cvq_shape, make_shape  # noqa: F401

__all__ = ["make_shape", "shape_of", "qtable", "decode_attn", "decode_attn_gqa", "combine",
           "attend", "naive_dequant", "naive_decode", "encode_append", "split_tokens",
           "suggest_splits", "partials_alloc", "group_dim_of", "attend_fused", "workspace_alloc",
           "fault_status", "CvqError"]


def _ptr(t):
    # a plain int (or None) converts to the c_void_p argument without a ctypes object
    return t.data_ptr() if t is not None else None


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _require(t, name, dtype=None, device=True):
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _q_dtype(q):
    if q.dtype == torch.float32:
        return CVQ_F32
    if q.dtype == torch.bfloat16:
        return CVQ_BF16
    raise ValueError(f"q must be float32 or bfloat16, got {q.dtype}")


def _head_stride(cb, kind):
    """Head stride in floats of a codebook tensor.  With a leading KV-head dim
    (key [Hkv, 16, R, 256, 4, 2], value [Hkv, 16, R, 256, 8]) it is one head's size;
    without it (key [16, R, 256, 4, 2], value [16, R, 256, 8]) the codebook is shared
    by every KV head and the stride is 0."""
    per_head_dims = 6 if kind == "key" else 5
    if cb.dim() == per_head_dims:
        return cb.numel() // cb.shape[0]
    if cb.dim() == per_head_dims - 1:
        return 0
    raise ValueError(f"{kind} codebook has {cb.dim()} dims")


def group_dim_of(key_cb):
    """Scalars per quantization group, read off a key codebook [(Hkv,) NG, R, NC, PPG, 2]:
    8 (PPG = 4, 256 codewords) or 64 (PPG = 32, 64 codewords)."""
    return 2 * int(key_cb.shape[-2])


def shape_of(q, key_codes, rope_base=500000.0, group_dim=8, code_bits=0):
    """cvq_shape from q [B, Hq, 128] and key_codes: [B, Hkv, T_cap, R, 16] (group_dim 8),
    planar [B, Hkv, 2, R, T_cap] (group_dim 64) or, with code_bits 6, packed planar
    [B, Hkv, 2, R, 3 T_cap / 4]."""
    B, Hq, D = q.shape
    if group_dim == 64:
        _, Hkv, _, R, T = key_codes.shape
        if code_bits == 6:
            T = T * 4 // 3
    else:
        _, Hkv, T, R, _ = key_codes.shape
    return make_shape(B, Hq, Hkv, R, T, rope_base, D, group_dim, code_bits)


def pack_codes6(shape, codes, out=None, stream=None):
    """cvq_pack_codes6: planar one-byte codes [B, Hkv, 2, R, T_cap] -> packed 6-bit
    [B, Hkv, 2, R, 3 T_cap / 4] uint8 (shape: group_dim 64, code_bits 6)."""
    _require(codes, "codes", torch.uint8)
    if out is None:
        out = torch.empty((*codes.shape[:-1], codes.shape[-1] // 4 * 3), dtype=torch.uint8,
                          device=codes.device)
    st = _b.lib.cvq_pack_codes6(ctypes.byref(shape), _ptr(codes), _ptr(out), _stream(stream))
    _b.check(st, "cvq_pack_codes6")
    return out


def kv_head_range(n_kv_heads, rank, world):
    """The contiguous slice [h0, h1) of KV heads that rank `rank` of `world` decodes when a
    layer is partitioned by KV head (balanced: the first n_kv_heads % world ranks take one
    head more).  KV heads are independent units of the decode -- each with its own query
    heads, codes and codebooks -- so the ranks exchange no data."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    base, extra = divmod(n_kv_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_kv_heads(inputs, n_q_heads, n_kv_heads, rank, world):
    """This rank's share of one layer's inputs: every tensor restricted to its KV heads
    (and their query heads), made contiguous.  `inputs` holds q [B, Hq, 128], key_cb and
    val_cb [Hkv, ...], key_codes and val_codes [B, Hkv, ...] and seq_lens [B] (torch tensors
    or numpy arrays); codebooks shared by all heads (leading dim 1) are kept whole.
    Returns (shard, (h0, h1))."""
    h0, h1 = kv_head_range(n_kv_heads, rank, world)
    g = n_q_heads // n_kv_heads

    def contig(x):
        return x.contiguous() if hasattr(x, "contiguous") else x.copy()

    out = dict(inputs)
    out["q"] = contig(inputs["q"][:, h0 * g:h1 * g])
    for k in ("key_cb", "val_cb"):
        if inputs[k].shape[0] != 1:
            out[k] = contig(inputs[k][h0:h1])
    for k in ("key_codes", "val_codes"):
        out[k] = contig(inputs[k][:, h0:h1])
    return out, (h0, h1)


def split_tokens(shape, n_splits):
    return _b.lib.cvq_split_tokens(ctypes.byref(shape), n_splits)


def suggest_splits(shape, sm_count=None):
    if sm_count is None:
        sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return _b.lib.cvq_suggest_splits(ctypes.byref(shape), sm_count)


def qtable(shape, q, key_cb, ptable=None, stream=None):
    _require(q, "q", (torch.float32, torch.bfloat16))
    _require(key_cb, "key_cb", torch.float32)
    if ptable is None:
        ptable = torch.empty((shape.batch, shape.n_q_heads, 16, shape.R, 256, 4, 2),
                             dtype=torch.float32, device=q.device)
    _require(ptable, "ptable", torch.float32)
    st = _b.lib.cvq_qtable(ctypes.byref(shape), _ptr(q), _q_dtype(q), _ptr(key_cb),
                           _head_stride(key_cb, "key"), _ptr(ptable),
                           _stream(stream))
    _b.check(st, "cvq_qtable")
    return ptable


def partials_alloc(shape, n_splits, device):
    B, Hq = shape.batch, shape.n_q_heads
    part_o = torch.empty((B, Hq, n_splits, 128), dtype=torch.float32, device=device)
    part_m = torch.empty((B, Hq, n_splits), dtype=torch.float32, device=device)
    part_l = torch.empty((B, Hq, n_splits), dtype=torch.float32, device=device)
    return part_o, part_m, part_l


def _codes_check(key_codes, val_codes, seq_lens, val_cb):
    _require(key_codes, "key_codes", torch.uint8)
    _require(val_codes, "val_codes", torch.uint8)
    _require(seq_lens, "seq_lens", torch.int32)
    _require(val_cb, "val_cb", torch.float32)


def decode_attn(shape, ptable, key_codes, val_codes, seq_lens, val_cb, n_splits, partials=None,
                stream=None):
    """Table form: gathers from the P table of cvq_qtable."""
    _require(ptable, "ptable", torch.float32)
    _codes_check(key_codes, val_codes, seq_lens, val_cb)
    part_o, part_m, part_l = partials or partials_alloc(shape, n_splits, key_codes.device)
    st = _b.lib.cvq_decode_attn(ctypes.byref(shape), _ptr(ptable), _ptr(key_codes),
                                _ptr(val_codes), _ptr(seq_lens), _ptr(val_cb),
                                _head_stride(val_cb, "val"), n_splits,
                                _ptr(part_o), _ptr(part_m), _ptr(part_l), _stream(stream))
    _b.check(st, "cvq_decode_attn")
    return part_o, part_m, part_l


def decode_attn_gqa(shape, q, key_cb, key_codes, val_codes, seq_lens, val_cb, n_splits,
                    partials=None, stream=None):
    """GQA form: one codeword gather + rotation per token, shared by the query heads of
    a KV head."""
    _require(q, "q", (torch.float32, torch.bfloat16))
    _require(key_cb, "key_cb", torch.float32)
    _codes_check(key_codes, val_codes, seq_lens, val_cb)
    part_o, part_m, part_l = partials or partials_alloc(shape, n_splits, key_codes.device)
    st = _b.lib.cvq_decode_attn_gqa(ctypes.byref(shape), _ptr(q), _q_dtype(q), _ptr(key_cb),
                                    _head_stride(key_cb, "key"),
                                    _ptr(key_codes), _ptr(val_codes), _ptr(seq_lens), _ptr(val_cb),
                                    _head_stride(val_cb, "val"), n_splits,
                                    _ptr(part_o), _ptr(part_m), _ptr(part_l), _stream(stream))
    _b.check(st, "cvq_decode_attn_gqa")
    return part_o, part_m, part_l


def workspace_alloc(shape, n_splits, device):
    """Zeroed workspace for attend_fused (the partial states and the arrival counters,
    which every call leaves zero again)."""
    n = _b.lib.cvq_attend_workspace_bytes(ctypes.byref(shape), n_splits)
    if n == 0:
        raise ValueError("invalid shape or n_splits for cvq_attend_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def attend_fused(shape, q, key_cb, key_codes, val_codes, seq_lens, val_cb, n_splits,
                 workspace=None, out=None, lse=None, stream=None):
    """GQA decode with the split merge fused into its last CTA per work unit: one launch
    (cvq_attend).  Returns (out [B, Hq, 128], lse [B, Hq])."""
    _require(q, "q", (torch.float32, torch.bfloat16))
    _require(key_cb, "key_cb", torch.float32)
    _codes_check(key_codes, val_codes, seq_lens, val_cb)
    dev = key_codes.device
    if workspace is None:
        workspace = workspace_alloc(shape, n_splits, dev)
    if out is None:
        out = torch.empty((shape.batch, shape.n_q_heads, 128), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((shape.batch, shape.n_q_heads), dtype=torch.float32, device=dev)
    st = _b.lib.cvq_attend(ctypes.byref(shape), _ptr(q), _q_dtype(q), _ptr(key_cb),
                           _head_stride(key_cb, "key"), _ptr(key_codes), _ptr(val_codes),
                           _ptr(seq_lens), _ptr(val_cb), _head_stride(val_cb, "val"), n_splits,
                           _ptr(workspace), _ptr(out), _ptr(lse), _stream(stream))
    _b.check(st, "cvq_attend")
    return out, lse


def fault_status(clear=False, device=None):
    """The device fault word of the current (or given) CUDA device: 0, or CVQ_FAULT_* bits
    set by a kernel whose bounded wait on a codebook copy gave up.  Synchronizes the device."""
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        st = _b.lib.cvq_fault_status(ctypes.byref(flags), 1 if clear else 0)
    _b.check(st, "cvq_fault_status")
    return int(flags.value)


def combine(shape, n_splits, part_o, part_m, part_l, out=None, lse=None, stream=None):
    if out is None:
        out = torch.empty((shape.batch, shape.n_q_heads, 128), dtype=torch.float32,
                          device=part_o.device)
    if lse is None:
        lse = torch.empty((shape.batch, shape.n_q_heads), dtype=torch.float32, device=part_o.device)
    st = _b.lib.cvq_combine(ctypes.byref(shape), n_splits, _ptr(part_o), _ptr(part_m),
                            _ptr(part_l), _ptr(out), _ptr(lse), _stream(stream))
    _b.check(st, "cvq_combine")
    return out, lse


def naive_dequant(shape, key_cb, val_cb, key_codes, val_codes, seq_lens, k_out=None, v_out=None,
                  stream=None):
    """The naive path's first half: every cached key (rotated by RoPE) and value decoded
    into fp16 tensors [B, Hkv, t_cap, 128]."""
    _require(key_cb, "key_cb", torch.float32)
    _codes_check(key_codes, val_codes, seq_lens, val_cb)
    dims = (shape.batch, shape.n_kv_heads, shape.t_cap, 128)
    k_out = k_out if k_out is not None else torch.zeros(dims, dtype=torch.float16, device=key_codes.device)
    v_out = v_out if v_out is not None else torch.zeros(dims, dtype=torch.float16, device=key_codes.device)
    st = _b.lib.cvq_naive_dequant(ctypes.byref(shape), _ptr(key_cb), _head_stride(key_cb, "key"),
                                  _ptr(key_codes), _ptr(val_codes), _ptr(seq_lens), _ptr(val_cb),
                                  _head_stride(val_cb, "val"), _ptr(k_out), _ptr(v_out),
                                  _stream(stream))
    _b.check(st, "cvq_naive_dequant")
    return k_out, v_out


def encode_append(shape, keys, values, key_cb, val_cb, positions, key_codes, val_codes,
                  stream=None):
    """The write side of a decode step: codes of keys / values [B, Hkv, 128] (fp32,
    pre-RoPE keys) written in place at [b, h, positions[b]] of key_codes / val_codes
    [B, Hkv, t_cap, R, 16]; a position outside [0, t_cap) writes nothing."""
    _require(keys, "keys", torch.float32)
    _require(values, "values", torch.float32)
    _require(key_cb, "key_cb", torch.float32)
    _require(positions, "positions", torch.int32)
    _codes_check(key_codes, val_codes, positions, val_cb)
    st = _b.lib.cvq_encode_append(ctypes.byref(shape), _ptr(keys), _ptr(values), _ptr(key_cb),
                                  _head_stride(key_cb, "key"), _ptr(val_cb),
                                  _head_stride(val_cb, "val"), _ptr(positions),
                                  _ptr(key_codes), _ptr(val_codes), _stream(stream))
    _b.check(st, "cvq_encode_append")
    return key_codes, val_codes


def naive_decode(shape, q, k, v, seq_lens, n_splits, partials=None, stream=None):
    """The naive path's second half: split-T decode attention over fp16 keys / values."""
    _require(q, "q", (torch.float32, torch.bfloat16))
    _require(k, "k", torch.float16)
    _require(v, "v", torch.float16)
    _require(seq_lens, "seq_lens", torch.int32)
    part_o, part_m, part_l = partials or partials_alloc(shape, n_splits, k.device)
    st = _b.lib.cvq_naive_decode(ctypes.byref(shape), _ptr(q), _q_dtype(q), _ptr(k), _ptr(v),
                                 _ptr(seq_lens), n_splits, _ptr(part_o), _ptr(part_m),
                                 _ptr(part_l), _stream(stream))
    _b.check(st, "cvq_naive_decode")
    return part_o, part_m, part_l


def attend(q, key_cb, val_cb, key_codes, val_codes, seq_lens, rope_base=500000.0, n_splits=None,
           form="gqa", stream=None, code_bits=0):
    """One decode step: (out [B, Hq, 128], lse [B, Hq]) in fp32.

    form="gqa":   cvq_attend (decode with the merge fused in: one launch)
    form="gqa_split": cvq_decode_attn_gqa + cvq_combine
    form="table": cvq_qtable + cvq_decode_attn + cvq_combine
    form="naive": cvq_naive_dequant + cvq_naive_decode + cvq_combine (the comparison path)
    code_bits=6: the codes are packed 6-bit rows (64-scalar groups; see pack_codes6).
    """
    shape = shape_of(q, key_codes, rope_base, group_dim_of(key_cb), code_bits)
    if n_splits is None:
        n_splits = suggest_splits(shape)
    if form == "table":
        P = qtable(shape, q, key_cb, stream=stream)
        parts = decode_attn(shape, P, key_codes, val_codes, seq_lens, val_cb, n_splits, stream=stream)
    elif form == "naive":
        kh, vh = naive_dequant(shape, key_cb, val_cb, key_codes, val_codes, seq_lens, stream=stream)
        parts = naive_decode(shape, q, kh, vh, seq_lens, n_splits, stream=stream)
    elif form == "gqa":
        return attend_fused(shape, q, key_cb, key_codes, val_codes, seq_lens, val_cb, n_splits,
                            stream=stream)
    elif form == "gqa_split":
        parts = decode_attn_gqa(shape, q, key_cb, key_codes, val_codes, seq_lens, val_cb, n_splits,
                                stream=stream)
    else:
        raise ValueError(form)
    return combine(shape, n_splits, *parts, stream=stream)
