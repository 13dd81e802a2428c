"""Thin ctypes binding over ``libgqa_attn.so`` (C ABI in ``include/gqa_attn.h``).

Argument marshalling only: every step of the attention path runs in the CUDA
kernels behind the C entry points.  The functions take torch tensors for
convenience, pass their device pointers and the current CUDA stream, and raise
``AttnError`` on a non-OK status.  There is no fallback: if the library is
missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# GQA_ATTN_DEBUG=1 selects the checked build (every TMA coordinate and global
# index range-checked in the kernels; built with `... build --debug`).
CHECKED = os.environ.get("GQA_ATTN_DEBUG", "0") == "1"
LIBRARY = os.path.join(_HERE, "libgqa_attn_debug.so" if CHECKED else "libgqa_attn.so")

if not os.path.exists(LIBRARY):
    raise ImportError(f"{LIBRARY} is not built; run `python -m gqa_attention_flash_b200.build"
                      f"{' --debug' if CHECKED else ''}`")

lib = ctypes.CDLL(LIBRARY)

ATTN_OK = 0
STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_NULL", 2: "ATTN_ERR_INVALID", 3: "ATTN_ERR_UNSUPPORTED",
          4: "ATTN_ERR_CUDA", 5: "ATTN_ERR_TIMEOUT", 6: "ATTN_ERR_DEVICE_BOUNDS",
          7: "ATTN_ERR_SCRATCH_LIMIT"}

_p = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

lib.attn_fwd.restype = _i
lib.attn_fwd.argtypes = [_p, _p, _p, _p, _p] + [_i] * 6 + [_f, _i, _i, _i, _p, _p]
lib.attn_fwd_varlen.restype = _i
lib.attn_fwd_varlen.argtypes = [_p, _p, _p, _p, _p] + [_i] * 6 + [_f, _i, _i, _i, _p, _p, _p]
lib.attn_fwd_flex.restype = _i
lib.attn_fwd_flex.argtypes = [_p, _p, _p, _p, _p] + [_i] * 6 + [_f, _i, _i, _i, _p, _p, _f, _p, _p,
                                                                _p, _p, _i, _p]
lib.attn_bwd.restype = _i
lib.attn_bwd.argtypes = [_p] * 8 + [_p] + [_i] * 6 + [_f, _i, _i, _i, _p, _p, _p]
lib.attn_rbs_block_mask.restype = _i
lib.attn_rbs_block_mask.argtypes = [_p, _p, _p, _p, _p] + [_i] * 6 + [_f, _f, _i, _p]
_KEEP = ctypes.CFUNCTYPE(_i, _i, _i, _p)
lib.attn_block_mask_build.restype = _i
lib.attn_block_mask_build.argtypes = [_p, _i, _i, _i, _KEEP, _p]
lib.attn_block_mask_document.restype = _i
lib.attn_block_mask_document.argtypes = [_p, _i, _i, _i, _i, _i, _p, _p]
lib.attn_decode.restype = _i
lib.attn_decode.argtypes = [_p, _p, _p, _p, _p, _i, _p] + [_i] * 5
lib.attn_decode_paged.restype = _i
lib.attn_decode_paged.argtypes = [_p, _p, _p, _p, _p, _p, _i, _p] + [_i] * 7
lib.attn_decode_noalloc.restype = _i
lib.attn_decode_noalloc.argtypes = [_p, _p, _p, _p, _p, _i, _p] + [_i] * 5
lib.attn_status_string.restype = ctypes.c_char_p
lib.attn_status_string.argtypes = [_i]
lib.attn_last_device_status.restype = _i
lib.attn_last_device_status.argtypes = [_p]
lib.attn_check_bounded_wait.restype = _i
lib.attn_check_bounded_wait.argtypes = [_i, _p]


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.attn_status_string(status).decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# The C ABI sees raw pointers and sizes only: it cannot tell a transposed view, a
# float16 tensor or a tensor on another device from the layout it expects.  The
# wrappers therefore refuse such tensors here, before any call into the library.
def _tensor(t, name, dtype, shape):
    """Check dtype, shape (entries of None are free) and row-major contiguity;
    returns the shape."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != len(shape) or any(w is not None and w != g for g, w in zip(t.shape, shape)):
        want = "(" + ", ".join("*" if w is None else str(w) for w in shape) + ")"
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major); call .contiguous()")
    return tuple(t.shape)


def _same_device(**tensors):
    """Every given tensor on the current CUDA device (the one whose stream the
    kernels are launched on)."""
    cur = None
    for name, t in tensors.items():
        if t is None:
            continue
        idx = t.get_device()
        if idx < 0:
            raise ValueError(f"{name} must be a CUDA tensor, got device {t.device}")
        if cur is None:
            cur = torch.cuda.current_device()
        if idx != cur:
            raise ValueError(f"{name} is on {t.device}, but the current device is "
                             f"cuda:{cur}")


def _check_prefill(O, Q, K, V, LSE, k_lengths, q_lengths):
    B, Hq, Sq, D = _tensor(Q, "Q", torch.bfloat16, (None,) * 4)
    _, Hkv, Sk, _ = _tensor(K, "K", torch.bfloat16, (B, None, None, D))
    _tensor(V, "V", torch.bfloat16, (B, Hkv, Sk, D))
    _tensor(O, "O", torch.bfloat16, (B, Hq, Sq, D))
    if LSE is not None:
        _tensor(LSE, "LSE", torch.float32, (B, Hq, Sq))
    if k_lengths is not None:
        _tensor(k_lengths, "k_lengths", torch.int32, (B,))
    if q_lengths is not None:
        _tensor(q_lengths, "q_lengths", torch.int32, (B,))
    return B, Hq, Hkv, Sq, Sk, D


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != ATTN_OK:
        raise AttnError(rc, where)


def status_string(status: int) -> str:
    return lib.attn_status_string(status).decode()


def attn_fwd(O, Q, K, V, LSE, scale, causal=False, window=0, input_pos=0, k_lengths=None,
             q_lengths=None, stream=None):
    """Fill O (B,Hq,Sq,D) bf16 and LSE (B,Hq,Sq) fp32 (or None) in place.

    Shapes are read from the tensors: Q (B,Hq,Sq,D), K/V (B,Hkv,Sk,D).  Calls
    ``attn_fwd_varlen`` when q_lengths is given, else ``attn_fwd``.
    """
    B, Hq, Hkv, Sq, Sk, D = _check_prefill(O, Q, K, V, LSE, k_lengths, q_lengths)
    _same_device(O=O, Q=Q, K=K, V=V, LSE=LSE, k_lengths=k_lengths, q_lengths=q_lengths)
    args = [_ptr(O), _ptr(Q), _ptr(K), _ptr(V), _ptr(LSE), B, Hq, Hkv, Sq, Sk, D, float(scale),
            int(causal), int(window), int(input_pos), _ptr(k_lengths)]
    if q_lengths is not None:
        rc = lib.attn_fwd_varlen(*args, _ptr(q_lengths), _stream(stream))
        _check(rc, "attn_fwd_varlen")
    else:
        rc = lib.attn_fwd(*args, _stream(stream))
        _check(rc, "attn_fwd")


def attn_fwd_flex(O, Q, K, V, LSE, scale, causal=False, window=0, input_pos=0, k_lengths=None,
                  q_lengths=None, softcap=0.0, alibi_slopes=None, doc_q=None, doc_kv=None,
                  block_mask=None, stream=None):
    """flex_attention! forward: attn_fwd plus SoftCapScore (softcap > 0) or
    AliBiScore (alibi_slopes, fp32 (Hq,)), DocumentMask (doc_q int32 (Sq,), doc_kv
    int32 (Sk,)) and a BlockMask (uint8 (ceil(Sq/64), ceil(Sk/64)), or one per
    (batch, query head) as a 4-D (B, Hq, ., .) tensor), all on the device."""
    B, Hq, Hkv, Sq, Sk, D = _check_prefill(O, Q, K, V, LSE, k_lengths, q_lengths)
    if alibi_slopes is not None:
        _tensor(alibi_slopes, "alibi_slopes", torch.float32, (Hq,))
    if doc_q is not None:
        _tensor(doc_q, "doc_q", torch.int32, (Sq,))
    if doc_kv is not None:
        _tensor(doc_kv, "doc_kv", torch.int32, (Sk,))
    if block_mask is not None:
        nqb, nkb = block_mask_shape(Sq, Sk)
        _tensor(block_mask, "block_mask", torch.uint8,
                (B, Hq, nqb, nkb) if block_mask.dim() == 4 else (nqb, nkb))
    _same_device(O=O, Q=Q, K=K, V=V, LSE=LSE, k_lengths=k_lengths, q_lengths=q_lengths,
                 alibi_slopes=alibi_slopes, doc_q=doc_q, doc_kv=doc_kv, block_mask=block_mask)
    rc = lib.attn_fwd_flex(_ptr(O), _ptr(Q), _ptr(K), _ptr(V), _ptr(LSE), B, Hq, Hkv, Sq, Sk, D,
                           float(scale), int(causal), int(window), int(input_pos),
                           _ptr(k_lengths), _ptr(q_lengths), float(softcap), _ptr(alibi_slopes),
                           _ptr(doc_q), _ptr(doc_kv), _ptr(block_mask),
                           1 if block_mask is not None and block_mask.dim() == 4 else 0,
                           _stream(stream))
    _check(rc, "attn_fwd_flex")


def rbs_block_mask(Q, K, alpha_base=0.22, alpha_rescue=0.18, diagonal=1, want_scores=False,
                   stream=None):
    """Block-sparse prefill mask from the RBS block scores: uint8 (B, Hq, nqb, nkb)
    device tensor (2 = keep, 0 = skip), plus the (base, rescue) scores if asked."""
    B, Hq, Sq, D = _tensor(Q, "Q", torch.bfloat16, (None,) * 4)
    _, Hkv, Sk, _ = _tensor(K, "K", torch.bfloat16, (B, None, None, D))
    _same_device(Q=Q, K=K)
    shape = (B, Hq, (Sq + 63) // 64, (Sk + 63) // 64)
    mask = torch.empty(shape, dtype=torch.uint8, device=Q.device)
    base = torch.empty(shape, dtype=torch.float32, device=Q.device) if want_scores else None
    resc = torch.empty(shape, dtype=torch.float32, device=Q.device) if want_scores else None
    rc = lib.attn_rbs_block_mask(_ptr(mask), _ptr(base), _ptr(resc), _ptr(Q), _ptr(K), B, Hq,
                                 Hkv, Sq, Sk, D, float(alpha_base), float(alpha_rescue),
                                 int(diagonal), _stream(stream))
    _check(rc, "attn_rbs_block_mask")
    return (mask, base, resc) if want_scores else mask


def attn_bwd(dQ, dK, dV, dO, Q, K, V, O, LSE, scale, causal=False, window=0, input_pos=0,
             k_lengths=None, q_lengths=None, stream=None):
    """Backward of attn_fwd: fill dQ (like Q) and dK, dV (like K, V) in place from dO,
    the forward's inputs, output O and LSE."""
    B, Hq, Hkv, Sq, Sk, D = _check_prefill(O, Q, K, V, LSE, k_lengths, q_lengths)
    if LSE is None:
        raise ValueError("LSE (the forward's saved statistics) is required")
    _tensor(dO, "dO", torch.bfloat16, (B, Hq, Sq, D))
    _tensor(dQ, "dQ", torch.bfloat16, (B, Hq, Sq, D))
    _tensor(dK, "dK", torch.bfloat16, (B, Hkv, Sk, D))
    _tensor(dV, "dV", torch.bfloat16, (B, Hkv, Sk, D))
    _same_device(dQ=dQ, dK=dK, dV=dV, dO=dO, Q=Q, K=K, V=V, O=O, LSE=LSE, k_lengths=k_lengths,
                 q_lengths=q_lengths)
    rc = lib.attn_bwd(_ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dO), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                      _ptr(LSE), B, Hq, Hkv, Sq, Sk, D, float(scale), int(causal), int(window),
                      int(input_pos), _ptr(k_lengths), _ptr(q_lengths), _stream(stream))
    _check(rc, "attn_bwd")


def block_mask_shape(Sq: int, Sk: int):
    return ((Sq + 63) // 64, (Sk + 63) // 64)


def block_mask_document(Sq, Sk, doc_q, doc_kv, causal=False, window=0, input_pos=0):
    """Host uint8 BlockMask for DocumentMask (+ causal / window): doc_q, doc_kv are
    int32 CPU tensors of lengths Sq and Sk.  Returns a CPU uint8 tensor."""
    out = torch.empty(block_mask_shape(Sq, Sk), dtype=torch.uint8)
    dq = doc_q.to(torch.int32).contiguous()
    dk = doc_kv.to(torch.int32).contiguous()
    assert dq.numel() == Sq and dk.numel() == Sk and not dq.is_cuda and not dk.is_cuda
    rc = lib.attn_block_mask_document(_ptr(out), int(Sq), int(Sk), int(input_pos), int(causal),
                                      int(window), _ptr(dq), _ptr(dk))
    _check(rc, "attn_block_mask_document")
    return out


def block_mask_build(Sq, Sk, keep, input_pos=0):
    """Host uint8 BlockMask from a Python predicate keep(q, kv) -> bool on absolute
    query position q and key position kv (the page's build_block_mask)."""
    out = torch.empty(block_mask_shape(Sq, Sk), dtype=torch.uint8)
    cb = _KEEP(lambda q, kv, ctx: 1 if keep(q, kv) else 0)
    rc = lib.attn_block_mask_build(_ptr(out), int(Sq), int(Sk), int(input_pos), cb, None)
    _check(rc, "attn_block_mask_build")
    return out


def _check_decode(O, Q, K, V, lengths):
    B, Hq, D = _tensor(Q, "Q", torch.bfloat16, (None,) * 3)
    _, Hkv, S_cap, _ = _tensor(K, "K", torch.bfloat16, (B, None, None, D))
    _tensor(V, "V", torch.bfloat16, (B, Hkv, S_cap, D))
    _tensor(O, "O", torch.bfloat16, (B, Hq, D))
    _tensor(lengths, "lengths", torch.int32, (B,))
    _same_device(O=O, Q=Q, K=K, V=V, lengths=lengths)
    return B, Hq, Hkv, S_cap, D


def attn_decode(O, Q, K, V, lengths, n_splits=8, stream=None):
    """Fill O (B,Hq,D) bf16 in place; Q (B,Hq,D), K/V caches (B,Hkv,S_cap,D)."""
    B, Hq, Hkv, S_cap, D = _check_decode(O, Q, K, V, lengths)
    rc = lib.attn_decode(_ptr(O), _ptr(Q), _ptr(K), _ptr(V), _ptr(lengths), int(n_splits),
                         _stream(stream), B, Hq, Hkv, S_cap, D)
    _check(rc, "attn_decode")


def attn_decode_paged(O, Q, K_cache, V_cache, block_tables, seq_lens, n_splits=8, stream=None):
    """Decode from a paged cache: Q (B,Hq,D); K/V caches (num_blocks, block_size, Hkv, D);
    block_tables int32 (B, max_blocks); seq_lens int32 (B,); O (B,Hq,D) filled in place."""
    B, Hq, D = _tensor(Q, "Q", torch.bfloat16, (None,) * 3)
    num_blocks, block_size, Hkv, _ = _tensor(K_cache, "K_cache", torch.bfloat16,
                                             (None, None, None, D))
    _tensor(V_cache, "V_cache", torch.bfloat16, (num_blocks, block_size, Hkv, D))
    _tensor(O, "O", torch.bfloat16, (B, Hq, D))
    _tensor(block_tables, "block_tables", torch.int32, (B, None))
    _tensor(seq_lens, "seq_lens", torch.int32, (B,))
    _same_device(O=O, Q=Q, K_cache=K_cache, V_cache=V_cache, block_tables=block_tables,
                 seq_lens=seq_lens)
    rc = lib.attn_decode_paged(_ptr(O), _ptr(Q), _ptr(K_cache), _ptr(V_cache), _ptr(block_tables),
                               _ptr(seq_lens), int(n_splits), _stream(stream), B, Hq, Hkv,
                               num_blocks, block_size, int(block_tables.shape[1]), D)
    _check(rc, "attn_decode_paged")


def attn_decode_noalloc(O, Q, K, V, lengths, n_splits=8, stream=None):
    """attn_decode without any allocation: the workspace lives in the library's
    fixed 16 MiB device array (for callers that cannot allocate device memory;
    calls that overlap on the GPU share that array and must be ordered)."""
    B, Hq, Hkv, S_cap, D = _check_decode(O, Q, K, V, lengths)
    rc = lib.attn_decode_noalloc(_ptr(O), _ptr(Q), _ptr(K), _ptr(V), _ptr(lengths),
                                 int(n_splits), _stream(stream), B, Hq, Hkv, S_cap, D)
    _check(rc, "attn_decode_noalloc")


def last_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return lib.attn_last_device_status(_stream(stream))


def check_bounded_wait(limit_us: int, stream=None):
    _check(lib.attn_check_bounded_wait(int(limit_us), _stream(stream)), "attn_check_bounded_wait")
