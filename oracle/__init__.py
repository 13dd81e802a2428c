"""Python front end of the fp64 CPU oracle (``oracle/oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the entry module's smoke check and
the benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports this package, and this package imports nothing from the CUDA library.

Arrays cross the boundary as C-contiguous float64 / int32 numpy arrays; the
oracle itself does all of the arithmetic in C (see the citations there).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")


def build(source: str = SOURCE, output: str = LIBRARY, extra_flags=()) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE double semantics)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *extra_flags,
           source, "-o", output, "-lm"]
    subprocess.run(cmd, check=True)
    return output


def _needs_build(lib: str, src: str) -> bool:
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)


def _dptr(a):
    return None if a is None else a.ctypes.data_as(_D)


def _iptr(a):
    return None if a is None else a.ctypes.data_as(_I)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.int32))


class Oracle:
    """ctypes handle on one compiled oracle library (the real one by default)."""

    def __init__(self, library: str | None = None):
        if library is None:
            if _needs_build(LIBRARY, SOURCE):
                build()
            library = LIBRARY
        self.lib = ctypes.CDLL(library)
        L = self.lib
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_causal_mask.argtypes = [_D, ctypes.c_int, ctypes.c_int]
        L.oracle_sliding_window_mask.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.oracle_attn_fwd.restype = ctypes.c_int
        L.oracle_attn_fwd.argtypes = [_D, _D, _D, _D, _D] + [ctypes.c_int] * 6 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I, _I, _I, ctypes.c_int]
        L.oracle_flex_fwd.restype = ctypes.c_int
        L.oracle_flex_fwd.argtypes = [_D, _D, _D, _D, _D] + [ctypes.c_int] * 6 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I, _I, _I, ctypes.c_int,
            ctypes.c_double, _D, _I, _I, ctypes.c_void_p]
        L.oracle_rbs_block_scores.restype = ctypes.c_int
        L.oracle_rbs_block_scores.argtypes = [_D, _D, _D, _D] + [ctypes.c_int] * 6
        L.oracle_rbs_block_mask.restype = ctypes.c_int
        L.oracle_rbs_block_mask.argtypes = [ctypes.c_void_p, _D, _D, ctypes.c_long, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                            ctypes.c_int]
        L.oracle_decode_paged.restype = ctypes.c_int
        L.oracle_decode_paged.argtypes = [_D, _D, _D, _D, _D, _I, _I] + [ctypes.c_int] * 7
        L.oracle_attn_bwd.restype = ctypes.c_int
        L.oracle_attn_bwd.argtypes = [_D] * 7 + [ctypes.c_int] * 6 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I, _I]
        L.oracle_attn_visible.restype = ctypes.c_int
        L.oracle_attn_visible.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 6 + [_I, _I, _I,
                                                                                 ctypes.c_int]
        L.oracle_decode.restype = ctypes.c_int
        L.oracle_decode.argtypes = [_D, _D, _D, _D, _D] + [ctypes.c_int] * 5 + [_I]

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    # -- mlx-arsenal "Attention" page mask builders ---------------------------------
    def causal_mask(self, seq_len: int, offset: int = 0) -> np.ndarray:
        """Additive mask of shape (1, 1, seq_len, offset + seq_len), 0 / -inf."""
        out = np.empty((seq_len, offset + seq_len), dtype=np.float64)
        self.lib.oracle_causal_mask(_dptr(out), seq_len, offset)
        return out.reshape(1, 1, seq_len, offset + seq_len)

    def sliding_window_mask(self, seq_len: int, window_size: int, offset: int = 0) -> np.ndarray:
        out = np.empty((seq_len, offset + seq_len), dtype=np.float64)
        self.lib.oracle_sliding_window_mask(_dptr(out), seq_len, window_size, offset)
        return out.reshape(1, 1, seq_len, offset + seq_len)

    # -- Tylo.jl "Primitives" page, attention! ----------------------------------------
    def attn_fwd(self, Q, K, V, scale, causal=False, window=0, input_pos=0,
                 k_lengths=None, q_lengths=None, rows=None, Sq=None):
        """O (B,Hq,n,D) float64 and LSE (B,Hq,n) float64.

        Q is (B, Hq, n, D).  When ``rows`` is given, Q holds only those query
        rows (absolute indices into a sequence of ``Sq`` rows); otherwise Q is
        the whole (B, Hq, Sq, D) tensor.
        """
        Q, K, V = _f64(Q), _f64(K), _f64(V)
        B, Hq, n, D = Q.shape
        Bk, Hkv, Sk, Dk = K.shape
        assert Bk == B and Dk == D and V.shape == K.shape
        rows_a = _i32(rows)
        if rows_a is None:
            Sq = n
        else:
            assert rows_a.shape == (n,) and Sq is not None
        kl, ql = _i32(k_lengths), _i32(q_lengths)
        O = np.empty((B, Hq, n, D), dtype=np.float64)
        LSE = np.empty((B, Hq, n), dtype=np.float64)
        rc = self.lib.oracle_attn_fwd(_dptr(O), _dptr(LSE), _dptr(Q), _dptr(K), _dptr(V),
                                      B, Hq, Hkv, Sq, Sk, D, float(scale), int(causal),
                                      int(window), int(input_pos), _iptr(kl), _iptr(ql),
                                      _iptr(rows_a), n)
        if rc != 0:
            raise ValueError("oracle_attn_fwd rejected its arguments")
        return O, LSE

    def attn_visible(self, B, Sq, Sk, causal=False, window=0, input_pos=0, k_lengths=None,
                     q_lengths=None, rows=None):
        """uint8 (B, n, Sk): 1 where query row i of batch b sees key j under the
        masks of attn_fwd (the same mask rows its scores get), else 0.  ``rows``
        selects absolute query rows (default: all Sq).  The decode key set is
        ``attn_visible(B, 1, S_cap, k_lengths=lengths)``."""
        rows_a = _i32(rows)
        n = Sq if rows_a is None else rows_a.shape[0]
        kl, ql = _i32(k_lengths), _i32(q_lengths)
        out = np.empty((B, n, Sk), dtype=np.uint8)
        rc = self.lib.oracle_attn_visible(out.ctypes.data_as(ctypes.c_void_p), int(B), int(Sq),
                                          int(Sk), int(causal), int(window), int(input_pos),
                                          _iptr(kl), _iptr(ql), _iptr(rows_a), n)
        if rc != 0:
            raise ValueError("oracle_attn_visible rejected its arguments")
        return out

    # -- Tylo.jl "Primitives" page, flex_attention! -----------------------------------
    def flex_fwd(self, Q, K, V, scale, causal=False, window=0, input_pos=0,
                 k_lengths=None, q_lengths=None, rows=None, Sq=None,
                 softcap=0.0, alibi_slopes=None, doc_q=None, doc_kv=None, block_keep=None):
        """attn_fwd with SoftCapScore / AliBiScore, DocumentMask and block sparsity.

        ``doc_q`` has one id per local query row (length Sq), ``doc_kv`` one per
        key (length Sk); ``alibi_slopes`` one slope per query head; ``block_keep``
        (B, Hq, ceil(Sq/64), ceil(Sk/64)) flags of the kept 64x64 blocks.
        """
        Q, K, V = _f64(Q), _f64(K), _f64(V)
        B, Hq, n, D = Q.shape
        Bk, Hkv, Sk, Dk = K.shape
        assert Bk == B and Dk == D and V.shape == K.shape
        rows_a = _i32(rows)
        if rows_a is None:
            Sq = n
        else:
            assert rows_a.shape == (n,) and Sq is not None
        kl, ql = _i32(k_lengths), _i32(q_lengths)
        sl = None if alibi_slopes is None else _f64(alibi_slopes)
        if sl is not None:
            assert sl.shape == (Hq,)
        dq, dk = _i32(doc_q), _i32(doc_kv)
        if dq is not None:
            assert dq.shape == (Sq,) and dk is not None and dk.shape == (Sk,)
        bk = None
        if block_keep is not None:
            bk = np.ascontiguousarray(np.asarray(block_keep, dtype=np.uint8))
            assert bk.shape == (B, Hq, (Sq + 63) // 64, (Sk + 63) // 64)
        O = np.empty((B, Hq, n, D), dtype=np.float64)
        LSE = np.empty((B, Hq, n), dtype=np.float64)
        rc = self.lib.oracle_flex_fwd(_dptr(O), _dptr(LSE), _dptr(Q), _dptr(K), _dptr(V),
                                      B, Hq, Hkv, Sq, Sk, D, float(scale), int(causal),
                                      int(window), int(input_pos), _iptr(kl), _iptr(ql),
                                      _iptr(rows_a), n, float(softcap), _dptr(sl),
                                      _iptr(dq), _iptr(dk),
                                      None if bk is None else bk.ctypes.data_as(ctypes.c_void_p))
        if rc != 0:
            raise ValueError("oracle_flex_fwd rejected its arguments")
        return O, LSE

    # -- Tylo.jl "Primitives" page, decode_attention! ---------------------------------
    def decode(self, Q, K, V, lengths):
        """O (B,Hq,D) and LSE (B,Hq) float64; Q (B,Hq,D), K/V (B,Hkv,S_cap,D)."""
        Q, K, V = _f64(Q), _f64(K), _f64(V)
        B, Hq, D = Q.shape
        _, Hkv, S_cap, _ = K.shape
        ln = _i32(lengths)
        O = np.empty((B, Hq, D), dtype=np.float64)
        LSE = np.empty((B, Hq), dtype=np.float64)
        rc = self.lib.oracle_decode(_dptr(O), _dptr(LSE), _dptr(Q), _dptr(K), _dptr(V),
                                    B, Hq, Hkv, S_cap, D, _iptr(ln))
        if rc != 0:
            raise ValueError("oracle_decode rejected its arguments")
        return O, LSE


    # -- Tylo.jl "Primitives" page, ∇attention! ---------------------------------------
    def attn_bwd(self, Q, K, V, dO, scale, causal=False, window=0, input_pos=0,
                 k_lengths=None, q_lengths=None):
        """(dQ, dK, dV) float64 for the output gradient dO (shapes of Q, K, V, O)."""
        Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
        B, Hq, Sq, D = Q.shape
        _, Hkv, Sk, _ = K.shape
        assert dO.shape == Q.shape and V.shape == K.shape
        kl, ql = _i32(k_lengths), _i32(q_lengths)
        dQ, dK, dV = np.empty_like(Q), np.empty_like(K), np.empty_like(V)
        rc = self.lib.oracle_attn_bwd(_dptr(dQ), _dptr(dK), _dptr(dV), _dptr(Q), _dptr(K),
                                      _dptr(V), _dptr(dO), B, Hq, Hkv, Sq, Sk, D, float(scale),
                                      int(causal), int(window), int(input_pos), _iptr(kl),
                                      _iptr(ql))
        if rc != 0:
            raise ValueError("oracle_attn_bwd rejected its arguments")
        return dQ, dK, dV

    # -- mlx-arsenal RBS page: block scores and the block mask --------------------------
    def rbs_block_scores(self, Q, K):
        """(base, rescue) log block scores, each (B, Hq, ceil(Sq/64), ceil(Sk/64))."""
        Q, K = _f64(Q), _f64(K)
        B, Hq, Sq, D = Q.shape
        _, Hkv, Sk, _ = K.shape
        nqb, nkb = (Sq + 63) // 64, (Sk + 63) // 64
        base = np.empty((B, Hq, nqb, nkb), dtype=np.float64)
        rescue = np.empty_like(base)
        rc = self.lib.oracle_rbs_block_scores(_dptr(base), _dptr(rescue), _dptr(Q), _dptr(K),
                                              B, Hq, Hkv, Sq, Sk, D)
        if rc != 0:
            raise ValueError("oracle_rbs_block_scores rejected its arguments")
        return base, rescue

    def rbs_block_mask(self, base, rescue, alpha_base=0.22, alpha_rescue=0.18, diagonal=1):
        """uint8 keep flags of the RBS recipe (union of both branches and the band)."""
        base, rescue = _f64(base), _f64(rescue)
        *lead, nqb, nkb = base.shape
        keep = np.empty(base.shape, dtype=np.uint8)
        rows = int(np.prod(lead)) * nqb
        rc = self.lib.oracle_rbs_block_mask(keep.ctypes.data_as(ctypes.c_void_p), _dptr(base),
                                            _dptr(rescue), rows, nqb, nkb, float(alpha_base),
                                            float(alpha_rescue), int(diagonal))
        if rc != 0:
            raise ValueError("oracle_rbs_block_mask rejected its arguments")
        return keep

    # -- vllm-mlx paged KV cache + decode_attention! ------------------------------------
    def decode_paged(self, Q, K_cache, V_cache, block_tables, seq_lens):
        """vllm-mlx paged KV cache decode: O (B,Hq,D) and LSE (B,Hq) float64.

        Q (B, Hq, D); K_cache / V_cache (num_blocks, block_size, Hkv, D);
        block_tables int (B, max_blocks); seq_lens int (B,).
        """
        Q, K, V = _f64(Q), _f64(K_cache), _f64(V_cache)
        B, Hq, D = Q.shape
        num_blocks, block_size, Hkv, Dk = K.shape
        assert Dk == D and V.shape == K.shape
        bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
        assert bt.ndim == 2 and bt.shape[0] == B
        ln = _i32(seq_lens)
        O = np.empty((B, Hq, D), dtype=np.float64)
        LSE = np.empty((B, Hq), dtype=np.float64)
        rc = self.lib.oracle_decode_paged(_dptr(O), _dptr(LSE), _dptr(Q), _dptr(K), _dptr(V),
                                          _iptr(bt), _iptr(ln), B, Hq, Hkv, num_blocks, block_size,
                                          bt.shape[1], D)
        if rc != 0:
            raise ValueError("oracle_decode_paged rejected its arguments")
        return O, LSE


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``oracle/oracle.c`` (compiled on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
