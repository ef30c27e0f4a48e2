"""Python view of the CPU oracle (liboracle.so).

TEST INFRASTRUCTURE ONLY.  The oracle is a plain, slow, obviously-correct C implementation of
the LLVQ index decode (shell -> class -> Golay refinement r, sign pattern s, lexicographic
arrangement rank I''), of the fp64 GEMV/GEMM on packed words and of the nearest-point search
over the shell union (angular and Euclidean criteria, with a brute-force search beside it).  Only the tests, the
package's smoke check and the bench's CPU-baseline leg import this module; the product path
never does.  Indices wider than 64 bits travel as (lo, hi) uint64 pairs.

Method source: "Leech Lattice Vector Quantization for Efficient LLM Compression",
papernotes.org notes, 方法详解 / 关键设计 1-2 and 4; gist.science summary, Methodik 1-3.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None

u64p = C.POINTER(C.c_uint64)
i32p = C.POINTER(C.c_int32)
i8p = C.POINTER(C.c_int8)
u16p = C.POINTER(C.c_uint16)
u32p = C.POINTER(C.c_uint32)
f64p = C.POINTER(C.c_double)


class ClassInfo(C.Structure):
    _fields_ = [("m", C.c_int32), ("odd", C.c_int32), ("k", C.c_int32), ("nvals", C.c_int32),
                ("vals", C.c_int32 * 24), ("cnts", C.c_int32 * 24), ("A", C.c_uint32),
                ("B", C.c_int32), ("P_lo", C.c_uint64), ("P_hi", C.c_uint64),
                ("size_lo", C.c_uint64), ("size_hi", C.c_uint64),
                ("offset_lo", C.c_uint64), ("offset_hi", C.c_uint64)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        L.ora_golay_by_mask.argtypes = [u32p]
        L.ora_golay_by_weight.argtypes = [u32p, i32p]
        L.ora_in_leech.argtypes = [i32p]
        L.ora_shell_enumerate.argtypes = [C.c_int32, i32p, C.c_uint64]
        L.ora_shell_enumerate.restype = C.c_uint64
        L.ora_shell_counts_dp.argtypes = [C.c_int32, u64p, u64p]
        L.ora_unrank_arrangement.argtypes = [C.c_int32, i32p, C.c_uint64, C.c_uint64, i32p]
        L.ora_rank_arrangement.argtypes = [C.c_int32, i32p, C.c_int32, i32p, u64p, u64p]
        L.ora_codec_create.argtypes = [C.c_int32]
        L.ora_codec_create.restype = C.c_void_p
        L.ora_codec_destroy.argtypes = [C.c_void_p]
        L.ora_codec_max_shell.argtypes = [C.c_void_p]
        L.ora_codec_npoints.argtypes = [C.c_void_p, u64p, u64p]
        L.ora_codec_shell_offset.argtypes = [C.c_void_p, C.c_int32, u64p, u64p]
        L.ora_codec_shell_nclasses.argtypes = [C.c_void_p, C.c_int32]
        L.ora_codec_shell_nclasses.restype = C.c_int64
        L.ora_codec_shell_class.argtypes = [C.c_void_p, C.c_int32, C.c_int64, C.POINTER(ClassInfo)]
        L.ora_decode.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, i32p]
        L.ora_encode.argtypes = [C.c_void_p, i32p, u64p, u64p]
        L.ora_decode_batch_shell.argtypes = [C.c_void_p, C.c_int64, u64p, u64p, i8p, i32p]
        L.ora_decode_batch_shell.restype = C.c_int64
        L.ora_gemm.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_int32, C.c_int64,
                               C.c_int32, u16p, u16p, C.c_int32, f64p]
        L.ora_gemm.restype = C.c_int64
        L.ora_gemm_mt.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_int32,
                                  C.c_int64, C.c_int32, u16p, u16p, C.c_int32, f64p, C.c_int32]
        L.ora_gemm_mt.restype = C.c_int64
        f32p = C.POINTER(C.c_float)
        L.ora_search.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_double, f64p, i32p, f64p]
        L.ora_search_batch.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_double, C.c_int64, f32p,
                                       i8p, f64p, C.c_int32]
        L.ora_search_brute.argtypes = [C.c_int32, C.c_int32, C.c_double, C.c_int64, f32p, i8p, f64p,
                                       C.c_int32]
        L.ora_search_brute.restype = C.c_int64
        L.ora_class_best.argtypes = [C.c_void_p, C.c_int32, C.c_int64, C.c_uint32, f64p, i32p, f64p]
        L.ora_spherical_gptq.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, f64p, f64p, i8p, f64p]
        L.ora_gptq_block_matrix.argtypes = [C.c_int32, f64p, C.c_int32, f64p]
        L.ora_half_to_double.argtypes = [C.c_uint16]
        L.ora_half_to_double.restype = C.c_double
        _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


def _u128(lo: int, hi: int) -> int:
    return (int(hi) << 64) | int(lo)


def golay_by_mask() -> np.ndarray:
    out = np.zeros(4096, np.uint32)
    lib().ora_golay_by_mask(_p(out, u32p))
    return out


def golay_by_weight():
    out = np.zeros(4096, np.uint32)
    base = np.zeros(26, np.int32)
    lib().ora_golay_by_weight(_p(out, u32p), _p(base, i32p))
    return out, base


def in_leech(x) -> bool:
    a = np.ascontiguousarray(x, dtype=np.int32)
    return bool(lib().ora_in_leech(_p(a, i32p)))


def shell_enumerate(m: int, store: bool = True):
    """All points of shell m (direct search) as int8 [n, 24], or just the count."""
    L = lib()
    if not store:
        return int(L.ora_shell_enumerate(m, None, 0))
    n = int(L.ora_shell_enumerate(m, None, 0))
    out = np.zeros((n, 24), np.int32)
    L.ora_shell_enumerate(m, _p(out, i32p), n)
    return out


def shell_counts_dp(mmax: int) -> list[int]:
    lo = np.zeros(mmax + 1, np.uint64)
    hi = np.zeros(mmax + 1, np.uint64)
    if lib().ora_shell_counts_dp(mmax, _p(lo, u64p), _p(hi, u64p)):
        raise RuntimeError("shell count DP failed")
    return [_u128(a, b) for a, b in zip(lo, hi)]


def unrank_arrangement(cnts, rank: int) -> list[int]:
    c = np.ascontiguousarray(cnts, np.int32)
    seq = np.zeros(int(c.sum()), np.int32)
    if lib().ora_unrank_arrangement(len(c), _p(c, i32p), rank & (2**64 - 1), rank >> 64,
                                    _p(seq, i32p)):
        raise ValueError("rank out of range")
    return seq.tolist()


def rank_arrangement(cnts, seq) -> int:
    c = np.ascontiguousarray(cnts, np.int32)
    s = np.ascontiguousarray(seq, np.int32)
    lo, hi = C.c_uint64(), C.c_uint64()
    if lib().ora_rank_arrangement(len(c), _p(c, i32p), len(s), _p(s, i32p), C.byref(lo),
                                  C.byref(hi)):
        raise ValueError("not an arrangement of the multiset")
    return _u128(lo.value, hi.value)


@dataclass
class Class:
    m: int
    odd: bool
    k: int
    vals: list
    cnts: list
    A: int
    B: int
    P: int
    size: int
    offset: int


class Codec:
    """The oracle's codec for one index budget (48, 72 or 96 bits)."""

    def __init__(self, index_bits: int):
        self.index_bits = index_bits
        self._h = lib().ora_codec_create(index_bits)
        if not self._h:
            raise RuntimeError(f"oracle codec create failed for {index_bits} bits")
        self.max_shell = int(lib().ora_codec_max_shell(self._h))
        lo, hi = C.c_uint64(), C.c_uint64()
        lib().ora_codec_npoints(self._h, C.byref(lo), C.byref(hi))
        self.n_points = _u128(lo.value, hi.value)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:
            _lib.ora_codec_destroy(h)
            self._h = None

    def shell_offset(self, m: int) -> int:
        lo, hi = C.c_uint64(), C.c_uint64()
        lib().ora_codec_shell_offset(self._h, m, C.byref(lo), C.byref(hi))
        return _u128(lo.value, hi.value)

    def shell_nclasses(self, m: int) -> int:
        return int(lib().ora_codec_shell_nclasses(self._h, m))

    def shell_class(self, m: int, j: int) -> Class:
        ci = ClassInfo()
        if lib().ora_codec_shell_class(self._h, m, j, C.byref(ci)):
            raise IndexError((m, j))
        nv = ci.nvals
        return Class(ci.m, bool(ci.odd), ci.k, list(ci.vals[:nv]), list(ci.cnts[:nv]), ci.A, ci.B,
                     _u128(ci.P_lo, ci.P_hi), _u128(ci.size_lo, ci.size_hi),
                     _u128(ci.offset_lo, ci.offset_hi))

    def classes(self):
        for m in range(2, self.max_shell + 1):
            for j in range(self.shell_nclasses(m)):
                yield self.shell_class(m, j)

    def decode(self, index: int) -> list[int]:
        x = np.zeros(24, np.int32)
        if lib().ora_decode(self._h, index & (2**64 - 1), index >> 64, _p(x, i32p)):
            raise ValueError(f"index {index} out of range")
        return x.tolist()

    def encode(self, x) -> int:
        a = np.ascontiguousarray(x, np.int32)
        lo, hi = C.c_uint64(), C.c_uint64()
        if lib().ora_encode(self._h, _p(a, i32p), C.byref(lo), C.byref(hi)):
            raise ValueError("not a coded lattice point")
        return _u128(lo.value, hi.value)

    def decode_batch(self, lo: np.ndarray, hi: np.ndarray | None = None, with_shell=False):
        lo = np.ascontiguousarray(lo, np.uint64)
        n = lo.shape[0]
        hi_a = None if hi is None else np.ascontiguousarray(hi, np.uint64)
        out = np.zeros((n, 24), np.int8)
        shell = np.zeros(n, np.int32)
        bad = lib().ora_decode_batch_shell(self._h, n, _p(lo, u64p),
                                           None if hi_a is None else _p(hi_a, u64p),
                                           _p(out, i8p), _p(shell, i32p))
        if with_shell:
            return out, shell, int(bad)
        return out

    def search(self, X, m_max: int, mode: int, scale: float = 1.0, threads: int = 1):
        """Best point of shells 2..m_max for each row of X (fp32 [n, 24]) under the angular
        (mode 0) or Euclidean (mode 1, reconstruction scale * v) criterion.
        Returns (points int8 [n, 24], <x, v> fp64 [n])."""
        X, n, V, d = _search_args(X)
        if lib().ora_search_batch(self._h, m_max, mode, scale, n, X.ctypes.data_as(C.POINTER(C.c_float)),
                                  _p(V, i8p), _p(d, f64p), threads):
            raise ValueError("bad search arguments")
        return V, d

    def class_best(self, m: int, j: int, word: int, y):
        """Best point of class j of shell m with codeword word (1-mod-4 set of an odd class,
        2-mod-4 set of an even one) for target y; returns (point, <y, v>)."""
        yy = np.ascontiguousarray(y, np.float64)
        v = np.zeros(24, np.int32)
        d = C.c_double()
        if lib().ora_class_best(self._h, m, j, word, _p(yy, f64p), _p(v, i32p), C.byref(d)):
            raise ValueError("no such class, or the word does not fit it")
        return v, d.value

    def spherical_gptq(self, W, U, max_shell: int):
        """One Spherical GPTQ pass: returns (W after the pass, points int8 [rows, nb, 24], norms
        [rows, nb]); W fp64 [rows, cols], U fp64 [cols, cols] upper triangular, H^-1 = U^T U."""
        W = np.array(W, np.float64, order="C", copy=True)
        U = np.ascontiguousarray(U, np.float64)
        rows, cols = W.shape
        nb = cols // 24
        P = np.zeros((rows, nb, 24), np.int8)
        Nr = np.zeros((rows, nb), np.float64)
        if lib().ora_spherical_gptq(self._h, max_shell, rows, cols, _p(W, f64p), _p(U, f64p), _p(P, i8p), _p(Nr, f64p)):
            raise ValueError("bad Spherical GPTQ arguments")
        return W, P, Nr

    def gemm(self, words: np.ndarray, nb: int, gain_mode: int, gains: np.ndarray, x: np.ndarray,
             batch: int, row_pitch_words: int | None = None, threads: int = 1) -> np.ndarray:
        """fp64 y[batch, rows] from packed words [rows, pitch] (uint64, or uint64 pairs for
        16-byte words given as [rows, pitch, 2]), fp16 gains and fp16 x [batch, nb*24]."""
        words = np.ascontiguousarray(words)
        word_bytes = 16 if words.ndim == 3 else 8
        rows = words.shape[0]
        pitch = words.shape[1] if row_pitch_words is None else row_pitch_words
        g = np.ascontiguousarray(gains).view(np.uint16)
        xx = np.ascontiguousarray(x).view(np.uint16)
        assert xx.size == batch * nb * 24
        y = np.zeros((batch, rows), np.float64)
        if threads > 1:
            bad = lib().ora_gemm_mt(self._h, rows, nb, words.ctypes.data_as(C.c_void_p), word_bytes,
                                    pitch, gain_mode, _p(g, u16p), _p(xx, u16p), batch,
                                    _p(y, f64p), threads)
        else:
            bad = lib().ora_gemm(self._h, rows, nb, words.ctypes.data_as(C.c_void_p), word_bytes,
                                 pitch, gain_mode, _p(g, u16p), _p(xx, u16p), batch, _p(y, f64p))
        if bad < 0:
            raise ValueError("word size does not match the index budget")
        return y


ANGULAR, EUCLIDEAN = 0, 1


def _search_args(X):
    X = np.ascontiguousarray(X, np.float32).reshape(-1, 24)
    n = X.shape[0]
    return X, n, np.zeros((n, 24), np.int8), np.zeros(n, np.float64)


def search_brute(X, m_max: int, mode: int, scale: float = 1.0, threads: int = 1):
    """Best point of shells 2..m_max for each row of X by enumerating every point from the
    congruences (no classes).  Returns (points int8 [n, 24], <x, v> [n], points visited)."""
    X, n, V, d = _search_args(X)
    visited = lib().ora_search_brute(m_max, mode, scale, n, X.ctypes.data_as(C.POINTER(C.c_float)),
                                     _p(V, i8p), _p(d, f64p), threads)
    if visited < 0:
        raise ValueError("bad search arguments")
    return V, d, int(visited)


def gptq_block_matrix(U, b: int):
    """G_B = U_BB^-1 U_B,rest of block b ([24, cols], zero before the later columns)."""
    U = np.ascontiguousarray(U, np.float64)
    cols = U.shape[0]
    G = np.zeros((24, cols), np.float64)
    if lib().ora_gptq_block_matrix(cols, _p(U, f64p), b, _p(G, f64p)):
        raise ValueError("bad block")
    return G


def search_objective(mode: int, scale: float, dot, norm2):
    """The quantity each search mode maximizes, from <x, v> and |v|^2 (scaled coordinates)."""
    dot = np.asarray(dot, np.float64)
    norm2 = np.asarray(norm2, np.float64)
    if mode == ANGULAR:
        return dot / np.sqrt(norm2)
    return 2.0 * scale * dot - scale * scale * norm2


def half_to_double(h: int) -> float:
    return float(lib().ora_half_to_double(h))
