"""LLVQ (Leech lattice vector quantization) decode and fused decode-and-multiply on B200.

A thin ctypes binding over libllvq.so (the C ABI in include/llvq.h).  Every step of the
decode, the products, the encoder, the nearest-point search and the Spherical GPTQ pass runs in
the library's CUDA kernels; this module only marshals arguments (device pointers of torch
tensors, the current CUDA stream; a workspace tensor for the GPTQ pass when none is given).  There is no CPU
fallback: importing the binding fails if libllvq.so is missing or cannot be loaded.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libllvq.so")

LLVQ_OK = 0
LLVQ_ERR_ARG = 1
LLVQ_ERR_UNSUPPORTED = 2
LLVQ_ERR_CUDA = 3
LLVQ_ERR_DEVICE_FLAG = 4
LLVQ_GAIN_FP16_DIRECT = 0
LLVQ_GAIN_U8_TABLE = 1
LLVQ_FLAG_INDEX_RANGE = 0x1
LLVQ_FLAG_WAIT_TIMEOUT = 0x2
LLVQ_FLAG_NOT_CODED = 0x4
LLVQ_FLAG_SEARCH_INPUT = 0x8
LLVQ_SEARCH_ANGULAR = 0
LLVQ_SEARCH_EUCLIDEAN = 1


class llvq_weight(C.Structure):
    _fields_ = [("rows", C.c_int32), ("cols", C.c_int32), ("blocks_per_row", C.c_int32),
                ("index_bits", C.c_int32), ("word_bytes", C.c_int32), ("gain_mode", C.c_int32),
                ("row_pitch_words", C.c_int64), ("words", C.c_void_p), ("gains", C.c_void_p)]


class llvq_class96(C.Structure):
    _fields_ = [("start_lo", C.c_uint64), ("start_hi", C.c_uint32), ("meta", C.c_uint32),
                ("rcp_lo", C.c_uint64), ("rcp_hi", C.c_uint64), ("cum", C.c_uint32 * 4),
                ("vals", C.c_uint32 * 4)]


class LLVQError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = lib().llvq_last_error_message().decode()
        super().__init__(f"{what}: {llvq_status_string(status)} ({status})" + (f": {msg}" if msg else ""))
        self.status = status


_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libllvq.so not built at {LIB_PATH}; run codebook_free_lattice_b200/build.py")
        L = C.CDLL(LIB_PATH)
        L.llvq_status_string.argtypes = [C.c_int]
        L.llvq_status_string.restype = C.c_char_p
        L.llvq_codec_create.argtypes = [C.c_int32, C.POINTER(C.c_void_p)]
        L.llvq_codec_destroy.argtypes = [C.c_void_p]
        L.llvq_codec_destroy.restype = None
        L.llvq_codec_info.argtypes = [C.c_void_p, C.POINTER(C.c_int32), C.POINTER(C.c_uint64),
                                      C.POINTER(C.c_uint64), C.POINTER(C.c_int64)]
        L.llvq_decode.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_int64, C.c_void_p, C.c_void_p]
        L.llvq_gemv.argtypes = [C.c_void_p, C.POINTER(llvq_weight), C.c_void_p, C.c_void_p, C.c_void_p]
        L.llvq_gemm_smallbatch.argtypes = [C.c_void_p, C.POINTER(llvq_weight), C.c_void_p, C.c_int32,
                                           C.c_void_p, C.c_void_p]
        L.llvq_get_error.argtypes = [C.c_void_p, C.c_void_p, C.POINTER(C.c_uint32)]
        L.llvq_decode_noalloc.argtypes = [C.c_int32, C.c_void_p, C.c_int32, C.c_int64, C.c_void_p, C.c_void_p]
        L.llvq_encode.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_int32, C.c_void_p]
        L.llvq_search.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_double, C.c_void_p, C.c_int64,
                                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p]
        L.llvq_spherical_gptq_workspace.argtypes = [C.c_int32, C.c_int32]
        L.llvq_spherical_gptq_workspace.restype = C.c_size_t
        L.llvq_spherical_gptq.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                                          C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
        L.llvq_set_wait_polls.argtypes = [C.c_uint32, C.c_uint32]
        L.llvq_set_wait_polls.restype = None
        L.llvq_last_error_message.argtypes = []
        L.llvq_last_error_message.restype = C.c_char_p
        L.llvq_class_table96.argtypes = [C.c_int32, C.c_void_p, C.c_int64, C.POINTER(C.c_int64)]
        for f in ("llvq_codec_create", "llvq_codec_info", "llvq_decode", "llvq_gemv",
                  "llvq_gemm_smallbatch", "llvq_get_error", "llvq_decode_noalloc", "llvq_class_table96",
                  "llvq_encode", "llvq_search", "llvq_spherical_gptq"):
            getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


EXPORTED = ("llvq_codec_create", "llvq_codec_destroy", "llvq_codec_info", "llvq_decode",
            "llvq_gemv", "llvq_gemm_smallbatch", "llvq_get_error", "llvq_status_string",
            "llvq_decode_noalloc", "llvq_class_table96", "llvq_last_error_message", "llvq_encode",
            "llvq_set_wait_polls", "llvq_search", "llvq_spherical_gptq", "llvq_spherical_gptq_workspace")


def llvq_set_wait_polls(table_polls: int = 0xFFFFFFFF, mma_polls: int = 0xFFFFFFFF) -> None:
    """Limits of the kernels' first bounded waits (tests of the timeout paths); defaults restore."""
    lib().llvq_set_wait_polls(table_polls, mma_polls)


def llvq_status_string(status: int) -> str:
    return lib().llvq_status_string(status).decode()


def llvq_decode_noalloc(words, out, n: int | None = None, stream=None):
    """48-bit decode through the entry point that allocates no device memory (its tables live
    in a static device array; see include/llvq.h).  words: device int64 words; out: int8 [n, 24]."""
    n = out.shape[0] if n is None else n
    _check(lib().llvq_decode_noalloc(48, C.c_void_p(words.data_ptr()), 8, n, C.c_void_p(out.data_ptr()),
                                     _stream(stream)), "llvq_decode_noalloc")


def class_table96(m: int):
    """Host-side 96-bit class records of shell m (no device needed), as a numpy structured array
    with the fields of llvq_class96 (include/llvq.h)."""
    import numpy as np
    n = C.c_int64()
    _check(lib().llvq_class_table96(m, None, 0, C.byref(n)), f"llvq_class_table96({m})")
    dt = np.dtype([("start_lo", "<u8"), ("start_hi", "<u4"), ("meta", "<u4"), ("rcp_lo", "<u8"),
                   ("rcp_hi", "<u8"), ("cum", "u1", 16), ("vals", "u1", 16)])
    assert dt.itemsize == C.sizeof(llvq_class96) == 64
    out = np.zeros(n.value, dt)
    _check(lib().llvq_class_table96(m, out.ctypes.data_as(C.c_void_p), n.value, C.byref(n)),
           f"llvq_class_table96({m})")
    return out


def _check(status: int, what: str):
    if status != LLVQ_OK:
        raise LLVQError(status, what)


def _stream(stream) -> C.c_void_p:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


class Codec:
    """Decode and encode tables of one index budget (48, 72 or 96 bits) on the current CUDA device.
    close() (or leaving a `with` block) releases them at once; the 96-bit tables hold 23.6 GB."""

    def __init__(self, index_bits: int = 48):
        h = C.c_void_p()
        _check(lib().llvq_codec_create(index_bits, C.byref(h)), f"llvq_codec_create({index_bits})")
        self._h = h
        self.index_bits = index_bits
        M, lo, hi, nc = C.c_int32(), C.c_uint64(), C.c_uint64(), C.c_int64()
        _check(lib().llvq_codec_info(h, C.byref(M), C.byref(lo), C.byref(hi), C.byref(nc)), "llvq_codec_info")
        self.max_shell = M.value
        self.n_points = (hi.value << 64) | lo.value
        self.n_classes = nc.value
        self.word_bytes = 8 if index_bits == 48 else 16

    @property
    def handle(self) -> C.c_void_p:
        return self._h

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            lib().llvq_codec_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
        return False

    def weight(self, words, gains, rows: int, cols: int, gain_mode: int,
               row_pitch_words: int | None = None) -> llvq_weight:
        nb = -(-cols // 24)
        pitch = nb if row_pitch_words is None else row_pitch_words
        return llvq_weight(rows, cols, nb, self.index_bits, self.word_bytes, gain_mode, pitch,
                           words.data_ptr(), gains.data_ptr())

    def decode(self, words, out, n: int | None = None, stream=None):
        """words: device tensor of packed words; out: device int8 [n, 24]."""
        n = out.shape[0] if n is None else n
        _check(lib().llvq_decode(self._h, C.c_void_p(words.data_ptr()), self.word_bytes, n,
                                 C.c_void_p(out.data_ptr()), _stream(stream)), "llvq_decode")

    def encode(self, vectors, words, n: int | None = None, stream=None):
        """vectors: device int8 [n, 24] lattice points; words: device int64 [n] (48-bit budget),
        written with the packed indices (gain code 0)."""
        n = vectors.shape[0] if n is None else n
        _check(lib().llvq_encode(self._h, C.c_void_p(vectors.data_ptr()), n, C.c_void_p(words.data_ptr()),
                                 self.word_bytes, _stream(stream)), "llvq_encode")

    def search(self, X, points, max_shell: int, mode: int, scale: float = 1.0, dots=None,
               levels=None, codes=None, n: int | None = None, stream=None):
        """Nearest point of shells 2..max_shell for each row of X (device fp32 [n, 24]) into points
        (device int8 [n, 24]); dots (device fp64 [n]) receives <x, v>; with levels (device fp64)
        and codes (device uint8 [n]) the angular criterion also picks the nearest gain level."""
        n = X.shape[0] if n is None else n
        ptr = lambda t: None if t is None else C.c_void_p(t.data_ptr())
        _check(lib().llvq_search(self._h, max_shell, mode, scale, ptr(X), n, ptr(points), ptr(dots),
                                 ptr(levels), 0 if levels is None else levels.numel(), ptr(codes),
                                 _stream(stream)), "llvq_search")

    def spherical_gptq(self, W, U, points, norms, max_shell: int, workspace=None, stream=None):
        """One Spherical GPTQ pass in place on W (device fp64 [rows, cols]) with U (device fp64
        [cols, cols], upper, H^-1 = U^T U); points (device int8 [rows, cols/24, 24]) and norms
        (device fp64 [rows, cols/24]) receive v and |w| per block.  workspace: a device uint8 tensor
        of at least spherical_gptq_workspace(rows, cols) bytes (allocated here when None)."""
        import torch
        rows, cols = W.shape
        need = lib().llvq_spherical_gptq_workspace(rows, cols)
        if workspace is None:
            workspace = torch.empty(max(int(need), 256), dtype=torch.uint8, device=W.device)
        _check(lib().llvq_spherical_gptq(self._h, max_shell, rows, cols, C.c_void_p(W.data_ptr()),
                                         C.c_void_p(U.data_ptr()), C.c_void_p(points.data_ptr()),
                                         C.c_void_p(norms.data_ptr()), C.c_void_p(workspace.data_ptr()),
                                         workspace.numel(), _stream(stream)), "llvq_spherical_gptq")
        return workspace

    def gemv(self, w: llvq_weight, x, y, stream=None):
        _check(lib().llvq_gemv(self._h, C.byref(w), C.c_void_p(x.data_ptr()), C.c_void_p(y.data_ptr()),
                               _stream(stream)), "llvq_gemv")

    def gemm(self, w: llvq_weight, X, Y, batch: int, stream=None):
        _check(lib().llvq_gemm_smallbatch(self._h, C.byref(w), C.c_void_p(X.data_ptr()), batch,
                                          C.c_void_p(Y.data_ptr()), _stream(stream)), "llvq_gemm_smallbatch")

    def get_error(self, stream=None) -> int:
        flags = C.c_uint32()
        st = lib().llvq_get_error(self._h, _stream(stream), C.byref(flags))
        if st not in (LLVQ_OK, LLVQ_ERR_DEVICE_FLAG):
            raise LLVQError(st, "llvq_get_error")
        return flags.value
