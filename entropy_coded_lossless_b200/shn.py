"""ctypes binding of libshn.so (include/shn.h) — argument marshalling only.

Every step of the codec runs in the library's CUDA kernels; this module only passes device
pointers (from torch tensors), host segment arrays and the current CUDA stream. There is no CPU
fallback: if the library is missing or a call is made with CPU tensors, it raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libshn.so")

SHN_OK = 0
SHN_ERR_INVALID_ARG = 1
SHN_ERR_CAPACITY = 2
SHN_ERR_CORRUPT = 3
SHN_ERR_CUDA = 4
SHN_ERR_TIMEOUT = 5
SHN_ERR_UNSUPPORTED = 6
SHN_ERR_WORKSPACE = 7
TABLE_BYTES = 11264
TABLE_PUBLIC_BYTES = 800

EXPORTED = [
    "shn_version", "shn_status_string", "shn_check_params", "shn_table_bytes", "shn_encode_bound",
    "shn_encode_workspace_bytes", "shn_encode_workspace_bytes_min", "shn_decode_workspace_bytes", "shn_histogram", "shn_build_tables",
    "shn_encode", "shn_decode", "shn_decode_bf16", "shn_decode_from_host", "shn_offload_workspace_bytes",
    "shn_offload", "shn_get_device_status", "shn_encode_static_max_chunks", "shn_encode_static",
]


class ShnError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class Segment(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_uint64), ("length", ctypes.c_uint64)]


class Params(ctypes.Structure):
    _fields_ = [("K", ctypes.c_uint32), ("log2L", ctypes.c_uint32), ("chunk_symbols", ctypes.c_uint32),
                ("states_per_chunk", ctypes.c_uint32)]


@dataclass(frozen=True)
class CodecParams:
    K: int = 16
    log2L: int = 7
    chunk_symbols: int = 4096
    states_per_chunk: int = 4

    def c(self) -> Params:
        return Params(self.K, self.log2L, self.chunk_symbols, self.states_per_chunk)


_lib = None


def lib():
    """Load libshn.so from the package directory (built by entropy_coded_lossless_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libshn.so not built at {LIB_PATH}; run python -m entropy_coded_lossless_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        u32, u64, i32, vp, sz = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        P = ctypes.POINTER(Params)
        sigs = {
            "shn_version": (u32, []),
            "shn_status_string": (ctypes.c_char_p, [i32]),
            "shn_check_params": (i32, [P]),
            "shn_table_bytes": (sz, [P]),
            "shn_encode_bound": (sz, [P, vp, u32]),
            "shn_encode_workspace_bytes": (sz, [P, vp, u32]),
            "shn_encode_workspace_bytes_min": (sz, [P, vp, u32]),
            "shn_decode_workspace_bytes": (sz, [P]),
            "shn_histogram": (i32, [vp, vp, u32, vp, vp]),
            "shn_build_tables": (i32, [vp, u32, P, vp, vp]),
            "shn_encode": (i32, [vp, vp, u32, vp, P, vp, sz, vp, sz, vp, vp]),
            "shn_decode": (i32, [vp, sz, P, vp, sz, vp, sz, vp]),
            "shn_decode_bf16": (i32, [vp, sz, P, vp, sz, u32, vp, sz, vp, sz, vp]),
            "shn_offload_workspace_bytes": (sz, [P, vp, ctypes.POINTER(u32), u32]),
            "shn_offload": (i32, [vp, vp, ctypes.POINTER(u32), u32, P, vp, sz, vp, sz, ctypes.POINTER(sz),
                                  ctypes.POINTER(sz), vp, vp]),
            "shn_decode_from_host": (i32, [ctypes.POINTER(vp), ctypes.POINTER(sz), u32, P, vp, sz, vp, sz, vp,
                                           ctypes.POINTER(sz), sz, vp, vp]),
            "shn_get_device_status": (i32, [vp, ctypes.POINTER(u32), ctypes.POINTER(u32), vp]),
            "shn_encode_static_max_chunks": (u64, []),
            "shn_encode_static": (i32, [vp, vp, u32, vp, P, vp, sz, vp, vp, vp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().shn_status_string(int(code)).decode()
    except Exception:  # pragma: no cover - library missing
        return "unknown"


def _check(code: int, what: str):
    if code != SHN_OK:
        raise ShnError(code, what)


class Segments:
    """A segment list marshalled once into the C array the ABI takes (reused on every call)."""

    def __init__(self, segments):
        self.pairs = [(int(o), int(n)) for o, n in segments]
        self.arr = (Segment * max(1, len(self.pairs)))()
        for i, (o, n) in enumerate(self.pairs):
            self.arr[i].offset, self.arr[i].length = o, n

    def __len__(self):
        return len(self.pairs)

    def __iter__(self):
        return iter(self.pairs)


def _segments(segments):
    if isinstance(segments, Segments):
        return segments.arr
    return Segments(segments).arr


def _dev(t: torch.Tensor, name: str, host_ok: bool = False) -> int:
    """Device address of t; with host_ok, pinned host memory (mapped into the device address space)
    is accepted too."""
    if not isinstance(t, torch.Tensor) or not (t.is_cuda or (host_ok and t.is_pinned())):
        raise ValueError(f"{name} must be a CUDA tensor" + (" or pinned host memory" if host_ok else ""))
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _bytes_view(x: torch.Tensor) -> torch.Tensor:
    if x.dtype in (torch.int8, torch.uint8):
        return x.reshape(-1)
    raise ValueError("expected an int8/uint8 tensor")


# --------------------------------------------------------------------------------------------
# queries


def version() -> int:
    return int(lib().shn_version())


def check_params(p: CodecParams) -> int:
    return int(lib().shn_check_params(ctypes.byref(p.c())))


def table_bytes(p: CodecParams) -> int:
    return int(lib().shn_table_bytes(ctypes.byref(p.c())))


def encode_bound(p: CodecParams, segments) -> int:
    return int(lib().shn_encode_bound(ctypes.byref(p.c()), _segments(segments), len(segments)))


def encode_workspace_bytes(p: CodecParams, segments) -> int:
    """Workspace for the single-pass encoder (one worst-case slot per chunk)."""
    return int(lib().shn_encode_workspace_bytes(ctypes.byref(p.c()), _segments(segments), len(segments)))


def encode_workspace_bytes_min(p: CodecParams, segments) -> int:
    """Smallest encoder workspace (two-pass mode)."""
    return int(lib().shn_encode_workspace_bytes_min(ctypes.byref(p.c()), _segments(segments), len(segments)))


def decode_workspace_bytes(p: CodecParams) -> int:
    return int(lib().shn_decode_workspace_bytes(ctypes.byref(p.c())))


# --------------------------------------------------------------------------------------------
# the four calls, one-to-one with the C ABI


def shn_histogram(x: torch.Tensor, segments, hist: torch.Tensor, stream=None):
    xb = _bytes_view(x)
    _check(lib().shn_histogram(_dev(xb, "x"), _segments(segments), len(segments), _dev(hist, "hist"),
                               _stream(stream)), "shn_histogram")


def shn_build_tables(hist: torch.Tensor, n_tables: int, p: CodecParams, tables: torch.Tensor, stream=None):
    _check(lib().shn_build_tables(_dev(hist, "hist"), n_tables, ctypes.byref(p.c()), _dev(tables, "tables"),
                                  _stream(stream)), "shn_build_tables")


def shn_encode(x: torch.Tensor, segments, tables: torch.Tensor, p: CodecParams, work: torch.Tensor,
               out: torch.Tensor, out_bytes: torch.Tensor, stream=None):
    xb = _bytes_view(x)
    _check(lib().shn_encode(_dev(xb, "x") if xb.numel() else (xb.data_ptr() or None), _segments(segments),
                            len(segments), _dev(tables, "tables") if tables.numel() else None, ctypes.byref(p.c()),
                            _dev(work, "work"), work.numel(), _dev(out, "out", host_ok=True), out.numel(),
                            _dev(out_bytes, "out_bytes"), _stream(stream)), "shn_encode")


def shn_encode_static(x: torch.Tensor, segments, tables: torch.Tensor, p: CodecParams, out: torch.Tensor,
                      out_bytes: torch.Tensor, status: torch.Tensor, stream=None):
    """shn_encode with the library's built-in scratch array instead of a caller workspace."""
    xb = _bytes_view(x)
    _check(lib().shn_encode_static(_dev(xb, "x") if xb.numel() else None, _segments(segments), len(segments),
                                   _dev(tables, "tables") if tables.numel() else None, ctypes.byref(p.c()),
                                   _dev(out, "out"), out.numel(), _dev(out_bytes, "out_bytes"),
                                   _dev(status, "status"), _stream(stream)), "shn_encode_static")


def encode_static_max_chunks() -> int:
    return int(lib().shn_encode_static_max_chunks())


def shn_decode(comp: torch.Tensor, comp_bytes: int, p: CodecParams, work: torch.Tensor, out: torch.Tensor,
               stream=None):
    _check(lib().shn_decode(_dev(comp, "comp"), int(comp_bytes), ctypes.byref(p.c()), _dev(work, "work"),
                            work.numel(), _dev(out, "out") if out.numel() else None, out.numel(),
                            _stream(stream)), "shn_decode")


def shn_decode_bf16(comp: torch.Tensor, comp_bytes: int, p: CodecParams, scales: torch.Tensor, log2_group: int,
                    work: torch.Tensor, out: torch.Tensor, stream=None):
    """Decode fused with dequantisation: out (bfloat16) = int8 value x scales[i >> log2_group]."""
    if scales.dtype != torch.float32 or out.dtype != torch.bfloat16:
        raise ValueError("scales must be float32 and out bfloat16")
    _check(lib().shn_decode_bf16(_dev(comp, "comp"), int(comp_bytes), ctypes.byref(p.c()), _dev(scales, "scales"),
                                 scales.numel(), int(log2_group), _dev(work, "work"), work.numel(),
                                 _dev(out, "out") if out.numel() else None, out.numel(), _stream(stream)),
           "shn_decode_bf16")


def offload_workspace_bytes(p: CodecParams, segments, batch_ends) -> int:
    ends = (ctypes.c_uint32 * len(batch_ends))(*[int(e) for e in batch_ends])
    return int(lib().shn_offload_workspace_bytes(ctypes.byref(p.c()), _segments(segments), ends, len(batch_ends)))


def shn_offload(x: torch.Tensor, segments, batch_ends, p: CodecParams, work: torch.Tensor, h_out: torch.Tensor,
                stream=None, copy_stream=None):
    """Offload x as one SHN1 stream per batch of segments into pinned host memory h_out; returns
    (offsets, sizes) of the streams in h_out. Blocks until the last batch is encoded."""
    if h_out.device.type != "cpu" or h_out.dtype != torch.uint8:
        raise ValueError("h_out must be a uint8 CPU tensor")
    nb = len(batch_ends)
    ends = (ctypes.c_uint32 * nb)(*[int(e) for e in batch_ends])
    offs, sizes = (ctypes.c_size_t * nb)(), (ctypes.c_size_t * nb)()
    xb = _bytes_view(x)
    _check(lib().shn_offload(_dev(xb, "x"), _segments(segments), ends, nb, ctypes.byref(p.c()), _dev(work, "work"),
                             work.numel(), h_out.data_ptr(), h_out.numel(), offs, sizes, _stream(stream),
                             _stream(copy_stream if copy_stream is not None else stream)), "shn_offload")
    return list(offs), list(sizes)


def shn_decode_from_host(h_streams, stream_bytes, p: CodecParams, staging: torch.Tensor, work: torch.Tensor,
                         out: torch.Tensor, out_offsets, stream=None, copy_stream=None):
    """Pipelined reload: copy each host stream (pinned uint8 tensors) to `staging` on copy_stream
    while the previous one decodes into out[out_offsets[i]:] on stream."""
    n = len(h_streams)
    for t in h_streams:
        if t.device.type != "cpu" or t.dtype != torch.uint8:
            raise ValueError("host streams must be uint8 CPU tensors")
    ptrs = (ctypes.c_void_p * n)(*[t.data_ptr() for t in h_streams])
    sizes = (ctypes.c_size_t * n)(*[int(b) for b in stream_bytes])
    offs = (ctypes.c_size_t * n)(*[int(o) for o in out_offsets])
    _check(lib().shn_decode_from_host(ptrs, sizes, n, ctypes.byref(p.c()), _dev(staging, "staging"), staging.numel(),
                                      _dev(work, "work"), work.numel(), _dev(out, "out"), offs, out.numel(),
                                      _stream(stream), _stream(copy_stream if copy_stream is not None else stream)),
           "shn_decode_from_host")


def shn_get_device_status(work: torch.Tensor, stream=None):
    st, det = ctypes.c_uint32(0), ctypes.c_uint32(0)
    _check(lib().shn_get_device_status(_dev(work, "work"), ctypes.byref(st), ctypes.byref(det), _stream(stream)),
           "shn_get_device_status")
    return int(st.value), int(det.value)


# --------------------------------------------------------------------------------------------
# buffers and a convenience round trip built only from the calls above


def empty_aligned(nbytes: int, device, align: int = 256) -> torch.Tensor:
    """uint8 device buffer whose data pointer is `align`-byte aligned (torch's allocator gives 512)."""
    t = torch.empty(max(1, nbytes) + align, dtype=torch.uint8, device=device)
    off = (-t.data_ptr()) % align
    return t[off:off + nbytes]


class Codec:
    """Holds the device buffers for repeated encode/decode of one segment layout."""

    def __init__(self, segments, p: CodecParams = CodecParams(), device="cuda", single_pass=True):
        """single_pass: allocate the encoder workspace that lets every chunk be coded once into its
        own slot (about the stream bound); otherwise the minimal one (two-pass encoder)."""
        self.p = p
        self.segments = Segments(segments)  # marshalled once: the calls below reuse the C array
        self.device = torch.device(device)
        ns = len(self.segments)
        self.hist = torch.zeros(max(1, ns) * 256, dtype=torch.int64, device=self.device)
        self.tables = empty_aligned(max(1, ns) * TABLE_BYTES, self.device)
        wsize = encode_workspace_bytes if single_pass else encode_workspace_bytes_min
        self.work_enc = empty_aligned(wsize(p, self.segments), self.device)
        self.work_dec = empty_aligned(decode_workspace_bytes(p), self.device)
        self.bound = encode_bound(p, self.segments)
        if self.bound == 0:
            raise ShnError(SHN_ERR_INVALID_ARG, "encode_bound")
        self.stream_buf = empty_aligned(self.bound, self.device, 16)
        self.out_bytes = torch.zeros(1, dtype=torch.int64, device=self.device)
        self.n_symbols = sum(n for _, n in self.segments)

    def histogram(self, x, stream=None):
        shn_histogram(x, self.segments, self.hist, stream)

    def build(self, stream=None):
        shn_build_tables(self.hist, len(self.segments), self.p, self.tables, stream)

    def encode(self, x, stream=None):
        shn_encode(x, self.segments, self.tables, self.p, self.work_enc, self.stream_buf, self.out_bytes, stream)

    def compress(self, x, stream=None):
        """histogram → tables → encode, all on the device; returns nothing (stream_buf/out_bytes)."""
        self.histogram(x, stream)
        self.build(stream)
        self.encode(x, stream)

    def decode(self, comp, comp_bytes, out, stream=None):
        shn_decode(comp, comp_bytes, self.p, self.work_dec, out, stream)

    def status(self, which="enc", stream=None):
        return shn_get_device_status(self.work_enc if which == "enc" else self.work_dec, stream)

    def table_fields(self, i: int):
        """Public fields of table record i (host copy): K, log2L, status, w_max, dp_cost, n, f, lo."""
        rec = self.tables[i * TABLE_BYTES:i * TABLE_BYTES + TABLE_PUBLIC_BYTES].cpu()
        hdr = rec[:16].view(torch.int32)
        dp_cost = int(rec[16:24].view(torch.int64)[0])
        n = int(rec[24:32].view(torch.int64)[0])
        f = rec[32:544].view(torch.int16).to(torch.int32) & 0xFFFF
        lo = rec[544:800].to(torch.int32)
        K = int(hdr[0])
        return dict(K=K, log2L=int(hdr[1]), status=int(hdr[2]), w_max=int(hdr[3]), dp_cost=dp_cost, n=n,
                    f=f[:K].tolist(), lo=lo[:K].tolist())
