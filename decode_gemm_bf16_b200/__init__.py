"""Python binding of libunweight (argument marshalling only).

Every function forwards to the C ABI declared in ``include/unweight.h``; all
work runs in the library's CUDA kernels.  torch provides device memory and
streams.  There is no CPU fallback: if the shared library is missing the
import of a function raises.

The method: "Cloudflare推出Unweight無損壓縮系統，將LLM模型大小壓縮15-22%"
(easyvibecoding.app) -- §BF16權重壓縮原理 (format), §四種執行管道 (pipelines),
§重建矩陣乘法核心運作 (reconstructive GEMM), §自動調優機制 (autotuner).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libunweight.so")

UW_OK = 0
STATUS = {0: "UW_OK", 1: "UW_ERR_INVALID_ARG", 2: "UW_ERR_SHAPE", 3: "UW_ERR_CORRUPT",
          4: "UW_ERR_UNSUPPORTED", 5: "UW_ERR_WORKSPACE", 6: "UW_ERR_CUDA", 7: "UW_ERR_TIMEOUT",
          8: "UW_ERR_DEVICE"}
UW_PIPE_AUTO, UW_PIPE_FULL, UW_PIPE_EXPONENT, UW_PIPE_TRANSCODE, UW_PIPE_DIRECT_PALETTE = -1, 0, 1, 2, 3
UW_PIPE_FUSED_HUFFMAN = 4
PIPELINES = {"full": 0, "exponent": 1, "transcode": 2, "direct_palette": 3, "fused_huffman": 4}
UW_VARIANT_AUTO, UW_VARIANT_TENSOR, UW_VARIANT_GEMV = 0, 1, 2
VARIANTS = {"auto": 0, "tensor": 1, "gemv": 2}
UW_FORM_HUFFMAN, UW_FORM_PALETTE = 1, 2
SECTIONS = ["sm", "vbits", "vpre", "vexp", "vcol", "idx", "stream", "chunk_off", "seg_rel", "lut"]

# every entry point of include/unweight.h
EXPORTS = ["uw_status_str", "uw_version", "uw_last_device_status", "uw_compress_scratch_bytes",
           "uw_compress_query", "uw_compress_commit", "uw_blob_info_get", "uw_blob_section",
           "uw_blob_serialized_bytes", "uw_blob_serialize", "uw_blob_device_bytes",
           "uw_blob_deserialize", "uw_blob_free", "uw_decode_full", "uw_decode_exponent",
           "uw_transcode_palette", "uw_gemm_workspace", "uw_gemm", "uw_dense_gemm_workspace",
           "uw_dense_gemm", "uw_autotune", "uw_gemm_direct_palette_noalloc", "uw_plan_resolve",
           "uw_plan_load_json", "uw_gemm_swiglu_workspace", "uw_gemm_swiglu",
           "uw_sequence_workspace", "uw_gemm_sequence"]


class UnweightError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class BlobInfo(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("G", ctypes.c_int64), ("V", ctypes.c_int64),
                ("nseg", ctypes.c_int64), ("nchunk", ctypes.c_int64), ("forms", ctypes.c_uint32),
                ("palette", ctypes.c_uint8 * 16), ("code_len", ctypes.c_uint8 * 16),
                ("freq", ctypes.c_uint64 * 16), ("hist", ctypes.c_uint64 * 256),
                ("total_bits", ctypes.c_uint64), ("bytes_huffman_form", ctypes.c_uint64),
                ("bytes_palette_form", ctypes.c_uint64), ("device_bytes", ctypes.c_uint64),
                ("mean_code_len", ctypes.c_double), ("exponent_entropy", ctypes.c_double),
                ("palette_coverage", ctypes.c_double), ("section_offset", ctypes.c_uint64 * 10),
                ("section_bytes", ctypes.c_uint64 * 10)]


class SeqItem(ctypes.Structure):
    _fields_ = [("blob", ctypes.c_void_p), ("X", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("hard", ctypes.c_int32)]


class PlanEntry(ctypes.Structure):
    _fields_ = [("blob_index", ctypes.c_int32), ("M", ctypes.c_int64), ("pipeline", ctypes.c_int32),
                ("variant", ctypes.c_int32), ("sm_dec", ctypes.c_int32), ("grid", ctypes.c_int32),
                ("split_k", ctypes.c_int32), ("us", ctypes.c_double), ("layer_us", ctypes.c_double)]


class GemmOpts(ctypes.Structure):
    _fields_ = [("pipeline", ctypes.c_int32), ("sm_dec", ctypes.c_int32), ("grid", ctypes.c_int32),
                ("out_f32", ctypes.c_int32), ("variant", ctypes.c_int32), ("split_k", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("projection", ctypes.c_int32),
                ("plan", ctypes.POINTER(PlanEntry)), ("plan_entries", ctypes.c_int32),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


_lib = None


def lib():
    """Loads libunweight.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libunweight.so not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        sig = {
            "uw_status_str": ([I32], ctypes.c_char_p),
            "uw_version": ([], I32),
            "uw_last_device_status": ([P], I32),
            "uw_compress_scratch_bytes": ([I64, I64, ctypes.POINTER(SZ)], I32),
            "uw_compress_query": ([P, I64, I64, ctypes.c_uint32, P, SZ, P, ctypes.POINTER(P),
                                   ctypes.POINTER(SZ)], I32),
            "uw_compress_commit": ([P, P, P, SZ, P, SZ, P], I32),
            "uw_blob_info_get": ([P, ctypes.POINTER(BlobInfo)], I32),
            "uw_blob_section": ([P, I32, ctypes.POINTER(P), ctypes.POINTER(SZ)], I32),
            "uw_blob_serialized_bytes": ([P, ctypes.POINTER(SZ)], I32),
            "uw_blob_serialize": ([P, P, SZ, ctypes.POINTER(SZ), P], I32),
            "uw_blob_device_bytes": ([P, SZ, ctypes.POINTER(SZ)], I32),
            "uw_blob_deserialize": ([P, SZ, P, SZ, P, ctypes.POINTER(P)], I32),
            "uw_blob_free": ([P], None),
            "uw_decode_full": ([P, P, P], I32),
            "uw_decode_exponent": ([P, P, P], I32),
            "uw_transcode_palette": ([P, P, P], I32),
            "uw_gemm_workspace": ([P, I64, ctypes.POINTER(GemmOpts), ctypes.POINTER(SZ)], I32),
            "uw_gemm": ([P, I64, P, P, ctypes.POINTER(GemmOpts), P], I32),
            "uw_plan_resolve": ([ctypes.POINTER(GemmOpts), I64, ctypes.POINTER(GemmOpts)], I32),
            "uw_gemm_swiglu_workspace": ([P, P, I64, ctypes.POINTER(GemmOpts), ctypes.POINTER(SZ)], I32),
            "uw_gemm_swiglu": ([P, I64, P, P, P, ctypes.POINTER(GemmOpts), P], I32),
            "uw_sequence_workspace": ([ctypes.POINTER(SeqItem), I32, I64, ctypes.POINTER(SZ)], I32),
            "uw_gemm_sequence": ([ctypes.POINTER(SeqItem), I32, I64, I32, I32, P, SZ, P], I32),
            "uw_dense_gemm_workspace": ([I64, I64, I64, I32, I32, I32, ctypes.POINTER(SZ)], I32),
            "uw_dense_gemm": ([P, I64, P, I64, I64, P, I32, I32, I32, I32, P, SZ, P], I32),
            "uw_gemm_direct_palette_noalloc": ([P, I64, P, P, I32, P], I32),
            "uw_autotune": ([ctypes.POINTER(P), I32, I32, ctypes.POINTER(I64), I32, ctypes.POINTER(P),
                             ctypes.POINTER(P), P, SZ, I32, ctypes.POINTER(PlanEntry), ctypes.c_char_p, P], I32),
            "uw_plan_load_json": ([ctypes.c_char_p, ctypes.POINTER(PlanEntry), I32, ctypes.POINTER(I32)], I32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(st: int, what: str):
    if st != UW_OK:
        raise UnweightError(what, st)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _bits16(t: torch.Tensor) -> torch.Tensor:
    """Accepts bf16 / int16 / uint16 CUDA tensors; returns the same storage."""
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise ValueError(f"expected 16-bit BF16 bit patterns, got {t.dtype}")
    return t.contiguous()


def status_str(st: int) -> str:
    return lib().uw_status_str(st).decode()


def uw_version() -> int:
    return lib().uw_version()


def uw_last_device_status(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the device status word."""
    return lib().uw_last_device_status(_stream(stream))


class Blob:
    """A compressed weight matrix: the library handle plus its device image."""

    def __init__(self, handle: ctypes.c_void_p, dev: torch.Tensor):
        self._h = handle
        self.dev = dev
        self.info = uw_blob_info_get(self)
        self.N, self.K = self.info["N"], self.info["K"]

    @property
    def handle(self):
        return self._h

    def section(self, name: str) -> torch.Tensor:
        """Device bytes of one section (uint8 view into the device image)."""
        k = SECTIONS.index(name)
        ptr = ctypes.c_void_p()
        n = ctypes.c_size_t()
        _check(lib().uw_blob_section(self._h, k, ctypes.byref(ptr), ctypes.byref(n)), "uw_blob_section")
        off = (ptr.value or 0) - self.dev.data_ptr()
        return self.dev[off:off + n.value]

    def __del__(self):
        try:
            if self._h:
                lib().uw_blob_free(self._h)
                self._h = None
        except Exception:
            pass


def uw_blob_info_get(blob: Blob) -> dict:
    info = BlobInfo()
    _check(lib().uw_blob_info_get(blob.handle, ctypes.byref(info)), "uw_blob_info_get")
    out = {}
    for name, _ in BlobInfo._fields_:
        v = getattr(info, name)
        out[name] = list(v) if hasattr(v, "__len__") else v
    out["sections"] = {SECTIONS[i]: (info.section_offset[i], info.section_bytes[i]) for i in range(10)}
    return out


def uw_compress(W: torch.Tensor, forms: int = UW_FORM_HUFFMAN | UW_FORM_PALETTE, stream=None) -> Blob:
    """Compresses a device BF16 matrix W[N, K] (query + commit, torch-allocated)."""
    W = _bits16(W)
    N, K = W.shape
    L = lib()
    sb = ctypes.c_size_t()
    _check(L.uw_compress_scratch_bytes(N, K, ctypes.byref(sb)), "uw_compress_scratch_bytes")
    scratch = torch.empty(sb.value, dtype=torch.uint8, device=W.device)
    h = ctypes.c_void_p()
    db = ctypes.c_size_t()
    s = _stream(stream)
    _check(L.uw_compress_query(_ptr(W), N, K, forms, _ptr(scratch), sb.value, s, ctypes.byref(h),
                               ctypes.byref(db)), "uw_compress_query")
    dev = torch.empty(db.value, dtype=torch.uint8, device=W.device)
    st = L.uw_compress_commit(h, _ptr(W), _ptr(scratch), sb.value, _ptr(dev), db.value, s)
    if st != UW_OK:
        L.uw_blob_free(h)
        raise UnweightError("uw_compress_commit", st)
    return Blob(h, dev)


def uw_decode_full(blob: Blob, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(blob.N, blob.K, dtype=torch.bfloat16, device=blob.dev.device)
    _check(lib().uw_decode_full(blob.handle, _ptr(out), _stream(stream)), "uw_decode_full")
    return out


def uw_decode_exponent(blob: Blob, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(blob.N * blob.K, dtype=torch.uint8, device=blob.dev.device)
    _check(lib().uw_decode_exponent(blob.handle, _ptr(out), _stream(stream)), "uw_decode_exponent")
    return out


def uw_transcode_palette(blob: Blob, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(blob.N * blob.K // 2, dtype=torch.uint8, device=blob.dev.device)
    _check(lib().uw_transcode_palette(blob.handle, _ptr(out), _stream(stream)), "uw_transcode_palette")
    return out


def _variant(v) -> int:
    return VARIANTS[v] if isinstance(v, str) else int(v)


class Plan:
    """Autotuner entries held in host memory (the array uw_gemm reads under
    UW_PIPE_AUTO)."""

    def __init__(self, entries: Sequence[dict]):
        self.entries = list(entries)
        self._arr = (PlanEntry * max(1, len(self.entries)))()
        for i, e in enumerate(self.entries):
            a = self._arr[i]
            a.blob_index, a.M = int(e["projection"]), int(e["M"])
            p = e["pipeline"]
            a.pipeline = PIPELINES[p] if isinstance(p, str) else int(p)
            a.variant, a.sm_dec = int(e.get("variant", 0)), int(e.get("sm_dec", 0))
            a.grid, a.split_k = int(e.get("grid", 0)), int(e.get("split_k", 0))
            a.us, a.layer_us = float(e.get("us", 0.0)), float(e.get("layer_us", 0.0))

    def __len__(self):
        return len(self.entries)


def _opts(pipeline, sm_dec=0, grid=0, out_f32=False, ws: Optional[torch.Tensor] = None, variant=0,
          split_k=0, stages=0, plan: Optional[Plan] = None, projection: int = 0) -> GemmOpts:
    o = GemmOpts()
    if pipeline == "auto":
        pipeline = UW_PIPE_AUTO
    o.pipeline = PIPELINES[pipeline] if isinstance(pipeline, str) else int(pipeline)
    o.sm_dec = int(sm_dec)
    o.grid = int(grid)
    o.out_f32 = 1 if out_f32 else 0
    o.variant = _variant(variant)
    o.split_k = int(split_k)
    o.stages = int(stages)
    o.projection = int(projection)
    if plan is not None:
        o.plan = ctypes.cast(plan._arr, ctypes.POINTER(PlanEntry))
        o.plan_entries = len(plan)
    o.workspace = ws.data_ptr() if ws is not None else None
    o.workspace_bytes = ws.numel() if ws is not None else 0
    return o


def uw_gemm_workspace(blob: Blob, M: int, pipeline="direct_palette", sm_dec=0, grid=0, variant=0, split_k=0,
                      plan: Optional[Plan] = None, projection: int = 0) -> int:
    o = _opts(pipeline, sm_dec, grid, variant=variant, split_k=split_k, plan=plan, projection=projection)
    n = ctypes.c_size_t()
    _check(lib().uw_gemm_workspace(blob.handle, int(M), ctypes.byref(o), ctypes.byref(n)), "uw_gemm_workspace")
    return n.value


def uw_plan_resolve(plan: Plan, projection: int, M: int) -> dict:
    """The options UW_PIPE_AUTO takes for (projection, M) under `plan`."""
    o = _opts("auto", plan=plan, projection=projection)
    r = GemmOpts()
    _check(lib().uw_plan_resolve(ctypes.byref(o), int(M), ctypes.byref(r)), "uw_plan_resolve")
    names = {v: k for k, v in PIPELINES.items()}
    return dict(pipeline=names[r.pipeline], variant=r.variant, sm_dec=r.sm_dec, grid=r.grid, split_k=r.split_k)


_ws_cache = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device workspace of at least nbytes, cached per device (contents do not matter)."""
    key = (str(device),)
    t = _ws_cache.get(key)
    if t is None or t.numel() < nbytes:
        t = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = t
    return t


def uw_gemm(X: torch.Tensor, blob: Blob, pipeline="direct_palette", out: Optional[torch.Tensor] = None,
            out_f32: bool = False, ws: Optional[torch.Tensor] = None, sm_dec: int = 0, grid: int = 0,
            variant=0, split_k: int = 0, stages: int = 0, plan: Optional[Plan] = None, projection: int = 0,
            stream=None) -> torch.Tensor:
    """Y[M, N] = X[M, K] . W^T with W compressed in `blob`.  pipeline "auto"
    takes the plan's choice for (projection, M).  Tensor cores, except batch 1
    on a projection with few 128-row tiles (or variant "gemv"): the library's
    CUDA-core GEMV."""
    X = _bits16(X)
    M = X.shape[0]
    if out is None:
        out = torch.empty(M, blob.N, dtype=torch.float32 if out_f32 else torch.bfloat16, device=X.device)
    if ws is None:
        ws = workspace(uw_gemm_workspace(blob, M, pipeline, sm_dec, grid, variant, split_k, plan, projection),
                       X.device)
    o = _opts(pipeline, sm_dec, grid, out_f32, ws, variant, split_k, stages, plan, projection)
    _check(lib().uw_gemm(_ptr(X), M, blob.handle, _ptr(out), ctypes.byref(o), _stream(stream)), "uw_gemm")
    return out


def uw_gemm_swiglu_workspace(gate: Blob, up: Blob, M: int, grid: int = 0, split_k: int = 0, variant=0) -> int:
    o = _opts("direct_palette", 0, grid, variant=variant, split_k=split_k)
    n = ctypes.c_size_t()
    _check(lib().uw_gemm_swiglu_workspace(gate.handle, up.handle, int(M), ctypes.byref(o), ctypes.byref(n)),
           "uw_gemm_swiglu_workspace")
    return n.value


def uw_gemm_swiglu(X: torch.Tensor, gate: Blob, up: Blob, out: Optional[torch.Tensor] = None, out_f32: bool = False,
                   ws: Optional[torch.Tensor] = None, grid: int = 0, split_k: int = 0, stages: int = 0, variant=0,
                   pipeline="direct_palette", stream=None) -> torch.Tensor:
    """H[M, N] = silu(X . Wg^T) * (X . Wu^T) in one launch from the palette
    forms of the gate and up projections."""
    X = _bits16(X)
    M = X.shape[0]
    if out is None:
        out = torch.empty(M, gate.N, dtype=torch.float32 if out_f32 else torch.bfloat16, device=X.device)
    if ws is None:
        ws = workspace(uw_gemm_swiglu_workspace(gate, up, M, grid, split_k, variant), X.device)
    o = _opts(pipeline, 0, grid, out_f32, ws, variant, split_k, stages)
    _check(lib().uw_gemm_swiglu(_ptr(X), M, gate.handle, up.handle, _ptr(out), ctypes.byref(o), _stream(stream)),
           "uw_gemm_swiglu")
    return out


def _seq_items(items):
    arr = (SeqItem * len(items))()
    for i, (blob, X, Y, hard) in enumerate(items):
        h = blob.handle
        arr[i].blob = h.value if hasattr(h, "value") else h
        arr[i].X = X.data_ptr()
        arr[i].Y = Y.data_ptr()
        arr[i].hard = 1 if hard else 0
    return arr


def uw_sequence_workspace(items, M: int) -> int:
    """items: sequence of (blob, X, Y, hard)."""
    arr = _seq_items(items)
    n = ctypes.c_size_t()
    _check(lib().uw_sequence_workspace(arr, len(items), int(M), ctypes.byref(n)), "uw_sequence_workspace")
    return n.value


def uw_gemm_sequence(items, M: int, out_f32: bool = False, dec_ctas: int = 0, ws: Optional[torch.Tensor] = None,
                     stream=None):
    """Runs (blob, X, Y, hard) items in order; hard items' transcodes run ahead
    on a side stream (§跨層管道化)."""
    arr = _seq_items(items)
    if ws is None:
        ws = workspace(uw_sequence_workspace(items, M), items[0][1].device)
    _check(lib().uw_gemm_sequence(arr, len(items), int(M), 1 if out_f32 else 0, int(dec_ctas), _ptr(ws), ws.numel(),
                                  _stream(stream)), "uw_gemm_sequence")


def uw_gemm_direct_palette_noalloc(X: torch.Tensor, blob: Blob, out: Optional[torch.Tensor] = None,
                                   out_f32: bool = False, stream=None) -> torch.Tensor:
    """Direct-palette GEMM whose scratch is a fixed array inside the library,
    for callers that cannot allocate device memory at call time (see the
    header).  `out` should be preallocated by such callers."""
    X = _bits16(X)
    M = X.shape[0]
    if out is None:
        out = torch.empty(M, blob.N, dtype=torch.float32 if out_f32 else torch.bfloat16, device=X.device)
    _check(lib().uw_gemm_direct_palette_noalloc(_ptr(X), M, blob.handle, _ptr(out), 1 if out_f32 else 0,
                                                _stream(stream)), "uw_gemm_direct_palette_noalloc")
    return out


def uw_dense_gemm_workspace(M: int, N: int, K: int, grid: int = 0, variant=0, split_k: int = 0) -> int:
    n = ctypes.c_size_t()
    _check(lib().uw_dense_gemm_workspace(int(M), int(N), int(K), _variant(variant), int(grid), int(split_k),
                                         ctypes.byref(n)), "uw_dense_gemm_workspace")
    return n.value


def uw_dense_gemm(X: torch.Tensor, W: torch.Tensor, out: Optional[torch.Tensor] = None, out_f32: bool = False,
                  ws: Optional[torch.Tensor] = None, grid: int = 0, variant=0, split_k: int = 0,
                  stream=None) -> torch.Tensor:
    """The uncompressed baseline: the same GEMM (tensor cores, or the GEMV where
    uw_gemm would use it) on plain BF16 W[N, K]."""
    X = _bits16(X)
    W = _bits16(W)
    M, K = X.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32 if out_f32 else torch.bfloat16, device=X.device)
    if ws is None:
        ws = workspace(uw_dense_gemm_workspace(M, N, K, grid, variant, split_k), X.device)
    _check(lib().uw_dense_gemm(_ptr(X), M, _ptr(W), N, K, _ptr(out), 1 if out_f32 else 0, _variant(variant),
                               int(grid), int(split_k), _ptr(ws), ws.numel(), _stream(stream)), "uw_dense_gemm")
    return out


def uw_blob_serialize(blob: Blob, stream=None) -> bytes:
    n = ctypes.c_size_t()
    _check(lib().uw_blob_serialized_bytes(blob.handle, ctypes.byref(n)), "uw_blob_serialized_bytes")
    buf = ctypes.create_string_buffer(n.value)
    w = ctypes.c_size_t()
    _check(lib().uw_blob_serialize(blob.handle, buf, n.value, ctypes.byref(w), _stream(stream)),
           "uw_blob_serialize")
    return buf.raw[:w.value]


def uw_blob_device_bytes(data: bytes) -> int:
    n = ctypes.c_size_t()
    _check(lib().uw_blob_device_bytes(data, len(data), ctypes.byref(n)), "uw_blob_device_bytes")
    return n.value


def uw_blob_deserialize(data: bytes, device="cuda", stream=None) -> Blob:
    nb = uw_blob_device_bytes(data)
    dev = torch.empty(nb, dtype=torch.uint8, device=device)
    h = ctypes.c_void_p()
    _check(lib().uw_blob_deserialize(data, len(data), _ptr(dev), nb, _stream(stream), ctypes.byref(h)),
           "uw_blob_deserialize")
    return Blob(h, dev)


def uw_autotune(blobs: Sequence[Blob], Ms: Sequence[int], X: Sequence[torch.Tensor], Y: Sequence[torch.Tensor],
                ws: torch.Tensor, reps: int = 5, plan_json_path: Optional[str] = None, copies: int = 1,
                stream=None) -> list:
    """Coordinate-descent choice of pipeline, variant, grid and decoder split
    per projection and batch size.  `blobs` holds `copies` copies of every
    projection, copy-major ([copy0: p0, p1, ...], [copy1: ...]); X and Y one
    buffer per projection."""
    nb = len(blobs)
    assert nb % copies == 0
    nproj, nm = nb // copies, len(Ms)
    H = (ctypes.c_void_p * nb)(*[b.handle.value if hasattr(b.handle, "value") else b.handle for b in blobs])
    Ms_c = (ctypes.c_int64 * nm)(*[int(m) for m in Ms])
    Xp = (ctypes.c_void_p * nproj)(*[x.data_ptr() for x in X])
    Yp = (ctypes.c_void_p * nproj)(*[y.data_ptr() for y in Y])
    plan = (PlanEntry * (nproj * nm))()
    _check(lib().uw_autotune(H, nproj, copies, Ms_c, nm, Xp, Yp, _ptr(ws), ws.numel(), int(reps), plan,
                             plan_json_path.encode() if plan_json_path else None, _stream(stream)), "uw_autotune")
    return [_entry_dict(p) for p in plan]


def _entry_dict(p: PlanEntry) -> dict:
    names = {v: k for k, v in PIPELINES.items()}
    return dict(projection=p.blob_index, M=p.M, pipeline=names[p.pipeline], variant=p.variant, sm_dec=p.sm_dec,
                grid=p.grid, split_k=p.split_k, us=p.us, layer_us=p.layer_us)


def uw_plan_load_json(path: str, cap: int = 4096) -> list:
    """The plan entries of a JSON file written by uw_autotune."""
    arr = (PlanEntry * cap)()
    n = ctypes.c_int32()
    _check(lib().uw_plan_load_json(path.encode(), arr, cap, ctypes.byref(n)), "uw_plan_load_json")
    return [_entry_dict(arr[i]) for i in range(min(n.value, cap))]
