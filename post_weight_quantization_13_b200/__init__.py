"""Python binding of libgptq.so, the B200 GPTQ layer solver.

Argument marshalling only: every step of the solve runs in the library's
CUDA kernels.  PyTorch provides device memory and the stream.  The functions
carry the C ABI's names (``include/gptq.h``):

    gptq_hessian_accumulate(S, X, n_accum=None, stream=None)
    gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws, stream=None)
    gptq_quantize_layer(W, U, perm, dead, cfg, scales, zeros, g_idx, ws, ...)
    gptq_quantize_layer_noalloc(W, U, perm, dead, cfg, scales, zeros, g_idx, ...)

plus ``solve_layer`` which allocates the outputs and workspace and makes the
three calls in order.  If the shared library is missing the import fails: there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

__all__ = [
    "GptqConfig", "GptqError", "LIB_PATH", "lib", "GPTQ_OK",
    "gptq_abi_version", "gptq_last_error", "gptq_kernel_launches", "gptq_validate_config",
    "gptq_workspace_bytes", "gptq_hessian_accumulate", "gptq_prepare_hinv",
    "gptq_quantize_layer", "gptq_quantize_layer_noalloc", "GPTQ_STATIC_SCRATCH_BYTES",
    "gptq_workspace_status", "gptq_quantize_layer_noalloc_status",
    "gptq_dequantize_layer", "gptq_export_checkpoint", "gptq_selftest_wait_timeout",
    "gptq_selftest_quotient",
    "solve_layer", "solve_block", "export_checkpoint", "STATUS_NAMES",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptq.so")

GPTQ_OK = 0
STATUS_NAMES = {
    0: "GPTQ_OK", 1: "GPTQ_ERR_INVALID_ARG", 2: "GPTQ_ERR_NOT_PD",
    3: "GPTQ_ERR_NONFINITE", 4: "GPTQ_ERR_WORKSPACE", 5: "GPTQ_ERR_CUDA",
    6: "GPTQ_ERR_TIMEOUT", 7: "GPTQ_ERR_UNSUPPORTED",
}
_DTYPES = {"float16": 0, "bfloat16": 1, "float32": 2}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python post_weight_quantization_13_b200/build.py` (there is no CPU fallback)")

lib = ctypes.CDLL(LIB_PATH)


class _Config(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("sym", ctypes.c_int32), ("desc_act", ctypes.c_int32),
                ("damp_percent", ctypes.c_float), ("block_size", ctypes.c_int32)]


_p = ctypes.c_void_p
_i64 = ctypes.c_int64
lib.gptq_abi_version.restype = ctypes.c_int
lib.gptq_last_error.restype = ctypes.c_char_p
lib.gptq_kernel_launches.restype = ctypes.c_uint64
lib.gptq_validate_config.argtypes = [ctypes.POINTER(_Config), _i64, _i64]
lib.gptq_validate_config.restype = ctypes.c_int
lib.gptq_workspace_bytes.argtypes = [_i64, _i64, ctypes.POINTER(_Config)]
lib.gptq_workspace_bytes.restype = ctypes.c_size_t
lib.gptq_hessian_accumulate.argtypes = [_p, _i64, _p, ctypes.c_int, _i64, _i64,
                                        ctypes.POINTER(_i64), _p]
lib.gptq_hessian_accumulate.restype = ctypes.c_int
lib.gptq_prepare_hinv.argtypes = [_p, _i64, _i64, ctypes.POINTER(_Config), _p, _p, _p,
                                  _p, ctypes.c_size_t, _p]
lib.gptq_prepare_hinv.restype = ctypes.c_int
lib.gptq_quantize_layer.argtypes = [_p, ctypes.c_int, _i64, _i64, _i64, _p, _p, _p,
                                    ctypes.POINTER(_Config), _p, _p, _p, _p, _p, _p,
                                    _p, ctypes.c_size_t, _p]
lib.gptq_quantize_layer.restype = ctypes.c_int
lib.gptq_quantize_layer_noalloc.argtypes = [_p, ctypes.c_int, _i64, _i64, _i64, _p, _p, _p,
                                            ctypes.POINTER(_Config), _p, _p, _p, _p, _p, _p, _p]
lib.gptq_quantize_layer_noalloc.restype = ctypes.c_int
lib.gptq_workspace_status.argtypes = [_p, ctypes.c_size_t, _p]
lib.gptq_workspace_status.restype = ctypes.c_int
lib.gptq_quantize_layer_noalloc_status.argtypes = [_p]
lib.gptq_quantize_layer_noalloc_status.restype = ctypes.c_int

lib.gptq_dequantize_layer.argtypes = [_p, _p, _p, _p, _i64, _i64, ctypes.c_int, ctypes.c_int, _p,
                                      ctypes.c_int, _i64, _p]
lib.gptq_dequantize_layer.restype = ctypes.c_int

lib.gptq_export_checkpoint.argtypes = [_p, _p, _p, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _p, _p, _p, _p]
lib.gptq_export_checkpoint.restype = ctypes.c_int

lib.gptq_selftest_wait_timeout.argtypes = [ctypes.c_uint64, _p]
lib.gptq_selftest_wait_timeout.restype = ctypes.c_int
lib.gptq_selftest_quotient.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint64),
                                       ctypes.POINTER(ctypes.c_uint64), _p]
lib.gptq_selftest_quotient.restype = ctypes.c_int

# bytes of the library's static scratch (GPTQ_STATIC_SCRATCH_BYTES in gptq.h)
GPTQ_STATIC_SCRATCH_BYTES = 32 << 20


class GptqError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


@dataclass
class GptqConfig:
    """The pages' BaseQuantizeConfig fields plus ``sym`` and ``block_size``."""
    bits: int = 4
    group_size: int = 128
    sym: bool = False
    desc_act: bool = False
    damp_percent: float = 0.01
    block_size: int = 128

    def c(self) -> _Config:
        return _Config(int(self.bits), int(self.group_size), int(bool(self.sym)),
                       int(bool(self.desc_act)), float(self.damp_percent), int(self.block_size))

    @classmethod
    def of(cls, cfg) -> "GptqConfig":
        if isinstance(cfg, GptqConfig):
            return cfg
        if isinstance(cfg, dict):
            return cls(**cfg)
        return cls(**{k: getattr(cfg, k) for k in cls.__dataclass_fields__})


def _check(status: int):
    if status != GPTQ_OK:
        raise GptqError(status, lib.gptq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dt(t) -> int:
    name = str(t.dtype).replace("torch.", "")
    if name not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _DTYPES[name]


def _rowmajor(t, name):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with contiguous rows")


def gptq_abi_version() -> int:
    return lib.gptq_abi_version()


def gptq_kernel_launches() -> int:
    return int(lib.gptq_kernel_launches())


def gptq_last_error() -> str:
    return lib.gptq_last_error().decode()


def gptq_validate_config(cfg, out: int, in_: int) -> None:
    c = GptqConfig.of(cfg).c()
    _check(lib.gptq_validate_config(ctypes.byref(c), out, in_))


def gptq_workspace_bytes(out: int, in_: int, cfg) -> int:
    c = GptqConfig.of(cfg).c()
    return int(lib.gptq_workspace_bytes(out, in_, ctypes.byref(c)))


def gptq_hessian_accumulate(S, X, n_accum=None, stream=None) -> int:
    """S (in x in fp32, upper triangle) += X X^T for X (in x tokens).
    Returns the updated token count (n_accum + tokens)."""
    _rowmajor(S, "S")
    _rowmajor(X, "X")
    n = _i64(0 if n_accum is None else int(n_accum))
    _check(lib.gptq_hessian_accumulate(_ptr(S), S.shape[0], _ptr(X), _dt(X), X.shape[1],
                                       X.stride(0), ctypes.byref(n), _stream(stream)))
    return n.value


def gptq_prepare_hinv(S, n: int, cfg, U, perm, dead, ws, stream=None) -> None:
    c = GptqConfig.of(cfg).c()
    _check(lib.gptq_prepare_hinv(_ptr(S), int(n), S.shape[0], ctypes.byref(c), _ptr(U),
                                 _ptr(perm), _ptr(dead), _ptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream)))


def gptq_quantize_layer(W, U, perm, dead, cfg, scales, zeros, g_idx, ws, codes=None,
                        qweight=None, loss=None, stream=None) -> None:
    _rowmajor(W, "W")
    c = GptqConfig.of(cfg).c()
    _check(lib.gptq_quantize_layer(_ptr(W), _dt(W), W.shape[0], W.shape[1], W.stride(0),
                                   _ptr(U), _ptr(perm), _ptr(dead), ctypes.byref(c),
                                   _ptr(codes), _ptr(qweight), _ptr(scales), _ptr(zeros),
                                   _ptr(g_idx), _ptr(loss), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)))


def gptq_quantize_layer_noalloc(W, U, perm, dead, cfg, scales, zeros, g_idx, codes=None,
                                qweight=None, loss=None, stream=None) -> None:
    """gptq_quantize_layer on the library's static device scratch: allocates
    nothing, for layers whose workspace fits GPTQ_STATIC_SCRATCH_BYTES.  Calls
    on one device share that scratch and must not overlap in time."""
    _rowmajor(W, "W")
    c = GptqConfig.of(cfg).c()
    _check(lib.gptq_quantize_layer_noalloc(_ptr(W), _dt(W), W.shape[0], W.shape[1], W.stride(0),
                                           _ptr(U), _ptr(perm), _ptr(dead), ctypes.byref(c),
                                           _ptr(codes), _ptr(qweight), _ptr(scales), _ptr(zeros),
                                           _ptr(g_idx), _ptr(loss), _stream(stream)))


def gptq_workspace_status(ws, stream=None) -> None:
    """Wait for the stream and raise GptqError if the last prepare or
    quantize call on workspace ``ws`` raised a device-side status (a bounded
    wait that gave up, NaN/Inf in S, a non-positive pivot)."""
    _check(lib.gptq_workspace_status(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def gptq_quantize_layer_noalloc_status(stream=None) -> None:
    """The same for the last gptq_quantize_layer_noalloc call on this device."""
    _check(lib.gptq_quantize_layer_noalloc_status(_stream(stream)))


def gptq_dequantize_layer(qweight, scales, zeros, g_idx, bits, Wq, stream=None) -> None:
    """Wq (out x in; f16, bf16 or f32) <- scales * (code - zeros) from the
    packed codes gptq_quantize_layer wrote."""
    _rowmajor(Wq, "Wq")
    out, in_ = Wq.shape
    _check(lib.gptq_dequantize_layer(_ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(g_idx), out, in_,
                                     int(bits), scales.shape[1], _ptr(Wq), _dt(Wq), Wq.stride(0),
                                     _stream(stream)))


def gptq_export_checkpoint(qweight, scales, zeros, out: int, in_: int, bits: int, ngroups: int,
                           zero_offset: int, qweight_t=None, qzeros=None, scales_h=None,
                           stream=None) -> None:
    """The solver's outputs in the loaders' checkpoint layout: qweight_t
    (in*bits/32 x out), qzeros (ngroups x out*bits/32), scales_h (float16,
    ngroups x out).  Any output may be None to skip it."""
    _check(lib.gptq_export_checkpoint(_ptr(qweight), _ptr(scales), _ptr(zeros), int(out), int(in_),
                                      int(bits), int(ngroups), int(zero_offset), _ptr(qweight_t),
                                      _ptr(qzeros), _ptr(scales_h), _stream(stream)))


def gptq_selftest_quotient(n: int, seed: int = 1, stream=None) -> tuple[int, int]:
    """Check the sweep's divide-free quotient against IEEE division on n
    pseudo-random pairs; returns (pairs checked, mismatches)."""
    c, m = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(lib.gptq_selftest_quotient(int(n), int(seed), ctypes.byref(c), ctypes.byref(m), _stream(stream)))
    return c.value, m.value


def gptq_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    """Run the bounded-wait timeout path once; returns the status code
    (GPTQ_ERR_TIMEOUT = 6 when the path works)."""
    return lib.gptq_selftest_wait_timeout(int(limit_ns), _stream(stream))


def solve_layer(W, X=None, cfg=None, S=None, n=None, with_codes=True, stream=None):
    """One layer solve on the GPU: Hessian from X (or the given (S, n)),
    prepare, quantize.  Allocates outputs and workspace with torch and
    returns a dict of device tensors."""
    import torch
    cfg = GptqConfig.of(cfg or GptqConfig())
    dev = W.device
    out, in_ = W.shape
    if S is None:
        S = torch.zeros((in_, in_), dtype=torch.float32, device=dev)
        n = gptq_hessian_accumulate(S, X, 0, stream)
    ws = torch.empty(gptq_workspace_bytes(out, in_, cfg), dtype=torch.uint8, device=dev)
    U = torch.empty((in_, in_), dtype=torch.float32, device=dev)
    perm = torch.empty(in_, dtype=torch.int32, device=dev)
    dead = torch.empty(in_, dtype=torch.uint8, device=dev)
    gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws, stream)
    ng = 1 if cfg.group_size == -1 else in_ // cfg.group_size
    scales = torch.empty((out, ng), dtype=torch.float32, device=dev)
    zeros = torch.empty((out, ng), dtype=torch.int32, device=dev)
    g_idx = torch.empty(in_, dtype=torch.int32, device=dev)
    loss = torch.empty(out, dtype=torch.float32, device=dev)
    codes = torch.empty((out, in_), dtype=torch.int32, device=dev) if with_codes else None
    qweight = None
    if (in_ * cfg.bits) % 32 == 0:
        qweight = torch.empty((out, in_ * cfg.bits // 32), dtype=torch.int32, device=dev)
    gptq_quantize_layer(W, U, perm, dead, cfg, scales, zeros, g_idx, ws, codes=codes,
                        qweight=qweight, loss=loss, stream=stream)
    return dict(S=S, n=n, U=U, perm=perm, dead=dead, scales=scales, zeros=zeros, g_idx=g_idx,
                loss=loss, codes=codes, qweight=qweight)


def export_checkpoint(res, bits: int, zero_offset: int = 1, stream=None):
    """A solve_layer result in the loaders' checkpoint layout: a dict of
    device tensors qweight (int32, in*bits/32 x out), qzeros (int32,
    ngroups x out*bits/32), scales (float16, ngroups x out) and g_idx."""
    import torch
    scales, zeros, qweight = res["scales"], res["zeros"], res["qweight"]
    if qweight is None:
        raise ValueError("the result has no packed qweight (in * bits is not a multiple of 32)")
    out, ng = scales.shape
    in_ = res["g_idx"].shape[0]
    dev = scales.device
    qweight_t = torch.empty((in_ * bits // 32, out), dtype=torch.int32, device=dev)
    qzeros = torch.empty((ng, out * bits // 32), dtype=torch.int32, device=dev)
    scales_h = torch.empty((ng, out), dtype=torch.float16, device=dev)
    gptq_export_checkpoint(qweight, scales, zeros, out, in_, bits, ng, zero_offset,
                           qweight_t, qzeros, scales_h, stream)
    return dict(qweight=qweight_t, qzeros=qzeros, scales=scales_h, g_idx=res["g_idx"])


def solve_block(layers, activations=None, cfg=None, streams=True, hessians=None):
    """Quantize the linear layers of one decoder block.

    layers: list of (name, W, site) with W an (out x in) device tensor and
      site the name of the activation stream feeding it (layers that read the
      same activations, e.g. q/k/v or gate/up, share one site).
    activations: dict site -> X (in x tokens device tensor) or an iterable of
      such token batches.
    hessians: optional dict site -> (S, n), an accumulated S (in x in fp32
      device tensor, upper triangle) and its token count, used instead of
      accumulating from activations for that site.

    For each site the Hessian is accumulated and prepared (U, perm, dead)
    once; every layer of the site is then quantized against that shared U.
    The Hessians of all sites run first, back to back on the caller's stream
    (the Hessian kernel is persistent and wants every SM).  Each site's
    prepare follows on that stream, and with ``streams`` the layers of a site
    are then quantized concurrently on side streams, which overlap the
    following sites' prepares.  Every workspace and output allocated for a
    side stream is recorded on it, so its memory is not reused before that
    stream's work is done.  Returns {name: dict(...)} as solve_layer does,
    plus {"site:" + site: dict(S, n, U, perm, dead)}; synchronises the device.
    """
    import torch
    cfg = GptqConfig.of(cfg or GptqConfig())
    hessians = hessians or {}
    sites = {}
    for name, W, site in layers:
        sites.setdefault(site, []).append((name, W))
    dev = layers[0][1].device
    main = torch.cuda.current_stream(dev)
    results = {}
    # 1. the Hessians, one site after another on the caller's stream
    acc = {}
    for site, members in sites.items():
        in_ = members[0][1].shape[1]
        if site in hessians:
            acc[site] = hessians[site]
            continue
        S = torch.zeros((in_, in_), dtype=torch.float32, device=dev)
        n = 0
        X = activations[site]
        for Xb in ([X] if torch.is_tensor(X) else X):
            n = gptq_hessian_accumulate(S, Xb, n, main)
        acc[site] = (S, n)
    # 2. per site: prepare on the caller's stream, then its layers
    side = []
    for site, members in sites.items():
        S, n = acc[site]
        in_ = members[0][1].shape[1]
        ws = torch.empty(gptq_workspace_bytes(0, in_, cfg), dtype=torch.uint8, device=dev)
        U = torch.empty((in_, in_), dtype=torch.float32, device=dev)
        perm = torch.empty(in_, dtype=torch.int32, device=dev)
        dead = torch.empty(in_, dtype=torch.uint8, device=dev)
        gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws, main)
        del ws
        results["site:" + site] = dict(S=S, n=n, U=U, perm=perm, dead=dead)
        ng = 1 if cfg.group_size == -1 else in_ // cfg.group_size
        for name, W in members:
            s_layer = torch.cuda.Stream(dev) if streams else main
            s_layer.wait_stream(main)
            out = W.shape[0]
            wsq = torch.empty(gptq_workspace_bytes(out, in_, cfg), dtype=torch.uint8, device=dev)
            r = dict(scales=torch.empty((out, ng), dtype=torch.float32, device=dev),
                     zeros=torch.empty((out, ng), dtype=torch.int32, device=dev),
                     g_idx=torch.empty(in_, dtype=torch.int32, device=dev),
                     loss=torch.empty(out, dtype=torch.float32, device=dev),
                     codes=torch.empty((out, in_), dtype=torch.int32, device=dev),
                     qweight=(torch.empty((out, in_ * cfg.bits // 32), dtype=torch.int32, device=dev)
                              if (in_ * cfg.bits) % 32 == 0 else None))
            if s_layer is not main:
                for t in [wsq, W, U, perm, dead] + [v for v in r.values() if v is not None]:
                    t.record_stream(s_layer)
            gptq_quantize_layer(W, U, perm, dead, cfg, r["scales"], r["zeros"], r["g_idx"], wsq,
                                codes=r["codes"], qweight=r["qweight"], loss=r["loss"], stream=s_layer)
            r.update(perm=perm, dead=dead, U=U, n=n, ws=wsq, stream=s_layer)
            results[name] = r
            side.append(s_layer)
    for s_layer in side:
        main.wait_stream(s_layer)
    torch.cuda.synchronize(dev)
    for name, _, _ in layers:
        r = results[name]
        ws = r.pop("ws")
        s_layer = r.pop("stream")
        gptq_workspace_status(ws, s_layer)
    return results
