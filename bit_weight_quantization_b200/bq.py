"""Thin ctypes binding of the C ABI in ``libbq.so`` (declared in include/bq.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels. Torch tensors may be passed wherever the C call takes a device
pointer (their ``data_ptr()`` is used); the stream defaults to torch's current
CUDA stream. If the shared library is missing this module raises at import.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libbq.so not built at {LIB_PATH}; run bit_weight_quantization_b200.build.build()")
_lib = ctypes.CDLL(LIB_PATH)

BQ_OK, BQ_ERR_INVALID_ARG, BQ_ERR_UNSUPPORTED, BQ_ERR_SIZE = 0, 1, 2, 3
BQ_ERR_CUDA, BQ_ERR_BAD_PACKED, BQ_ERR_DEVICE_CHECK = 4, 5, 6
BQ_FMT_RABIT2, BQ_FMT_BITNET_W1A8, BQ_FMT_TERNARY_A8, BQ_FMT_ABQ, BQ_FMT_BVSR4, BQ_FMT_RABIT3 = 1, 2, 3, 4, 5, 6
FORMATS = {"rabit": 1, "bitnet": 2, "ternary": 3, "abq": 4, "bvsr": 5, "rabit3": 6}


class bq_pack_desc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("w_bits", ctypes.c_int32), ("a_bits", ctypes.c_int32),
                ("lora_rank", ctypes.c_int32), ("lora_alpha", ctypes.c_float), ("h2", ctypes.c_void_p),
                ("lora_A", ctypes.c_void_p), ("lora_B", ctypes.c_void_p), ("rabit_svid_rounds", ctypes.c_int32),
                ("abq_bit_balance", ctypes.c_int32), ("abq_comp_a", ctypes.c_void_p),
                ("abq_comp_b", ctypes.c_void_p), ("h3", ctypes.c_void_p), ("bvsr_cluster_rounds", ctypes.c_int32)]


class bq_plan_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("tokens_per_cta", "token_groups", "ctas_per_group",
                                              "warps_per_row_block", "tiles_per_warp", "ring_stages",
                                              "tiles_per_stage", "x_chunks_per_thread")] + \
               [("shared_bytes", ctypes.c_uint32)]


class bq_layer(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("N_pad", ctypes.c_int32), ("K_pad", ctypes.c_int32), ("w_bits", ctypes.c_int32),
                ("a_bits", ctypes.c_int32), ("lora_rank", ctypes.c_int32),
                ("packed_bytes", ctypes.c_uint64), ("packed", ctypes.c_void_p)]


_P = ctypes.c_void_p
_SIGS = {
    "bq_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "bq_version": (ctypes.c_int32, []),
    "bq_packed_bytes": (ctypes.c_int, [ctypes.POINTER(bq_pack_desc), ctypes.c_int32, ctypes.c_int32,
                                       ctypes.POINTER(ctypes.c_size_t)]),
    "bq_pack_weights": (ctypes.c_int, [ctypes.POINTER(bq_pack_desc), _P, ctypes.c_int32, ctypes.c_int32, _P,
                                       ctypes.c_size_t, _P, ctypes.POINTER(bq_layer)]),
    "bq_packed_validate": (ctypes.c_int, [_P, ctypes.c_size_t, _P, ctypes.POINTER(bq_layer)]),
    "bq_act_bytes": (ctypes.c_int, [ctypes.POINTER(bq_layer), ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]),
    "bq_quantize_act": (ctypes.c_int, [ctypes.POINTER(bq_layer), _P, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "bq_gemv": (ctypes.c_int, [ctypes.POINTER(bq_layer), _P, _P, _P, _P]),
    "bq_gemm": (ctypes.c_int, [ctypes.POINTER(bq_layer), _P, ctypes.c_int32, _P, _P, _P]),
    "bq_linear_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(bq_layer), ctypes.c_int32,
                                                 ctypes.POINTER(ctypes.c_size_t)]),
    "bq_linear": (ctypes.c_int, [ctypes.POINTER(bq_layer), _P, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]),
    "bq_linear_static_scratch": (ctypes.c_int, [ctypes.POINTER(bq_layer), _P, ctypes.c_int32, _P, _P, _P]),
    "bq_linear_plan": (ctypes.c_int, [ctypes.POINTER(bq_layer), ctypes.c_int32, ctypes.c_int32,
                                      ctypes.POINTER(bq_plan_info)]),
    "bq_linear_group": (ctypes.c_int, [ctypes.POINTER(bq_layer), ctypes.c_int32, _P, ctypes.c_int32,
                                       ctypes.POINTER(_P), ctypes.POINTER(_P), _P]),
    "bq_device_check": (ctypes.c_int, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args

EXPORTED = tuple(_SIGS)

# the struct layouts below are those of this ABI version of include/bq.h
BQ_ABI_VERSION = 4
if _lib.bq_version() != BQ_ABI_VERSION:
    raise ImportError(f"{LIB_PATH} has ABI version {_lib.bq_version()}, this binding needs {BQ_ABI_VERSION}; "
                      "rebuild it with bit_weight_quantization_b200.build.build(force=True)")


class BQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {bq_status_str(status)} (status {status})")


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else int(stream.cuda_stream)
    import torch
    return int(torch.cuda.current_stream().cuda_stream)


def _check(st: int, where: str):
    if st != BQ_OK:
        raise BQError(st, where)


def bq_status_str(status: int) -> str:
    return _lib.bq_status_str(status).decode()


def bq_version() -> int:
    return _lib.bq_version()


def make_desc(fmt, w_bits=0, a_bits=0, lora_rank=0, lora_alpha=0.1, h2=None, lora_A=None, lora_B=None,
              rabit_svid_rounds=0, abq_bit_balance=0, abq_comp_a=None, abq_comp_b=None, h3=None,
              bvsr_cluster_rounds=0):
    return bq_pack_desc(FORMATS.get(fmt, fmt), w_bits, a_bits, lora_rank, lora_alpha,
                        _ptr(h2), _ptr(lora_A), _ptr(lora_B), rabit_svid_rounds, abq_bit_balance,
                        _ptr(abq_comp_a), _ptr(abq_comp_b), _ptr(h3), bvsr_cluster_rounds)


def bq_packed_bytes(desc: bq_pack_desc, N: int, K: int) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.bq_packed_bytes(ctypes.byref(desc), N, K, ctypes.byref(out)), "bq_packed_bytes")
    return out.value


def bq_pack_weights(desc: bq_pack_desc, W, N: int, K: int, packed, packed_bytes: int, stream=None) -> bq_layer:
    layer = bq_layer()
    _check(_lib.bq_pack_weights(ctypes.byref(desc), _ptr(W), N, K, _ptr(packed), packed_bytes,
                                _stream(stream), ctypes.byref(layer)), "bq_pack_weights")
    return layer


def bq_packed_validate(packed_host: bytes, packed_dev) -> bq_layer:
    layer = bq_layer()
    buf = ctypes.create_string_buffer(bytes(packed_host), len(packed_host))
    _check(_lib.bq_packed_validate(buf, len(packed_host), _ptr(packed_dev), ctypes.byref(layer)),
           "bq_packed_validate")
    return layer


def bq_act_bytes(layer: bq_layer, M: int) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.bq_act_bytes(ctypes.byref(layer), M, ctypes.byref(out)), "bq_act_bytes")
    return out.value


def bq_quantize_act(layer: bq_layer, x_bf16, M: int, act, act_bytes: int, stream=None) -> None:
    _check(_lib.bq_quantize_act(ctypes.byref(layer), _ptr(x_bf16), M, _ptr(act), act_bytes, _stream(stream)),
           "bq_quantize_act")


def bq_gemv(layer: bq_layer, act, y, acc_dbg=None, stream=None) -> None:
    _check(_lib.bq_gemv(ctypes.byref(layer), _ptr(act), _ptr(y), _ptr(acc_dbg), _stream(stream)), "bq_gemv")


def bq_gemm(layer: bq_layer, act, M: int, y, acc_dbg=None, stream=None) -> None:
    _check(_lib.bq_gemm(ctypes.byref(layer), _ptr(act), M, _ptr(y), _ptr(acc_dbg), _stream(stream)), "bq_gemm")


def bq_linear_workspace_bytes(layer: bq_layer, M: int) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.bq_linear_workspace_bytes(ctypes.byref(layer), M, ctypes.byref(out)), "bq_linear_workspace_bytes")
    return out.value


def bq_linear_plan(layer: bq_layer, M: int, fused: bool = True) -> dict:
    """The work split of bq_linear (fused) or bq_gemm for `layer` and M tokens (host only)."""
    info = bq_plan_info()
    _check(_lib.bq_linear_plan(ctypes.byref(layer), M, int(fused), ctypes.byref(info)), "bq_linear_plan")
    return {n: getattr(info, n) for n, _ in bq_plan_info._fields_}


BQ_STATIC_SCRATCH_BYTES = 1 << 20
BQ_MAX_GROUP = 4


def bq_linear_group(layers, x_bf16, M: int, ys, accs=None, stream=None) -> None:
    """Several layers sharing the input x in one launch (bq_linear_group)."""
    n = len(layers)
    arr = (bq_layer * n)(*layers)
    yp = (_P * n)(*[_ptr(y) for y in ys])
    ap = None if accs is None else (_P * n)(*[_ptr(a) for a in accs])
    _check(_lib.bq_linear_group(arr, n, _ptr(x_bf16), M, yp, ap, _stream(stream)), "bq_linear_group")


def bq_linear_static_scratch(layer: bq_layer, x_bf16, M: int, y, acc_dbg=None, stream=None) -> None:
    """bq_linear with the library's fixed scratch array instead of a workspace."""
    _check(_lib.bq_linear_static_scratch(ctypes.byref(layer), _ptr(x_bf16), M, _ptr(y), _ptr(acc_dbg),
                                         _stream(stream)), "bq_linear_static_scratch")


def bq_linear(layer: bq_layer, x_bf16, M: int, y, acc_dbg=None, workspace=None, workspace_bytes: int = 0,
              stream=None) -> None:
    _check(_lib.bq_linear(ctypes.byref(layer), _ptr(x_bf16), M, _ptr(y), _ptr(acc_dbg), _ptr(workspace),
                          workspace_bytes, _stream(stream)), "bq_linear")


def bq_device_check() -> None:
    _check(_lib.bq_device_check(), "bq_device_check")


def raw_status(name: str, *args) -> int:
    """Call an ABI function and return its status code without raising (for fault tests)."""
    return getattr(_lib, name)(*args)


class QuantLinear:
    """Device buffers (torch allocations) for one packed layer plus the calls on them.

    Owns: the packed buffer. Per call: an activation buffer for M tokens and y.
    All arithmetic happens in the library."""

    def __init__(self, fmt, W, *, w_bits=0, a_bits=0, lora_rank=0, lora_alpha=0.1, h2=None,
                 lora_A=None, lora_B=None, rabit_svid_rounds=0, abq_bit_balance=0, abq_comp_a=None,
                 abq_comp_b=None, h3=None, bvsr_cluster_rounds=0, stream=None):
        import torch
        N, K = W.shape
        self.desc = make_desc(fmt, w_bits, a_bits, lora_rank, lora_alpha, h2, lora_A, lora_B, rabit_svid_rounds,
                              abq_bit_balance, abq_comp_a, abq_comp_b, h3, bvsr_cluster_rounds)
        nbytes = bq_packed_bytes(self.desc, N, K)
        self.packed = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
        self.layer = bq_pack_weights(self.desc, W, N, K, self.packed, nbytes, stream)
        # the pack reads W, h2, h3, the LoRA matrices and a, b asynchronously: wait before the caller may free them
        torch.cuda.synchronize(W.device)
        self.N, self.K = N, K
        self._acts = {}

    def act_buffer(self, M):
        import torch
        if M not in self._acts:
            n = bq_act_bytes(self.layer, M)
            self._acts[M] = torch.empty(n, dtype=torch.uint8, device=self.packed.device)
        return self._acts[M]

    def quantize_act(self, x_bf16, stream=None):
        M = x_bf16.shape[0]
        act = self.act_buffer(M)
        bq_quantize_act(self.layer, x_bf16, M, act, act.numel(), stream)
        return act

    def workspace(self, M):
        import torch
        key = ("ws", M)
        if key not in self._acts:
            n = bq_linear_workspace_bytes(self.layer, M)
            self._acts[key] = torch.empty(max(n, 256), dtype=torch.uint8, device=self.packed.device)
        return self._acts[key]

    def linear(self, x_bf16, y=None, acc_dbg=None, stream=None):
        """Fused activation quantization + layer (bq_linear)."""
        import torch
        M = x_bf16.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float32, device=x_bf16.device)
        ws = self.workspace(M)
        bq_linear(self.layer, x_bf16, M, y, acc_dbg, ws, ws.numel(), stream)
        return y

    def forward(self, x_bf16, y=None, acc_dbg=None, stream=None):
        import torch
        M = x_bf16.shape[0]
        act = self.quantize_act(x_bf16, stream)
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float32, device=x_bf16.device)
        if M == 1:
            bq_gemv(self.layer, act, y, acc_dbg, stream)
        else:
            bq_gemm(self.layer, act, M, y, acc_dbg, stream)
        return y


class StepGraph:
    """A fixed sequence of this library's calls, captured once into a CUDA graph and replayed.

    This is how a decode loop avoids paying the host cost of every call on every step: the
    calls in ``issue()`` (which enqueue on torch's current stream, the default of every call
    here) are captured on ``stream`` after ``warmup`` eager runs. The buffers they read and
    write are fixed in the graph, so a step refreshes their contents (e.g. one copy into the
    input buffer), calls ``replay()``, and reads the outputs. ``replay()`` enqueues the whole
    step on torch's current stream. The library allocates nothing and never synchronizes in
    its compute calls, which is what makes them capturable. ``issue()`` may fork work onto other
    streams and join it back before returning (e.g. read each call's outputs back to pinned host
    memory on a copy stream while the later calls run)."""

    def __init__(self, issue, stream=None, warmup: int = 1):
        import torch
        s = stream if stream is not None else torch.cuda.Stream()
        with torch.cuda.stream(s):
            for _ in range(warmup):
                issue()
        s.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=s):
            issue()
        s.synchronize()

    def replay(self) -> None:
        self.graph.replay()
