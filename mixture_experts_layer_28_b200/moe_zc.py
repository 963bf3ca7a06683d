"""ctypes binding of libmoe_zc.so (include/moe_zc.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
fallback: if the library is missing or the tensors are not on a CUDA device,
the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_zc.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "moe_zc.h")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_OOM = -4
ERR_TIMEOUT = -5
ERR_NO_RESULT = -6

MAX_K = 32      # largest K the library accepts
MAX_E = 1024    # largest N + Z the library accepts


class MoeZcError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class Pid(ctypes.Structure):
    """moe_zc_pid: set-point and gains of the bias controller."""
    _fields_ = [("target_zero_frac", ctypes.c_float), ("kp", ctypes.c_float),
                ("ki", ctypes.c_float), ("kd", ctypes.c_float), ("max_shift", ctypes.c_float)]


class LaunchPlan(ctypes.Structure):
    """moe_zc_launch_plan (include/moe_zc.h)."""
    _fields_ = [("kernels", ctypes.c_int32), ("router_grid", ctypes.c_int32),
                ("router_token_tile", ctypes.c_int32), ("router_k_slices", ctypes.c_int32),
                ("expert_gemms_one_grid", ctypes.c_int32), ("expert_grid", ctypes.c_int32),
                ("one_grid_step", ctypes.c_int32)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m mixture_experts_layer_28_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.moe_zc_forward.argtypes = [vp] * 6 + [i64, i32, i32, i32, i32, i32, vp, vp]
        L.moe_zc_forward.restype = ctypes.c_int
        L.moe_zc_forward_ex.argtypes = [vp] * 6 + [i64, i32, i32, i32, i32, i32, vp, vp, vp]
        L.moe_zc_forward_ex.restype = ctypes.c_int
        L.moe_zc_forward_host.argtypes = [vp] * 6 + [i64, i32, i32, i32, i32, i32, vp, vp, i64, vp]
        L.moe_zc_forward_host.restype = ctypes.c_int
        L.moe_zc_expert_load.argtypes = [vp]
        L.moe_zc_expert_load.restype = ctypes.c_int
        L.moe_zc_last_routing.argtypes = [vp, vp]
        L.moe_zc_last_routing.restype = ctypes.c_int
        L.moe_zc_last_expert.argtypes = [i32, i32, vp, vp, vp, vp]
        L.moe_zc_last_expert.restype = ctypes.c_int
        L.moe_zc_synchronize.argtypes = []
        L.moe_zc_synchronize.restype = ctypes.c_int
        L.moe_zc_reserve.argtypes = [i64, i32, i32, i32, i32, i32]
        L.moe_zc_reserve.restype = ctypes.c_int
        L.moe_zc_release.argtypes = []
        L.moe_zc_release.restype = None
        L.moe_zc_status_string.argtypes = [ctypes.c_int]
        L.moe_zc_status_string.restype = ctypes.c_char_p
        L.moe_zc_profile.argtypes = [i32]
        L.moe_zc_profile.restype = ctypes.c_int
        L.moe_zc_profile_read.argtypes = [vp, i32, vp]
        L.moe_zc_profile_read.restype = ctypes.c_int
        L.moe_zc_stage_name.argtypes = [i32]
        L.moe_zc_stage_name.restype = ctypes.c_char_p
        L.moe_zc_route_noalloc.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32,
                                           vp, vp, vp, vp, vp]
        L.moe_zc_route_noalloc.restype = ctypes.c_int
        L.moe_zc_bias_controller_init.argtypes = [vp, i32, vp]
        L.moe_zc_bias_controller_init.restype = ctypes.c_int
        L.moe_zc_bias_controller_step.argtypes = [vp, i32, i32, i64, i32,
                                                  ctypes.POINTER(Pid), vp, vp]
        L.moe_zc_bias_controller_step.restype = ctypes.c_int
        L.moe_zc_test_inject.argtypes = [i32, i64]
        L.moe_zc_test_inject.restype = None
        L.moe_zc_fp8_quantize.argtypes = [vp, i64, i64, i32, vp, vp]
        L.moe_zc_fp8_quantize.restype = ctypes.c_int
        L.moe_zc_plan.argtypes = [i64, i32, i32, i32, i32, i32, i32, i32,
                                  ctypes.POINTER(LaunchPlan)]
        L.moe_zc_plan.restype = ctypes.c_int
        L.moe_zc_test_one_grid.argtypes = [i32]
        L.moe_zc_test_one_grid.restype = None
        L.moe_zc_fp8_quantize_weights.argtypes = [vp, i64, i32, vp, vp, vp]
        L.moe_zc_fp8_quantize_weights.restype = ctypes.c_int
        L.moe_zc_forward_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, i32,
                                         i32, i32, vp, vp, vp]
        L.moe_zc_forward_fp8.restype = ctypes.c_int
        L.moe_zc_forward_host_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i32, i32,
                                              i32, i32, i32, vp, vp, i64, vp]
        L.moe_zc_forward_host_fp8.restype = ctypes.c_int
        L.moe_zc_route.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp]
        L.moe_zc_route.restype = ctypes.c_int
        L.moe_zc_dispatch.argtypes = [vp, vp, vp, i64, i32, i32, i32, vp, vp, vp, vp]
        L.moe_zc_dispatch.restype = ctypes.c_int
        L.moe_zc_experts.argtypes = [vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, vp, vp]
        L.moe_zc_experts.restype = ctypes.c_int
        L.moe_zc_combine.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, vp, vp]
        L.moe_zc_combine.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_zc_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise MoeZcError(status, what)


def _dev_ptr(t: Optional[torch.Tensor], dtype, name: str) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def forward(x: torch.Tensor, W_r: torch.Tensor, b: torch.Tensor,
            W_gate: Optional[torch.Tensor], W_up: Optional[torch.Tensor],
            W_down: Optional[torch.Tensor], N: int, Z: int, K: int,
            out: Optional[torch.Tensor] = None,
            logit_offset: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_zc_forward(_ex) on CUDA tensors; returns out [T, d] bf16."""
    T, d = x.shape
    I = int(W_gate.shape[1]) if (W_gate is not None and N > 0) else 0
    if out is None:
        out = torch.empty_like(x)
    bf = torch.bfloat16
    args = [_dev_ptr(x, bf, "x"), _dev_ptr(W_r, bf, "W_r"), _dev_ptr(b, torch.float32, "b"),
            _dev_ptr(W_gate, bf, "W_gate"), _dev_ptr(W_up, bf, "W_up"),
            _dev_ptr(W_down, bf, "W_down"), T, d, N, Z, K, I]
    o = _dev_ptr(out, bf, "out")
    s = _stream_ptr(stream)
    if logit_offset is None:
        st = lib().moe_zc_forward(*args, o, s)
    else:
        st = lib().moe_zc_forward_ex(*args, _dev_ptr(logit_offset, torch.float32, "logit_offset"),
                                     o, s)
    _check(st, "moe_zc_forward")
    return out


class Fp8Weight:
    """A weight matrix quantised by moe_zc_fp8_quantize_weights: E4M3 codes
    (uint8, the matrix's shape) and UE8M0 scales in 512-byte atoms (uint8)."""

    def __init__(self, codes: torch.Tensor, scales: torch.Tensor):
        self.codes, self.scales = codes, scales


def fp8_quantize_weights(W: torch.Tensor, stream=None) -> Fp8Weight:
    """moe_zc_fp8_quantize_weights of a CUDA bf16 tensor, taken as [rows, cols]
    with cols its last dimension (e.g. W_gate [N, I, d] as [N * I, d])."""
    cols = int(W.shape[-1])
    rows = W.numel() // cols
    codes = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
    scales = torch.empty(rows * cols // 32, dtype=torch.uint8, device=W.device)
    _check(lib().moe_zc_fp8_quantize_weights(_dev_ptr(W, torch.bfloat16, "W"), rows, cols,
                                             codes.data_ptr(), scales.data_ptr(),
                                             _stream_ptr(stream)),
           "moe_zc_fp8_quantize_weights")
    return Fp8Weight(codes, scales)


def forward_fp8(x: torch.Tensor, W_r: torch.Tensor, b: torch.Tensor, W_gate: Fp8Weight,
                W_up: Fp8Weight, W_down: torch.Tensor, N: int, Z: int, K: int,
                out: Optional[torch.Tensor] = None,
                logit_offset: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_zc_forward_fp8: gate/up in block-scaled FP8 (weights from
    fp8_quantize_weights), down in bf16; returns out [T, d] bf16."""
    T, d = x.shape
    I = int(W_gate.codes.shape[1]) if N > 0 else 0
    if out is None:
        out = torch.empty_like(x)
    bf, u8 = torch.bfloat16, torch.uint8
    st = lib().moe_zc_forward_fp8(
        _dev_ptr(x, bf, "x"), _dev_ptr(W_r, bf, "W_r"), _dev_ptr(b, torch.float32, "b"),
        _dev_ptr(W_gate.codes, u8, "W_gate codes"), _dev_ptr(W_gate.scales, u8, "W_gate scales"),
        _dev_ptr(W_up.codes, u8, "W_up codes"), _dev_ptr(W_up.scales, u8, "W_up scales"),
        _dev_ptr(W_down, bf, "W_down"), T, d, N, Z, K, I,
        _dev_ptr(logit_offset, torch.float32, "logit_offset"), _dev_ptr(out, bf, "out"),
        _stream_ptr(stream))
    _check(st, "moe_zc_forward_fp8")
    return out


def forward_host_fp8(x_host: torch.Tensor, W_r: torch.Tensor, b: torch.Tensor,
                     W_gate: Fp8Weight, W_up: Fp8Weight, W_down: torch.Tensor, N: int, Z: int,
                     K: int, out_host: Optional[torch.Tensor] = None,
                     logit_offset: Optional[torch.Tensor] = None, chunk_tokens: int = 0,
                     stream=None) -> torch.Tensor:
    """moe_zc_forward_host_fp8: forward_fp8 on CPU tensors x_host / out_host
    (pin them for overlap).  Asynchronous on `stream`."""
    if x_host.is_cuda or x_host.dtype != torch.bfloat16 or not x_host.is_contiguous():
        raise ValueError("x_host must be a contiguous bf16 CPU tensor")
    T, d = x_host.shape
    I = int(W_gate.codes.shape[1]) if N > 0 else 0
    if out_host is None:
        out_host = torch.empty_like(x_host, pin_memory=x_host.is_pinned())
    if out_host.is_cuda or out_host.dtype != torch.bfloat16 or not out_host.is_contiguous():
        raise ValueError("out_host must be a contiguous bf16 CPU tensor")
    bf, u8 = torch.bfloat16, torch.uint8
    st = lib().moe_zc_forward_host_fp8(
        x_host.data_ptr(), _dev_ptr(W_r, bf, "W_r"), _dev_ptr(b, torch.float32, "b"),
        _dev_ptr(W_gate.codes, u8, "W_gate codes"), _dev_ptr(W_gate.scales, u8, "W_gate scales"),
        _dev_ptr(W_up.codes, u8, "W_up codes"), _dev_ptr(W_up.scales, u8, "W_up scales"),
        _dev_ptr(W_down, bf, "W_down"), T, d, N, Z, K, I,
        _dev_ptr(logit_offset, torch.float32, "logit_offset"), out_host.data_ptr(),
        chunk_tokens, _stream_ptr(stream))
    _check(st, "moe_zc_forward_host_fp8")
    return out_host


def route(x: torch.Tensor, W_r: torch.Tensor, b: torch.Tensor, N: int, Z: int, K: int,
          logit_offset: Optional[torch.Tensor] = None, stream=None):
    """moe_zc_route: (idx int32 [T, K], gate fp32 [T, K], zsum fp32 [T],
    counts int32 [E]) as CUDA tensors."""
    T, d = x.shape
    dev = x.device
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    gate = torch.empty(T, K, dtype=torch.float32, device=dev)
    zsum = torch.empty(T, dtype=torch.float32, device=dev)
    counts = torch.empty(N + Z, dtype=torch.int32, device=dev)
    _check(lib().moe_zc_route(_dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(W_r, torch.bfloat16, "W_r"),
                              _dev_ptr(b, torch.float32, "b"),
                              _dev_ptr(logit_offset, torch.float32, "logit_offset"), T, d, N, Z, K,
                              idx.data_ptr(), gate.data_ptr(), zsum.data_ptr(), counts.data_ptr(),
                              _stream_ptr(stream)), "moe_zc_route")
    return idx, gate, zsum, counts


def dispatch(x: torch.Tensor, idx: torch.Tensor, counts: torch.Tensor, N: int, rows: int,
             stream=None):
    """moe_zc_dispatch: (slot int32 [T, K], send bf16 [rows, d], send_expert
    int32 [rows]); rows = the FFN picks, sum(counts[:N]) (known to the caller
    from the histogram)."""
    T, d = x.shape
    K = int(idx.shape[1])
    slot = torch.empty(T, K, dtype=torch.int32, device=x.device)
    send = torch.empty(max(rows, 1), d, dtype=torch.bfloat16, device=x.device)
    send_expert = torch.empty(max(rows, 1), dtype=torch.int32, device=x.device)
    _check(lib().moe_zc_dispatch(_dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(idx, torch.int32, "idx"),
                                 _dev_ptr(counts, torch.int32, "counts"), T, d, N, K,
                                 slot.data_ptr(), send.data_ptr(), send_expert.data_ptr(),
                                 _stream_ptr(stream)), "moe_zc_dispatch")
    return slot, send[:rows], send_expert[:rows]


def experts(x_rows: torch.Tensor, expert: torch.Tensor, expert_base: int, W_gate: torch.Tensor,
            W_up: torch.Tensor, W_down: torch.Tensor, stream=None) -> torch.Tensor:
    """moe_zc_experts: y [R, d], row i = SwiGLU expert (expert[i] - expert_base)
    of the given shard applied to x_rows[i]."""
    R, d = x_rows.shape
    N, I = int(W_gate.shape[0]), int(W_gate.shape[1])
    y = torch.empty_like(x_rows)
    bf = torch.bfloat16
    _check(lib().moe_zc_experts(_dev_ptr(x_rows, bf, "x_rows") if R else None,
                                _dev_ptr(expert, torch.int32, "expert") if R else None,
                                expert_base, R, d, N, I, _dev_ptr(W_gate, bf, "W_gate"),
                                _dev_ptr(W_up, bf, "W_up"), _dev_ptr(W_down, bf, "W_down"),
                                y.data_ptr() if R else None, _stream_ptr(stream)), "moe_zc_experts")
    return y


def combine(x: torch.Tensor, y_rows: torch.Tensor, slot: torch.Tensor, gate: torch.Tensor,
            zsum: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_zc_combine: out_t = zsum_t x_t + sum_k gate_{t,k} y_rows[slot_{t,k}]."""
    T, d = x.shape
    K = int(slot.shape[1])
    if out is None:
        out = torch.empty_like(x)
    yp = y_rows.data_ptr() if y_rows.numel() else None
    if yp is not None:
        _dev_ptr(y_rows, torch.bfloat16, "y_rows")
    _check(lib().moe_zc_combine(_dev_ptr(x, torch.bfloat16, "x"), yp,
                                _dev_ptr(slot, torch.int32, "slot"),
                                _dev_ptr(gate, torch.float32, "gate"),
                                _dev_ptr(zsum, torch.float32, "zsum"), T, d, K,
                                _dev_ptr(out, torch.bfloat16, "out"), _stream_ptr(stream)),
           "moe_zc_combine")
    return out


def forward_host(x_host: torch.Tensor, W_r: torch.Tensor, b: torch.Tensor,
                 W_gate: Optional[torch.Tensor], W_up: Optional[torch.Tensor],
                 W_down: Optional[torch.Tensor], N: int, Z: int, K: int,
                 out_host: Optional[torch.Tensor] = None,
                 logit_offset: Optional[torch.Tensor] = None, chunk_tokens: int = 0,
                 stream=None) -> torch.Tensor:
    """moe_zc_forward_host: x_host and out_host are CPU tensors (pin them for
    overlap); the weights are CUDA tensors.  Asynchronous on `stream`."""
    if x_host.is_cuda:
        raise ValueError("x_host must be a CPU tensor")
    if x_host.dtype != torch.bfloat16 or not x_host.is_contiguous():
        raise ValueError("x_host must be contiguous bf16")
    T, d = x_host.shape
    I = int(W_gate.shape[1]) if (W_gate is not None and N > 0) else 0
    if out_host is None:
        out_host = torch.empty_like(x_host, pin_memory=x_host.is_pinned())
    if out_host.is_cuda or out_host.dtype != torch.bfloat16 or not out_host.is_contiguous():
        raise ValueError("out_host must be a contiguous bf16 CPU tensor")
    bf = torch.bfloat16
    st = lib().moe_zc_forward_host(
        x_host.data_ptr(), _dev_ptr(W_r, bf, "W_r"), _dev_ptr(b, torch.float32, "b"),
        _dev_ptr(W_gate, bf, "W_gate"), _dev_ptr(W_up, bf, "W_up"), _dev_ptr(W_down, bf, "W_down"),
        T, d, N, Z, K, I, _dev_ptr(logit_offset, torch.float32, "logit_offset"),
        out_host.data_ptr(), chunk_tokens, _stream_ptr(stream))
    _check(st, "moe_zc_forward_host")
    return out_host


def expert_load(E: int) -> np.ndarray:
    counts = np.zeros(E, dtype=np.int32)
    _check(lib().moe_zc_expert_load(counts.ctypes.data), "moe_zc_expert_load")
    return counts


def last_routing(T: int, K: int):
    idx = np.zeros((T, K), dtype=np.int32)
    gate = np.zeros((T, K), dtype=np.float32)
    _check(lib().moe_zc_last_routing(idx.ctypes.data, gate.ctypes.data), "moe_zc_last_routing")
    return idx, gate


def last_expert(e: int, d: int, I: int, max_rows: int):
    """(tokens int32 [n], H bf16 [n, I], Y bf16 [n, d]) of FFN expert e, last forward."""
    n = ctypes.c_int32(0)
    tokens = np.zeros(max_rows, dtype=np.int32)
    H = torch.zeros(max_rows, I, dtype=torch.bfloat16)
    Y = torch.zeros(max_rows, d, dtype=torch.bfloat16)
    _check(lib().moe_zc_last_expert(e, max_rows, ctypes.byref(n), tokens.ctypes.data,
                                    H.data_ptr(), Y.data_ptr()), "moe_zc_last_expert")
    k = min(n.value, max_rows)
    return tokens[:k], H[:k], Y[:k], n.value


def synchronize() -> None:
    _check(lib().moe_zc_synchronize(), "moe_zc_synchronize")


def reserve(T: int, d: int, N: int, Z: int, K: int, I: int) -> None:
    _check(lib().moe_zc_reserve(T, d, N, Z, K, I), "moe_zc_reserve")


def release() -> None:
    lib().moe_zc_release()


NOALLOC_SCRATCH_BYTES = 4 << 20


def route_noalloc(x: torch.Tensor, W_r: torch.Tensor, b: torch.Tensor, N: int, Z: int, K: int,
                  idx: torch.Tensor, gate: torch.Tensor, counts: torch.Tensor,
                  status: torch.Tensor, logit_offset: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    """moe_zc_route_noalloc: routing into caller-owned device tensors
    (idx int32 [T, K], gate fp32 [T, K], counts int32 [E]) with no device
    allocation by the library; status (int32 [1], device) is cleared by the
    call and set non-zero on the device if a bounded wait runs out."""
    T, d = x.shape
    st = lib().moe_zc_route_noalloc(
        _dev_ptr(x, torch.bfloat16, "x"), _dev_ptr(W_r, torch.bfloat16, "W_r"),
        _dev_ptr(b, torch.float32, "b"), _dev_ptr(logit_offset, torch.float32, "logit_offset"),
        T, d, N, Z, K, _dev_ptr(idx, torch.int32, "idx"), _dev_ptr(gate, torch.float32, "gate"),
        _dev_ptr(counts, torch.int32, "counts"), _dev_ptr(status, torch.int32, "status"),
        _stream_ptr(stream))
    _check(st, "moe_zc_route_noalloc")


STAGES = 7


def profile(enable: bool) -> None:
    _check(lib().moe_zc_profile(1 if enable else 0), "moe_zc_profile")


def profile_read() -> tuple[dict, int]:
    """({stage name: summed ms}, forwards recorded) since profile(True)."""
    ms = np.zeros(STAGES, dtype=np.float32)
    n = ctypes.c_int32(0)
    _check(lib().moe_zc_profile_read(ms.ctypes.data, STAGES, ctypes.byref(n)),
           "moe_zc_profile_read")
    names = [lib().moe_zc_stage_name(i).decode() for i in range(STAGES)]
    return dict(zip(names, ms.tolist())), n.value


class BiasController:
    """Host-side PID controller of the expert biases (moe_zc_bias_controller_*).

    step(counts) takes an expert-load histogram over `tokens` tokens and
    returns the new biases (numpy float32 [E]).
    """

    def __init__(self, b0, N: int, Z: int, K: int, target_zero_frac: float,
                 kp: float, ki: float, kd: float = 0.0, max_shift: float = 0.0):
        self.N, self.Z, self.K = N, Z, K
        self.pid = Pid(target_zero_frac, kp, ki, kd, max_shift)
        self.b = np.ascontiguousarray(np.asarray(b0, dtype=np.float32)).copy()
        self.state = np.zeros(3 * (N + Z), dtype=np.float32)
        _check(lib().moe_zc_bias_controller_init(self.b.ctypes.data, N + Z,
                                                 self.state.ctypes.data),
               "moe_zc_bias_controller_init")

    def step(self, counts, tokens: int) -> np.ndarray:
        c = np.ascontiguousarray(np.asarray(counts, dtype=np.int32))
        _check(lib().moe_zc_bias_controller_step(c.ctypes.data, self.N, self.Z, tokens, self.K,
                                                 ctypes.byref(self.pid), self.state.ctypes.data,
                                                 self.b.ctypes.data),
               "moe_zc_bias_controller_step")
        return self.b.copy()


FP8_BLOCK128 = 0   # 128 x 128 blocks, fp32 scale amax / 448
FP8_MX32 = 1       # 1 x 32 blocks along a row, power-of-two scales


def fp8_quantize(W: torch.Tensor, mode: int = FP8_BLOCK128):
    """E4M3 codes (numpy uint8 [rows, cols]) and block scales (numpy float32)
    of a host bf16 matrix (moe_zc_fp8_quantize)."""
    if W.device.type != "cpu" or W.dtype != torch.bfloat16 or W.dim() != 2:
        raise ValueError("W must be a 2-D bf16 CPU tensor")
    W = W.contiguous()
    rows, cols = W.shape
    br, bc = (128, 128) if mode == FP8_BLOCK128 else (1, 32)
    codes = np.zeros((rows, cols), dtype=np.uint8)
    scales = np.zeros(((rows + br - 1) // br, (cols + bc - 1) // bc), dtype=np.float32)
    _check(lib().moe_zc_fp8_quantize(W.data_ptr(), rows, cols, mode, codes.ctypes.data,
                                     scales.ctypes.data), "moe_zc_fp8_quantize")
    return codes, scales


def allreduce_expert_load(counts: np.ndarray, group=None) -> np.ndarray:
    """Sum an expert-load histogram over the ranks of a torch.distributed
    group (exact: int64 counts), so a controller on every rank sees the
    global usage."""
    import torch.distributed as dist
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.as_tensor(np.asarray(counts, dtype=np.int64), device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t.cpu().numpy()


def test_inject(fail_allocs: int = 0, wait_limit_ns: int = 0) -> None:
    lib().moe_zc_test_inject(fail_allocs, wait_limit_ns)


def plan(T: int, d: int, N: int, Z: int, K: int, I: int, sms: int = 148,
         resident_blocks: int = 148) -> dict:
    """moe_zc_plan: how a forward of these sizes is launched (host only)."""
    p = LaunchPlan()
    _check(lib().moe_zc_plan(T, d, N, Z, K, I, sms, resident_blocks, ctypes.byref(p)),
           "moe_zc_plan")
    return {name: getattr(p, name) for name, _ in LaunchPlan._fields_}


def test_one_grid(off: bool = False, step: bool = True) -> None:
    """Test hook for batches of at most 64 tokens: off keeps them off the
    one-grid expert GEMMs; step=False keeps route, dispatch and combine out
    of that grid."""
    lib().moe_zc_test_one_grid(1 if off else (0 if step else 2))


def declared_symbols() -> list[str]:
    """Function names declared in include/moe_zc.h."""
    import re
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|void|const char\*)\s+(moe_zc_\w+)\s*\(", text, re.M)))
