"""Python binding of libmilo (include/milo.h): argument marshalling only.

Every step of the int3 + low-rank-compensator MoE forward runs in the sm_100a
kernels of ``libmilo.so``; this module passes torch tensors' device pointers
and the current CUDA stream through ctypes.  torch is used for device memory
and streams only.  There is no CPU fallback: if the library is missing or no
GPU is present the calls raise.

The operation is the inference hot path of "MiLo: Efficient Quantized MoE
Inference with Mixture of Low-Rank Compensators" (W_out = W_quant + U V with
int3 W_quant, routed over a Mixtral-style top-k MoE layer).
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MILO_LIBRARY=checked loads the checked build (range checks in every kernel,
# MILO_DEV_BOUNDS on a violation), built by `python -m int3_gemm_rank_b200.build
# --checked`.
LIB_PATH = os.path.join(_HERE, "libmilo_checked.so" if os.environ.get("MILO_LIBRARY") == "checked"
                        else "libmilo.so")

MILO_F16, MILO_BF16, MILO_F32 = 0, 1, 2
MILO_OK, MILO_ERR_INVALID_ARG, MILO_ERR_UNSUPPORTED_SHAPE, MILO_ERR_WORKSPACE, MILO_ERR_CUDA = range(5)
MILO_LORC_F16, MILO_LORC_INT3 = 0, 1
MILO_DEV_BAD_EXPERT_ID, MILO_DEV_NONFINITE, MILO_DEV_FP16_RANGE, MILO_DEV_TIMEOUT, MILO_DEV_BOUNDS = 1, 2, 4, 8, 16
MILO_ROUTE_RENORM, MILO_ROUTE_IDS_GIVEN = 1, 2
MILO_GEMM_AUTO, MILO_GEMM_MMA, MILO_GEMM_TC = 0, 1, 2
MILO_GROUP, MILO_MAX_RANK = 64, 64

# The C ABI symbols of include/milo.h (checked by the tests).
EXPORTS = ("milo_status_str", "milo_last_error", "milo_version", "milo_pack", "milo_unpack",
           "milo_route", "milo_table_bytes", "milo_linear_prepare", "milo_layer_prepare",
           "milo_linear_workspace_bytes", "milo_moe_workspace_bytes", "milo_grouped_linear",
           "milo_moe_forward", "milo_moe_h_offset", "milo_set_profile_events",
           "milo_grouped_linear_noalloc", "milo_packed_bytes", "milo_hqq_pack",
           "milo_quantize_lorc_workspace", "milo_quantize_lorc", "milo_kurtosis_workspace", "milo_kurtosis",
           "milo_assign_ranks", "milo_selftest_wait_timeout", "milo_set_gemm_path", "milo_dequantize")


class MiloError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"milo status {status}: {msg}")
        self.status = status


class milo_qweight(C.Structure):
    _fields_ = [("packed", C.c_void_p), ("U", C.c_void_p), ("V", C.c_void_p), ("rank", C.c_int32),
                ("lorc_format", C.c_int32)]


class milo_expert(C.Structure):
    _fields_ = [("w1", milo_qweight), ("w3", milo_qweight), ("w2", milo_qweight)]


class milo_linear(C.Structure):
    _fields_ = [("N", C.c_int32), ("K", C.c_int32), ("n_experts", C.c_int32), ("group", C.c_int32),
                ("max_rank", C.c_int32), ("table", C.c_void_p)]


class milo_moe_layer(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_routed", C.c_int32),
                ("n_shared", C.c_int32), ("top_k", C.c_int32), ("group", C.c_int32),
                ("max_rank", C.c_int32), ("table", C.c_void_p)]


_lib = None


class milo_lorc_params(C.Structure):
    _fields_ = [("rank", C.c_int32), ("rounds", C.c_int32), ("sketch", C.c_int32),
                ("power_iters", C.c_int32), ("hqq_iters", C.c_int32), ("hqq_beta", C.c_float),
                ("hqq_kappa", C.c_float)]


def lib() -> C.CDLL:
    """Load libmilo.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m int3_gemm_rank_b200.build` (nvcc, sm_100a; --checked "
                               "for the checked build)")
        L = C.CDLL(LIB_PATH)
        vp, i32, u32, sz = C.c_void_p, C.c_int32, C.c_uint32, C.c_size_t
        L.milo_status_str.argtypes = [C.c_int]; L.milo_status_str.restype = C.c_char_p
        L.milo_last_error.argtypes = []; L.milo_last_error.restype = C.c_char_p
        L.milo_version.argtypes = []; L.milo_version.restype = i32
        L.milo_pack.argtypes = [vp, i32, i32, i32, vp, vp, vp]; L.milo_pack.restype = C.c_int
        L.milo_unpack.argtypes = [vp, i32, i32, vp, vp]; L.milo_unpack.restype = C.c_int
        L.milo_packed_bytes.argtypes = [i32, i32, C.POINTER(sz)]
        L.milo_packed_bytes.restype = C.c_int
        L.milo_route.argtypes = [vp, i32, i32, i32, u32, vp, vp, vp, vp, vp, vp, vp]
        L.milo_route.restype = C.c_int
        L.milo_table_bytes.argtypes = [i32, C.POINTER(sz)]; L.milo_table_bytes.restype = C.c_int
        L.milo_linear_prepare.argtypes = [C.POINTER(milo_linear), C.POINTER(milo_qweight), vp, sz]
        L.milo_linear_prepare.restype = C.c_int
        L.milo_layer_prepare.argtypes = [C.POINTER(milo_moe_layer), C.POINTER(milo_expert), vp, sz]
        L.milo_layer_prepare.restype = C.c_int
        L.milo_linear_workspace_bytes.argtypes = [C.POINTER(milo_linear), i32, i32, C.POINTER(sz)]
        L.milo_linear_workspace_bytes.restype = C.c_int
        L.milo_moe_workspace_bytes.argtypes = [C.POINTER(milo_moe_layer), i32, C.POINTER(sz)]
        L.milo_moe_workspace_bytes.restype = C.c_int
        L.milo_grouped_linear.argtypes = [C.POINTER(milo_linear), vp, C.c_int, i32, i32, vp, vp, vp,
                                          C.c_int, vp, sz, vp, vp]
        L.milo_grouped_linear.restype = C.c_int
        L.milo_moe_forward.argtypes = [C.POINTER(milo_moe_layer), vp, C.c_int, i32, vp, vp, vp, vp,
                                       vp, C.c_int, vp, sz, vp, vp]
        L.milo_moe_forward.restype = C.c_int
        L.milo_moe_h_offset.argtypes = [C.POINTER(milo_moe_layer), i32]
        L.milo_moe_h_offset.restype = sz
        L.milo_set_profile_events.argtypes = [C.POINTER(C.c_void_p), i32]
        L.milo_set_profile_events.restype = C.c_int
        L.milo_grouped_linear_noalloc.argtypes = [C.POINTER(milo_linear), vp, C.c_int, i32, i32, vp, vp,
                                                  vp, C.c_int, vp, vp]
        L.milo_grouped_linear_noalloc.restype = C.c_int
        f32 = C.c_float
        L.milo_hqq_pack.argtypes = [vp, vp, vp, i32, i32, i32, i32, f32, f32, vp, vp, vp, vp]
        L.milo_hqq_pack.restype = C.c_int
        L.milo_quantize_lorc_workspace.argtypes = [i32, i32, C.POINTER(milo_lorc_params), C.POINTER(sz)]
        L.milo_quantize_lorc_workspace.restype = C.c_int
        L.milo_quantize_lorc.argtypes = [vp, i32, i32, C.POINTER(milo_lorc_params), vp, vp, vp, vp, vp, vp, sz,
                                         vp, vp]
        L.milo_quantize_lorc.restype = C.c_int
        L.milo_kurtosis_workspace.argtypes = [C.POINTER(sz)]; L.milo_kurtosis_workspace.restype = C.c_int
        L.milo_kurtosis.argtypes = [vp, C.c_int64, vp, vp, sz, vp, vp]; L.milo_kurtosis.restype = C.c_int
        L.milo_assign_ranks.argtypes = [C.POINTER(C.c_double), i32, i32, i32, C.POINTER(i32)]
        L.milo_assign_ranks.restype = C.c_int
        L.milo_selftest_wait_timeout.argtypes = [vp, vp]; L.milo_selftest_wait_timeout.restype = C.c_int
        L.milo_set_gemm_path.argtypes = [i32]; L.milo_set_gemm_path.restype = C.c_int
        L.milo_dequantize.argtypes = [vp, i32, i32, vp, vp]; L.milo_dequantize.restype = C.c_int
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != MILO_OK:
        msg = lib().milo_last_error().decode() or lib().milo_status_str(status).decode()
        raise MiloError(status, f"{what}: {msg}")


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    return {torch.float16: MILO_F16, torch.bfloat16: MILO_BF16, torch.float32: MILO_F32}[t.dtype]


def _cuda(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


_ACT = (torch.float16, torch.bfloat16)               # activations x
_OUT = (torch.float16, torch.bfloat16, torch.float32)  # outputs y


def _dname(d) -> str:
    return str(d).replace("torch.", "")


def _arg(t, name: str, dtypes=None, shape=None, min_numel: int | None = None, device=None):
    """Check a tensor before its pointer crosses the C ABI.  The library reads
    and writes through the raw pointer with the sizes the call states, so a
    tensor of another dtype or size would be read or written out of bounds.
    dtype and size are checked first (they need no device), then contiguity,
    then that the tensor is a CUDA tensor on the call's device."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, not {type(t).__name__}")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} must be {' or '.join(_dname(d) for d in dtypes)}, not {_dname(t.dtype)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} must hold at least {min_numel} elements, not {t.numel()}")
    _cuda(t, name)
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}; the call's other tensors are on {device}")


def _rows_arg(x, name: str, width: int):
    """Activation rows [T, width] in fp16 or bf16; returns their device."""
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, not {type(x).__name__}")
    if x.dim() != 2 or x.shape[1] != width:
        raise ValueError(f"{name} must be [T, {width}], not {tuple(x.shape)}")
    _arg(x, name, _ACT)
    return x.device


def _weight_arg(W):
    """A weight matrix W [N, K] in fp16 (the quantiser and packer read N*K
    halves)."""
    if not isinstance(W, torch.Tensor) or W.dim() != 2:
        raise ValueError("W must be a [N, K] tensor")
    _arg(W, "W", (torch.float16,))


def _status_arg(dev_status, device):
    if dev_status is not None:
        _arg(dev_status, "dev_status", (torch.int32,), min_numel=1, device=device)


def _ws_arg(ws, device) -> tuple:
    """The 256-byte-aligned start of a caller's workspace and the bytes from
    there to its end (0 when the buffer ends before that boundary)."""
    _arg(ws, "ws", device=device)
    start = ws.data_ptr()
    off = (-start) % 256
    return start + off, max(0, ws.numel() * ws.element_size() - off)


def milo_set_profile_events(events: list | None):
    """Record torch.cuda.Event objects around the grouped GEMM launches (None disables)."""
    if not events:
        _check(lib().milo_set_profile_events(None, 0), "milo_set_profile_events")
        return
    arr = (C.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().milo_set_profile_events(arr, len(events)), "milo_set_profile_events")


def milo_set_gemm_path(path: str):
    """Which grouped GEMM kernel the forward calls use: "auto", "mma" (mma.sync)
    or "tc" (tcgen05); process-wide."""
    mode = {"auto": MILO_GEMM_AUTO, "mma": MILO_GEMM_MMA, "tc": MILO_GEMM_TC}[path]
    _check(lib().milo_set_gemm_path(mode), "milo_set_gemm_path")


def new_status(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


# ---------------------------------------------------------------------------
# packing
# ---------------------------------------------------------------------------

def milo_packed_bytes(N: int, K: int) -> int:
    """Bytes of the packed blob of a weight [N, K]."""
    nb = C.c_size_t()
    _check(lib().milo_packed_bytes(N, K, C.byref(nb)), "milo_packed_bytes")
    return nb.value


def milo_pack(W: torch.Tensor, group: int = MILO_GROUP, dev_status: torch.Tensor | None = None):
    """Quantise W fp16 [N, K] to int3 and pack it: the device blob (uint8 tensor) of milo.h."""
    _weight_arg(W)
    N, K = W.shape
    _status_arg(dev_status, W.device)
    nbytes = milo_packed_bytes(N, K) if K > 0 and K % 128 == 0 and N > 0 else 16
    blob = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _check(lib().milo_pack(_ptr(W), N, K, group, _ptr(blob), _ptr(dev_status), _stream()), "milo_pack")
    return blob


def milo_dequantize(packed: torch.Tensor, N: int, K: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp16 [N, K] dequantised weights (q - z) s of a packed blob."""
    _arg(packed, "packed", (torch.uint8,), min_numel=milo_packed_bytes(N, K))
    if out is None:
        W = torch.empty((N, K), dtype=torch.float16, device=packed.device)
    else:
        _arg(out, "out", (torch.float16,), shape=(N, K), device=packed.device)
        W = out
    with torch.cuda.device(packed.device):
        _check(lib().milo_dequantize(_ptr(packed), N, K, _ptr(W), _stream()), "milo_dequantize")
    return W


def milo_unpack(packed: torch.Tensor, N: int, K: int) -> torch.Tensor:
    """Codes u8 [N, K] of a packed blob."""
    _arg(packed, "packed", (torch.uint8,), min_numel=milo_packed_bytes(N, K))
    codes = torch.empty((N, K), dtype=torch.uint8, device=packed.device)
    with torch.cuda.device(packed.device):
        _check(lib().milo_unpack(_ptr(packed), N, K, _ptr(codes), _stream()), "milo_unpack")
    return codes


# ---------------------------------------------------------------------------
# offline MiLo quantiser
# ---------------------------------------------------------------------------

HQQ_ITERS, HQQ_BETA, HQQ_KAPPA = 20, 10.0, 1.01


def milo_hqq_pack(W: torch.Tensor, U: torch.Tensor | None = None, V: torch.Tensor | None = None,
                  iters: int = HQQ_ITERS, beta: float = HQQ_BETA, kappa: float = HQQ_KAPPA,
                  residual: bool = False, dev_status: torch.Tensor | None = None):
    """HQQ-quantise W - U V (fp16 W [N, K], U [N, r], V [r, K]) and pack it.
    Returns (blob uint8, residual f32 [N, K] = W - W_hat, or None)."""
    _weight_arg(W)
    N, K = W.shape
    if (U is None) != (V is None):
        raise ValueError("milo_hqq_pack: give both U and V, or neither")
    r = 0 if U is None or U.dim() != 2 else U.shape[1]
    if U is not None:
        _arg(U, "U", (torch.float16,), shape=(N, r), device=W.device)
        _arg(V, "V", (torch.float16,), shape=(r, K), device=W.device)
    _status_arg(dev_status, W.device)
    nbytes = milo_packed_bytes(N, K) if K > 0 and K % 128 == 0 and N > 0 else 16
    blob = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    R = torch.empty((N, K), dtype=torch.float32, device=W.device) if residual else None
    _check(lib().milo_hqq_pack(_ptr(W), _ptr(U), _ptr(V), r, N, K, iters, beta, kappa, _ptr(blob), _ptr(R),
                               _ptr(dev_status), _stream()), "milo_hqq_pack")
    return blob, R


def lorc_params(rank: int, rounds: int = 3, sketch: int | None = None, power_iters: int = 2,
                iters: int = HQQ_ITERS, beta: float = HQQ_BETA, kappa: float = HQQ_KAPPA) -> milo_lorc_params:
    if sketch is None:
        sketch = min(128, max(16, 2 * rank)) if rank > 0 else 0
    return milo_lorc_params(rank, rounds, sketch, power_iters, iters, beta, kappa)


def milo_quantize_lorc_workspace(N: int, K: int, params: milo_lorc_params) -> int:
    nb = C.c_size_t()
    _check(lib().milo_quantize_lorc_workspace(N, K, C.byref(params), C.byref(nb)), "milo_quantize_lorc_workspace")
    return nb.value


def milo_quantize_lorc(W: torch.Tensor, params: milo_lorc_params, omega: torch.Tensor | None = None,
                       dev_status: torch.Tensor | None = None):
    """The offline MiLo quantiser of W fp16 [N, K]: HQQ, the rank-r compensator of
    the residual, and params.rounds refinement rounds.  omega: f32 [K, sketch],
    the random test matrix.  Returns (QWeight with fp16 U, V of the best round,
    per-round errors f32 [rounds + 1])."""
    _weight_arg(W)
    N, K = W.shape
    _status_arg(dev_status, W.device)
    r = params.rank
    if r > 0:
        if omega is None or omega.dtype != torch.float32 or tuple(omega.shape) != (K, params.sketch):
            raise ValueError("omega must be float32 [K, sketch]")
        _cuda(omega, "omega")
    nbytes = milo_packed_bytes(N, K) if K > 0 and K % 128 == 0 and N > 0 else 16
    blob = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    U = torch.empty((N, r), dtype=torch.float16, device=W.device) if r > 0 else None
    V = torch.empty((r, K), dtype=torch.float16, device=W.device) if r > 0 else None
    n_err = params.rounds + 1 if r > 0 else 1
    err = torch.empty(n_err, dtype=torch.float32, device=W.device)
    ws_bytes = milo_quantize_lorc_workspace(N, K, params)
    ws = torch.empty(ws_bytes + 256, dtype=torch.uint8, device=W.device)
    wp, _ = _aligned_view(ws, 256, ws_bytes)
    _check(lib().milo_quantize_lorc(_ptr(W), N, K, C.byref(params), _ptr(omega), _ptr(blob), _ptr(U), _ptr(V),
                                    _ptr(err), C.c_void_p(wp), ws_bytes, _ptr(dev_status), _stream()),
           "milo_quantize_lorc")
    return QWeight(blob, N, K, U, V, rank=r), err


def milo_kurtosis(W: torch.Tensor, dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """Pearson kurtosis of all entries of an fp16 CUDA tensor: a device fp64 scalar tensor."""
    _cuda(W, "W")
    if W.dtype != torch.float16:
        raise ValueError("W must be float16")
    nb = C.c_size_t()
    _check(lib().milo_kurtosis_workspace(C.byref(nb)), "milo_kurtosis_workspace")
    ws = torch.empty(nb.value // 8, dtype=torch.float64, device=W.device)
    out = torch.empty(1, dtype=torch.float64, device=W.device)
    _check(lib().milo_kurtosis(_ptr(W), W.numel(), _ptr(out), _ptr(ws), nb.value, _ptr(dev_status), _stream()),
           "milo_kurtosis")
    return out


def milo_assign_ranks(scores, avg_rank: int, max_rank: int = MILO_MAX_RANK) -> list:
    """Ranks (multiples of 8) for matrices with the given scores, within n * avg_rank in total."""
    n = len(scores)
    sc = (C.c_double * max(n, 1))(*[float(x) for x in scores])
    out = (C.c_int32 * max(n, 1))()
    _check(lib().milo_assign_ranks(sc, n, int(avg_rank), int(max_rank), out), "milo_assign_ranks")
    return [int(out[i]) for i in range(n)]


def quantize_experts(experts: list, avg_rank: int, max_rank: int = MILO_MAX_RANK, rounds: int = 3,
                     power_iters: int = 2, score: str = "kurtosis", activation_counts=None, seed: int = 0,
                     dev_status: torch.Tensor | None = None):
    """The offline MiLo pipeline for a layer's experts.

    experts: list of dict(w1=, w3=, w2=) fp16 CUDA weights ([I, H], [I, H], [H, I]).
    Ranks: a budget of avg_rank per projection split by score (milo_assign_ranks),
    the score being each projection's kurtosis (milo_kurtosis) or, with
    score="activation", its expert's entry of activation_counts.  Then each
    projection goes through milo_quantize_lorc (HQQ, rank-r compensator,
    `rounds` refinement rounds) with a standard-normal test matrix drawn from a
    generator seeded with `seed`.  Host synchronisation happens only to read the
    kurtosis values.  Returns (list of dict(w1=, w3=, w2=) QWeight, ranks in
    projection order w1, w3, w2 of expert 0, 1, ...)."""
    names = ("w1", "w3", "w2")
    mats = [e[n] for e in experts for n in names]
    if score == "kurtosis":
        scores = [float(milo_kurtosis(W, dev_status).item()) for W in mats]
    elif score == "activation":
        if activation_counts is None or len(activation_counts) != len(experts):
            raise ValueError("activation_counts needs one count per expert")
        scores = [float(c) for c in activation_counts for _ in names]
    else:
        raise ValueError("score must be 'kurtosis' or 'activation'")
    ranks = milo_assign_ranks(scores, avg_rank, max_rank)
    gen = torch.Generator(device=mats[0].device)
    gen.manual_seed(seed)
    out = []
    for i, W in enumerate(mats):
        p = lorc_params(ranks[i], rounds=rounds, power_iters=power_iters)
        omega = (torch.randn(W.shape[1], p.sketch, generator=gen, device=W.device, dtype=torch.float32)
                 if ranks[i] > 0 else None)
        qw, _ = milo_quantize_lorc(W, p, omega, dev_status)
        if i % 3 == 0:
            out.append({})
        out[-1][names[i % 3]] = qw
    return out, ranks


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

def milo_route(logits: torch.Tensor | None, k: int, renorm: bool, E: int | None = None,
               ids: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
               out: dict | None = None) -> dict:
    """Top-k router + grouping.  With `ids` given ([T, k] int32) the top-k is skipped.
    `out` (the dict a previous call returned, or one with the same keys and
    sizes) receives the results in place, e.g. inside a CUDA graph capture."""
    flags = MILO_ROUTE_RENORM if renorm else 0
    if ids is not None:
        flags |= MILO_ROUTE_IDS_GIVEN
        if E is None:
            raise ValueError("milo_route: E (the number of experts) is required when ids are given")
        if not isinstance(ids, torch.Tensor) or ids.dim() != 2 or ids.shape[1] != k:
            raise ValueError(f"milo_route: ids must be [T, {k}]")
        _arg(ids, "ids", (torch.int32,))
        T = ids.shape[0]
        dev = ids.device
        w = None
    else:
        if not isinstance(logits, torch.Tensor) or logits.dim() != 2:
            raise ValueError("milo_route: logits must be a [T, E] tensor")
        _arg(logits, "logits", (torch.float16,))
        T, E = logits.shape
        dev = logits.device
        if out:
            _arg(out["ids"], "out['ids']", (torch.int32,), shape=(T, k), device=dev)
            _arg(out["w"], "out['w']", (torch.float32,), shape=(T, k), device=dev)
        ids = out["ids"] if out else torch.empty((T, k), dtype=torch.int32, device=dev)
        w = out["w"] if out else torch.empty((T, k), dtype=torch.float32, device=dev)
    _status_arg(dev_status, dev)
    if out:
        for name, t, n in (("offsets", out["offsets"], E + 1), ("perm", out["perm"], T * k),
                           ("inv_perm", out["inv_perm"], T * k)):
            if t.dtype != torch.int32 or not t.is_contiguous() or t.numel() < n:
                raise MiloError(MILO_ERR_INVALID_ARG, f"milo_route: out[{name!r}] must be int32[{n}]")
            _arg(t, f"out[{name!r}]", device=dev)
        off, perm, inv = out["offsets"], out["perm"], out["inv_perm"]
    else:
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
        inv = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().milo_route(_ptr(logits), T, E, k, flags, _ptr(ids), _ptr(w), _ptr(off), _ptr(perm),
                                _ptr(inv), _ptr(dev_status), _stream()), "milo_route")
    return {"ids": ids, "w": w, "offsets": off, "perm": perm[:T * k], "inv_perm": inv[:T * k]}


# ---------------------------------------------------------------------------
# projections and layers
# ---------------------------------------------------------------------------

class QWeight:
    """A packed projection W [N, K] on the device: the blob of milo.h (codes,
    scales, zeros) and the compensator, fp16 U [N, r] and V [r, K], or
    (lorc_int3) the blobs of U^T [r, N] and V [r, K]."""

    def __init__(self, packed, N: int, K: int, U=None, V=None, rank: int | None = None, lorc_int3: bool = False):
        self.packed = packed
        self.N, self.K = int(N), int(K)
        if rank is None:
            rank = 0 if U is None or U.numel() == 0 else int(U.shape[1])
        self.rank = int(rank)
        self.U = U if self.rank else None
        self.V = V if self.rank else None
        self.lorc_int3 = bool(lorc_int3) and self.rank > 0

    @classmethod
    def quantize(cls, W: torch.Tensor, U=None, V=None, dev_status=None, lorc_int3: bool = False):
        """Pack W (and, with lorc_int3, U^T and V) with milo_pack."""
        packed = milo_pack(W, dev_status=dev_status)
        if lorc_int3 and U is not None and U.numel():
            r = int(U.shape[1])
            return cls(packed, W.shape[0], W.shape[1], milo_pack(U.t().contiguous(), dev_status=dev_status),
                       milo_pack(V, dev_status=dev_status), rank=r, lorc_int3=True)
        return cls(packed, W.shape[0], W.shape[1], U, V)

    def check(self):
        """Checks the pieces' dtypes and sizes against N, K and the rank before
        their pointers go into a layer table: the kernels read each piece
        with the sizes the shape implies.  Int3 factors need N and K to be
        multiples of 128 (the packed format's rows); milo_packed_bytes
        refuses other sizes with UNSUPPORTED_SHAPE."""
        _arg(self.packed, "packed", (torch.uint8,), min_numel=milo_packed_bytes(self.N, self.K))
        dev = self.packed.device
        if not self.rank:
            return
        if self.lorc_int3:
            nu, nv = milo_packed_bytes(self.rank, self.N), milo_packed_bytes(self.rank, self.K)
            _arg(self.U, "U (int3 blob of U^T)", (torch.uint8,), min_numel=nu, device=dev)
            _arg(self.V, "V (int3 blob)", (torch.uint8,), min_numel=nv, device=dev)
        else:
            _arg(self.U, "U", (torch.float16,), shape=(self.N, self.rank), device=dev)
            _arg(self.V, "V", (torch.float16,), shape=(self.rank, self.K), device=dev)

    def cstruct(self) -> milo_qweight:
        self.check()
        return milo_qweight(self.packed.data_ptr(), self.U.data_ptr() if self.rank else None,
                            self.V.data_ptr() if self.rank else None, self.rank,
                            MILO_LORC_INT3 if self.lorc_int3 else MILO_LORC_F16)


# ---------------------------------------------------------------------------
# saving packed experts (the quantiser is offline and slow; a saved layer
# loads in seconds)
# ---------------------------------------------------------------------------

SAVE_FORMAT = 1


def _qweight_shapes(qw: QWeight) -> dict:
    """Expected host array shapes and dtypes of a projection's pieces."""
    out = {"packed": ((milo_packed_bytes(qw.N, qw.K),), "uint8")}
    if qw.rank and qw.lorc_int3:
        out["U"] = ((milo_packed_bytes(qw.rank, qw.N),), "uint8")
        out["V"] = ((milo_packed_bytes(qw.rank, qw.K),), "uint8")
    elif qw.rank:
        out["U"] = ((qw.N, qw.rank), "float16")
        out["V"] = ((qw.rank, qw.K), "float16")
    return out


def save_experts(path, experts: list) -> None:
    """Write packed experts (list of dict(w1=, w3=, w2=) QWeight, as
    quantize_experts returns them) to an .npz file: each projection's blob,
    its shape and rank, and its compensator (fp16 U and V, or their int3
    blobs), copied to the host."""
    import json

    import numpy as np
    arrays, meta = {}, []
    for e, d in enumerate(experts):
        for name, qw in d.items():
            key = f"e{e}.{name}"
            pieces = {"packed": qw.packed}
            if qw.rank:
                pieces.update(U=qw.U, V=qw.V)
            for part, (shape, dt) in _qweight_shapes(qw).items():
                a = pieces[part].detach().cpu().numpy()
                if a.shape != shape or a.dtype != np.dtype(dt):
                    raise ValueError(f"{key}.{part}: {a.dtype}{list(a.shape)}, expected {dt}{list(shape)}")
                arrays[f"{key}.{part}"] = a
            meta.append({"expert": e, "name": name, "N": qw.N, "K": qw.K, "rank": qw.rank,
                         "lorc_int3": qw.lorc_int3})
    arrays["meta"] = np.frombuffer(json.dumps({"format": SAVE_FORMAT, "projections": meta}).encode(), np.uint8)
    np.savez(path, **arrays)


def load_experts(path, device="cuda") -> list:
    """The experts save_experts wrote, as QWeights on `device` (sizes checked
    against the packed layout of milo.h)."""
    import json

    import numpy as np
    with np.load(path, allow_pickle=False) as f:
        meta = json.loads(bytes(f["meta"]).decode())
        if meta.get("format") != SAVE_FORMAT:
            raise ValueError(f"{path}: unknown format {meta.get('format')}")
        experts = []
        for m in meta["projections"]:
            key = f"e{m['expert']}.{m['name']}"
            probe = QWeight(None, m["N"], m["K"], rank=m["rank"], lorc_int3=m["lorc_int3"])
            got = {}
            for part, (shape, dt) in _qweight_shapes(probe).items():
                a = f[f"{key}.{part}"]
                if a.shape != shape or a.dtype != np.dtype(dt):
                    raise ValueError(f"{path}: {key}.{part} is {a.dtype}{list(a.shape)}, expected {dt}{list(shape)}")
                got[part] = torch.from_numpy(np.ascontiguousarray(a)).to(device)
            while len(experts) <= m["expert"]:
                experts.append({})
            experts[m["expert"]][m["name"]] = QWeight(got["packed"], m["N"], m["K"], got.get("U"), got.get("V"),
                                                      rank=m["rank"], lorc_int3=m["lorc_int3"])
    return experts


def _table(n_proj: int, device) -> torch.Tensor:
    nb = C.c_size_t()
    _check(lib().milo_table_bytes(n_proj, C.byref(nb)), "milo_table_bytes")
    return torch.empty(nb.value + 64, dtype=torch.uint8, device=device)


def _aligned_view(buf: torch.Tensor, align: int, nbytes: int) -> tuple:
    off = (-buf.data_ptr()) % align
    return buf.data_ptr() + off, nbytes


class GroupedLinear:
    """milo_grouped_linear over n_experts packed projections of shape [N, K]."""

    def __init__(self, weights: list, device="cuda"):
        self.weights = weights
        self.cs = milo_linear(weights[0].N, weights[0].K, len(weights), MILO_GROUP, 0, None)
        arr = (milo_qweight * len(weights))(*[w.cstruct() for w in weights])
        self._table = _table(len(weights), device)
        ptr, nb = _aligned_view(self._table, 64, self._table.numel() - 64)
        _check(lib().milo_linear_prepare(C.byref(self.cs), arr, C.c_void_p(ptr), nb), "milo_linear_prepare")
        self._ws = None

    def workspace_bytes(self, T: int, k: int) -> int:
        nb = C.c_size_t()
        _check(lib().milo_linear_workspace_bytes(C.byref(self.cs), T, k, C.byref(nb)),
               "milo_linear_workspace_bytes")
        return nb.value

    def workspace(self, T: int, k: int, device="cuda") -> torch.Tensor:
        need = self.workspace_bytes(T, k) + 256
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=device)
        return self._ws

    def __call__(self, x: torch.Tensor, offsets: torch.Tensor, perm: torch.Tensor | None, k: int = 1,
                 out_dtype=torch.float32, dev_status=None, y=None, ws=None) -> torch.Tensor:
        return milo_grouped_linear(self, x, offsets, perm, k, out_dtype, dev_status, y, ws)


def _linear_args(lin: GroupedLinear, x, offsets, perm, k, out_dtype, dev_status, y):
    """Checks the tensors of a grouped-linear call against the projection's
    shape; returns (T, device, y)."""
    dev = _rows_arg(x, "x", lin.cs.K)
    T = x.shape[0]
    if T > 0:
        _arg(offsets, "offsets", (torch.int32,), min_numel=lin.cs.n_experts + 1, device=dev)
        if perm is not None:
            _arg(perm, "perm", (torch.int32,), min_numel=T * k, device=dev)
    if y is None:
        y = torch.empty((T * k, lin.cs.N), dtype=out_dtype, device=dev)
    else:
        _arg(y, "y", _OUT, shape=(T * k, lin.cs.N), device=dev)
    _status_arg(dev_status, dev)
    return T, dev, y


def milo_grouped_linear(lin: GroupedLinear, x, offsets, perm, k=1, out_dtype=torch.float32,
                        dev_status=None, y=None, ws=None) -> torch.Tensor:
    T, dev, y = _linear_args(lin, x, offsets, perm, k, out_dtype, dev_status, y)
    if ws is None:
        ws = lin.workspace(T, k, dev)
    wp, wn = _ws_arg(ws, dev)
    with torch.cuda.device(dev):
        _check(lib().milo_grouped_linear(C.byref(lin.cs), _ptr(x), _dt(x), T, k, _ptr(offsets), _ptr(perm),
                                         _ptr(y), _dt(y), C.c_void_p(wp), wn, _ptr(dev_status), _stream()),
               "milo_grouped_linear")
    return y


def milo_grouped_linear_noalloc(lin: GroupedLinear, x, offsets, perm, k=1, out_dtype=torch.float32,
                                dev_status=None, y=None) -> torch.Tensor:
    """milo_grouped_linear without a workspace argument: for callers that cannot
    allocate device memory; the scratch is the library's built-in buffer."""
    T, dev, y = _linear_args(lin, x, offsets, perm, k, out_dtype, dev_status, y)
    with torch.cuda.device(dev):
        _check(lib().milo_grouped_linear_noalloc(C.byref(lin.cs), _ptr(x), _dt(x), T, k, _ptr(offsets),
                                                 _ptr(perm), _ptr(y), _dt(y), _ptr(dev_status), _stream()),
               "milo_grouped_linear_noalloc")
    return y


class MoELayer:
    """milo_moe_forward over routed + shared SwiGLU experts (list of dict(w1=, w3=, w2=) QWeights)."""

    def __init__(self, experts: list, n_routed: int, n_shared: int, top_k: int, device="cuda"):
        self.experts = experts
        H = experts[0]["w2"].N
        I = experts[0]["w1"].N
        self.cs = milo_moe_layer(H, I, n_routed, n_shared, top_k, MILO_GROUP, 0, None)
        arr = (milo_expert * len(experts))(*[milo_expert(e["w1"].cstruct(), e["w3"].cstruct(),
                                                         e["w2"].cstruct()) for e in experts])
        self._table = _table(3 * len(experts), device)
        ptr, nb = _aligned_view(self._table, 64, self._table.numel() - 64)
        _check(lib().milo_layer_prepare(C.byref(self.cs), arr, C.c_void_p(ptr), nb), "milo_layer_prepare")
        self._ws = None

    def workspace_bytes(self, T: int) -> int:
        nb = C.c_size_t()
        _check(lib().milo_moe_workspace_bytes(C.byref(self.cs), T, C.byref(nb)), "milo_moe_workspace_bytes")
        return nb.value

    def workspace(self, T: int, device="cuda") -> torch.Tensor:
        need = self.workspace_bytes(T) + 256
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=device)
        return self._ws

    def h_view(self, T: int, ws: torch.Tensor | None = None) -> torch.Tensor:
        """The fp16 SwiGLU activations [T*k + S*T, I] left in the workspace by the last forward."""
        ws = self._ws if ws is None else ws
        wp, _ = _aligned_view(ws, 256, 0)
        off = (wp - ws.data_ptr()) + lib().milo_moe_h_offset(C.byref(self.cs), T)
        R = T * self.cs.top_k + self.cs.n_shared * T
        return ws[off:off + R * self.cs.inter * 2].view(torch.float16).view(R, self.cs.inter)

    def __call__(self, x, route: dict, out_dtype=torch.float32, dev_status=None, y=None, ws=None):
        return milo_moe_forward(self, x, route, out_dtype, dev_status, y, ws)


def milo_moe_forward(layer: MoELayer, x, route: dict, out_dtype=torch.float32, dev_status=None,
                     y=None, ws=None) -> torch.Tensor:
    dev = _rows_arg(x, "x", layer.cs.hidden)
    T = x.shape[0]
    Tk = T * layer.cs.top_k
    if T > 0:
        # milo_route's outputs over the routed experts (k = top_k)
        for key, dt, n in (("w", torch.float32, Tk), ("offsets", torch.int32, layer.cs.n_routed + 1),
                           ("perm", torch.int32, Tk), ("inv_perm", torch.int32, Tk)):
            if route.get(key) is None:
                raise ValueError(f"route[{key!r}] is required")
            _arg(route[key], f"route[{key!r}]", (dt,), min_numel=n, device=dev)
    if y is None:
        y = torch.empty((T, layer.cs.hidden), dtype=out_dtype, device=dev)
    else:
        _arg(y, "y", _OUT, shape=(T, layer.cs.hidden), device=dev)
    _status_arg(dev_status, dev)
    if ws is None:
        ws = layer.workspace(T, dev)
    wp, wn = _ws_arg(ws, dev)
    with torch.cuda.device(dev):
        _check(lib().milo_moe_forward(C.byref(layer.cs), _ptr(x), _dt(x), T, _ptr(route.get("w")),
                                      _ptr(route.get("offsets")), _ptr(route.get("perm")),
                                      _ptr(route.get("inv_perm")), _ptr(y), _dt(y), C.c_void_p(wp), wn,
                                      _ptr(dev_status), _stream()),
               "milo_moe_forward")
    return y
