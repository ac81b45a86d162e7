"""CPU oracle for the int3 + low-rank-compensator MoE forward (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
(``cpu_baseline`` and ``--impl reference``) may import this package.  The
CUDA library never calls it and shares no code with it.

The arithmetic lives in ``milo_oracle.c`` (plain C, fp64, scalar loops); this
module only marshals numpy arrays through ctypes.  See the header of that file
for the passages of "MiLo: Efficient Quantized MoE Inference with Mixture of
Low-Rank Compensators" that each function follows and the readings taken where
the pages are silent.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "milo_oracle.c")
_LIB = os.path.join(_HERE, "libmilo_oracle.so")

NONFINITE = 2
FP16_RANGE = 4
BAD_EXPERT = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -ffp-contract=off, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp,
                               "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


class Proj(C.Structure):
    _fields_ = [("Q", C.c_void_p), ("scale", C.c_void_p), ("zero", C.c_void_p),
                ("U", C.c_void_p), ("V", C.c_void_p), ("rank", C.c_int32),
                ("Uq", C.c_void_p), ("Us", C.c_void_p), ("Uz", C.c_void_p),
                ("Vq", C.c_void_p), ("Vs", C.c_void_p), ("Vz", C.c_void_p)]


def lib():
    global _lib
    if _lib is None:
        # MILO_ORACLE_LIB lets the mutation tests load a deliberately broken copy.
        L = C.CDLL(os.environ.get("MILO_ORACLE_LIB") or build())
        vp, i, d = C.c_void_p, C.c_int, C.c_double
        L.milo_ref_h2d.argtypes = [C.c_uint16]; L.milo_ref_h2d.restype = d
        L.milo_ref_d2h.argtypes = [d]; L.milo_ref_d2h.restype = C.c_uint16
        L.milo_ref_f2h.argtypes = [C.c_float]; L.milo_ref_f2h.restype = C.c_uint16
        L.milo_ref_quantize.argtypes = [vp, i, i, i, vp, vp, vp]; L.milo_ref_quantize.restype = i
        L.milo_ref_pack.argtypes = [vp, i, i, vp]; L.milo_ref_pack.restype = None
        L.milo_ref_unpack.argtypes = [vp, i, i, vp]; L.milo_ref_unpack.restype = None
        L.milo_ref_code_bit.argtypes = [i, i, C.POINTER(i), C.POINTER(i)]
        L.milo_ref_tile_pack.argtypes = [vp, vp, vp, i, i, vp]; L.milo_ref_tile_pack.restype = None
        L.milo_ref_dequant.argtypes = [vp, vp, vp, i, i, i, vp]; L.milo_ref_dequant.restype = None
        L.milo_ref_group.argtypes = [vp, i, i, i, vp, vp, vp]; L.milo_ref_group.restype = i
        L.milo_ref_route.argtypes = [vp, i, i, i, i, vp, vp, vp, vp, vp]; L.milo_ref_route.restype = i
        L.milo_ref_linear.argtypes = [vp, i, i, C.POINTER(Proj), i, i, vp, i]
        L.milo_ref_linear.restype = None
        L.milo_ref_silu.argtypes = [d]; L.milo_ref_silu.restype = d
        L.milo_ref_moe_forward.argtypes = [vp, i, i, i, i, i, i, i, i, vp, vp, C.POINTER(Proj),
                                           C.POINTER(Proj), C.POINTER(Proj), vp, vp, i]
        L.milo_ref_moe_forward.restype = i
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------

def h2d(bits) -> np.ndarray:
    f = np.vectorize(lambda b: lib().milo_ref_h2d(int(b)), otypes=[np.float64])
    return f(np.asarray(bits, dtype=np.uint16))


def d2h(vals) -> np.ndarray:
    f = np.vectorize(lambda v: lib().milo_ref_d2h(float(v)), otypes=[np.uint16])
    return f(np.asarray(vals, dtype=np.float64))


def quantize(W_bits: np.ndarray, group: int = 64):
    """RTN asymmetric int3 quantisation.  Returns (q u8 [N,K], scale, zero fp16 bits [G,N], status)."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    q = np.zeros((N, K), np.uint8)
    s = np.zeros((K // group, N), np.uint16)
    z = np.zeros((K // group, N), np.uint16)
    st = lib().milo_ref_quantize(_p(W), N, K, group, _p(q), _p(s), _p(z))
    return q, s, z, st


def pack(q: np.ndarray) -> np.ndarray:
    q = _c(q, np.uint8)
    N, K = q.shape
    assert K % 128 == 0
    Q = np.zeros((N, 3 * K // 32), np.uint32)
    lib().milo_ref_pack(_p(q), N, K, _p(Q))
    return Q


def unpack(Q: np.ndarray, K: int) -> np.ndarray:
    Q = _c(Q, np.uint32)
    N = Q.shape[0]
    q = np.zeros((N, K), np.uint8)
    lib().milo_ref_unpack(_p(Q), N, K, _p(q))
    return q


def tile_pack(Q: np.ndarray, scale: np.ndarray, zero: np.ndarray, K: int) -> np.ndarray:
    """Row-major words [N, 3K/32] and group-major scale, zero [K/64, N] -> the device
    blob (u8, ceil(N/64) * K/128 * 3584 bytes)."""
    Q = _c(Q, np.uint32); s = _c(scale, np.uint16); z = _c(zero, np.uint16)
    N = Q.shape[0]
    blob = np.zeros(((N + 63) // 64) * (K // 128) * 3584, np.uint8)
    lib().milo_ref_tile_pack(_p(Q), _p(s), _p(z), N, K, _p(blob))
    return blob


def code_bit(k: int, beta: int):
    w, b = C.c_int(), C.c_int()
    lib().milo_ref_code_bit(k, beta, C.byref(w), C.byref(b))
    return w.value, b.value


def dequant(q, scale, zero, group: int = 64) -> np.ndarray:
    q = _c(q, np.uint8); s = _c(scale, np.uint16); z = _c(zero, np.uint16)
    N, K = q.shape
    out = np.zeros((N, K), np.float64)
    lib().milo_ref_dequant(_p(q), _p(s), _p(z), N, K, group, _p(out))
    return out


def group(ids: np.ndarray, E: int):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    off = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    inv = np.zeros(T * k, np.int32)
    st = lib().milo_ref_group(_p(ids), T, k, E, _p(off), _p(perm), _p(inv))
    return off, perm, inv, st


def route(logits_bits: np.ndarray, k: int, renorm: bool):
    """Top-k softmax router.  Returns (ids [T,k], w f64 [T,k], offsets, perm, inv_perm, status)."""
    L = _c(logits_bits, np.uint16)
    T, E = L.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    off = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    inv = np.zeros(T * k, np.int32)
    st = lib().milo_ref_route(_p(L), T, E, k, int(renorm), _p(ids), _p(w), _p(off), _p(perm),
                              _p(inv))
    return ids, w, off, perm, inv, st


class PackedProj:
    """A quantised projection as the oracle sees it (all host arrays).  With
    `lorc3` = (Uq, Us, Uz, Vq, Vs, Vz) the compensator is int3: U^T [r, N] and
    V [r, K] packed like weights (groups of 64 along N and K)."""

    def __init__(self, Q, scale, zero, U, V, lorc3=None):
        self.Q = _c(Q, np.uint32)
        self.scale = _c(scale, np.uint16)
        self.zero = _c(zero, np.uint16)
        self.U = _c(U, np.uint16)
        self.V = _c(V, np.uint16)
        self.rank = int(self.U.shape[1]) if self.U.ndim == 2 else 0
        self.N = self.Q.shape[0]
        self.K = self.Q.shape[1] * 32 // 3
        self.lorc3 = None if lorc3 is None or self.rank == 0 else tuple(
            _c(a, t) for a, t in zip(lorc3, (np.uint32, np.uint16, np.uint16) * 2))

    def cstruct(self) -> Proj:
        l3 = [a.ctypes.data for a in self.lorc3] if self.lorc3 else [None] * 6
        return Proj(self.Q.ctypes.data, self.scale.ctypes.data, self.zero.ctypes.data,
                    self.U.ctypes.data if self.U.size else None,
                    self.V.ctypes.data if self.V.size else None, self.rank, *l3)


def quantize_projection(W_bits, U_bits, V_bits, group_size: int = 64, lorc_int3: bool = False) -> PackedProj:
    """W quantised and packed; with lorc_int3 the compensator too: U^T [r, N]
    and V [r, K] through the same quantiser (groups along N and K)."""
    q, s, z, _ = quantize(W_bits, group_size)
    lorc3 = None
    if lorc_int3 and U_bits is not None and np.asarray(U_bits).size:
        uq, us, uz, _ = quantize(np.ascontiguousarray(np.asarray(U_bits).T), group_size)
        vq, vs, vz, _ = quantize(np.asarray(V_bits), group_size)
        lorc3 = (pack(uq), us, uz, pack(vq), vs, vz)
    return PackedProj(pack(q), s, z, U_bits, V_bits, lorc3)


def linear(X: np.ndarray, P: PackedProj, group_size: int = 64, nthreads: int = 0) -> np.ndarray:
    """Y [M, N] = X w_hat^T + (X V^T) U^T in fp64."""
    X = _c(X, np.float64)
    M, K = X.shape
    assert K == P.K
    Y = np.zeros((M, P.N), np.float64)
    cs = P.cstruct()
    lib().milo_ref_linear(_p(X), M, K, C.byref(cs), P.N, group_size, _p(Y), nthreads)
    return Y


def silu(a: float) -> float:
    return lib().milo_ref_silu(float(a))


def moe_forward(x_bits: np.ndarray, x_is_bf16: bool, ids: np.ndarray, w: np.ndarray,
                experts: list, n_routed: int, n_shared: int, hidden: int, inter: int,
                group_size: int = 64, want_h: bool = False, nthreads: int = 0):
    """Full layer.  experts: list (n_routed + n_shared) of dict(w1=, w3=, w2=) PackedProj.

    Returns (y f64 [T, H], h fp16 bits [(T*k + S*T), I] or None, status).
    """
    x = _c(x_bits, np.uint16)
    T = x.shape[0]
    ids = _c(ids, np.int32)
    k = ids.shape[1] if ids.ndim == 2 else 1
    w = _c(w, np.float64)
    E, S = n_routed, n_shared
    arr = {name: (Proj * (E + S))(*[experts[e][name].cstruct() for e in range(E + S)])
           for name in ("w1", "w3", "w2")}
    y = np.zeros((T, hidden), np.float64)
    h = np.zeros(((T * k + S * T), inter), np.uint16) if want_h else None
    st = lib().milo_ref_moe_forward(_p(x), int(x_is_bf16), T, hidden, inter, E, S, k, group_size,
                                    _p(ids), _p(w), arr["w1"], arr["w3"], arr["w2"], _p(y),
                                    _p(h) if want_h else None, nthreads)
    return y, h, st
