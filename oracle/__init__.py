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
        f = C.c_float
        L.milo_ref_hqq.argtypes = [vp, i, i, i, f, f, vp, vp, vp, i]; L.milo_ref_hqq.restype = i
        L.milo_ref_hqq_trace.argtypes = [vp, i, f, f, vp, vp, vp, vp, vp]
        L.milo_ref_hqq_trace.restype = i
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


# ---------------------------------------------------------------------------
# Offline MiLo quantiser ("MiLo Algorithm: Mixture of Low-Rank Compensators":
# HQQ initial quantisation, a rank-r compensator from the SVD of the residual,
# and rounds that re-quantise W - U V and recompute U V from the new residual).

HQQ_ITERS, HQQ_BETA, HQQ_KAPPA = 20, 10.0, 1.01


def hqq(T: np.ndarray, iters: int = HQQ_ITERS, beta: float = HQQ_BETA, kappa: float = HQQ_KAPPA,
        nthreads: int = 0):
    """HQQ int3 quantisation of an fp32 target [N, K] (groups of 64 along K),
    rows over `nthreads` host threads (0: all cores; the result is the same).
    Returns (q u8 [N, K], scale, zero fp16 bits [K/64, N], status)."""
    T = _c(T, np.float32)
    N, K = T.shape
    assert K % 64 == 0
    q = np.zeros((N, K), np.uint8)
    sc = np.zeros((K // 64, N), np.uint16)
    ze = np.zeros((K // 64, N), np.uint16)
    st = lib().milo_ref_hqq(_p(T), N, K, int(iters), float(beta), float(kappa), _p(q), _p(sc), _p(ze),
                            int(nthreads))
    return q, sc, ze, st


def hqq_trace(t: np.ndarray, iters: int, beta: float, kappa: float):
    """One group of 64 fp32 targets.  Returns (q, s bits, z bits, z before each
    iteration and after the last [iters + 1], L1 error of each iteration [iters])."""
    t = _c(t, np.float32)
    assert t.shape == (64,)
    q = np.zeros(64, np.uint8)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    zt = np.zeros(iters + 1, np.float32)
    et = np.zeros(max(iters, 1), np.float32)
    lib().milo_ref_hqq_trace(_p(t), int(iters), float(beta), float(kappa), _p(q), _p(s), _p(z),
                             _p(zt), _p(et))
    return q, int(s[0]), int(z[0]), zt, et[:iters]


def _f16(bits) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float32)


def lorc_target(W_bits: np.ndarray, U_bits=None, V_bits=None) -> np.ndarray:
    """The quantisation target W - U V in fp32: starting from W, one rank term
    U[:, p] V[p, :] at a time, each product and difference rounded to fp32."""
    T = _f16(W_bits)
    if U_bits is None or np.asarray(U_bits).size == 0:
        return T
    U = _f16(U_bits)
    V = _f16(V_bits)
    for p in range(U.shape[1]):
        T = (T - (U[:, p:p + 1] * V[p:p + 1, :]).astype(np.float32)).astype(np.float32)
    return T


def residual(W_bits: np.ndarray, q: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """R = W - (q - z) s in fp32 (the residual the compensator approximates)."""
    N, K = q.shape
    s = np.repeat(_f16(scale).T, 64, axis=1)
    z = np.repeat(_f16(zero).T, 64, axis=1)
    d = ((q.astype(np.float32) - z).astype(np.float32) * s).astype(np.float32)
    return (_f16(W_bits) - d).astype(np.float32)


def _orth(Y: np.ndarray) -> np.ndarray:
    return np.linalg.qr(Y, mode="reduced")[0]


def _split(Y: np.ndarray, B: np.ndarray, r: int):
    """Rayleigh-Ritz on R ~ Y B (Y orthonormal columns): the top-r singular
    triplets of B, returned balanced as U = Y P_r S^(1/2), V = S^(-1/2) P_r^T B."""
    lam, P = np.linalg.eigh(B @ B.T)
    order = np.argsort(-lam, kind="stable")
    m = min(r, lam.size)
    lam, P = lam[order][:m], P[:, order][:, :m]
    sig = np.sqrt(np.clip(lam, 0.0, None))
    live = sig > (sig[0] * 1e-12 if m and sig[0] > 0 else np.inf)
    root = np.where(live, np.sqrt(sig), 0.0)
    inv = np.where(live, 1.0 / np.where(live, np.sqrt(sig), 1.0), 0.0)
    U = np.zeros((Y.shape[0], r))
    V = np.zeros((r, B.shape[1]))
    U[:, :m] = (Y @ P) * root[None, :]
    V[:m] = (P.T @ B) * inv[:, None]
    return U, V   # fewer than r directions (a thin R) leave zero columns / rows


def rsvd(R: np.ndarray, r: int, omega: np.ndarray, power_iters: int):
    """Rank-r compensator of R [N, K] by randomized subspace iteration (Halko,
    Martinsson and Tropp 2011): Y = orth(R omega), then power_iters times
    Z = orth(R^T Y), Y = orth(R Z); B = Y^T R; U, V from _split().  omega
    [K, l] (l >= r) is the random test matrix, an input.  fp64 throughout."""
    R = np.asarray(R, np.float64)
    Y = _orth(R @ np.asarray(omega, np.float64))
    for _ in range(power_iters):
        Y = _orth(R @ _orth(R.T @ Y))
    return _split(Y, Y.T @ R, r)


def svd_truncated(R: np.ndarray, r: int):
    """The exact rank-r truncated SVD of R, balanced like rsvd(); and the
    optimal error sqrt(sum_{i >= r} sigma_i^2) (Eckart-Young)."""
    u, sg, vt = np.linalg.svd(np.asarray(R, np.float64), full_matrices=False)
    root = np.sqrt(sg[:r])
    return u[:, :r] * root[None, :], vt[:r] * root[:, None], float(np.sqrt(np.sum(sg[r:] ** 2)))


def quantize_lorc(W_bits: np.ndarray, rank: int, rounds: int, omega: np.ndarray, power_iters: int = 2,
                  iters: int = HQQ_ITERS, beta: float = HQQ_BETA, kappa: float = HQQ_KAPPA):
    """The offline MiLo quantiser.  Round 0: HQQ(W), R = W - W_hat, (U, V) =
    rank-r compensator of R.  Each further round: HQQ(W - U V) with the fp16
    U, V of the previous round, a new residual and a new compensator.  Every
    round's error ||W - W_hat - U V||_F (fp16 U, V) is recorded; the round with
    the lowest error (the first on ties) is returned.

    Returns dict(q, scale, zero, U, V (fp16 bits), err [rounds + 1], best, status)."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    U16 = V16 = None
    errs, best, status = [], None, 0
    for rd in range(rounds + 1):
        T = lorc_target(W, U16, V16)
        q, sc, ze, st = hqq(T, iters, beta, kappa)
        status |= st
        R = residual(W, q, sc, ze)
        if rank > 0:
            U, V = rsvd(R, rank, omega, power_iters)
            U16 = U.astype(np.float16).view(np.uint16)
            V16 = V.astype(np.float16).view(np.uint16)
            E = R.astype(np.float64) - _f16(U16).astype(np.float64) @ _f16(V16).astype(np.float64)
        else:
            U16 = np.zeros((N, 0), np.uint16)
            V16 = np.zeros((0, K), np.uint16)
            E = R.astype(np.float64)
        errs.append(float(np.sqrt(np.sum(E * E))))
        if best is None or errs[-1] < errs[best["round"]]:
            best = dict(round=rd, q=q, scale=sc, zero=ze, U=U16, V=V16)
        if rank == 0:
            break
    return dict(q=best["q"], scale=best["scale"], zero=best["zero"], U=best["U"], V=best["V"],
                err=np.array(errs), best=best["round"], status=status)


# ---------------------------------------------------------------------------
# Adaptive ranks ("MiLo Algorithm: Mixture of Low-Rank Compensators": a higher
# rank for weights with a higher kurtosis, and for experts activated more often).

def kurtosis(W_bits: np.ndarray) -> float:
    """Pearson kurtosis m4 / m2^2 of all entries (fp64, centred moments); 0 for a constant matrix."""
    w = _f16(W_bits).astype(np.float64).ravel()
    d = w - w.mean()
    m2 = float(np.mean(d * d))
    return float(np.mean(d ** 4)) / (m2 * m2) if m2 > 0 else 0.0


def assign_ranks(scores, avg_rank: int, max_rank: int = 64) -> list:
    """Budget floor(n * avg_rank / 8) units of 8, capped at max_rank / 8 each:
    shares proportional to max(score, 0) (no positive score left -> equal),
    shares reaching the cap fixed there and the rest re-shared, floors, then the
    leftover units one at a time by decreasing fractional part (ties: higher
    score, lower index), pass after pass until used or all capped."""
    n = len(scores)
    cap = max_rank // 8
    units = min(n * avg_rank // 8, cap * n)
    s = [max(float(x), 0.0) for x in scores]
    if not sum(s) > 0.0:
        s = [1.0] * n
    share = [0.0] * n
    fixed = [False] * n
    eff = list(s)
    left = float(units)
    while True:
        active = 0.0
        for i in range(n):
            if not fixed[i]:
                active += eff[i]
        if not active > 0.0:          # only zero scores left: share the rest equally
            for i in range(n):
                if not fixed[i]:
                    eff[i] = 1.0
            active = 0.0
            for i in range(n):
                if not fixed[i]:
                    active += eff[i]
        changed = False
        for i in range(n):
            if fixed[i]:
                continue
            share[i] = left * eff[i] / active if active > 0.0 else 0.0
            if share[i] >= cap:
                share[i] = float(cap)
                fixed[i] = True
                left -= float(cap)
                changed = True
        if not changed:
            break
    u = [min(cap, int(np.floor(x))) for x in share]
    used = sum(u)
    frac = [x - np.floor(x) for x in share]
    order = sorted(range(n), key=lambda i: (-frac[i], -s[i], i))
    while used < units:               # passes until the budget is used or all are capped
        took = False
        for i in order:
            if used >= units:
                break
            if u[i] < cap:
                u[i] += 1
                used += 1
                took = True
        if not took:
            break
    return [8 * x for x in u]
