"""Python entry points of the fp64 eager oracle (oracle/eager.c) -- TEST INFRASTRUCTURE.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this.
``build()`` compiles eager.c with gcc (OpenMP, no fast-math) into
oracle/_eager_oracle.so; the functions below call it through ctypes on float64
numpy arrays.  See eager.c for the recurrences and their sources.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eager.c")
_LIB = os.path.join(_HERE, "_eager_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile eager.c -> _eager_oracle.so (skipped when up to date)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", _SRC, "-o", _LIB + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_mamba2_eager_step.argtypes = [i64, i64, i64, i64, i64, P, P, ctypes.c_int,
                                                 P, P, P, P, P, P]
        lib.oracle_mamba2_eager_step.restype = None
        lib.oracle_gdn_eager_step.argtypes = [i64, i64, i64, i64, P, P, P, P, P, P, P]
        lib.oracle_gdn_eager_step.restype = None
        lib.oracle_kda_eager_step.argtypes = [i64, i64, i64, i64, P, P, P, P, P, P, P]
        lib.oracle_kda_eager_step.restype = None
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def mamba2_step(S: np.ndarray, A, D, x, dt, Bm, Cm, dt_scales_input: bool = False) -> np.ndarray:
    """One eager Mamba-2 token for all (b,h). S[B,H,P,N] float64 is updated in place.

    x[B,H,P], dt[B,H], Bm/Cm[B,G,N], A/D[H].  Returns y[B,H,P].
    """
    lib = _load()
    assert S.dtype == np.float64 and S.flags.c_contiguous
    Bn, H, P, N = S.shape
    Bm = _f64(Bm)
    G = Bm.shape[1]
    x, dt, Cm, A, D = map(_f64, (x, dt, Cm, A, D))
    assert x.shape == (Bn, H, P) and dt.shape == (Bn, H) and Bm.shape == (Bn, G, N)
    assert Cm.shape == (Bn, G, N) and A.shape == (H,) and D.shape == (H,) and H % G == 0
    y = np.empty((Bn, H, P))
    lib.oracle_mamba2_eager_step(Bn, H, P, N, G, _p(A), _p(D), int(bool(dt_scales_input)),
                                 _p(S), _p(x), _p(dt), _p(Bm), _p(Cm), _p(y))
    return y


def gdn_step(S: np.ndarray, q, k, v, alpha, beta) -> np.ndarray:
    """One eager Gated DeltaNet token for all (b,h). S[B,H,d_v,d_k] updated in place.

    q,k[B,H,d_k], v[B,H,d_v], alpha/beta[B,H].  Returns o[B,H,d_v].
    """
    lib = _load()
    assert S.dtype == np.float64 and S.flags.c_contiguous
    Bn, H, P, N = S.shape
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    assert q.shape == (Bn, H, N) and k.shape == (Bn, H, N) and v.shape == (Bn, H, P)
    assert alpha.shape == (Bn, H) and beta.shape == (Bn, H)
    o = np.empty((Bn, H, P))
    lib.oracle_gdn_eager_step(Bn, H, P, N, _p(S), _p(q), _p(k), _p(v), _p(alpha), _p(beta),
                              _p(o))
    return o


def kda_step(S: np.ndarray, q, k, v, alpha, beta) -> np.ndarray:
    """One eager Kimi Delta Attention token for all (b,h). S[B,H,d_v,d_k] updated in place.

    q,k[B,H,d_k], v[B,H,d_v], alpha[B,H,d_k] (a gate per key channel), beta[B,H].
    Returns o[B,H,d_v].
    """
    lib = _load()
    assert S.dtype == np.float64 and S.flags.c_contiguous
    Bn, H, P, N = S.shape
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    assert q.shape == (Bn, H, N) and k.shape == (Bn, H, N) and v.shape == (Bn, H, P)
    assert alpha.shape == (Bn, H, N) and beta.shape == (Bn, H)
    o = np.empty((Bn, H, P))
    lib.oracle_kda_eager_step(Bn, H, P, N, _p(S), _p(q), _p(k), _p(v), _p(alpha), _p(beta),
                              _p(o))
    return o


def step(kind: str, S: np.ndarray, tok: dict, params: dict | None = None,
         dt_scales_input: bool = False) -> np.ndarray:
    """Dispatch one eager token of a layer kind ("mamba2" | "gdn" | "kda"; tok: one token, [B,...] arrays)."""
    if kind == "mamba2":
        return mamba2_step(S, params["A"], params["D"], tok["x"], tok["dt"], tok["B"], tok["C"],
                           dt_scales_input)
    if kind == "kda":
        return kda_step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
    return gdn_step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
