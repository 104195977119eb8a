"""float64 CPU oracle of the DART forward path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. It wraps ``oracle/dart_oracle.c`` (plain C, float64,
compiled by :func:`build` with gcc) through ctypes, and it never touches the
CUDA library. Each function follows one passage of "DART: Decoded Attention
over Recurrent States" (arXiv 2608.02032):

* :func:`recurrence`   -- §2 eq (2): H_t = a_t H_{t-1} + B_t^T X_t, Y_t = C_t H_t
* :func:`chunk_states` -- §3 eq (5): chunk state memories by direct summation
* :func:`sma`          -- §3 eq (8)-(10): state-memory attention by explicit loops; with
                          ``norm_eps`` the normalised score branch of App. B.1 eq (25)-(27)
* :func:`sma_bwd`      -- gradients of SMA's readout R w.r.t. Q, C, E and the chunk memories by the chain
                          rule, the weights recomputed (§4 "Efficient Training"; App. C eq (32)-(35))
* :func:`combine`      -- §3 eq (11): out_t = Y_t + g_t R_t
* :func:`decode`       -- single new token over cached chunk memories (§4 "Inference Cache")
* :func:`decode_step`  -- one decode step with its state maintenance: the recurrence of eq (2)
                          in recurrent form, the open chunk's memory accumulated token by token
                          and appended to the cache when the chunk closes (§4 "Inference Cache")
* :func:`layer`        -- the recurrence, chunk memories, SMA and combine in sequence.

Arrays are float64 numpy arrays in the layouts of ``dart_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dart_oracle.c")
_LIB = os.path.join(_HERE, "libdart_oracle.so")

_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64
_i64p = ctypes.POINTER(ctypes.c_int64)


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE semantics: no -ffast-math)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, src, "-lm", "-lpthread"])
    os.replace(tmp, out)
    return out


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(_f64p)


def _c64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


class Oracle:
    """Bound instance of a compiled oracle library (tests may load a variant)."""

    def __init__(self, lib_path: Optional[str] = None):
        self.path = lib_path or build()
        self.lib = ctypes.CDLL(self.path)
        L = self.lib
        L.dart_oracle_recurrence.argtypes = [_i64] * 7 + [_f64p] * 7 + [ctypes.c_int]
        L.dart_oracle_chunk_states.argtypes = [_i64] * 7 + [_f64p] * 4 + [ctypes.c_int]
        L.dart_oracle_sma.argtypes = [_i64] * 7 + [_f64p] * 4 + [_i64p, _i64] + [_f64p] * 2 + [ctypes.c_int]
        L.dart_oracle_combine.argtypes = [_i64] * 4 + [_f64p] * 3 + [_i64] * 3 + [_f64p]
        L.dart_oracle_decode.argtypes = [_i64] * 7 + [_f64p] * 5 + [_i64] * 2 + [_f64p] * 3 + [ctypes.c_int]
        L.dart_oracle_sma_norm.argtypes = ([_i64] * 7 + [ctypes.c_double] + [_f64p] * 4 + [_i64p, _i64] + [_f64p] * 2
                                           + [ctypes.c_int])
        L.dart_oracle_decode_step.argtypes = ([_i64] * 7 + [ctypes.c_int] + [_f64p] * 7 + [_i64] * 2 + [_f64p] * 5
                                              + [ctypes.c_int])
        L.dart_oracle_sma_bwd.argtypes = [_i64] * 7 + [_f64p] * 9 + [ctypes.c_int]
        L.dart_oracle_sma_bwd_tokens.argtypes = [_i64] * 7 + [_f64p] * 5 + [_i64p, _i64] + [_f64p] * 3 + [ctypes.c_int]
        L.dart_oracle_sma_bwd_ddh.argtypes = [_i64] * 7 + [_f64p] * 5 + [_i64p, _i64, _f64p, ctypes.c_int]
        L.dart_oracle_sma_bwd_norm_tokens.argtypes = ([_i64] * 7 + [ctypes.c_double] + [_f64p] * 5 + [_i64p, _i64]
                                                      + [_f64p] * 3 + [ctypes.c_int])
        L.dart_oracle_sma_bwd_norm_ddh.argtypes = ([_i64] * 7 + [ctypes.c_double] + [_f64p] * 5
                                                   + [_i64p, _i64, _f64p, ctypes.c_int])
        L.dart_oracle_sma_bwd_tokens.restype = None
        L.dart_oracle_sma_bwd_norm.argtypes = [_i64] * 7 + [ctypes.c_double] + [_f64p] * 9 + [ctypes.c_int]
        L.dart_oracle_sma_bwd_norm.restype = None
        L.dart_oracle_sma_bwd_ddh.restype = None
        for f in ("dart_oracle_recurrence", "dart_oracle_chunk_states", "dart_oracle_sma", "dart_oracle_combine",
                  "dart_oracle_decode", "dart_oracle_decode_step", "dart_oracle_sma_norm", "dart_oracle_sma_bwd"):
            getattr(L, f).restype = None

    # -- eq (2) -------------------------------------------------------------
    def recurrence(self, X, B, C, logA, S: int, want_hend: bool = True, threads: Optional[int] = None):
        """Token-by-token recurrence. Returns (Y [b,L,H,P], Hend [b,H,M,N,P] or None, Hfinal [b,H,N,P])."""
        X, B, C, logA = _c64(X), _c64(B), _c64(C), _c64(logA)
        Bt, L, H, P = X.shape
        G, N = B.shape[2], B.shape[3]
        M = -(-L // S)
        Y = np.empty_like(X)
        Hend = np.empty((Bt, H, M, N, P)) if want_hend else None
        Hfinal = np.empty((Bt, H, N, P))
        self.lib.dart_oracle_recurrence(Bt, L, H, G, N, P, S, _p(X), _p(B), _p(C), _p(logA), _p(Y), _p(Hend),
                                        _p(Hfinal), threads or default_threads())
        return Y, Hend, Hfinal

    # -- eq (5) -------------------------------------------------------------
    def chunk_states(self, X, B, logA, S: int, threads: Optional[int] = None) -> np.ndarray:
        X, B, logA = _c64(X), _c64(B), _c64(logA)
        Bt, L, H, P = X.shape
        G, N = B.shape[2], B.shape[3]
        M = -(-L // S)
        dH = np.empty((Bt, H, M, N, P))
        self.lib.dart_oracle_chunk_states(Bt, L, H, G, N, P, S, _p(X), _p(B), _p(logA), _p(dH),
                                          threads or default_threads())
        return dH

    # -- eq (8)-(10) --------------------------------------------------------
    def sma(self, Q, C, E, dH, S: int, tokens: Optional[Sequence[int]] = None, threads: Optional[int] = None,
            norm_eps: Optional[float] = None):
        """State-memory attention. Returns (R, lse).

        tokens None: R [b, L, H, P], lse [b, H, L]. Otherwise the token axis is the
        sample axis: R [b, len(tokens), H, P], lse [b, H, len(tokens)].
        norm_eps: the normalised score branch of App. B.1 with that epsilon.
        """
        Q, C, E, dH = _c64(Q), _c64(C), _c64(E), _c64(dH)
        Bt, L, H, P = E.shape
        G, N = Q.shape[2], Q.shape[3]
        assert dH.shape[:2] == (Bt, H) and dH.shape[2] == -(-L // S), "dH must hold every chunk of the sequence"
        if tokens is None:
            tok = None
            nt = L
        else:
            tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
            assert tok.ndim == 1 and (tok.size == 0 or (tok.min() >= 0 and tok.max() < L))
            nt = tok.size
        R = np.empty((Bt, nt, H, P))
        lse = np.empty((Bt, H, nt))
        tp = None if tok is None else tok.ctypes.data_as(_i64p)
        if norm_eps is None:
            self.lib.dart_oracle_sma(Bt, L, H, G, N, P, S, _p(Q), _p(C), _p(E), _p(dH), tp, nt, _p(R), _p(lse),
                                     threads or default_threads())
        else:
            self.lib.dart_oracle_sma_norm(Bt, L, H, G, N, P, S, float(norm_eps), _p(Q), _p(C), _p(E), _p(dH), tp, nt,
                                          _p(R), _p(lse), threads or default_threads())
        return R, lse

    # -- backward of eq (8)-(10) (§4 "Efficient Training", App. C eq (32)-(35)) --
    def sma_bwd(self, Q, C, E, dH, dR, S: int, threads: Optional[int] = None,
                norm_eps: Optional[float] = None) -> Dict[str, np.ndarray]:
        """Gradients of a loss through R given dR = dLoss/dR [b, L, H, P]; with norm_eps, of the
        normalised score branch (App. B.1).

        Returns dQ, dC [b, L, G, N], dE [b, L, H, P] and ddH [b, H, M, N, P]."""
        Q, C, E, dH, dR = _c64(Q), _c64(C), _c64(E), _c64(dH), _c64(dR)
        Bt, L, H, P = E.shape
        G, N = Q.shape[2], Q.shape[3]
        M = -(-L // S)
        assert dH.shape == (Bt, H, M, N, P) and dR.shape == E.shape
        dQ, dC = np.empty_like(Q), np.empty_like(C)
        dE, ddH = np.empty_like(E), np.empty_like(dH)
        if norm_eps is None:
            self.lib.dart_oracle_sma_bwd(Bt, L, H, G, N, P, S, _p(Q), _p(C), _p(E), _p(dH), _p(dR), _p(dQ), _p(dC),
                                         _p(dE), _p(ddH), threads or default_threads())
        else:
            self.lib.dart_oracle_sma_bwd_norm(Bt, L, H, G, N, P, S, float(norm_eps), _p(Q), _p(C), _p(E), _p(dH),
                                              _p(dR), _p(dQ), _p(dC), _p(dE), _p(ddH), threads or default_threads())
        return dict(dQ=dQ, dC=dC, dE=dE, ddH=ddH)

    def sma_bwd_tokens(self, Q, C, E, dH, dR, S: int, tokens: Sequence[int], threads: Optional[int] = None,
                       norm_eps: Optional[float] = None):
        """The per-token gradients of sma_bwd at the listed tokens only (every batch row, every head):
        dQ, dC [b, ntok, G, N] and dE [b, ntok, H, P]; with norm_eps, of the normalised score branch."""
        Q, C, E, dH, dR = _c64(Q), _c64(C), _c64(E), _c64(dH), _c64(dR)
        Bt, L, H, P = E.shape
        G, N = Q.shape[2], Q.shape[3]
        tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
        assert tok.ndim == 1 and tok.size > 0 and tok.min() >= 0 and tok.max() < L
        dQ, dC = np.empty((Bt, tok.size, G, N)), np.empty((Bt, tok.size, G, N))
        dE = np.empty((Bt, tok.size, H, P))
        if norm_eps is None:
            self.lib.dart_oracle_sma_bwd_tokens(Bt, L, H, G, N, P, S, _p(Q), _p(C), _p(E), _p(dH), _p(dR),
                                                tok.ctypes.data_as(_i64p), tok.size, _p(dQ), _p(dC), _p(dE),
                                                threads or default_threads())
        else:
            self.lib.dart_oracle_sma_bwd_norm_tokens(Bt, L, H, G, N, P, S, float(norm_eps), _p(Q), _p(C), _p(E),
                                                     _p(dH), _p(dR), tok.ctypes.data_as(_i64p), tok.size, _p(dQ),
                                                     _p(dC), _p(dE), threads or default_threads())
        return dict(dQ=dQ, dC=dC, dE=dE)

    def sma_bwd_ddh(self, Q, C, E, dH, dR, S: int, triples: Sequence[Sequence[int]], threads: Optional[int] = None,
                    norm_eps: Optional[float] = None):
        """ddH of sma_bwd for the listed (batch row, head, chunk) triples only: [n, N, P]; with norm_eps, of
        the normalised score branch."""
        Q, C, E, dH, dR = _c64(Q), _c64(C), _c64(E), _c64(dH), _c64(dR)
        Bt, L, H, P = E.shape
        G, N = Q.shape[2], Q.shape[3]
        tr = np.ascontiguousarray(np.asarray(triples, dtype=np.int64).reshape(-1, 3))
        out = np.empty((tr.shape[0], N, P))
        if norm_eps is None:
            self.lib.dart_oracle_sma_bwd_ddh(Bt, L, H, G, N, P, S, _p(Q), _p(C), _p(E), _p(dH), _p(dR),
                                             tr.ctypes.data_as(_i64p), tr.shape[0], _p(out),
                                             threads or default_threads())
        else:
            self.lib.dart_oracle_sma_bwd_norm_ddh(Bt, L, H, G, N, P, S, float(norm_eps), _p(Q), _p(C), _p(E), _p(dH),
                                                  _p(dR), tr.ctypes.data_as(_i64p), tr.shape[0], _p(out),
                                                  threads or default_threads())
        return out

    # -- eq (11) ------------------------------------------------------------
    def combine(self, Y, R, g, g_strides) -> np.ndarray:
        Y, R, g = _c64(Y), _c64(R), _c64(g)
        Bt, L, H, P = Y.shape
        out = np.empty_like(Y)
        sb, st, sh = g_strides
        self.lib.dart_oracle_combine(Bt, L, H, P, _p(Y), _p(R), _p(g), sb, st, sh, _p(out))
        return out

    # -- decode -------------------------------------------------------------
    def decode(self, Q, C, E, Y, g, g_strides, cache, n_chunks: Optional[int] = None, threads: Optional[int] = None):
        """One new token over cached chunk memories. cache [b, H, cs, N, P]. Returns (out, lse)."""
        Q, C, E, Y, g, cache = _c64(Q), _c64(C), _c64(E), _c64(Y), _c64(g), _c64(cache)
        Bt, G, N = Q.shape
        H, P = E.shape[1], E.shape[2]
        cs = cache.shape[2]
        n = cs if n_chunks is None else n_chunks
        assert 0 <= n <= cs
        out = np.empty_like(Y)
        lse = np.empty((Bt, H))
        sb, sh = g_strides
        self.lib.dart_oracle_decode(Bt, H, G, N, P, n, cs, _p(Q), _p(C), _p(E), _p(Y), _p(g), sb, sh, _p(cache),
                                    _p(out), _p(lse), threads or default_threads())
        return out, lse

    def decode_step(self, X, B, C, Q, E, logA, g, g_strides, state, acc, cache, n_chunks: int, close: bool,
                    threads: Optional[int] = None):
        """One decode step for one new token per batch row.

        X, E [b, H, P]; B, C, Q [b, G, N]; logA [b, H]. state, acc [b, H, N, P] and cache
        [b, H, cs, N, P] are float64 arrays updated in place: state and acc take the token
        (acc is the memory of the open chunk), and when ``close`` the token ends its chunk:
        acc is appended at cache index n_chunks and reset. Returns (out, lse) [b, H, P], [b, H].
        """
        for a in (state, acc, cache):
            assert a.dtype == np.float64 and a.flags.c_contiguous
        X, B, C, Q, E, logA, g = _c64(X), _c64(B), _c64(C), _c64(Q), _c64(E), _c64(logA), _c64(g)
        Bt, G, N = Q.shape
        H, P = E.shape[1], E.shape[2]
        cs = cache.shape[2]
        assert 0 <= n_chunks <= cs and (not close or n_chunks < cs)
        out = np.empty((Bt, H, P))
        lse = np.empty((Bt, H))
        sb, sh = g_strides
        self.lib.dart_oracle_decode_step(Bt, H, G, N, P, n_chunks, cs, 1 if close else 0, _p(X), _p(B), _p(C), _p(Q),
                                         _p(E), _p(logA), _p(g), sb, sh, _p(state), _p(acc), _p(cache), _p(out),
                                         _p(lse), threads or default_threads())
        return out, lse

    # -- the whole forward --------------------------------------------------
    def layer(self, X, B, C, Q, E, logA, g, g_strides, S: int, sma_tokens=None,
              threads: Optional[int] = None) -> Dict[str, np.ndarray]:
        """Recurrence (Y, final state) + direct-sum chunk memories + SMA (+ combine when dense)."""
        Y, _, Hfinal = self.recurrence(X, B, C, logA, S, want_hend=False, threads=threads)
        dH = self.chunk_states(X, B, logA, S, threads=threads)
        R, lse = self.sma(Q, C, E, dH, S, tokens=sma_tokens, threads=threads)
        res = dict(Y=Y, dH=dH, R=R, lse=lse, Hfinal=Hfinal)
        if sma_tokens is None:
            res["out"] = self.combine(Y, R, g, g_strides)
        else:
            tok = np.asarray(sma_tokens, dtype=np.int64)
            sb, st, sh = g_strides
            gg = np.asarray(g, dtype=np.float64).reshape(-1)
            Bt, L, H, P = np.shape(X)
            b = np.arange(Bt)[:, None, None]
            h = np.arange(H)[None, None, :]
            gsel = gg[b * sb + tok[None, :, None] * st + h * sh]
            res["out"] = Y[:, tok] + gsel[..., None] * R
        return res


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def recurrence(*a, **k):
    return get().recurrence(*a, **k)


def chunk_states(*a, **k):
    return get().chunk_states(*a, **k)


def sma(*a, **k):
    return get().sma(*a, **k)


def combine(*a, **k):
    return get().combine(*a, **k)


def decode(*a, **k):
    return get().decode(*a, **k)


def decode_step(*a, **k):
    return get().decode_step(*a, **k)


def layer(*a, **k):
    return get().layer(*a, **k)
