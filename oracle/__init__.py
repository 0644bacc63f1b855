"""CPU oracle of the RLT recurrent decoder -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It never imports the CUDA package and the
CUDA package never imports it; both receive the same seeded inputs.

The arithmetic lives in ``rlt_oracle.c`` (plain loops, one floating type per
build: ``f64`` for parity, ``f32`` for the timed baseline). This module only
marshals numpy arrays through ctypes. Citations are in the C source.

Pinned by ``tests/test_oracle_*.py`` (textbook pieces against torch CPU
routines, closed forms, brute force and the invariants the pages fix).
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

MAX_LAYERS = 64
_LIBS = {}


def load_library(path: str):
    """Load an oracle build from an explicit path (used by the mutation pins)."""
    lib = C.CDLL(path)
    _declare(lib)
    return lib


def _lib(precision: str):
    if precision not in _LIBS:
        # a planted-mistake build under test replaces the library wholesale
        override = os.environ.get(f"RLT_ORACLE_LIB_{precision.upper()}")
        path = override or _build.lib_path(precision)
        if not override and (not os.path.exists(path)
                             or os.path.getmtime(path) < os.path.getmtime(_build.SRC)):
            _build.build()
        lib = C.CDLL(path)
        _declare(lib)
        _LIBS[precision] = lib
    return _LIBS[precision]


class _Cfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "d", "n_heads", "head_dim", "n_enc", "n_dec", "ffn_dim", "ffn_kind",
        "vocab", "window", "mem_groups")] + [
        ("alpha", C.c_double), ("rms_eps", C.c_double), ("rope_theta", C.c_double)]


_PER_ENC = ("enc_ln1", "enc_wqkv", "enc_wo", "enc_ln2", "enc_w1", "enc_wb", "enc_w2")
_PER_DEC = ("dec_ln1", "dec_wqkv", "dec_wo", "dec_ln2", "dec_wqx", "dec_wox",
            "dec_ln3", "dec_w1", "dec_wb", "dec_w2")


class _W(C.Structure):
    _fields_ = ([("embed", C.c_void_p)]
                + [(n, C.c_void_p * MAX_LAYERS) for n in _PER_ENC]
                + [("enc_lnf", C.c_void_p)]
                + [("mem_wk", C.c_void_p * MAX_LAYERS), ("mem_wv", C.c_void_p * MAX_LAYERS)]
                + [("gate_w", C.c_void_p), ("gate_b", C.c_void_p), ("sstar", C.c_void_p)]
                + [(n, C.c_void_p * MAX_LAYERS) for n in _PER_DEC]
                + [("dec_lnf", C.c_void_p)])


def _declare(lib):
    P = C.c_void_p
    lib.orc_real_bytes.restype = C.c_int
    lib.orc_rmsnorm.argtypes = [P, P, C.c_int, C.c_double, P]
    lib.orc_linear.argtypes = [P, P, C.c_int, C.c_int, P]
    lib.orc_rope.argtypes = [P, C.c_int, C.c_long, C.c_double]
    lib.orc_attend_dense.argtypes = [P, P, P, C.c_int, C.c_int, P]
    for f in ("orc_gelu", "orc_silu", "orc_sigmoid"):
        getattr(lib, f).argtypes = [C.c_double]
        getattr(lib, f).restype = C.c_double
    lib.orc_encode.argtypes = [P, P, P, C.c_int, P, P, C.c_int]
    lib.orc_encode.restype = C.c_int
    lib.orc_step.argtypes = [P, P, P, P, C.c_int, C.c_long, P, P]
    lib.orc_decode.argtypes = [P, P, P, P, C.c_int, C.c_long, C.c_long, P, P, P]
    lib.orc_init_state.argtypes = [P, P, P, P]
    lib.orc_run.argtypes = [P, P, P, C.c_int, P, P, P]
    lib.orc_run.restype = C.c_int
    lib.orc_decode_bruteforce.argtypes = [P, P, P, P, C.c_int, C.c_int, P]
    lib.orc_decode_parallel_nofeedback.argtypes = [P, P, P, P, C.c_int, C.c_int, P]
    lib.orc_run_batch.argtypes = [P, P, P, C.c_int, P, C.c_int, C.c_int, P]
    lib.orc_run_batch.restype = C.c_int
    lib.orc_lm_head.argtypes = [P, P, P, P]
    lib.orc_sample.argtypes = [P, C.c_int, C.c_double, C.c_double]
    lib.orc_sample.restype = C.c_int


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


class Oracle:
    """The oracle bound to one model's weights.

    ``cfg`` is any object with the RLT config attributes (d, n_heads, head_dim,
    n_enc, n_dec, ffn_dim, ffn_kind, vocab, window, mem_groups, alpha,
    rms_eps, rope_theta); ``weights`` maps the generator's tensor names to
    float arrays (row-major [out][in]).
    """

    def __init__(self, cfg, weights, precision: str = "f64", lib=None):
        self.cfg = cfg
        self.precision = precision
        self.dt = np.float64 if precision == "f64" else np.float32
        self.lib = lib if lib is not None else _lib(precision)
        assert cfg.n_enc <= MAX_LAYERS and cfg.n_dec <= MAX_LAYERS
        assert cfg.mem_groups <= MAX_LAYERS
        self._c = _Cfg(cfg.d, cfg.n_heads, cfg.head_dim, cfg.n_enc, cfg.n_dec,
                       cfg.ffn_dim, cfg.ffn_kind, cfg.vocab, cfg.window,
                       cfg.mem_groups, float(cfg.alpha), float(cfg.rms_eps),
                       float(cfg.rope_theta))
        self._keep = {}
        conv = {}

        def arr(name):
            src = weights[name]
            key = id(src)
            if key not in conv:  # tied names share one converted array
                conv[key] = np.ascontiguousarray(src, dtype=self.dt)
            self._keep[name] = conv[key]
            return conv[key].ctypes.data

        w = _W()
        w.embed = arr("embed")
        swiglu = cfg.ffn_kind == 1
        for l in range(cfg.n_enc):
            w.enc_ln1[l] = arr(f"enc.{l}.ln1")
            w.enc_wqkv[l] = arr(f"enc.{l}.wqkv")
            w.enc_wo[l] = arr(f"enc.{l}.wo")
            w.enc_ln2[l] = arr(f"enc.{l}.ln2")
            w.enc_w1[l] = arr(f"enc.{l}.wa" if swiglu else f"enc.{l}.w1")
            if swiglu:
                w.enc_wb[l] = arr(f"enc.{l}.wb")
            w.enc_w2[l] = arr(f"enc.{l}.w2")
        w.enc_lnf = arr("enc.lnf")
        for g in range(cfg.mem_groups):
            w.mem_wk[g] = arr(f"mem.{g}.wk")
            w.mem_wv[g] = arr(f"mem.{g}.wv")
        w.gate_w = arr("gate.w")
        w.gate_b = arr("gate.b")
        w.sstar = arr("sstar")
        for l in range(cfg.n_dec):
            w.dec_ln1[l] = arr(f"dec.{l}.ln1")
            w.dec_wqkv[l] = arr(f"dec.{l}.wqkv")
            w.dec_wo[l] = arr(f"dec.{l}.wo")
            w.dec_ln2[l] = arr(f"dec.{l}.ln2")
            w.dec_wqx[l] = arr(f"dec.{l}.wqx")
            w.dec_wox[l] = arr(f"dec.{l}.wox")
            w.dec_ln3[l] = arr(f"dec.{l}.ln3")
            w.dec_w1[l] = arr(f"dec.{l}.wa" if swiglu else f"dec.{l}.w1")
            if swiglu:
                w.dec_wb[l] = arr(f"dec.{l}.wb")
            w.dec_w2[l] = arr(f"dec.{l}.w2")
        w.dec_lnf = arr("dec.lnf")
        self._w = w

    # -- helpers -------------------------------------------------------
    def _a(self, x, shape=None):
        a = np.ascontiguousarray(x, dtype=self.dt)
        if shape is not None:
            assert a.shape == tuple(shape), (a.shape, shape)
        return a

    def _args(self):
        return C.byref(self._c), C.byref(self._w)

    @property
    def win_shape(self):
        c = self.cfg
        return (c.n_dec, 2, c.window - 1, c.d)

    # -- the method ----------------------------------------------------
    def init_state(self):
        s = np.zeros(self.cfg.d, self.dt)
        win = np.zeros(self.win_shape, self.dt)
        self.lib.orc_init_state(*self._args(), _ptr(s), _ptr(win))
        return s, win

    def encode(self, tokens):
        """e [T][d], mem [G][T][2][d] of one sequence."""
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        T = tok.shape[0]
        c = self.cfg
        e = np.zeros((max(T, 1), c.d), self.dt)
        mem = np.zeros((c.mem_groups, max(T, 1), 2, c.d), self.dt)
        rc = self.lib.orc_encode(*self._args(), _ptr(tok), T, _ptr(e), _ptr(mem), max(T, 1))
        assert rc == 0
        return e[:T], mem

    def step(self, e_t, mem, t, s, win):
        """One transition at position t; returns the new (s, win)."""
        mem = self._a(mem)
        s = self._a(s, (self.cfg.d,)).copy()
        win = self._a(win, self.win_shape).copy()
        e_t = self._a(e_t, (self.cfg.d,))
        assert mem.shape[1] > t
        self.lib.orc_step(*self._args(), _ptr(e_t), _ptr(mem), mem.shape[1], t,
                          _ptr(s), _ptr(win))
        return s, win

    def decode(self, e, mem, t0, t1, s, win):
        """Steps t0..t1-1; returns (s_out [t1-t0][d], s, win)."""
        e = self._a(e)
        mem = self._a(mem)
        assert mem.shape[1] >= t1 and e.shape[0] >= t1
        s = self._a(s, (self.cfg.d,)).copy()
        win = self._a(win, self.win_shape).copy()
        out = np.zeros((max(t1 - t0, 1), self.cfg.d), self.dt)
        self.lib.orc_decode(*self._args(), _ptr(e), _ptr(mem), mem.shape[1],
                            t0, t1, _ptr(s), _ptr(win), _ptr(out))
        return out[: t1 - t0], s, win

    def run(self, tokens):
        """Encoder + all decoder steps from s*; returns (s_out [T][d], s, win)."""
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        T = tok.shape[0]
        out = np.zeros((max(T, 1), self.cfg.d), self.dt)
        s = np.zeros(self.cfg.d, self.dt)
        win = np.zeros(self.win_shape, self.dt)
        rc = self.lib.orc_run(*self._args(), _ptr(tok), T, _ptr(out), _ptr(s), _ptr(win))
        assert rc == 0
        return out[:T], s, win

    def decode_bruteforce(self, e, mem, T):
        e = self._a(e)
        mem = self._a(mem)
        out = np.zeros((max(T, 1), self.cfg.d), self.dt)
        self.lib.orc_decode_bruteforce(*self._args(), _ptr(e), _ptr(mem),
                                       mem.shape[1], T, _ptr(out))
        return out[:T]

    def decode_parallel_nofeedback(self, e, mem, T):
        e = self._a(e)
        mem = self._a(mem)
        out = np.zeros((max(T, 1), self.cfg.d), self.dt)
        self.lib.orc_decode_parallel_nofeedback(*self._args(), _ptr(e), _ptr(mem),
                                                mem.shape[1], T, _ptr(out))
        return out[:T]

    def lm_head(self, s):
        """Next-token logits [V] read from s_t."""
        s = self._a(s, (self.cfg.d,))
        out = np.zeros(self.cfg.vocab, self.dt)
        self.lib.orc_lm_head(*self._args(), _ptr(s), _ptr(out))
        return out

    def run_batch(self, tokens, lengths, n_threads=0):
        """Full runs of B sequences in parallel; returns (s_final [B][d], threads)."""
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        lens = np.ascontiguousarray(lengths, dtype=np.int32)
        B = lens.shape[0]
        out = np.zeros((B, self.cfg.d), self.dt)
        used = self.lib.orc_run_batch(*self._args(), _ptr(tok), tok.shape[1],
                                      _ptr(lens), B, int(n_threads), _ptr(out))
        return out, used


# -- textbook pieces, exposed for the pins ------------------------------
def rmsnorm(x, gamma, eps, precision="f64"):
    lib = _lib(precision)
    dt = np.float64 if precision == "f64" else np.float32
    x = np.ascontiguousarray(x, dt)
    g = np.ascontiguousarray(gamma, dt)
    y = np.zeros_like(x)
    lib.orc_rmsnorm(_ptr(x), _ptr(g), x.shape[0], eps, _ptr(y))
    return y


def linear(W, x, precision="f64"):
    lib = _lib(precision)
    dt = np.float64 if precision == "f64" else np.float32
    W = np.ascontiguousarray(W, dt)
    x = np.ascontiguousarray(x, dt)
    y = np.zeros(W.shape[0], dt)
    lib.orc_linear(_ptr(W), _ptr(x), W.shape[0], W.shape[1], _ptr(y))
    return y


def rope(v, pos, theta=10000.0, precision="f64"):
    lib = _lib(precision)
    dt = np.float64 if precision == "f64" else np.float32
    v = np.ascontiguousarray(v, dt).copy()
    lib.orc_rope(_ptr(v), v.shape[0], int(pos), theta)
    return v


def attend(q, K, V, precision="f64"):
    lib = _lib(precision)
    dt = np.float64 if precision == "f64" else np.float32
    q = np.ascontiguousarray(q, dt)
    K = np.ascontiguousarray(K, dt)
    V = np.ascontiguousarray(V, dt)
    out = np.zeros(q.shape[0], dt)
    lib.orc_attend_dense(_ptr(q), _ptr(K), _ptr(V), K.shape[0], q.shape[0], _ptr(out))
    return out


def sample(logits, temperature, u, precision="f64"):
    """One token from logits (argmax at temperature 0, else inverse CDF at u)."""
    lib = _lib(precision)
    dt = np.float64 if precision == "f64" else np.float32
    lg = np.ascontiguousarray(logits, dt)
    return int(lib.orc_sample(_ptr(lg), lg.shape[0], float(temperature), float(u)))


def scalar(fn: str, x: float) -> float:
    return getattr(_lib("f64"), f"orc_{fn}")(float(x))
