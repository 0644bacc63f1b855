"""Python binding of the RLT C ABI (``include/rlt.h``): argument marshalling only.

Every step of the path runs in ``librlt.so``'s kernels. PyTorch provides the
device memory (weights, arena, outputs) and the CUDA streams. There is no CPU
fallback: if the library is missing, importing a model raises.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import Dict, Optional

import numpy as np

from .configs import BF16, SWIGLU, RLTConfig

MAX_LAYERS = 64
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librlt.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "rlt.h")

RLT_OK = 0
STATUS = {0: "RLT_OK", 1: "RLT_ERR_INVALID_ARG", 2: "RLT_ERR_UNSUPPORTED",
          3: "RLT_ERR_NOT_READY", 4: "RLT_ERR_CAPACITY", 5: "RLT_ERR_DUPLICATE_ID",
          6: "RLT_ERR_CUDA", 7: "RLT_ERR_TIMEOUT", 8: "RLT_ERR_DEVICE", 9: "RLT_ERR_STALE"}


class RLTError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} "
                         f"({_lib().rlt_status_string(status).decode()})")


class rlt_config(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "d", "n_heads", "head_dim", "n_enc_layers", "n_dec_layers", "ffn_dim",
        "ffn_kind", "vocab", "window", "mem_groups", "tied", "dtype", "max_seqs",
        "max_len", "max_prefill_tokens", "enc_cache")] + [
        ("alpha", C.c_float), ("rms_eps", C.c_float), ("rope_theta", C.c_float)]


_ENC = ("enc_ln1", "enc_wqkv", "enc_wo", "enc_ln2", "enc_w1", "enc_wb", "enc_w2")
_DEC = ("dec_ln1", "dec_wqkv", "dec_wo", "dec_ln2", "dec_wqx", "dec_wox", "dec_ln3",
        "dec_w1", "dec_wb", "dec_w2")


class rlt_weights(C.Structure):
    _fields_ = ([("embed", C.c_void_p)]
                + [(n, C.c_void_p * MAX_LAYERS) for n in _ENC]
                + [("enc_lnf", C.c_void_p)]
                + [("mem_wk", C.c_void_p * MAX_LAYERS), ("mem_wv", C.c_void_p * MAX_LAYERS)]
                + [("gate_w", C.c_void_p), ("gate_b", C.c_void_p), ("sstar", C.c_void_p)]
                + [(n, C.c_void_p * MAX_LAYERS) for n in _DEC]
                + [("dec_lnf", C.c_void_p)])


class rlt_grads(C.Structure):
    _fields_ = ([(n, C.c_void_p) for n in ("gate_w", "gate_b", "sstar", "dec_lnf")]
                + [(n, C.c_void_p * MAX_LAYERS) for n in _DEC]
                + [("mem_wk", C.c_void_p * MAX_LAYERS), ("mem_wv", C.c_void_p * MAX_LAYERS)])


K_XATTN, K_SWA, K_GEMM, K_OTHER, K_ENC, K_STEP = range(6)
FAULT_NONE, FAULT_SKIP_ATTN_PRODUCER = 0, 1
STEP_CHAIN, STEP_FUSED = 0, 1
K_NAMES = ("xattn", "swa", "gemm", "other", "encoder", "step")


class rlt_stats(C.Structure):
    _fields_ = [("launches", C.c_int64), ("kernel_launches", C.c_int64 * 6),
                ("kernel_ms", C.c_double * 6), ("kernel_bytes", C.c_double * 6),
                ("kernel_flops", C.c_double * 6)]


_LIB = None


def _declare(lib):
    P, I = C.c_void_p, C.c_int
    lib.rlt_check_config.argtypes = [P]
    lib.rlt_arena_bytes.argtypes = [P]
    lib.rlt_arena_bytes.restype = C.c_size_t
    lib.rlt_create.argtypes = [P, P, P, C.c_size_t, C.POINTER(P)]
    lib.rlt_destroy.argtypes = [P]
    lib.rlt_destroy.restype = None
    lib.rlt_reset_seq.argtypes = [P, I, P]
    lib.rlt_prefill_encoder.argtypes = [P, P, P, P, P, I, P]
    lib.rlt_decoder_step.argtypes = [P, P, I, P]
    lib.rlt_run_sequence.argtypes = [P, P, I, I, P]
    lib.rlt_decoder_parallel.argtypes = [P, P, I, I, P, P]
    lib.rlt_backward_workspace_bytes.argtypes = [P, I, I]
    lib.rlt_backward_workspace_bytes.restype = C.c_size_t
    lib.rlt_backward.argtypes = [P, P, I, I, P, P, P, P, P, P, C.c_size_t, P]
    lib.rlt_run_ragged.argtypes = [P, P, P, I, P]
    lib.rlt_plan_ragged.argtypes = [P, I, P, P, I, C.POINTER(I)]
    lib.rlt_get_state.argtypes = [P, I, P, P, C.POINTER(C.c_int64), P]
    lib.rlt_set_state.argtypes = [P, I, P, P, C.c_int64, P]
    lib.rlt_get_encoder_output.argtypes = [P, I, P, P, C.POINTER(C.c_int64), P]
    lib.rlt_poll_device_error.argtypes = [P]
    lib.rlt_set_fault.argtypes = [P, I, C.c_int64]
    lib.rlt_append_encoder.argtypes = [P, P, P, I, P]
    lib.rlt_lm_head.argtypes = [P, P, I, P, P]
    lib.rlt_sample.argtypes = [P, P, I, C.c_float, P, P, P]
    lib.rlt_serve_step.argtypes = [P, P, I, C.c_float, P, P, P, P]
    lib.rlt_snapshot_bytes.argtypes = [P, I]
    lib.rlt_snapshot_bytes.restype = C.c_size_t
    lib.rlt_get_snapshot.argtypes = [P, I, P, C.c_size_t, P]
    lib.rlt_set_snapshot.argtypes = [P, I, P, C.c_size_t, P]
    lib.rlt_model_fingerprint.argtypes = [P, C.POINTER(C.c_uint64)]
    lib.rlt_set_step_kernel.argtypes = [P, I]
    lib.rlt_get_step_kernel.argtypes = [P]
    lib.rlt_step_kernel_ctas.argtypes = [P]
    lib.rlt_set_step_trace.argtypes = [P, P, C.c_size_t]
    lib.rlt_attend_workspace_bytes.argtypes = [I, I, I, I]
    lib.rlt_attend_workspace_bytes.restype = C.c_size_t
    lib.rlt_attend.argtypes = [P, P, P, I, I, I, I, I, P, P, C.c_size_t, P]
    lib.rlt_profile.argtypes = [P, I]
    lib.rlt_get_stats.argtypes = [P, P]
    lib.rlt_status_string.argtypes = [I]
    lib.rlt_last_cuda_error.argtypes = [C.c_char_p, C.c_size_t]
    lib.rlt_status_string.restype = C.c_char_p


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"librlt.so not built ({LIB_PATH}); run "
                               "python -m token_recurrent_decoding_b200.build")
        lib = C.CDLL(LIB_PATH)
        _declare(lib)
        _LIB = lib
    return _LIB


def header_symbols():
    """Function names the public header declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RLT_API\s+[\w\s\*]+?\b(rlt_\w+)\s*\(", text)))


def _check(rc: int, what: str):
    if rc != RLT_OK:
        if rc == 6:  # RLT_ERR_CUDA
            buf = C.create_string_buffer(160)
            _lib().rlt_last_cuda_error(buf, 160)
            what = f"{what}: {buf.value.decode()}"
        raise RLTError(rc, what)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def make_config(cfg: RLTConfig, max_seqs: int, max_len: int, max_prefill_tokens: int = 0,
                enc_cache: bool = False):
    return rlt_config(cfg.d, cfg.n_heads, cfg.head_dim, cfg.n_enc, cfg.n_dec, cfg.ffn_dim,
                      cfg.ffn_kind, cfg.vocab, cfg.window, cfg.mem_groups, int(cfg.tied),
                      cfg.dtype, max_seqs, max_len, max_prefill_tokens, int(enc_cache),
                      float(cfg.alpha), float(cfg.rms_eps), float(cfg.rope_theta))


def check_config(cfg: RLTConfig, max_seqs: int, max_len: int) -> int:
    c = make_config(cfg, max_seqs, max_len)
    return _lib().rlt_check_config(C.byref(c))


def arena_bytes(cfg: RLTConfig, max_seqs: int, max_len: int, max_prefill_tokens: int = 0,
                enc_cache: bool = False) -> int:
    c = make_config(cfg, max_seqs, max_len, max_prefill_tokens, enc_cache)
    return int(_lib().rlt_arena_bytes(C.byref(c)))


def plan_ragged(steps):
    """Host-only scheduler plan: (order, tick sizes)."""
    st = _i32(steps)
    n = st.shape[0]
    order = np.zeros(max(n, 1), np.int32)
    tmax = int(st.max()) if n else 0
    sizes = np.zeros(max(tmax, 1), np.int32)
    nt = C.c_int(0)
    _check(_lib().rlt_plan_ragged(_p(st), n, _p(order), _p(sizes), max(tmax, 1), C.byref(nt)),
           "rlt_plan_ragged")
    return order[:n], sizes[: nt.value]


def attend_workspace_bytes(n: int, n_heads: int, head_dim: int, cap: int) -> int:
    return int(_lib().rlt_attend_workspace_bytes(n, n_heads, head_dim, cap))


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def attend(q, kv, lengths, out, workspace, stream=None):
    """rlt_attend: q [n][H][dh] fp32, kv [n][H][2][cap][dh] (bf16 or fp32),
    lengths (host ints) -> out [n][H][dh] (kv dtype). Torch tensors on the GPU."""
    import torch
    n, H, two, cap, dh = kv.shape
    assert two == 2 and q.shape == (n, H, dh) and out.shape == (n, H, dh)
    dtype = BF16 if kv.dtype == torch.bfloat16 else 0
    lens = _i32(lengths)
    _check(_lib().rlt_attend(C.c_void_p(q.data_ptr()), C.c_void_p(kv.data_ptr()), _p(lens), n, H,
                             dh, cap, dtype, C.c_void_p(out.data_ptr()),
                             C.c_void_p(workspace.data_ptr()), workspace.numel(),
                             _stream_handle(stream)), "rlt_attend")


class Model:
    """One RLT model bound to device weights and a device arena.

    ``weights`` maps the generator's tensor names to numpy float32 arrays (the
    bf16 values for bf16 models); they are uploaded once with torch.
    """

    def __init__(self, cfg: RLTConfig, weights: Dict[str, np.ndarray], max_seqs: int,
                 max_len: int, device: str = "cuda", max_prefill_tokens: int = 0,
                 stream=None, enc_cache: bool = False):
        import torch
        self.torch = torch
        self.cfg = cfg
        self.max_seqs, self.max_len = max_seqs, max_len
        self.device = torch.device(device)
        self.wdtype = torch.bfloat16 if cfg.dtype == BF16 else torch.float32
        self.stream = stream
        lib = _lib()
        self._c = make_config(cfg, max_seqs, max_len, max_prefill_tokens, enc_cache)
        self.enc_cache = bool(enc_cache)
        rc = lib.rlt_check_config(C.byref(self._c))
        _check(rc, "rlt_check_config")
        self.arena_bytes = int(lib.rlt_arena_bytes(C.byref(self._c)))
        self._dev = {}
        w = rlt_weights()

        def up(name, matrix=True):
            src = weights[name]
            key = id(src)
            if key not in self._dev:  # tied names share one device tensor
                t = torch.from_numpy(np.ascontiguousarray(src, dtype=np.float32))
                t = t.to(self.device)
                if matrix:
                    t = t.to(self.wdtype)
                self._dev[key] = t
            return self._dev[key].data_ptr()

        sw = cfg.ffn_kind == SWIGLU
        w.embed = up("embed")
        for l in range(cfg.n_enc):
            w.enc_ln1[l] = up(f"enc.{l}.ln1", False)
            w.enc_wqkv[l] = up(f"enc.{l}.wqkv")
            w.enc_wo[l] = up(f"enc.{l}.wo")
            w.enc_ln2[l] = up(f"enc.{l}.ln2", False)
            w.enc_w1[l] = up(f"enc.{l}.wa" if sw else f"enc.{l}.w1")
            if sw:
                w.enc_wb[l] = up(f"enc.{l}.wb")
            w.enc_w2[l] = up(f"enc.{l}.w2")
        w.enc_lnf = up("enc.lnf", False)
        for g in range(cfg.mem_groups):
            w.mem_wk[g] = up(f"mem.{g}.wk")
            w.mem_wv[g] = up(f"mem.{g}.wv")
        w.gate_w = up("gate.w")
        w.gate_b = up("gate.b", False)
        w.sstar = up("sstar", False)
        for l in range(cfg.n_dec):
            w.dec_ln1[l] = up(f"dec.{l}.ln1", False)
            w.dec_ln2[l] = up(f"dec.{l}.ln2", False)
            w.dec_ln3[l] = up(f"dec.{l}.ln3", False)
            w.dec_wqx[l] = up(f"dec.{l}.wqx")
            w.dec_wox[l] = up(f"dec.{l}.wox")
            if not cfg.tied:
                w.dec_wqkv[l] = up(f"dec.{l}.wqkv")
                w.dec_wo[l] = up(f"dec.{l}.wo")
                w.dec_w1[l] = up(f"dec.{l}.wa" if sw else f"dec.{l}.w1")
                if sw:
                    w.dec_wb[l] = up(f"dec.{l}.wb")
                w.dec_w2[l] = up(f"dec.{l}.w2")
        w.dec_lnf = up("dec.lnf", False)
        self._w = w
        self.arena = torch.empty(self.arena_bytes, dtype=torch.uint8, device=self.device)
        torch.cuda.synchronize(self.device)
        h = C.c_void_p()
        _check(lib.rlt_create(C.byref(self._c), C.byref(w), C.c_void_p(self.arena.data_ptr()),
                              self.arena_bytes, C.byref(h)), "rlt_create")
        self._h = h

    # ------------------------------------------------------------------
    def _st(self, stream=None):
        s = stream if stream is not None else self.stream
        if s is None:
            s = self.torch.cuda.current_stream(self.device)
        return C.c_void_p(s.cuda_stream)

    def close(self):
        if getattr(self, "_h", None):
            _lib().rlt_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- the C-ABI calls, same names ------------------------------------
    def reset_seq(self, seq: int, stream=None):
        _check(_lib().rlt_reset_seq(self._h, seq, self._st(stream)), "rlt_reset_seq")

    def prefill_encoder(self, tokens, seq_ids, offsets, lengths, stream=None):
        """tokens: torch int32 tensor (device or pinned host)."""
        ids, off, lens = _i32(seq_ids), _i32(offsets), _i32(lengths)
        self._tok_keep = tokens
        _check(_lib().rlt_prefill_encoder(self._h, C.c_void_p(tokens.data_ptr()), _p(ids),
                                          _p(off), _p(lens), ids.shape[0], self._st(stream)),
               "rlt_prefill_encoder")

    def decoder_step(self, ready_ids, stream=None):
        ids = _i32(ready_ids)
        _check(_lib().rlt_decoder_step(self._h, _p(ids), ids.shape[0], self._st(stream)),
               "rlt_decoder_step")

    def run_sequence(self, seq_ids, n_steps: int, stream=None):
        ids = _i32(seq_ids)
        _check(_lib().rlt_run_sequence(self._h, _p(ids), ids.shape[0], int(n_steps),
                                       self._st(stream)), "rlt_run_sequence")

    def decoder_parallel(self, seq_ids, n_steps: int, s_all=None, stream=None):
        """Token-parallel decoder pass of fresh sequences (alpha = 0 models);
        s_all: optional fp32 device tensor [n][n_steps][d] for every s_t."""
        ids = _i32(seq_ids)
        ptr = None
        if s_all is not None:
            assert s_all.is_cuda and s_all.dtype == self.torch.float32 and s_all.is_contiguous()
            assert tuple(s_all.shape) == (ids.shape[0], int(n_steps), self.cfg.d)
            ptr = C.c_void_p(s_all.data_ptr())
        _check(_lib().rlt_decoder_parallel(self._h, _p(ids), ids.shape[0], int(n_steps), ptr,
                                           self._st(stream)), "rlt_decoder_parallel")

    def grad_shapes(self) -> Dict[str, tuple]:
        """Name (the weight generator's) -> shape of every gradient rlt_backward
        accumulates."""
        c = self.cfg
        d, F = c.d, c.ffn_dim
        sw = c.ffn_kind == SWIGLU
        out = {"gate.w": (d, 2 * d), "gate.b": (d,), "sstar": (d,), "dec.lnf": (d,)}
        for l in range(c.n_dec):
            out[f"dec.{l}.ln1"] = (d,)
            out[f"dec.{l}.wqkv"] = (3 * d, d)
            out[f"dec.{l}.wo"] = (d, d)
            out[f"dec.{l}.ln2"] = (d,)
            out[f"dec.{l}.wqx"] = (d, d)
            out[f"dec.{l}.wox"] = (d, d)
            out[f"dec.{l}.ln3"] = (d,)
            out[f"dec.{l}.wa" if sw else f"dec.{l}.w1"] = (F, d)
            if sw:
                out[f"dec.{l}.wb"] = (F, d)
            out[f"dec.{l}.w2"] = (d, F)
        for g in range(c.mem_groups):
            out[f"mem.{g}.wk"] = (d, d)
            out[f"mem.{g}.wv"] = (d, d)
        return out

    def carry_floats(self) -> int:
        c = self.cfg
        return c.d * (1 + 2 * c.n_dec * (c.window - 1))

    def backward_workspace_bytes(self, n: int, n_steps: int) -> int:
        return int(_lib().rlt_backward_workspace_bytes(C.byref(self._c), int(n), int(n_steps)))

    def backward(self, seq_ids, sgrad, grads=None, egrad=None, carry_in=None, carry_out=True,
                 workspace=None, stream=None):
        """Backpropagation through time over the next sgrad.shape[1] positions of
        the listed sequences (rlt_backward): runs their forward, then the
        reverse traversal. sgrad: fp32 device [n][n_steps][d] = dL/ds_t.
        grads (name -> fp32 device tensor, accumulated) and egrad ([n][max_len][d],
        accumulated) are allocated zeroed when None. Returns (grads, egrad,
        carry_out or None)."""
        torch = self.torch
        ids = _i32(seq_ids)
        n, n_steps = ids.shape[0], int(sgrad.shape[1])
        c = self.cfg
        assert sgrad.is_cuda and sgrad.dtype == torch.float32 and sgrad.is_contiguous()
        assert tuple(sgrad.shape) == (n, n_steps, c.d)
        dev = self.device
        if grads is None:
            grads = {k: torch.zeros(v, dtype=torch.float32, device=dev)
                     for k, v in self.grad_shapes().items()}
        if egrad is None:
            egrad = torch.zeros((n, self.max_len, c.d), dtype=torch.float32, device=dev)
        g = rlt_grads()
        sw = c.ffn_kind == SWIGLU
        for k, fld in (("gate.w", "gate_w"), ("gate.b", "gate_b"), ("sstar", "sstar"),
                       ("dec.lnf", "dec_lnf")):
            setattr(g, fld, grads[k].data_ptr())
        for l in range(c.n_dec):
            for k, fld in (("ln1", "dec_ln1"), ("wqkv", "dec_wqkv"), ("wo", "dec_wo"),
                           ("ln2", "dec_ln2"), ("wqx", "dec_wqx"), ("wox", "dec_wox"),
                           ("ln3", "dec_ln3"), ("wa" if sw else "w1", "dec_w1"),
                           ("w2", "dec_w2")):
                getattr(g, fld)[l] = grads[f"dec.{l}.{k}"].data_ptr()
            if sw:
                g.dec_wb[l] = grads[f"dec.{l}.wb"].data_ptr()
        for q in range(c.mem_groups):
            g.mem_wk[q] = grads[f"mem.{q}.wk"].data_ptr()
            g.mem_wv[q] = grads[f"mem.{q}.wv"].data_ptr()
        cin = None
        if carry_in is not None:
            assert tuple(carry_in.shape) == (n, self.carry_floats())
            assert carry_in.dtype == torch.float32 and carry_in.is_contiguous()
            cin = C.c_void_p(carry_in.data_ptr())
        cout = None
        if carry_out:
            cout_t = torch.empty((n, self.carry_floats()), dtype=torch.float32, device=dev)
            cout = C.c_void_p(cout_t.data_ptr())
        if workspace is None:
            workspace = torch.empty(self.backward_workspace_bytes(n, n_steps),
                                    dtype=torch.uint8, device=dev)
        _check(_lib().rlt_backward(self._h, _p(ids), n, n_steps, C.c_void_p(sgrad.data_ptr()),
                                   cin, cout, C.c_void_p(egrad.data_ptr()), C.byref(g),
                                   C.c_void_p(workspace.data_ptr()), workspace.numel(),
                                   self._st(stream)), "rlt_backward")
        self._bw_keep = (workspace, grads, egrad, carry_in)
        return grads, egrad, (cout_t if carry_out else None)

    def run_ragged(self, seq_ids, steps, stream=None):
        ids, st = _i32(seq_ids), _i32(steps)
        _check(_lib().rlt_run_ragged(self._h, _p(ids), _p(st), ids.shape[0], self._st(stream)),
               "rlt_run_ragged")

    def get_state(self, seq: int, stream=None):
        """(s [d] float32, cache [L_D][2][W-1][d] model dtype, t) as device tensors."""
        torch = self.torch
        c = self.cfg
        s = torch.empty(c.d, dtype=torch.float32, device=self.device)
        cache = torch.zeros((c.n_dec, 2, max(c.window - 1, 0), c.d), dtype=self.wdtype,
                            device=self.device)
        t = C.c_int64(0)
        _check(_lib().rlt_get_state(self._h, seq, C.c_void_p(s.data_ptr()),
                                    C.c_void_p(cache.data_ptr()) if cache.numel() else None,
                                    C.byref(t), self._st(stream)), "rlt_get_state")
        return s, cache, int(t.value)

    def set_state(self, seq: int, s, cache, t: int, stream=None):
        self._set_keep = (s, cache)
        _check(_lib().rlt_set_state(self._h, seq,
                                    C.c_void_p(s.data_ptr()) if s is not None else None,
                                    C.c_void_p(cache.data_ptr()) if cache is not None and cache.numel() else None,
                                    int(t), self._st(stream)), "rlt_set_state")

    def get_encoder_output(self, seq: int, stream=None):
        """(e [t_enc][d], mem [G][t_enc][2][d]) device tensors in the model dtype."""
        torch = self.torch
        c = self.cfg
        t = C.c_int64(0)
        _check(_lib().rlt_get_encoder_output(self._h, seq, None, None, C.byref(t),
                                             self._st(stream)), "rlt_get_encoder_output")
        te = int(t.value)
        e = torch.empty((te, c.d), dtype=self.wdtype, device=self.device)
        mem = torch.empty((c.mem_groups, te, 2, c.d), dtype=self.wdtype, device=self.device)
        if te:
            _check(_lib().rlt_get_encoder_output(self._h, seq, C.c_void_p(e.data_ptr()),
                                                 C.c_void_p(mem.data_ptr()), C.byref(t),
                                                 self._st(stream)), "rlt_get_encoder_output")
        return e, mem

    # -- serving loop ---------------------------------------------------
    def append_encoder(self, tokens, seq_ids, stream=None):
        """tokens: int32 tensor [n] (device or pinned host), one per id."""
        ids = _i32(seq_ids)
        self._tok_keep = tokens
        _check(_lib().rlt_append_encoder(self._h, C.c_void_p(tokens.data_ptr()), _p(ids),
                                         ids.shape[0], self._st(stream)), "rlt_append_encoder")

    def lm_head(self, seq_ids, logits=None, stream=None):
        """Logits [n][V] (fp32 device tensor) from each sequence's s_t."""
        ids = _i32(seq_ids)
        if logits is None:
            logits = self.torch.empty((ids.shape[0], self.cfg.vocab), dtype=self.torch.float32,
                                      device=self.device)
        _check(_lib().rlt_lm_head(self._h, _p(ids), ids.shape[0],
                                  C.c_void_p(logits.data_ptr()), self._st(stream)), "rlt_lm_head")
        return logits

    def sample(self, logits, temperature: float, uniforms=None, out=None, stream=None):
        n = logits.shape[0]
        if out is None:
            out = self.torch.empty(n, dtype=self.torch.int32, device=self.device)
        up = C.c_void_p(uniforms.data_ptr()) if uniforms is not None else None
        _check(_lib().rlt_sample(self._h, C.c_void_p(logits.data_ptr()), n, float(temperature),
                                 up, C.c_void_p(out.data_ptr()), self._st(stream)), "rlt_sample")
        return out

    def serve_step(self, seq_ids, temperature: float, uniforms=None, logits=None, out=None,
                   stream=None):
        """One autoregressive step; returns (tokens int32 [n], logits [n][V])."""
        ids = _i32(seq_ids)
        n = ids.shape[0]
        torch = self.torch
        if logits is None:
            logits = torch.empty((n, self.cfg.vocab), dtype=torch.float32, device=self.device)
        if out is None:
            out = torch.empty(n, dtype=torch.int32, device=self.device)
        self._serve_keep = (uniforms, logits, out)
        up = C.c_void_p(uniforms.data_ptr()) if uniforms is not None else None
        _check(_lib().rlt_serve_step(self._h, _p(ids), n, float(temperature), up,
                                     C.c_void_p(logits.data_ptr()), C.c_void_p(out.data_ptr()),
                                     self._st(stream)), "rlt_serve_step")
        return out, logits

    # -- exact prefix snapshots ------------------------------------------
    def snapshot_bytes(self, seq: int) -> int:
        return int(_lib().rlt_snapshot_bytes(self._h, seq))

    def get_snapshot(self, seq: int, out=None, stream=None):
        """Slot `seq`'s snapshot into `out` (uint8 tensor on the device or in
        pinned host memory; allocated on the device if None); returns it."""
        n = self.snapshot_bytes(seq)
        if out is None:
            out = self.torch.empty(n, dtype=self.torch.uint8, device=self.device)
        _check(_lib().rlt_get_snapshot(self._h, seq, C.c_void_p(out.data_ptr()), out.numel(),
                                       self._st(stream)), "rlt_get_snapshot")
        return out

    def set_snapshot(self, seq: int, buf, stream=None):
        self._snap_keep = buf
        _check(_lib().rlt_set_snapshot(self._h, seq, C.c_void_p(buf.data_ptr()), buf.numel(),
                                       self._st(stream)), "rlt_set_snapshot")

    def fingerprint(self) -> int:
        v = C.c_uint64(0)
        _check(_lib().rlt_model_fingerprint(self._h, C.byref(v)), "rlt_model_fingerprint")
        return int(v.value)

    def profile(self, stride: int):
        """stride k > 0: profile every k-th decoder step (and every prefill); 0: off."""
        _check(_lib().rlt_profile(self._h, int(stride)), "rlt_profile")

    def get_stats(self) -> dict:
        st = rlt_stats()
        _check(_lib().rlt_get_stats(self._h, C.byref(st)), "rlt_get_stats")
        out = {"launches": int(st.launches)}
        for k, name in enumerate(K_NAMES):
            out[name] = {"launches": int(st.kernel_launches[k]), "ms": float(st.kernel_ms[k]),
                         "bytes": float(st.kernel_bytes[k]), "flops": float(st.kernel_flops[k])}
        return out

    def set_step_kernel(self, kind: int):
        """STEP_FUSED (one persistent launch per step) or STEP_CHAIN."""
        _check(_lib().rlt_set_step_kernel(self._h, int(kind)), "rlt_set_step_kernel")

    def get_step_kernel(self) -> int:
        return int(_lib().rlt_get_step_kernel(self._h))

    def step_kernel_ctas(self) -> int:
        return int(_lib().rlt_step_kernel_ctas(self._h))

    def set_step_trace(self, buf):
        """buf: int64 device tensor [ctas][cap][4] (None: off); see rlt_set_step_trace."""
        self._trace_keep = buf
        ptr = C.c_void_p(buf.data_ptr()) if buf is not None else None
        nbytes = buf.numel() * buf.element_size() if buf is not None else 0
        _check(_lib().rlt_set_step_trace(self._h, ptr, nbytes), "rlt_set_step_trace")

    def set_fault(self, fault: int, wait_limit_ns: int = 0):
        """Plant a fault (FAULT_*) in later decoder-attention launches and
        bound their device waits (0 = default); FAULT_NONE clears it."""
        _check(_lib().rlt_set_fault(self._h, int(fault), int(wait_limit_ns)), "rlt_set_fault")

    def poll_device_error(self) -> int:
        return int(_lib().rlt_poll_device_error(self._h))
