"""ctypes binding of librssm (include/rssm.h): argument marshalling only.

The module-level functions carry the C names and signatures; ``Layer`` is a
convenience owner of one handle whose workspace and outputs are torch CUDA
tensors, passing raw device pointers and ``torch.cuda.current_stream()``.
Every step of the decode path runs in librssm's kernels; there is no fallback:
loading fails loudly when the library is missing, and calls fail when no CUDA
device is present.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librssm.so")

RSSM_OK, RSSM_EINVAL, RSSM_ESTATE, RSSM_ECUDA, RSSM_EDEVICE = range(5)
RSSM_MAMBA2, RSSM_GDN, RSSM_KDA = 0, 1, 2
RSSM_REPLAY, RSSM_EAGER = 0, 1
RSSM_F32, RSSM_BF16, RSSM_FP8E4M3 = 0, 1, 2
RSSM_DEV_BAD_ACCEPT, RSSM_DEV_BAD_COUNTERS, RSSM_DEV_PIPE_TIMEOUT = 1, 2, 3
DTYPES = {"f32": RSSM_F32, "bf16": RSSM_BF16, "fp8": RSSM_FP8E4M3}
KINDS = {"mamba2": RSSM_MAMBA2, "gdn": RSSM_GDN, "kda": RSSM_KDA}
MODES = {"replay": RSSM_REPLAY, "eager": RSSM_EAGER}


class rssm_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "kind", "mode", "state_dtype", "input_dtype", "batch", "nheads", "headdim", "dstate",
        "ngroups", "window", "max_draft", "dt_scales_input")]


class rssm_workspace_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "error_off", "seq_pos_off", "ckpt_pos_off", "pending_off", "flush_count_off", "arrive_off",
        "A_off", "D_off", "ckpt_off", "ckpt_bytes", "rc_off", "rc_bytes", "rc_scale_off",
        "rc_scale_bytes", "ring", "ring_stride", "xbuf_off", "xbuf_bytes", "bbuf_off", "bbuf_bytes", "sbuf_off",
        "sbuf_bytes", "tbuf_off", "tbuf_bytes", "snap_off", "snap_bytes", "tq_max", "seqinfo_off",
        "seqinfo_bytes", "dec_off", "dec_bytes", "coef_off", "coef_bytes", "query_off", "query_bytes",
        "total_bytes")]


class rssm_inputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("x", "dt", "Bm", "Cm", "q", "k", "v", "alpha", "beta")]


class rssm_prefill_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "nheads", "headdim", "dstate", "ngroups", "T", "dt_scales_input")]


# C declarations: name -> (restype, argtypes)
_VP, _I32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_CFGP, _LAYP, _INP = ctypes.POINTER(rssm_config), ctypes.POINTER(rssm_workspace_layout), ctypes.POINTER(rssm_inputs)
_PCFGP = ctypes.POINTER(rssm_prefill_config)
SIGNATURES = {
    "rssm_workspace_bytes": (_SZ, [_CFGP]),
    "rssm_workspace_layout_of": (ctypes.c_int, [_CFGP, _LAYP]),
    "rssm_create": (ctypes.c_int, [_CFGP, _VP, _SZ, _VP, ctypes.POINTER(_VP)]),
    "rssm_destroy": (ctypes.c_int, [_VP]),
    "rssm_set_stream": (ctypes.c_int, [_VP, _VP]),
    "rssm_set_params": (ctypes.c_int, [_VP, _VP, _VP]),
    "rssm_import_state": (ctypes.c_int, [_VP, _VP]),
    "rssm_export_state": (ctypes.c_int, [_VP, _VP]),
    "rssm_decode": (ctypes.c_int, [_VP, _INP, _VP]),
    "rssm_decode_static_scratch": (ctypes.c_int, [_VP, _INP, _VP]),
    "rssm_verify": (ctypes.c_int, [_VP, _I32, _INP, _VP]),
    "rssm_commit": (ctypes.c_int, [_VP, _VP]),
    "rssm_flush": (ctypes.c_int, [_VP]),
    "rssm_read_counters": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP]),
    "rssm_status_word": (ctypes.c_int, [_VP, _VP]),
    "rssm_clear_status": (ctypes.c_int, [_VP]),
    "rssm_set_split_event": (ctypes.c_int, [_VP, _VP]),
    "rssm_launch_count": (ctypes.c_int64, [_VP]),
    "rssm_last_error": (ctypes.c_char_p, [_VP]),
    "rssm_mamba2_prefill": (ctypes.c_int, [_PCFGP, _VP, _VP, _VP, _INP, _VP, _VP, _VP, _VP]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librssm.so (built by checkpoint_input_replay_rssm_b200.build); no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"librssm.so not found at {path}: build it with "
                               "`python -m checkpoint_input_replay_rssm_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


class RssmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"rssm status {status}: {msg}")
        self.status = status


def _check(st: int, h=None):
    if st != RSSM_OK:
        msg = load().rssm_last_error(h)
        raise RssmError(st, msg.decode() if msg else "")


def make_config(kind="mamba2", mode="replay", state_dtype="bf16", input_dtype="bf16", batch=1,
                nheads=1, headdim=64, dstate=128, ngroups=1, window=16, max_draft=1,
                dt_scales_input=False) -> rssm_config:
    return rssm_config(KINDS[kind], MODES[mode], DTYPES[state_dtype], DTYPES[input_dtype], batch,
                       nheads, headdim, dstate, ngroups if kind == "mamba2" else nheads, window,
                       max_draft, int(bool(dt_scales_input)))


# ---------------------------------------------------------------- C names
def rssm_workspace_bytes(cfg: rssm_config) -> int:
    return int(load().rssm_workspace_bytes(ctypes.byref(cfg)))


def rssm_workspace_layout_of(cfg: rssm_config) -> rssm_workspace_layout:
    lay = rssm_workspace_layout()
    _check(load().rssm_workspace_layout_of(ctypes.byref(cfg), ctypes.byref(lay)))
    return lay


def rssm_create(cfg: rssm_config, workspace_ptr: int, nbytes: int, stream_ptr: int):
    h = _VP()
    _check(load().rssm_create(ctypes.byref(cfg), workspace_ptr, nbytes, stream_ptr, ctypes.byref(h)))
    return h


def rssm_destroy(h):
    _check(load().rssm_destroy(h))


def rssm_set_stream(h, stream_ptr: int):
    _check(load().rssm_set_stream(h, stream_ptr), h)


def rssm_set_params(h, A_ptr: int, D_ptr: int):
    _check(load().rssm_set_params(h, A_ptr, D_ptr), h)


def rssm_import_state(h, S_ptr: int):
    _check(load().rssm_import_state(h, S_ptr), h)


def rssm_export_state(h, S_ptr: int):
    _check(load().rssm_export_state(h, S_ptr), h)


def rssm_decode(h, inputs: rssm_inputs, y_ptr: int):
    _check(load().rssm_decode(h, ctypes.byref(inputs), y_ptr), h)


def rssm_decode_static_scratch(h, inputs: rssm_inputs, y_ptr: int):
    _check(load().rssm_decode_static_scratch(h, ctypes.byref(inputs), y_ptr), h)


def rssm_verify(h, K: int, inputs: rssm_inputs, y_ptr: int):
    _check(load().rssm_verify(h, K, ctypes.byref(inputs), y_ptr), h)


def rssm_commit(h, accept_ptr: int):
    _check(load().rssm_commit(h, accept_ptr), h)


def rssm_flush(h):
    _check(load().rssm_flush(h), h)


def rssm_read_counters(h, seq_pos, ckpt_pos, pending, flush_count):
    """Host numpy arrays (int64, int64, int32, int32) of length batch, filled in place."""
    p = lambda a: None if a is None else a.ctypes.data_as(_VP)
    _check(load().rssm_read_counters(h, p(seq_pos), p(ckpt_pos), p(pending), p(flush_count)), h)


def rssm_status_word(h):
    """Returns (status, [code, sequence, head, value])."""
    info = (ctypes.c_int32 * 4)()
    st = load().rssm_status_word(h, ctypes.cast(info, _VP))
    return st, list(info)


def rssm_clear_status(h):
    _check(load().rssm_clear_status(h), h)


def rssm_set_split_event(h, event_ptr):
    _check(load().rssm_set_split_event(h, event_ptr), h)


def rssm_launch_count(h) -> int:
    return int(load().rssm_launch_count(h))


def rssm_last_error(h=None) -> str:
    m = load().rssm_last_error(h)
    return m.decode() if m else ""


def rssm_mamba2_prefill(cfg: rssm_prefill_config, A_ptr: int, D_ptr: int, S0_ptr, inputs: rssm_inputs,
                        y_ptr: int, S_out_ptr: int, err_ptr, stream_ptr):
    st = load().rssm_mamba2_prefill(ctypes.byref(cfg), A_ptr, D_ptr, S0_ptr, ctypes.byref(inputs), y_ptr,
                                    S_out_ptr, err_ptr, stream_ptr)
    if st != RSSM_OK:
        raise RssmError(st, "rssm_mamba2_prefill refused its arguments" if st == RSSM_EINVAL
                        else "rssm_mamba2_prefill launch failed")


def prefill(x, dt, Bm, Cm, A, D, S0=None, dt_scales_input=False, y=None, S_out=None, err=None, stream=None):
    """Torch convenience over rssm_mamba2_prefill: x [B,T,H,P] bf16, dt [B,T,H] fp32,
    Bm/Cm [B,T,G,N] bf16, A/D [H] fp32, S0 [B,H,P,N] fp32 or None.  Returns (y, S_out)."""
    import torch

    Bn, T, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    for t, dty in ((x, torch.bfloat16), (Bm, torch.bfloat16), (Cm, torch.bfloat16), (dt, torch.float32),
                   (A, torch.float32), (D, torch.float32)):
        assert t.is_cuda and t.is_contiguous() and t.dtype == dty
    y = y if y is not None else torch.empty((Bn, T, H, P), dtype=torch.float32, device=x.device)
    S_out = S_out if S_out is not None else torch.empty((Bn, H, P, N), dtype=torch.float32, device=x.device)
    cfg = rssm_prefill_config(Bn, H, P, N, G, T, int(bool(dt_scales_input)))
    ins = rssm_inputs(x=x.data_ptr(), dt=dt.data_ptr(), Bm=Bm.data_ptr(), Cm=Cm.data_ptr())
    st = stream if stream is not None else torch.cuda.current_stream(x.device)
    rssm_mamba2_prefill(cfg, A.data_ptr(), D.data_ptr(), None if S0 is None else S0.data_ptr(), ins,
                        y.data_ptr(), S_out.data_ptr(), None if err is None else err.data_ptr(), st.cuda_stream)
    return y, S_out


# ---------------------------------------------------------------- torch owner
class Layer:
    """One SSM layer's decode state on the current CUDA device.

    The workspace is a torch uint8 CUDA tensor owned here; inputs are torch CUDA
    tensors in the configured dtypes (x/B/C or q/k/v in ``input_dtype``; dt,
    alpha, beta fp32), laid out [B, T, ...] as include/rssm.h states.
    """

    def __init__(self, cfg: rssm_config, device=None, stream=None):
        import torch

        if not torch.cuda.is_available():
            raise RuntimeError("librssm needs a CUDA device; none is visible")
        self.torch = torch
        self.cfg = cfg
        self.device = torch.device(device or "cuda")
        self.layout = rssm_workspace_layout_of(cfg)
        self.nbytes = int(self.layout.total_bytes)
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(self.nbytes, dtype=torch.uint8, device=self.device)
            self.stream = stream or torch.cuda.current_stream(self.device)
            self.h = rssm_create(cfg, self.workspace.data_ptr(), self.nbytes, self.stream.cuda_stream)
        self.B, self.H, self.P, self.N = cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate
        self.T_last = 0

    def close(self):
        if getattr(self, "h", None):
            rssm_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- marshalling helpers
    def _ptr(self, t, dtype=None):
        if t is None:
            return None
        assert t.is_cuda and t.is_contiguous(), "inputs must be contiguous CUDA tensors"
        if dtype is not None:
            assert t.dtype == dtype, f"expected {dtype}, got {t.dtype}"
        return t.data_ptr()

    def _inputs(self, d: dict) -> rssm_inputs:
        torch = self.torch
        wide = torch.bfloat16 if self.cfg.input_dtype == RSSM_BF16 else torch.float32
        f32 = torch.float32
        spec = {"x": wide, "dt": f32, "B": wide, "C": wide, "q": wide, "k": wide, "v": wide,
                "alpha": f32, "beta": f32}
        cname = {"B": "Bm", "C": "Cm"}
        kw = {cname.get(k, k): self._ptr(v, spec[k]) for k, v in d.items()}
        return rssm_inputs(**kw)

    def set_params(self, A, D):
        rssm_set_params(self.h, self._ptr(A, self.torch.float32), self._ptr(D, self.torch.float32))

    def import_state(self, S):
        rssm_import_state(self.h, self._ptr(S, self.torch.float32))

    def export_state(self, out=None):
        out = out if out is not None else self.torch.empty((self.B, self.H, self.P, self.N),
                                                           dtype=self.torch.float32, device=self.device)
        rssm_export_state(self.h, self._ptr(out))
        return out

    def decode(self, inputs: dict, y=None):
        y = y if y is not None else self.torch.empty((self.B, 1, self.H, self.P),
                                                     dtype=self.torch.float32, device=self.device)
        rssm_decode(self.h, self._inputs(inputs), self._ptr(y))
        return y

    def decode_static_scratch(self, inputs: dict, y=None):
        y = y if y is not None else self.torch.empty((self.B, 1, self.H, self.P),
                                                     dtype=self.torch.float32, device=self.device)
        rssm_decode_static_scratch(self.h, self._inputs(inputs), self._ptr(y))
        return y

    def verify(self, K: int, inputs: dict, y=None):
        y = y if y is not None else self.torch.empty((self.B, K, self.H, self.P),
                                                     dtype=self.torch.float32, device=self.device)
        rssm_verify(self.h, K, self._inputs(inputs), self._ptr(y))
        return y

    def commit(self, accept_len):
        rssm_commit(self.h, self._ptr(accept_len, self.torch.int32))

    def flush(self):
        rssm_flush(self.h)

    def counters(self):
        import numpy as np

        sp = np.zeros(self.B, np.int64)
        ck = np.zeros(self.B, np.int64)
        pe = np.zeros(self.B, np.int32)
        fc = np.zeros(self.B, np.int32)
        rssm_read_counters(self.h, sp, ck, pe, fc)
        return sp, ck, pe, fc

    def status(self):
        return rssm_status_word(self.h)

    def clear_status(self):
        rssm_clear_status(self.h)

    def launches(self) -> int:
        return rssm_launch_count(self.h)

    def region(self, off_name: str, bytes_name: str, dtype):
        """A torch view of one workspace region (for inspection in tests)."""
        off = getattr(self.layout, off_name)
        n = getattr(self.layout, bytes_name)
        return self.workspace[off:off + n].view(dtype)
