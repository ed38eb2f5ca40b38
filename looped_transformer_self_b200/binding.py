"""ctypes binding of liblooped_spec.so (argument marshalling only).

Every call goes to the CUDA library; there is no other implementation.  If
the shared library is missing, the import fails loudly.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblooped_spec.so")

LT_F32, LT_BF16 = 0, 1
ERRORS = {-1: "LT_ERR_ARG", -2: "LT_ERR_SHAPE", -3: "LT_ERR_CAPACITY", -4: "LT_ERR_CUDA",
          -5: "LT_ERR_DEVICE_CHECK", -6: "LT_ERR_STATE"}


class LoopedSpecError(RuntimeError):
    def __init__(self, code, msg=""):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run __graft_entry__.build() "
                              "(or python looped_transformer_self_b200/build.py)")
        _lib = ctypes.CDLL(LIB_PATH)
        _declare(_lib)
    return _lib


_vp, _sz, _i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int


class ModelConfigC(ctypes.Structure):
    _fields_ = [("dtype", _i), ("d_model", _i), ("n_heads", _i), ("head_dim", _i), ("ffn", _i),
                ("vocab", _i), ("n_prelude", _i), ("n_core", _i), ("n_coda", _i), ("R", _i),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("resid_scale", ctypes.c_float)]


class DecodeConfigC(ctypes.Structure):
    _fields_ = [("d1", _i), ("d2", _i), ("temperature", ctypes.c_float),
                ("top_p", ctypes.c_float), ("seed", ctypes.c_uint64), ("max_branches", _i),
                ("max_ctx", _i), ("max_new", _i), ("second_mode", _i), ("trace_steps", _i),
                ("copy_k", _i), ("copy_max_len", _i), ("copy_match_cap", _i),
                ("copy_reserve", _i), ("copy_tau", ctypes.c_float)]


class StatsC(ctypes.Structure):
    _fields_ = [(n, _i) for n in ("steps", "rows_sum", "rows_max", "n_first", "n_second",
                                   "n_fallback", "gate_checks", "gate_opens", "branches_created",
                                   "resid_fallback", "committed_len", "copy_chains",
                                   "copy_rows", "copy_cut", "n_copy")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


class StepInfoC(ctypes.Structure):
    _fields_ = [(n, _i) for n in ("step", "rows", "n_committed", "n_first", "n_second",
                                   "n_fallback", "n_copy", "gate_checks", "gate_opens",
                                   "branches_created", "committed_len", "finished")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


class ProfileC(ctypes.Structure):
    _fields_ = [("steps", _i), ("rows", _i), ("step_ms", ctypes.c_double),
                ("gemm_core_ms", ctypes.c_double), ("gemm_core_bytes", ctypes.c_double),
                ("gemm_core_launches", _i), ("gemm_other_ms", ctypes.c_double),
                ("gemm_other_launches", _i), ("gemm_other_bytes", ctypes.c_double),
                ("attn_ms", ctypes.c_double),
                ("attn_launches", _i), ("kv_bytes", ctypes.c_double),
                ("weight_bytes_core", ctypes.c_double)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


class InfoC(ctypes.Structure):
    _fields_ = [("kernels_per_step", _i), ("gemm_grid", _i), ("n_tags", _i), ("kv_slots", _i),
                ("workspace_bytes", ctypes.c_double), ("weight_bytes_core", ctypes.c_double),
                ("weight_bytes_prelude_coda", ctypes.c_double),
                ("weight_bytes_head", ctypes.c_double)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_ip = ctypes.POINTER(ctypes.c_int32)


def _declare(L):
    L.lt_gemm_scratch_bytes.argtypes = [_i, _i, _i, _i, ctypes.POINTER(_sz)]
    L.lt_gemm_rows.argtypes = [_i, _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]
    L.lt_gemm_rows_noalloc.argtypes = [_i, _vp, _vp, _vp, _i, _i, _i, _vp]
    L.lt_selftest_wait.argtypes = [_ip, _vp]
    L.lt_readout_tv.argtypes = [_vp, ctypes.c_longlong, _vp, ctypes.c_longlong, _i, _i,
                                ctypes.c_float, ctypes.c_float, _vp, _vp]
    L.lt_workspace_bytes.argtypes = [ctypes.POINTER(ModelConfigC), ctypes.POINTER(DecodeConfigC),
                                     ctypes.POINTER(_sz)]
    L.lt_create.argtypes = [ctypes.POINTER(ModelConfigC), ctypes.POINTER(DecodeConfigC), _vp, _sz,
                            _vp, ctypes.POINTER(_vp)]
    L.lt_load_weights.argtypes = [_vp, _vp, _vp, _vp, ctypes.POINTER(_vp)]
    L.lt_prefill.argtypes = [_vp, _ip, _i, _ip, _ip, _vp]
    L.lt_generate.argtypes = [_vp, _i, _i, _ip, ctypes.POINTER(StatsC)]
    L.lt_decode_step.argtypes = [_vp, _i, _ip, ctypes.POINTER(_i), ctypes.POINTER(StepInfoC)]
    L.lt_get_stats.argtypes = [_vp, ctypes.POINTER(StatsC)]
    L.lt_copy_screen_scores.argtypes = [_vp, _i, _i, _i, _vp, ctypes.c_longlong, _vp,
                                        ctypes.c_longlong, _i, ctypes.c_float, ctypes.c_float,
                                        _vp, _vp, _vp, _vp]
    L.lt_read_log.argtypes = [_vp, _ip, _ip, _ip, _i]
    L.lt_read_trace.argtypes = [_vp, _ip, _i]
    L.lt_read_committed.argtypes = [_vp, _ip, _ip, ctypes.POINTER(_i)]
    L.lt_read_branch_table.argtypes = [_vp, _ip]
    L.lt_read_readouts.argtypes = [_vp, _vp, _vp, _ip, _ip]
    L.lt_block_pass.argtypes = [_vp, _i, _ip, _ip, _vp, _ip, _vp, _i, ctypes.POINTER(ctypes.c_float)]
    L.lt_kv_pool.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_sz), ctypes.POINTER(_i),
                             ctypes.POINTER(_i), ctypes.POINTER(_i)]
    L.lt_rollback_branch.argtypes = [_vp, ctypes.c_int32]
    L.lt_commit_branch.argtypes = [_vp, ctypes.c_int32]
    L.lt_profile_steps.argtypes = [_vp, _i, _i, ctypes.POINTER(ProfileC)]
    L.lt_profile_gemms.argtypes = [_vp, _i, ctypes.POINTER(ctypes.c_double)]
    L.lt_get_info.argtypes = [_vp, ctypes.POINTER(InfoC)]
    L.lt_reset.argtypes = [_vp]
    L.lt_last_error.argtypes = [_vp]
    L.lt_last_error.restype = ctypes.c_char_p
    L.lt_destroy.argtypes = [_vp]
    L.lt_destroy.restype = None


def check(code: int, what: str = "") -> None:
    if code != 0:
        raise LoopedSpecError(code, what)


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def gemm_rows(w: torch.Tensor, x: torch.Tensor, scratch: torch.Tensor = None,
              stream=None) -> torch.Tensor:
    """Y[i][n] = sum_k x[i][k] w[n][k] through lt_gemm_rows (fp32 result)."""
    assert w.is_cuda and x.is_cuda and w.dtype == x.dtype
    dtype = LT_BF16 if w.dtype == torch.bfloat16 else LT_F32
    n_out, k = w.shape
    ncols = x.shape[0]
    need = _sz()
    check(lib().lt_gemm_scratch_bytes(dtype, n_out, k, ncols, ctypes.byref(need)))
    if scratch is None or scratch.numel() < need.value:
        scratch = torch.empty(need.value, dtype=torch.uint8, device=w.device)
    y = torch.empty(ncols, n_out, dtype=torch.float32, device=w.device)
    check(lib().lt_gemm_rows(dtype, _ptr(w), _ptr(x), _ptr(y), n_out, k, ncols, _ptr(scratch),
                             scratch.numel(), _stream(stream)), "lt_gemm_rows")
    return y


def gemm_rows_noalloc(w: torch.Tensor, x: torch.Tensor, stream=None) -> torch.Tensor:
    """Y[i][n] = sum_k x[i][k] w[n][k] through lt_gemm_rows_noalloc: bf16 only,
    scratch in the library's static device array (no allocation by the call)."""
    assert w.is_cuda and x.is_cuda and w.dtype == x.dtype == torch.bfloat16
    n_out, k = w.shape
    ncols = x.shape[0]
    y = torch.empty(ncols, n_out, dtype=torch.float32, device=w.device)
    check(lib().lt_gemm_rows_noalloc(LT_BF16, _ptr(w), _ptr(x), _ptr(y), n_out, k, ncols,
                                     _stream(stream)), "lt_gemm_rows_noalloc")
    return y


def readout_tv(za: torch.Tensor, zb: torch.Tensor, temperature: float, top_p: float,
               stream=None) -> torch.Tensor:
    """Per-row total variation between the readout distributions of two fp32
    logit matrices [n][V] (row stride free, unit column stride) through
    lt_readout_tv.  With temperature > 0 both inputs are overwritten with the
    processed distributions."""
    assert za.is_cuda and zb.is_cuda and za.dtype == zb.dtype == torch.float32
    assert za.dim() == zb.dim() == 2 and za.shape == zb.shape
    assert za.stride(1) == 1 and zb.stride(1) == 1
    n, V = za.shape
    tv = torch.empty(n, dtype=torch.float32, device=za.device)
    check(lib().lt_readout_tv(_ptr(za), za.stride(0), _ptr(zb), zb.stride(0), n, V,
                              float(temperature), float(top_p), _ptr(tv), _stream(stream)),
          "lt_readout_tv")
    return tv


def copy_screen_scores(tokens: torch.Tensor, z1: torch.Tensor, zR: torch.Tensor, k: int,
                       match_cap: int, temperature: float, top_p: float, stream=None):
    """lt_copy_screen_scores: per position of the committed text `tokens`
    (device int32 [n]) the first copied token of the decoder's lookup (-1:
    none), its depth-d1 screen score (softmax of z1 at T = 1) and its
    full-depth acceptance probability from zR (fp32 [n][V] views, unit column
    stride).  zR is overwritten with the processed distributions when
    temperature > 0.  Returns (tok, score, accept) device tensors."""
    assert tokens.is_cuda and tokens.dtype == torch.int32 and tokens.dim() == 1
    assert z1.dtype == zR.dtype == torch.float32 and z1.shape == zR.shape
    assert z1.stride(1) == 1 and zR.stride(1) == 1 and z1.shape[0] == tokens.shape[0]
    n, V = z1.shape
    tok = torch.empty(n, dtype=torch.int32, device=tokens.device)
    score = torch.empty(n, dtype=torch.float32, device=tokens.device)
    acc = torch.empty(n, dtype=torch.float32, device=tokens.device)
    check(lib().lt_copy_screen_scores(_ptr(tokens), n, k, match_cap, _ptr(z1), z1.stride(0),
                                      _ptr(zR), zR.stride(0), V, float(temperature),
                                      float(top_p), _ptr(tok), _ptr(score), _ptr(acc),
                                      _stream(stream)), "lt_copy_screen_scores")
    return tok, score, acc


def selftest_wait(stream=None) -> dict:
    """lt_selftest_wait: a bounded wait that nothing releases must give up
    (status 1), and the next kernel must still run."""
    import numpy as np
    out = np.zeros(3, dtype=np.int32)
    check(lib().lt_selftest_wait(out.ctypes.data_as(_ip), _stream(stream)), "lt_selftest_wait")
    return {"status": int(out[0]), "context_alive": bool(out[1]), "wait_ms": int(out[2])}


# ---------------------------------------------------------------------------
# decoder handle
# ---------------------------------------------------------------------------

def _i32p(a):
    return a.ctypes.data_as(_ip)


def model_config_c(cfg) -> ModelConfigC:
    return ModelConfigC(LT_F32 if cfg.dtype == "f32" else LT_BF16, cfg.d_model, cfg.n_heads,
                        cfg.head_dim, cfg.ffn, cfg.vocab, cfg.n_prelude, cfg.n_core, cfg.n_coda,
                        cfg.R, cfg.rms_eps, cfg.rope_theta, cfg.resid_scale)


@dataclasses.dataclass
class CopyConfig:
    """Context-copy proposals of lt_decode_config (k = 0: off)."""
    tau: float
    k: int = 4
    max_len: int = 16
    match_cap: int = 64
    reserve: int = 8


class Decoder:
    """One lt_handle: caller-side device memory (weights, workspace) and a
    non-default CUDA stream, owned by this object."""

    def __init__(self, cfg, dec, weights=None, max_branches=16, max_ctx=None, trace_steps=0,
                 second_mode=0, device="cuda", workspace_fill=None, copy=None):
        """workspace_fill: a byte value written over the whole workspace before
        lt_create (tests use it to show that no state is read before it is
        written); None leaves the allocation as it comes.  copy: context-copy
        proposals, a CopyConfig (None: off)."""
        import numpy as np
        self.np = np
        self.cfg, self.dec = cfg, dec
        self.device = torch.device(device)
        self.stream = torch.cuda.Stream(device=self.device)
        self.mc = model_config_c(cfg)
        cp = copy or CopyConfig(tau=0.0, k=0)
        self.dc = DecodeConfigC(dec.d1, dec.d2, dec.temperature, dec.top_p, dec.seed,
                                max_branches, max_ctx or 4096, dec.max_new, second_mode,
                                trace_steps, cp.k, cp.max_len, cp.match_cap, cp.reserve,
                                cp.tau)
        need = _sz()
        check(lib().lt_workspace_bytes(ctypes.byref(self.mc), ctypes.byref(self.dc),
                                       ctypes.byref(need)), "lt_workspace_bytes")
        self.workspace = torch.empty(need.value, dtype=torch.uint8, device=self.device)
        if workspace_fill is not None:
            self.workspace.fill_(workspace_fill)
            torch.cuda.synchronize(self.device)
        h = _vp()
        check(lib().lt_create(ctypes.byref(self.mc), ctypes.byref(self.dc),
                              self.workspace.data_ptr(), need.value, self.stream.cuda_stream,
                              ctypes.byref(h)), "lt_create")
        self.h = h
        self.n_tags = len({r for r in (dec.d1, dec.d2, cfg.R) if r > 0})
        self.weights = {}
        if weights is not None:
            self.load(weights)

    def _err(self):
        return lib().lt_last_error(self.h).decode()

    def _check(self, code, what):
        if code != 0:
            raise LoopedSpecError(code, f"{what}: {self._err()}")

    def load(self, weights) -> None:
        """weights: iterable of (name, numpy fp32 array) as produced by
        synthetic.iter_weights / make_weights (bf16 models hold bf16 values)."""
        dt = torch.float32 if self.cfg.dtype == "f32" else torch.bfloat16
        items = weights.items() if isinstance(weights, dict) else weights
        with torch.cuda.stream(self.stream):
            for name, a in items:
                self.weights[name] = torch.from_numpy(a).to(device=self.device, dtype=dt,
                                                            non_blocking=False)
        self.stream.synchronize()
        self.bind_weights()

    def bind_weights(self) -> None:
        """Hands the device tensors in self.weights to the library."""
        w = self.weights
        ptrs = []
        for ln in self.cfg.layer_names():
            for t in ("g1", "wqkv", "wo", "g2", "wgu", "wd"):
                ptrs.append(w[f"{ln}.{t}"].data_ptr())
        arr = (_vp * len(ptrs))(*ptrs)
        self._check(lib().lt_load_weights(self.h, w["embed"].data_ptr(),
                                          w["final_norm"].data_ptr(), w["head"].data_ptr(), arr),
                    "lt_load_weights")

    def prefill(self, tokens, argmax=False, logits=False):
        np = self.np
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        first = np.zeros(1, dtype=np.int32)
        am = np.zeros((len(tok), self.n_tags), dtype=np.int32) if argmax else None
        lg = (torch.empty(len(tok), self.n_tags, self.cfg.vocab, dtype=torch.float32,
                          device=self.device) if logits else None)
        self._check(lib().lt_prefill(self.h, _i32p(tok), len(tok), _i32p(first),
                                     _i32p(am) if am is not None else None,
                                     lg.data_ptr() if lg is not None else None), "lt_prefill")
        return int(first[0]), am, lg

    def generate(self, n, ar=False):
        np = self.np
        out = np.zeros(max(n, 1), dtype=np.int32)
        st = StatsC()
        self._check(lib().lt_generate(self.h, 1 if ar else 0, n, _i32p(out), ctypes.byref(st)),
                    "lt_generate")
        return out[:n].tolist(), st.as_dict()

    def step(self, ar=False, info=False):
        """One decode pass: the last token it committed (None if none); with
        info=True also the pass's lt_step_info as a dict."""
        tok = self.np.zeros(1, dtype=self.np.int32)
        n = _i()
        si = StepInfoC()
        self._check(lib().lt_decode_step(self.h, 1 if ar else 0, _i32p(tok), ctypes.byref(n),
                                         ctypes.byref(si)), "lt_decode_step")
        t = int(tok[0]) if n.value else None
        return (t, si.as_dict()) if info else t

    def stats(self):
        """lt_get_stats: running totals of the current (or last) decode."""
        st = StatsC()
        self._check(lib().lt_get_stats(self.h, ctypes.byref(st)), "lt_get_stats")
        return st.as_dict()

    def kv_pool(self):
        """(torch view of the KV pool [planes, slots, 2, d], plane of core layer 0)."""
        p, nb, npl, ns, pc0 = _vp(), _sz(), _i(), _i(), _i()
        self._check(lib().lt_kv_pool(self.h, ctypes.byref(p), ctypes.byref(nb), ctypes.byref(npl),
                                     ctypes.byref(ns), ctypes.byref(pc0)), "lt_kv_pool")
        dt = torch.float32 if self.cfg.dtype == "f32" else torch.bfloat16
        off = p.value - self.workspace.data_ptr()
        raw = self.workspace[off:off + nb.value]
        view = raw.view(dt).view(npl.value, ns.value, 2, self.cfg.d_model)
        return view, pc0.value

    def block_pass(self, depth, pos, lists, list_off, hidden, iters=1, timed=False):
        """One shared-block pass; lists: device int32 tensor; hidden: device fp32
        [n_rows, d] (updated in place).  Returns per-replay ms when timed."""
        np = self.np
        dep = np.ascontiguousarray(depth, dtype=np.int32)
        ps = np.ascontiguousarray(pos, dtype=np.int32)
        off = np.ascontiguousarray(list_off, dtype=np.int32)
        ms = (ctypes.c_float * iters)() if timed else None
        self._check(lib().lt_block_pass(self.h, len(dep), _i32p(dep), _i32p(ps), lists.data_ptr(),
                                        _i32p(off), hidden.data_ptr(), iters, ms), "lt_block_pass")
        return list(ms) if timed else None

    def rollback_branch(self, uid):
        self._check(lib().lt_rollback_branch(self.h, uid), "lt_rollback_branch")

    def commit_branch(self, uid):
        self._check(lib().lt_commit_branch(self.h, uid), "lt_commit_branch")

    def read_log(self, n):
        np = self.np
        t, s, k = (np.zeros(max(n, 1), dtype=np.int32) for _ in range(3))
        self._check(lib().lt_read_log(self.h, _i32p(t), _i32p(s), _i32p(k), n), "lt_read_log")
        return t[:n].tolist(), s[:n].tolist(), k[:n].tolist()

    def read_trace(self, n_steps):
        np = self.np
        tr = np.zeros((max(n_steps, 1), self.dc.max_branches, 4), dtype=np.int32)
        self._check(lib().lt_read_trace(self.h, _i32p(tr), n_steps), "lt_read_trace")
        return [[tuple(int(v) for v in row) for row in step if row[0] >= 0]
                for step in tr[:n_steps]]

    def read_committed(self):
        np = self.np
        t = np.zeros(self.dc.max_ctx, dtype=np.int32)
        s = np.zeros(self.dc.max_ctx, dtype=np.int32)
        L = _i()
        self._check(lib().lt_read_committed(self.h, _i32p(t), _i32p(s), ctypes.byref(L)),
                    "lt_read_committed")
        return t[:L.value].tolist(), s[:L.value].tolist()

    def read_table(self):
        np = self.np
        t = np.zeros((12, self.dc.max_branches), dtype=np.int32)
        self._check(lib().lt_read_branch_table(self.h, _i32p(t)), "lt_read_branch_table")
        return t

    def read_readouts(self):
        np = self.np
        C, V = self.dc.max_branches, self.cfg.vocab
        lg = np.zeros((C, V), dtype=np.float32)
        pr = np.zeros((C, V), dtype=np.float32)
        am = np.zeros(C, dtype=np.int32)
        self._check(lib().lt_read_readouts(self.h, lg.ctypes.data, pr.ctypes.data, _i32p(am), None),
                    "lt_read_readouts")
        return lg, pr, am

    def profile(self, n_steps, ar=False):
        p = ProfileC()
        self._check(lib().lt_profile_steps(self.h, 1 if ar else 0, n_steps, ctypes.byref(p)),
                    "lt_profile_steps")
        return p.as_dict()

    def profile_gemms(self, n_iters=20):
        """lt_profile_gemms: the pass's shared-block GEMMs replayed alone as a
        graph; resets the decode state."""
        out = (ctypes.c_double * 3)()
        self._check(lib().lt_profile_gemms(self.h, n_iters, out), "lt_profile_gemms")
        return {"ms": out[0], "bytes": out[1], "launches": int(out[2])}

    def info(self):
        i = InfoC()
        self._check(lib().lt_get_info(self.h, ctypes.byref(i)), "lt_get_info")
        return i.as_dict()

    def close(self):
        if getattr(self, "h", None):
            lib().lt_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
