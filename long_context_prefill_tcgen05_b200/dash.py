"""ctypes binding of libdash.so (include/dash.h, include/dash_ops.h).

Argument marshalling only: torch tensors are passed as raw device pointers
plus sizes, torch supplies memory and the current stream, and every step of
the path runs in the library's CUDA kernels.  There is no fallback: if the
library is missing, ``lib()`` raises.
"""
import ctypes
import os
import re

import torch

from .build import LIB, INCLUDE

c_i32, c_i64, c_f32, c_f64, c_vp, c_sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                          ctypes.c_double, ctypes.c_void_p, ctypes.c_size_t)

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "non-finite score",
          4: "workspace too small", 5: "CUDA error", 6: "device wait timed out",
          7: "index out of range"}
MODES = {"prune": 0, "halt": 1, "dense": 2}
SELECTS = {"topk": 0, "threshold": 1}


class DashError(RuntimeError):
    def __init__(self, status, what=""):
        super().__init__(f"{what}: dash status {status} ({STATUS.get(status, '?')})")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("n_layers", c_i32), ("d_model", c_i32), ("n_heads", c_i32), ("n_kv_heads", c_i32),
                ("head_dim", c_i32), ("ffn_dim", c_i32), ("rms_eps", c_f64), ("rope_theta", c_f64),
                ("dtype", c_i32)]


# dash_dtype codes of the 16-bit float formats a model may use
DTYPES = {torch.bfloat16: 0, torch.float16: 1}


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_gate", "w_up", "w_down")]


class Config(ctypes.Structure):
    _fields_ = [("halt_layer", c_i32), ("mode", c_i32), ("select", c_i32), ("score", c_i32),
                ("keep_ratio", c_f64), ("threshold", c_f32), ("keep_first", c_i32), ("keep_last", c_i32),
                ("monitor_layers", c_i32)]


class LaunchRecord(ctypes.Structure):
    _fields_ = [("kind", c_i32), ("layer", c_i32), ("m", c_i64), ("n", c_i64), ("k", c_i64), ("ms", c_f32),
                ("launches", c_i32)]


class HaltCtx(ctypes.Structure):
    _fields_ = [("active_idx", c_vp), ("halted_idx", c_vp), ("h_full", c_vp), ("T", c_i64)]


class KVCacheDesc(ctypes.Structure):
    _fields_ = [("k", c_vp), ("v", c_vp), ("pos", c_vp), ("capacity", c_i64), ("len", c_i64)]


_SIGS = {
    "dash_status_string": (ctypes.c_char_p, [c_i32]),
    "dash_device_error": (c_i32, []),
    "dash_score": (c_i32, [c_vp, c_vp, c_i64, c_i32, c_i32, c_vp, c_vp]),
    "dash_topk_count": (c_i64, [c_i64, c_f64, c_i32, c_i32]),
    "dash_select_workspace_size": (c_sz, [c_i64]),
    "dash_select": (c_i32, [c_vp, c_i64, c_i32, c_f64, c_f32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "dash_compact": (c_i32, [c_vp, c_i64, c_vp, c_i64, c_i32, c_vp, c_vp]),
    "dash_scatter": (c_i32, [c_vp, c_vp, c_i64, c_i32, c_vp, c_i64, c_vp]),
    "dash_layer_workspace_size": (c_sz, [ctypes.POINTER(Dims), c_i64, c_i64, c_i64]),
    "dash_layer_forward": (c_i32, [ctypes.POINTER(Dims), ctypes.POINTER(LayerWeights), c_vp, c_i64, c_vp, c_i64,
                                   ctypes.POINTER(HaltCtx), c_vp, c_i32, c_vp, c_sz, c_vp]),
    "dash_prefill_workspace_size": (c_sz, [ctypes.POINTER(Dims), c_i64, ctypes.POINTER(Config)]),
    "dash_prefill": (c_i32, [ctypes.POINTER(Dims), ctypes.POINTER(LayerWeights), c_vp, c_i64, ctypes.POINTER(Config),
                             c_vp, ctypes.POINTER(c_i64), c_vp, c_vp, c_sz, c_vp]),
    "dash_rmsnorm": (c_i32, [c_vp, c_i64, c_i32, c_vp, c_f64, c_vp, c_vp]),
    "dash_linear": (c_i32, [c_vp, c_i64, c_i32, c_vp, c_i32, c_vp, c_vp]),
    "dash_set_gemm_pairs": (c_i32, [c_i32]),
    "dash_set_decode_tensor_cores": (c_i32, [c_i32]),
    "dash_attention": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "dash_prefill_varlen_workspace_size": (c_sz, [ctypes.POINTER(Dims), c_i64, c_i32, ctypes.POINTER(Config)]),
    "dash_prefill_varlen": (c_i32, [ctypes.POINTER(Dims), ctypes.POINTER(LayerWeights), c_vp,
                                    ctypes.POINTER(c_i32), c_i32, ctypes.POINTER(Config), c_vp,
                                    ctypes.POINTER(c_i64), ctypes.POINTER(c_i32), c_vp, c_vp, c_sz, c_vp]),
    "dash_layer_forward_noalloc": (c_i32, [ctypes.POINTER(Dims), ctypes.POINTER(LayerWeights), c_vp, c_i64, c_vp,
                                           c_i64, ctypes.POINTER(HaltCtx), c_vp, c_i32, c_vp]),
    "dash_exp2_fma": (c_i32, [c_vp, c_i64, c_vp, c_vp]),
    "dash_prefill_kv": (c_i32, [ctypes.POINTER(Dims), ctypes.POINTER(LayerWeights), c_vp, c_i64,
                                ctypes.POINTER(Config), c_vp, ctypes.POINTER(c_i64), c_vp,
                                ctypes.POINTER(KVCacheDesc), c_vp, c_sz, c_vp]),
    "dash_prefill_varlen_kv": (c_i32, [ctypes.POINTER(Dims), ctypes.POINTER(LayerWeights), c_vp,
                                       ctypes.POINTER(c_i32), c_i32, ctypes.POINTER(Config), c_vp,
                                       ctypes.POINTER(c_i64), ctypes.POINTER(c_i32), c_vp,
                                       ctypes.POINTER(KVCacheDesc), c_vp, c_sz, c_vp]),
    "dash_decode_workspace_size": (c_sz, [ctypes.POINTER(Dims), c_i32]),
    "dash_decode_attention_workspace_size": (c_sz, [c_i32]),
    "dash_decode_attention": (c_i32, [c_vp, c_i32, ctypes.POINTER(KVCacheDesc), c_i32, c_i32, c_i32, c_vp, c_vp,
                                      c_sz, c_vp]),
    "dash_decode_step": (c_i32, [ctypes.POINTER(Dims), ctypes.POINTER(LayerWeights), c_vp, c_i32,
                                 ctypes.POINTER(c_i32), ctypes.POINTER(KVCacheDesc), c_vp, c_sz, c_vp]),
    "dash_selftest_wait_timeout": (c_i32, [c_vp]),
    "dash_timing_start": (c_i32, [c_i32]),
    "dash_timing_stop": (c_i32, [ctypes.POINTER(LaunchRecord), c_i32]),
    "dash_kernel_name": (ctypes.c_char_p, [c_i32]),
}

_LIB = None


def lib():
    """Loads libdash.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing; build it with "
                               "`python -m long_context_prefill_tcgen05_b200.build`")
        L = ctypes.CDLL(LIB)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def declared_symbols():
    """Every dash_* function declared in include/*.h."""
    names = set()
    for fn in os.listdir(INCLUDE):
        if fn.endswith(".h"):
            with open(os.path.join(INCLUDE, fn)) as f:
                names |= set(re.findall(r"\b(dash_[a-z_0-9]+)\s*\(", f.read()))
    return sorted(names)


def _check(status, what):
    if status != 0:
        raise DashError(status, what)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32


def _t(t, dtype, name, shape=None):
    """Pointer to a contiguous CUDA tensor of `dtype` (None passes through).
    The library takes row-major buffers whose sizes follow from the shape
    arguments, so a strided view, another dtype or a host tensor is refused
    here rather than read as something else.  `shape` entries that are None
    are not checked."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        what = f"{tuple(t.shape)} {t.dtype} {t.device}{'' if t.is_contiguous() else ' strided'}" \
            if isinstance(t, torch.Tensor) else type(t).__name__
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got {what}")
    if shape is not None and (t.dim() != len(shape) or any(w is not None and g != w for g, w in zip(t.shape, shape))):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _out(t, dtype, name, n):
    """Pointer to an output buffer of at least n elements (None passes through)."""
    if isinstance(t, torch.Tensor) and t.numel() < n:
        raise ValueError(f"{name}: needs at least {n} elements, has {t.numel()}")
    return _t(t, dtype, name)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def device_error():
    """Reads and clears the library's sticky device error (synchronises)."""
    return lib().dash_device_error()


def check_device():
    _check(device_error(), "device")


# --------------------------------------------------------- launch timing
def timing_start(capacity=1 << 16):
    _check(lib().dash_timing_start(capacity), "dash_timing_start")


def timing_stop(capacity=1 << 16):
    """Stops recording; returns a list of dicts (kind name, layer, m, n, k, ms)."""
    buf = (LaunchRecord * capacity)()
    n = lib().dash_timing_stop(buf, capacity)
    if n < 0:
        raise DashError(5, "dash_timing_stop")
    return [{"kind": lib().dash_kernel_name(r.kind).decode(), "layer": r.layer, "m": r.m, "n": r.n,
             "k": r.k, "ms": r.ms, "launches": r.launches} for r in buf[:n]]


# ----------------------------------------------------------- workspaces
_WS = {}


def workspace(nbytes, device):
    """A cached uint8 device buffer of at least nbytes (reused across calls)."""
    key = str(device)
    buf = _WS.get(key)
    if buf is None or buf.numel() < nbytes:
        _WS[key] = buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    return buf


def release_workspaces():
    _WS.clear()


# ------------------------------------------------------------- row ops
def score(U, H=None, relative=False, out=None, stream=None):
    T, d = U.shape
    out = torch.empty(T, dtype=torch.float32, device=U.device) if out is None else out
    _check(lib().dash_score(_t(U, BF16, "U"), _t(H, BF16, "H", (T, d)), T, d, int(relative),
                            _t(out, F32, "out", (T,)), _stream(stream)), "dash_score")
    return out


def topk_count(T, keep, keep_first=0, keep_last=0):
    return lib().dash_topk_count(T, keep, keep_first, keep_last)


def select(scores, kind="topk", keep=0.5, threshold=0.0, keep_first=0, keep_last=0, want_halted=False,
           stream=None):
    """Returns (idx [count] int32, halted [T-count] or None, count) after a sync."""
    T = scores.numel()
    dev = scores.device
    idx = torch.empty(max(T, 1), dtype=torch.int32, device=dev)
    halted = torch.empty(max(T, 1), dtype=torch.int32, device=dev) if want_halted else None
    count = torch.empty(1, dtype=torch.int32, device=dev)
    ws = workspace(lib().dash_select_workspace_size(T), dev)
    _check(lib().dash_select(_t(scores, F32, "scores"), T, SELECTS[kind], keep, threshold, keep_first, keep_last, _p(idx),
                             _p(halted), _p(count), _p(ws), ws.numel(), _stream(stream)), "dash_select")
    n = int(count.item())
    if n < 0:
        raise DashError(-n, "dash_select")
    return idx[:n], (halted[:T - n] if want_halted else None), n


def compact(X, idx, stream=None):
    K = idx.numel()
    Y = torch.empty(K, X.shape[1], dtype=X.dtype, device=X.device)
    x_dtype = X.dtype if X.dtype in DTYPES else BF16  # rows are copied bit for bit: either 16-bit format
    _check(lib().dash_compact(_t(X, x_dtype, "X"), X.shape[0], _t(idx, I32, "idx"), K, X.shape[1], _p(Y),
                              _stream(stream)), "dash_compact")
    return Y


def scatter(Y, idx, X, stream=None):
    x_dtype = X.dtype if X.dtype in DTYPES else BF16  # rows are copied bit for bit: either 16-bit format
    _check(lib().dash_scatter(_t(Y, x_dtype, "Y", (idx.numel(), X.shape[1])), _t(idx, I32, "idx"), idx.numel(),
                              X.shape[1], _t(X, x_dtype, "X"), X.shape[0], _stream(stream)), "dash_scatter")
    return X


def rmsnorm(X, g, eps, stream=None):
    Y = torch.empty_like(X)
    _check(lib().dash_rmsnorm(_t(X, BF16, "X"), X.shape[0], X.shape[1], _t(g, BF16, "g", (X.shape[1],)), eps, _p(Y),
                              _stream(stream)), "dash_rmsnorm")
    return Y


def linear(A, W, out=None, stream=None):
    M, K = A.shape
    N = W.shape[0]
    out = torch.empty(M, N, dtype=A.dtype, device=A.device) if out is None else out
    _check(lib().dash_linear(_t(A, BF16, "A"), M, K, _t(W, BF16, "W", (N, K)), N, _t(out, BF16, "out", (M, N)),
                             _stream(stream)), "dash_linear")
    return out


def set_gemm_pairs(enable):
    """Runs later GEMMs as 256x256 tiles on SM pairs (True, the default) or as
    single-SM tiles (False); returns the previous setting."""
    return bool(lib().dash_set_gemm_pairs(1 if enable else 0))


def set_decode_tensor_cores(enable):
    """Runs later generation steps' projections for 3 or more sequences on the
    tensor cores (True, the default) or as CUDA-core GEMVs (False); returns
    the previous setting."""
    return bool(lib().dash_set_decode_tensor_cores(1 if enable else 0))


def exp2_fma(x, stream=None):
    y = torch.empty_like(x)
    _check(lib().dash_exp2_fma(_t(x, F32, "x"), x.numel(), _p(y), _stream(stream)), "dash_exp2_fma")
    return y


def attention(Q, K, V, hq, hkv, hd, qpos=None, kstart=None, out=None, stream=None):
    M = Q.shape[0]
    out = torch.empty(M, hq * hd, dtype=Q.dtype, device=Q.device) if out is None else out
    T_kv = K.shape[0]
    _check(lib().dash_attention(_t(Q, BF16, "Q", (M, hq * hd)), _t(K, BF16, "K", (T_kv, hkv * hd)),
                                _t(V, BF16, "V", (T_kv, hkv * hd)), M, T_kv, hq, hkv, hd, _t(qpos, I32, "qpos", (M,)),
                                _t(kstart, I32, "kstart", (M,)), _t(out, BF16, "out", (M, hq * hd)),
                                _stream(stream)), "dash_attention")
    return out


# --------------------------------------------------------------- stack
class Stack:
    """A decoder stack's dims plus its weights laid out for the library
    (w_qkv = [wq; wk; wv] concatenated once, at load time).  The weights'
    torch dtype (bfloat16 or float16) is the model's 16-bit format; hidden
    states and caches passed with this stack must use it too."""

    def __init__(self, dims, layers):
        self.model = dims
        self.dtype = layers[0]["wq"].dtype
        if self.dtype not in DTYPES or any(t.dtype != self.dtype for w in layers for t in w.values()):
            raise ValueError(f"weights must all be bfloat16 or all float16, got {self.dtype}")
        self.dims = Dims(dims.n_layers if len(layers) == dims.n_layers else len(layers), dims.d_model,
                         dims.n_heads, dims.n_kv_heads, dims.head_dim, dims.ffn_dim, dims.rms_eps,
                         dims.rope_theta, DTYPES[self.dtype])
        self.tensors = []
        arr = (LayerWeights * len(layers))()
        for i, w in enumerate(layers):
            qkv = torch.cat([w["wq"], w["wk"], w["wv"]], 0).contiguous()
            keep = [w["attn_norm"].contiguous(), qkv, w["wo"].contiguous(), w["ffn_norm"].contiguous(),
                    w["wg"].contiguous(), w["wu"].contiguous(), w["wd"].contiguous()]
            self.tensors.append(keep)
            arr[i] = LayerWeights(*[t.data_ptr() for t in keep])
        self.layers = arr
        self.n_layers = len(layers)


def layer_forward(stack, l, H, pos=None, max_pos=None, halt=None, delta=None, relative=False, stream=None):
    """One block in place on H [M, d].  halt = (active_idx, halted_idx, h_full) or None."""
    M = H.shape[0]
    T_kv = M
    hctx = None
    if halt is not None:
        active, halted, h_full = halt
        T_kv = h_full.shape[0]
        _t(active, I32, "active_idx", (M,))
        _t(h_full, stack.dtype, "h_full", (T_kv, H.shape[1]))
        if halted.numel():
            _t(halted, I32, "halted_idx", (T_kv - M,))
        hctx = HaltCtx(active.data_ptr(), halted.data_ptr() if halted.numel() else None, h_full.data_ptr(), T_kv)
        pos = active
    if max_pos is None:
        max_pos = T_kv
    need = lib().dash_layer_workspace_size(ctypes.byref(stack.dims), M, T_kv, max_pos)
    ws = workspace(need, H.device)
    w = ctypes.pointer(stack.layers[l])
    _check(lib().dash_layer_forward(ctypes.byref(stack.dims), w, _t(H, stack.dtype, "H", (M, stack.dims.d_model)),
                                    M, _t(pos, I32, "pos", (M,)), max_pos,
                                    ctypes.byref(hctx) if hctx is not None else None, _out(delta, F32, "delta", M),
                                    int(relative),
                                    _p(ws), ws.numel(), _stream(stream)), "dash_layer_forward")
    return H


def make_config(halt_layer=0, mode="prune", select="topk", keep=0.5, threshold=0.0, relative=False,
                keep_first=0, keep_last=0, monitor_layers=1):
    return Config(halt_layer, MODES[mode], SELECTS[select], int(relative), keep, threshold, keep_first, keep_last,
                  monitor_layers)


def prefill_varlen(stack, H, cu_seqlens, cfg, idx_out=None, delta_out=None, stream=None):
    """dash_prefill_varlen in place on H [T, d] for the sequences cu_seqlens
    (host ints, length nseq + 1); returns (K, per-sequence active counts)."""
    cu = [int(x) for x in cu_seqlens]
    nseq = len(cu) - 1
    T = H.shape[0]
    need = lib().dash_prefill_varlen_workspace_size(ctypes.byref(stack.dims), T, nseq, ctypes.byref(cfg))
    ws = workspace(need, H.device)
    cu_arr = (c_i32 * (nseq + 1))(*cu)
    counts = (c_i32 * nseq)()
    K = c_i64(0)
    _check(lib().dash_prefill_varlen(ctypes.byref(stack.dims), stack.layers,
                                     _t(H, stack.dtype, "H", (T, stack.dims.d_model)),
                                     cu_arr, nseq, ctypes.byref(cfg), _out(idx_out, I32, "idx_out", T),
                                     ctypes.byref(K), counts, _out(delta_out, F32, "delta_out", T), _p(ws), ws.numel(),
                                     _stream(stream)), "dash_prefill_varlen")
    return K.value, list(counts)


def prefill(stack, H, cfg, idx_out=None, delta_out=None, stream=None):
    """Runs dash_prefill in place on H [T, d]; returns K (the active count)."""
    T = H.shape[0]
    need = lib().dash_prefill_workspace_size(ctypes.byref(stack.dims), T, ctypes.byref(cfg))
    ws = workspace(need, H.device)
    K = c_i64(0)
    _check(lib().dash_prefill(ctypes.byref(stack.dims), stack.layers, _t(H, stack.dtype, "H", (T, stack.dims.d_model)), T,
                              ctypes.byref(cfg), _out(idx_out, I32, "idx_out", T), ctypes.byref(K),
                              _out(delta_out, F32, "delta_out", T), _p(ws), ws.numel(), _stream(stream)),
           "dash_prefill")
    return K.value


# ------------------------------------------------------------- KV cache
class KVCache:
    """Caller-owned KV caches for nseq sequences x n_layers layers.

    capacity: rows per cache, one int for all, or a list per layer.  The
    descriptor array ``desc`` (dash_kv_cache[nseq * n_layers], sequence-
    major) is what the library reads and whose ``len`` fields it updates.
    """

    def __init__(self, stack, nseq=1, capacity=0, device="cuda", with_pos=True):
        L = stack.n_layers
        caps = [int(capacity)] * L if isinstance(capacity, int) else [int(c) for c in capacity]
        kvd = stack.dims.n_kv_heads * stack.dims.head_dim
        self.nseq, self.n_layers = nseq, L
        self.k, self.v, self.pos = [], [], []
        self.desc = (KVCacheDesc * (nseq * L))()
        for s in range(nseq):
            for l in range(L):
                k = torch.zeros(max(caps[l], 1), kvd, dtype=stack.dtype, device=device)
                v = torch.zeros_like(k)
                p = torch.full((max(caps[l], 1),), -1, dtype=torch.int32, device=device) if with_pos else None
                self.k.append(k)
                self.v.append(v)
                self.pos.append(p)
                self.desc[s * L + l] = KVCacheDesc(k.data_ptr(), v.data_ptr(), p.data_ptr() if with_pos else None,
                                                   caps[l], 0)

    def lens(self, s=0):
        return [self.desc[s * self.n_layers + l].len for l in range(self.n_layers)]

    def layer(self, s, l):
        """(k [len, kvd], v, pos [len] or None) of sequence s, layer l."""
        i = s * self.n_layers + l
        n = self.desc[i].len
        return self.k[i][:n], self.v[i][:n], (self.pos[i][:n] if self.pos[i] is not None else None)


def prefill_kv(stack, H, cfg, cache, idx_out=None, delta_out=None, stream=None):
    """dash_prefill_kv: dash_prefill that also fills cache (KVCache, nseq = 1); returns K."""
    T = H.shape[0]
    need = lib().dash_prefill_workspace_size(ctypes.byref(stack.dims), T, ctypes.byref(cfg))
    ws = workspace(need, H.device)
    K = c_i64(0)
    _check(lib().dash_prefill_kv(ctypes.byref(stack.dims), stack.layers, _t(H, stack.dtype, "H", (T, stack.dims.d_model)),
                                 T,
                                 ctypes.byref(cfg), _out(idx_out, I32, "idx_out", T), ctypes.byref(K),
                                 _out(delta_out, F32, "delta_out", T), cache.desc, _p(ws), ws.numel(),
                                 _stream(stream)), "dash_prefill_kv")
    return K.value


def prefill_varlen_kv(stack, H, cu_seqlens, cfg, cache, idx_out=None, delta_out=None, stream=None):
    """dash_prefill_varlen_kv; returns (K, per-sequence active counts)."""
    cu = [int(x) for x in cu_seqlens]
    nseq = len(cu) - 1
    T = H.shape[0]
    need = lib().dash_prefill_varlen_workspace_size(ctypes.byref(stack.dims), T, nseq, ctypes.byref(cfg))
    ws = workspace(need, H.device)
    cu_arr = (c_i32 * (nseq + 1))(*cu)
    counts = (c_i32 * nseq)()
    K = c_i64(0)
    _check(lib().dash_prefill_varlen_kv(ctypes.byref(stack.dims), stack.layers,
                                        _t(H, stack.dtype, "H", (T, stack.dims.d_model)), cu_arr, nseq, ctypes.byref(cfg),
                                        _out(idx_out, I32, "idx_out", T), ctypes.byref(K), counts,
                                        _out(delta_out, F32, "delta_out", T), cache.desc, _p(ws), ws.numel(),
                                        _stream(stream)), "dash_prefill_varlen_kv")
    return K.value, list(counts)


def decode_step(stack, X, pos, cache, stream=None):
    """dash_decode_step in place on X [nseq, d]: one new token per sequence at
    the host positions pos; appends to cache (KVCache)."""
    n = X.shape[0]
    need = lib().dash_decode_workspace_size(ctypes.byref(stack.dims), n)
    ws = workspace(need, X.device)
    pos_arr = (c_i32 * n)(*[int(p) for p in pos])
    _check(lib().dash_decode_step(ctypes.byref(stack.dims), stack.layers, _t(X, stack.dtype, "X", (n, stack.dims.d_model)),
                                  n, pos_arr, cache.desc, _p(ws), ws.numel(), _stream(stream)), "dash_decode_step")
    return X


def decode_attention(Q, kv, hq, hkv, hd, out=None, stream=None):
    """dash_decode_attention: Q [nseq, hq*hd]; kv = list of (K [len, hkv*hd], V) per sequence."""
    n = Q.shape[0]
    out = torch.empty_like(Q) if out is None else out
    desc = (KVCacheDesc * n)()
    for s, (k, v) in enumerate(kv):
        _t(k, BF16, f"K[{s}]", (None, hkv * hd))
        _t(v, BF16, f"V[{s}]", tuple(k.shape))
        desc[s] = KVCacheDesc(k.data_ptr(), v.data_ptr(), None, k.shape[0], k.shape[0])
    need = lib().dash_decode_attention_workspace_size(hd)
    ws = workspace(need, Q.device)
    _check(lib().dash_decode_attention(_t(Q, BF16, "Q", (n, hq * hd)), n, desc, hq, hkv, hd,
                                       _t(out, BF16, "out", (n, hq * hd)), _p(ws), ws.numel(), _stream(stream)),
           "dash_decode_attention")
    return out
