"""ctypes binding of libnc_b200.so (the C ABI in include/nc.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  Device buffers may be torch CUDA tensors (their
data_ptr() is passed) or raw integer device pointers; host buffers are
numpy arrays.  There is no CPU fallback: if the shared library is missing
or fails to load, every entry point raises.
"""
import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnc_b200.so")

NC_OK, NC_ERR_INVALID_ARG, NC_ERR_OOM, NC_ERR_CUDA, NC_ERR_TOKEN_RANGE, NC_ERR_TIMEOUT, \
    NC_ERR_UNSUPPORTED = range(7)
NC_INIT_SPEC, NC_INIT_ALL_RANDOM = 0, 1
(EPI_STORE_BF16, EPI_STORE_F32, EPI_RESID_F32, EPI_RELU2, EPI_RELU2_BWD, EPI_AXPBY_BF16,
 EPI_ACC_F32, EPI_ROPE_QKNORM) = range(8)


class NcError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("nc status %d: %s" % (status, msg))
        self.status = status


class TensorDesc(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("ndim", ctypes.c_int),
                ("shape", ctypes.c_int64 * 2), ("dtype", ctypes.c_int),
                ("data", ctypes.c_void_p), ("data_bf16", ctypes.c_void_p)]


class GemmDesc(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int),
                ("batch", ctypes.c_int),
                ("A", ctypes.c_void_p), ("lda", ctypes.c_int64), ("stride_a", ctypes.c_int64),
                ("a_kmajor", ctypes.c_int),
                ("B", ctypes.c_void_p), ("ldb", ctypes.c_int64), ("stride_b", ctypes.c_int64),
                ("b_kmajor", ctypes.c_int),
                ("D", ctypes.c_void_p), ("ldd", ctypes.c_int64), ("stride_d", ctypes.c_int64),
                ("aux", ctypes.c_void_p), ("ldaux", ctypes.c_int64),
                ("stride_aux", ctypes.c_int64),
                ("epi", ctypes.c_int), ("alpha", ctypes.c_float), ("beta", ctypes.c_float),
                ("split_k", ctypes.c_int), ("rope_T", ctypes.c_int), ("rope_H", ctypes.c_int),
                ("rope_tab", ctypes.c_void_p), ("rstd_q", ctypes.c_void_p),
                ("rstd_k", ctypes.c_void_p), ("rope_Hkv", ctypes.c_int),
                ("ab_type", ctypes.c_int), ("ab_scale", ctypes.c_void_p),
                ("amax_out", ctypes.c_void_p)]


class ModelConfig(ctypes.Structure):
    _fields_ = [("depth", ctypes.c_int), ("vocab", ctypes.c_int), ("seed", ctypes.c_uint64),
                ("flags", ctypes.c_int), ("n_kv_head", ctypes.c_int),
                ("window", ctypes.c_void_p), ("fp8", ctypes.c_int),
                ("lm_chunk_tokens", ctypes.c_int)]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


_lib = None
vp = ctypes.c_void_p
i64 = ctypes.c_int64
ci = ctypes.c_int
cf = ctypes.c_float


def lib():
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libnc_b200.so is missing: run pretraining_step_b200/build.py "
                           "(there is no fallback path)")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "nc_gpt_init": (ci, [ci, ci, ctypes.c_uint64, ctypes.POINTER(vp)]),
        "nc_gpt_init_ex": (ci, [ci, ci, ctypes.c_uint64, ci, ctypes.POINTER(vp)]),
        "nc_gpt_init_config": (ci, [ctypes.POINTER(ModelConfig), ctypes.POINTER(vp)]),
        "nc_params_free": (None, [vp]),
        "nc_set_stream": (ci, [vp, vp]),
        "nc_num_tensors": (ci, [vp]),
        "nc_tensor_info": (ci, [vp, ci, ctypes.POINTER(TensorDesc)]),
        "nc_tensor_write": (ci, [vp, ci, vp]),
        "nc_tensor_read": (ci, [vp, ci, vp]),
        "nc_momentum_read": (ci, [vp, ci, vp]),
        "nc_params_sync": (ci, [vp]),
        "nc_grads_create": (ci, [vp, ctypes.POINTER(vp)]),
        "nc_grads_free": (None, [vp]),
        "nc_grad_info": (ci, [vp, ci, ctypes.POINTER(TensorDesc)]),
        "nc_grad_read": (ci, [vp, ci, vp]),
        "nc_grad_write": (ci, [vp, ci, vp]),
        "nc_gpt_fwd_bwd": (ci, [vp, vp, vp, ci, ci, ctypes.POINTER(cf), vp]),
        "nc_gpt_fwd_bwd_async": (ci, [vp, vp, vp, ci, ci, vp, vp]),
        "nc_muon_step": (ci, [vp, vp, cf, cf]),
        "nc_adamw_step": (ci, [vp, vp, cf, cf, cf, cf, cf, cf]),
        "nc_step_capture": (ci, [vp, vp, vp, ci, ci, vp, vp, cf, cf]),
        "nc_step_replay": (ci, [vp]),
        "nc_sync": (ci, [vp]),
        "nc_debug_status_word": (vp, [vp]),
        "nc_op_gemm": (ci, [ctypes.POINTER(GemmDesc), vp]),
        "nc_op_rmsnorm": (ci, [vp, i64, ci, vp, vp, vp]),
        "nc_op_embed_gather": (ci, [vp, i64, vp, ci, ci, vp, vp]),
        "nc_op_exp2_poly": (ci, [vp, vp, i64, vp]),
        "nc_op_fp8_quantize": (ci, [vp, ci, i64, ci, i64, ci, vp, i64, vp, vp, vp]),
        "nc_op_fp8_quantize2": (ci, [vp, i64, ci, i64, vp, vp, vp, vp, vp]),
        "nc_op_sync": (ci, [vp]),
        "nc_debug_op_status_word": (vp, []),
        "nc_op_attention_fwd": (ci, [vp, vp, vp, i64, vp, i64, vp, ci, ci, ci, vp]),
        "nc_op_attention_bwd": (ci, [vp, vp, vp, i64, vp, vp, i64, vp, vp, vp, vp, i64, vp,
                                     ci, ci, ci, vp]),
        "nc_op_attention_bwd_noalloc": (ci, [vp, vp, vp, i64, vp, vp, i64, vp, vp, vp, vp,
                                             i64, ci, ci, ci, vp]),
        "nc_op_attention_fwd_ex": (ci, [vp, i64, vp, vp, i64, vp, i64, vp, ci, ci, ci, ci, ci,
                                        vp]),
        "nc_op_attention_bwd_ex": (ci, [vp, i64, vp, vp, i64, vp, vp, i64, vp, vp, vp, vp, i64,
                                        vp, ci, ci, ci, ci, ci, vp]),
        "nc_newton_schulz_scratch_bytes": (ctypes.c_size_t, [ci, ci, ci]),
        "nc_op_newton_schulz": (ci, [vp, vp, ci, ci, ci, ci, vp, vp]),
        "nc_profile_enable": (ci, [vp, ci]),
        "nc_profile_read": (ci, [vp, ctypes.POINTER(KernelStat), ci, ctypes.POINTER(ci)]),
        "nc_launch_count": (i64, [vp]),
        "nc_last_error": (ctypes.c_char_p, []),
        "nc_status_string": (ctypes.c_char_p, [ci]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(status):
    if status != NC_OK:
        raise NcError(status, lib().nc_last_error().decode())


def _ptr(x):
    """Device pointer of a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ model
def window_pattern(pattern, depth, short):
    """Per-layer windows from a short/long pattern such as "SSSL": layer l
    takes the letter l % len(pattern); 'S' is a left window of `short` keys,
    'L' full causal (-1)."""
    if not pattern or any(c not in "SL" for c in pattern):
        raise ValueError("pattern of 'S' and 'L'")
    return [short if pattern[l % len(pattern)] == "S" else -1 for l in range(depth)]


class GPT:
    """One model (nc_params) and its gradients (nc_grads).  n_kv_head: KV
    heads (0: one per query head); window: None or one causal left window
    per layer (negative: full causal)."""

    def __init__(self, depth, vocab=32768, seed=0, all_random=False, stream=None, n_kv_head=0,
                 window=None, fp8=False, lm_chunk_tokens=0):
        h = vp()
        cfg = ModelConfig(depth=depth, vocab=vocab, seed=seed,
                          flags=NC_INIT_ALL_RANDOM if all_random else NC_INIT_SPEC,
                          n_kv_head=n_kv_head, window=None, fp8=int(bool(fp8)),
                          lm_chunk_tokens=int(lm_chunk_tokens))
        win = None
        if window is not None:
            if len(window) != depth:
                raise ValueError("one window per layer")
            win = (ctypes.c_int32 * depth)(*[int(w) for w in window])
            cfg.window = ctypes.cast(win, ctypes.c_void_p)
        _check(lib().nc_gpt_init_config(ctypes.byref(cfg), ctypes.byref(h)))
        self.h = h
        g = vp()
        st = lib().nc_grads_create(self.h, ctypes.byref(g))
        if st != NC_OK:
            lib().nc_params_free(self.h)
            _check(st)
        self.g = g
        self.depth, self.vocab = depth, vocab
        self.n_kv_head, self.window = n_kv_head, None if window is None else list(window)
        if stream is not None:
            self.set_stream(stream)

    def close(self):
        if getattr(self, "g", None):
            lib().nc_grads_free(self.g)
            self.g = None
        if getattr(self, "h", None):
            lib().nc_params_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_stream(self, stream):
        _check(lib().nc_set_stream(self.h, _stream(stream)))

    def num_tensors(self):
        return lib().nc_num_tensors(self.h)

    def tensor_info(self, idx):
        t = TensorDesc()
        _check(lib().nc_tensor_info(self.h, idx, ctypes.byref(t)))
        return t

    def shapes(self):
        return [tuple(self.tensor_info(i).shape) for i in range(self.num_tensors())]

    def write(self, idx, arr):
        a = np.ascontiguousarray(arr, dtype=np.float32)
        assert a.shape == tuple(self.tensor_info(idx).shape)
        _check(lib().nc_tensor_write(self.h, idx, a.ctypes.data))

    def read(self, idx):
        t = self.tensor_info(idx)
        out = np.empty(tuple(t.shape), dtype=np.float32)
        _check(lib().nc_tensor_read(self.h, idx, out.ctypes.data))
        return out

    def load(self, params):
        for i, p in enumerate(params):
            self.write(i, p)

    def params(self):
        return [self.read(i) for i in range(self.num_tensors())]

    def grad(self, idx):
        t = self.tensor_info(idx)
        out = np.empty(tuple(t.shape), dtype=np.float32)
        _check(lib().nc_grad_read(self.g, idx, out.ctypes.data))
        return out

    def write_grad(self, idx, arr):
        a = np.ascontiguousarray(arr, dtype=np.float32)
        assert a.shape == tuple(self.tensor_info(idx).shape)
        _check(lib().nc_grad_write(self.g, idx, a.ctypes.data))

    def grads(self):
        return [self.grad(i) for i in range(self.num_tensors())]

    def momentum(self, idx):
        t = self.tensor_info(idx)
        out = np.empty(tuple(t.shape), dtype=np.float32)
        _check(lib().nc_momentum_read(self.h, idx, out.ctypes.data))
        return out

    def fwd_bwd(self, tokens, targets):
        """tokens/targets: numpy int32 [B, T] (host) or torch int32 CUDA tensors."""
        if isinstance(tokens, np.ndarray):
            tokens = np.ascontiguousarray(tokens, dtype=np.int32)
            targets = np.ascontiguousarray(targets, dtype=np.int32)
        B, T = tokens.shape
        loss = cf(0)
        _check(lib().nc_gpt_fwd_bwd(self.h, _ptr(tokens), _ptr(targets), B, T,
                                    ctypes.byref(loss), self.g))
        return loss.value

    def fwd_bwd_async(self, tokens, targets, loss_dev):
        B, T = tokens.shape
        _check(lib().nc_gpt_fwd_bwd_async(self.h, _ptr(tokens), _ptr(targets), B, T,
                                          _ptr(loss_dev), self.g))

    def muon_step(self, lr, momentum):
        _check(lib().nc_muon_step(self.h, self.g, lr, momentum))

    def capture_step(self, tokens, targets, loss_dev, lr, momentum):
        """Record fwd_bwd_async + muon_step as one CUDA graph (nothing runs).
        tokens, targets, loss_dev: device tensors kept alive by this object
        for as long as the graph may replay."""
        B, T = tokens.shape
        _check(lib().nc_step_capture(self.h, _ptr(tokens), _ptr(targets), B, T, _ptr(loss_dev),
                                     self.g, lr, momentum))
        self._graph_io = (tokens, targets, loss_dev)

    def replay_step(self):
        _check(lib().nc_step_replay(self.h))

    def adamw_step(self, lr_embed, lr_head, beta1, beta2, eps, weight_decay):
        """AdamW on the embedding and lm_head from the current gradients."""
        _check(lib().nc_adamw_step(self.h, self.g, lr_embed, lr_head, beta1, beta2, eps,
                                   weight_decay))

    def sync(self):
        _check(lib().nc_sync(self.h))

    def profile(self, on=True):
        _check(lib().nc_profile_enable(self.h, 1 if on else 0))

    def profile_read(self):
        arr = (KernelStat * 64)()
        n = ci(0)
        _check(lib().nc_profile_read(self.h, arr, 64, ctypes.byref(n)))
        return {arr[i].name.decode(): dict(launches=arr[i].launches, ms=arr[i].total_ms,
                                           flops=arr[i].flops, bytes=arr[i].bytes)
                for i in range(n.value)}

    def launch_count(self):
        return int(lib().nc_launch_count(self.h))


# ------------------------------------------------------------------ ops
def gemm(M, N, K, A, B, D, *, lda=None, ldb=None, ldd=None, a_kmajor=True, b_kmajor=True,
         batch=1, stride_a=0, stride_b=0, stride_d=0, epi=EPI_STORE_BF16, aux=None, ldaux=0,
         stride_aux=0, alpha=1.0, beta=0.0, split_k=1, ab_scale=None, amax_out=None, stream=None):
    """D = epi(A B^T) on the tensor cores; ab_scale (a device array of the
    two operands' fp8 scales) selects E4M3 operands (one byte each)."""
    d = GemmDesc()
    d.M, d.N, d.K, d.batch = M, N, K, batch
    d.A, d.B, d.D, d.aux = _ptr(A), _ptr(B), _ptr(D), _ptr(aux)
    d.lda = lda if lda is not None else (K if a_kmajor else M)
    d.ldb = ldb if ldb is not None else (K if b_kmajor else N)
    d.ldd = ldd if ldd is not None else N
    d.stride_a, d.stride_b, d.stride_d = stride_a, stride_b, stride_d
    d.a_kmajor, d.b_kmajor = int(bool(a_kmajor)), int(bool(b_kmajor))
    d.ldaux = ldaux if ldaux else d.ldd
    d.stride_aux = stride_aux
    d.epi, d.alpha, d.beta, d.split_k = epi, alpha, beta, split_k
    if ab_scale is not None:
        d.ab_type, d.ab_scale = 1, _ptr(ab_scale)
    if amax_out is not None:
        d.amax_out = _ptr(amax_out)
    _check(lib().nc_op_gemm(ctypes.byref(d), _stream(stream)))


def embed_gather(tokens, n, E, vocab, d, x, stream=None):
    """x[i] = E[tokens[i]] (fp32 rows, bit for bit); ids out of range are
    clamped and reported by op_sync."""
    _check(lib().nc_op_embed_gather(_ptr(tokens), n, _ptr(E), vocab, d, _ptr(x), _stream(stream)))


def fp8_quantize(x, rows, cols, q, scale, scratch, *, ldx=None, ldq=None, transpose=False, stream=None):
    """q = E4M3(x * s), s = 448 / amax(|x|) written to scale[0] (x bf16 or
    fp32 on the device; q uint8, transposed if asked)."""
    import torch as _t
    bf16 = x.dtype == _t.bfloat16
    ldx = ldx if ldx is not None else cols
    ldq = ldq if ldq is not None else (rows if transpose else cols)
    _check(lib().nc_op_fp8_quantize(_ptr(x), int(bf16), rows, cols, ldx, int(bool(transpose)), _ptr(q),
                                    ldq, _ptr(scale), _ptr(scratch), _stream(stream)))


def fp8_quantize2(x, rows, cols, q, qT, scale, scratch, *, ldx=None, stream=None):
    """Both layouts of the E4M3 quantisation of a bf16 matrix in one pass."""
    _check(lib().nc_op_fp8_quantize2(_ptr(x), rows, cols, ldx if ldx is not None else cols, _ptr(q),
                                     _ptr(qT), _ptr(scale), _ptr(scratch), _stream(stream)))


def exp2_poly(x, y, n, stream=None):
    """y = 2^x (fp32 device arrays of n elements) by the FMA-pipe exponential
    of the attention softmax."""
    _check(lib().nc_op_exp2_poly(_ptr(x), _ptr(y), n, _stream(stream)))


def op_sync(stream=None):
    """Wait for the stream and raise NcError if an op recorded a device-side
    error (the device's op status word is cleared)."""
    _check(lib().nc_op_sync(_stream(stream)))


def rmsnorm(x, y, rstd, rows, cols, stream=None):
    _check(lib().nc_op_rmsnorm(_ptr(x), rows, cols, _ptr(y), _ptr(rstd), _stream(stream)))


def attention_fwd(q, k, v, ld, o, ldo, lse, B, T, H, stream=None):
    _check(lib().nc_op_attention_fwd(_ptr(q), _ptr(k), _ptr(v), ld, _ptr(o), ldo, _ptr(lse),
                                     B, T, H, _stream(stream)))


def attention_bwd(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B, T, H,
                  stream=None):
    _check(lib().nc_op_attention_bwd(_ptr(q), _ptr(k), _ptr(v), ld, _ptr(o), _ptr(dout), ldo,
                                     _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), ldg, _ptr(delta),
                                     B, T, H, _stream(stream)))


def attention_fwd_ex(q, ldq, k, v, ldkv, o, ldo, lse, B, T, H, Hkv, window, stream=None):
    """Causal attention with Hkv KV heads shared by groups of query heads and a
    left window (window < 0: none)."""
    _check(lib().nc_op_attention_fwd_ex(_ptr(q), ldq, _ptr(k), _ptr(v), ldkv, _ptr(o), ldo,
                                        _ptr(lse), B, T, H, Hkv, window, _stream(stream)))


def attention_bwd_ex(q, ldq, k, v, ldkv, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B, T, H,
                     Hkv, window, stream=None):
    _check(lib().nc_op_attention_bwd_ex(_ptr(q), ldq, _ptr(k), _ptr(v), ldkv, _ptr(o),
                                        _ptr(dout), ldo, _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                                        ldg, _ptr(delta), B, T, H, Hkv, window, _stream(stream)))


def attention_bwd_noalloc(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, B, T, H,
                          stream=None):
    """Attention backward that allocates nothing (scratch inside the library)."""
    _check(lib().nc_op_attention_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), ld, _ptr(o),
                                             _ptr(dout), ldo, _ptr(lse), _ptr(dq), _ptr(dk),
                                             _ptr(dv), ldg, B, T, H, _stream(stream)))


def newton_schulz_scratch_bytes(count, rows, cols):
    return int(lib().nc_newton_schulz_scratch_bytes(count, rows, cols))


def newton_schulz(x, out, count, rows, cols, steps, scratch, stream=None):
    _check(lib().nc_op_newton_schulz(_ptr(x), _ptr(out), count, rows, cols, steps,
                                     _ptr(scratch), _stream(stream)))


def status_string(s):
    return lib().nc_status_string(s).decode()
