"""ctypes binding of libheal.so.  Argument marshalling only: every step of the hot
path runs in the library's CUDA kernels.  Functions carry the C names and take torch
CUDA tensors (PyTorch is used for device memory and streams only)."""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libheal.so")
# The same kernels built with HEAL_DEBUG: every global store index they compute is checked
# and a violation is reported by heal_get_device_status() instead of faulting.  A process
# selects it with use_debug_library() before its first call.
DEBUG_LIB_PATH = os.path.join(HERE, "libheal_debug.so")

HEAL_OK, HEAL_ERR_INVALID_ARGUMENT, HEAL_ERR_UNSUPPORTED, HEAL_ERR_CUDA, HEAL_ERR_TIMEOUT = range(5)
SPLIT_FP16_S11, SPLIT_BF16 = 0, 1
TILE_AUTO, TILE_128x128, TILE_256x256_PAIR, TILE_SKINNY_SPLITK, TILE_SKINNY_FULLK, TILE_SKINNY_CHAIN = -1, 0, 1, 2, 3, 4

# every symbol the public header declares
EXPORTED = ("heal_split", "heal_gemm_compensated", "heal_gemm_workspace_bytes", "heal_kv_quantize_int16",
            "heal_attention_int16", "heal_attention_workspace_bytes", "heal_attention_workspace_bytes_gqa",
            "heal_get_device_status",
            "heal_status_string", "heal_version", "heal_attention_int16_noalloc", "heal_embedding_gather",
            "heal_rmsnorm", "heal_rope", "heal_swiglu", "heal_add", "heal_argmax", "heal_probe_wait_timeout",
            "heal_heads_to_rows")


class HealError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class GemmOpts(ctypes.Structure):
    _fields_ = [("tile_config", ctypes.c_int), ("chan_exp", ctypes.c_void_p), ("b_layout", ctypes.c_int),
                ("b_presplit", ctypes.c_int), ("b_lo", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("b_static", ctypes.c_int),
                ("b_split_pass", ctypes.c_int), ("reserved", ctypes.c_int * 2)]


_lib = None
_vp, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


def use_debug_library():
    """Make this process load libheal_debug.so instead of libheal.so (before the first call)."""
    global LIB_PATH
    if _lib is not None:
        raise RuntimeError("the library is already loaded in this process")
    LIB_PATH = DEBUG_LIB_PATH


def lib():
    """Load libheal.so (raises if the CUDA extension has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build the CUDA extension first "
                           "(python -m error_compensated_gemm_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "heal_split": ([_vp, _vp, _vp, _i64, _i, _vp], _i),
        "heal_gemm_compensated": ([_i, _i, _i, _vp, _i64, _vp, _i64, _vp, _i64, _i, ctypes.POINTER(GemmOpts), _vp], _i),
        "heal_gemm_workspace_bytes": ([_i, _i, _i, ctypes.POINTER(GemmOpts)], _sz),
        "heal_kv_quantize_int16": ([_vp, _i, _i, _i, _i, _i, _i64, _i64, _i64, _vp, _vp, _i, _i, _vp], _i),
        "heal_attention_int16": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _f, _i, _vp, _vp, _sz,
                                  _vp, _vp], _i),
        "heal_attention_workspace_bytes": ([_i, _i, _i, _i], _sz),
        "heal_attention_workspace_bytes_gqa": ([_i, _i, _i, _i, _i], _sz),
        "heal_attention_int16_noalloc": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _f, _i, _vp,
                                          _vp, _vp], _i),
        "heal_get_device_status": ([_vp], _i),
        "heal_probe_wait_timeout": ([_i, _vp], _i),
        "heal_embedding_gather": ([_vp, _i, _i, _vp, _i, _vp, _vp], _i),
        "heal_rmsnorm": ([_vp, _vp, _i, _i, _f, _vp, _vp], _i),
        "heal_rope": ([_vp, _i, _i, _i, _i64, _vp, _vp, _vp, _vp], _i),
        "heal_swiglu": ([_vp, _i, _i, _vp, _vp], _i),
        "heal_add": ([_vp, _vp, _i64, _vp], _i),
        "heal_argmax": ([_vp, _i, _i, _vp, _vp], _i),
        "heal_heads_to_rows": ([_vp, _i, _i, _i, _i, _vp, _vp], _i),
        "heal_status_string": ([_i], ctypes.c_char_p),
        "heal_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def status_string(status):
    try:
        return lib().heal_status_string(int(status)).decode()
    except Exception:  # library missing: still give a message
        return "status %d" % status


def _check(status, where):
    if status != HEAL_OK:
        raise HealError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libheal takes CUDA tensors; got a CPU tensor")


def heal_split(x, hi, lo, fmt=SPLIT_FP16_S11, stream=None):
    _cuda(x, hi, lo)
    if not (x.is_contiguous() and hi.is_contiguous() and lo.is_contiguous()):
        raise ValueError("heal_split takes contiguous tensors")
    if hi.numel() != x.numel() or lo.numel() != x.numel() or hi.element_size() != 2 or lo.element_size() != 2:
        raise ValueError("hi/lo must be 16-bit tensors with x.numel() elements")
    _check(lib().heal_split(_ptr(x), _ptr(hi), _ptr(lo), x.numel(), int(fmt), _stream(stream)), "heal_split")


def gemm_opts(tile_config=TILE_AUTO, chan_exp=None, b_layout=0, b_lo=None, workspace=None, b_static=False,
              b_16bit=False, b_split_pass=False):
    o = GemmOpts()
    o.tile_config = int(tile_config)
    o.chan_exp = None if chan_exp is None else chan_exp.data_ptr()
    o.b_layout = int(b_layout)
    if b_16bit and b_lo is not None:
        raise ValueError("a 16-bit B has no lo part")
    o.b_presplit = 2 if b_16bit else (1 if b_lo is not None else 0)
    o.b_lo = None if b_lo is None else b_lo.data_ptr()
    o.workspace = None if workspace is None else workspace.data_ptr()
    o.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    o.b_static = 1 if b_static else 0
    o.b_split_pass = 1 if b_split_pass else 0
    return o


def heal_gemm_workspace_bytes(M, N, K, tile_config=TILE_AUTO, b_split_pass=False):
    o = gemm_opts(tile_config, b_split_pass=b_split_pass)
    return int(lib().heal_gemm_workspace_bytes(int(M), int(N), int(K), ctypes.byref(o)))


def heal_gemm_compensated(A, B, C, fmt=SPLIT_FP16_S11, tile_config=TILE_AUTO, chan_exp=None, b_layout=0,
                          b_lo=None, workspace=None, b_static=False, b_16bit=False, b_split_pass=False,
                          stream=None):
    """C[M,N] = A[M,K] . B with B [K,N] (b_layout 0) or [N,K] (b_layout 1); B may be the
    16-bit hi part with b_lo the lo part (pre-split weights), or a 16-bit matrix with
    b_16bit=True (two products: only A is split).  b_split_pass=True splits an FP32 B
    into the workspace with one pass before the product (same bits)."""
    _cuda(A, B, C, chan_exp, b_lo, workspace)
    if A.dim() != 2 or B.dim() != 2 or C.dim() != 2 or A.stride(1) != 1 or B.stride(1) != 1 or C.stride(1) != 1:
        raise ValueError("heal_gemm_compensated takes 2-D row-major tensors")
    M, K = A.shape
    N = C.shape[1]
    if C.shape[0] != M or (B.shape != ((K, N) if b_layout == 0 else (N, K))):
        raise ValueError("shape mismatch")
    o = gemm_opts(tile_config, chan_exp, b_layout, b_lo, workspace, b_static, b_16bit, b_split_pass)
    st = lib().heal_gemm_compensated(M, N, K, _ptr(A), A.stride(0), _ptr(B), B.stride(0), _ptr(C), C.stride(0),
                                     int(fmt), ctypes.byref(o), _stream(stream))
    _check(st, "heal_gemm_compensated")


def heal_kv_quantize_int16(x, q_cache, scale_cache, t_offset=0, stream=None):
    """x [B, T, H, D] (bf16 or fp32, last dim contiguous) -> q_cache [B, H, Tmax, D] int16 and
    scale_cache [B, H, Tmax] float32, rows t_offset..t_offset+T-1."""
    import torch
    _cuda(x, q_cache, scale_cache)
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("x must be [B, T, H, D] with a contiguous last dimension")
    B, T, H, D = x.shape
    Tmax = q_cache.shape[2]
    if tuple(q_cache.shape) != (B, H, Tmax, D) or tuple(scale_cache.shape) != (B, H, Tmax):
        raise ValueError("cache shape mismatch")
    if not (q_cache.is_contiguous() and scale_cache.is_contiguous()):
        raise ValueError("caches must be contiguous")
    if q_cache.dtype != torch.int16 or scale_cache.dtype != torch.float32:
        raise ValueError("cache dtypes must be int16 / float32")
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("x must be bf16 or float32")
    st = lib().heal_kv_quantize_int16(_ptr(x), 1 if x.dtype == torch.bfloat16 else 0, B, T, H, D, x.stride(0),
                                      x.stride(1), x.stride(2), _ptr(q_cache), _ptr(scale_cache), Tmax,
                                      int(t_offset), _stream(stream))
    _check(st, "heal_kv_quantize_int16")


def heal_attention_workspace_bytes(B, Hq, Tq, Tmax):
    return int(lib().heal_attention_workspace_bytes(int(B), int(Hq), int(Tq), int(Tmax)))


def heal_attention_workspace_bytes_gqa(B, Hq, Hkv, Tq, Tmax):
    return int(lib().heal_attention_workspace_bytes_gqa(int(B), int(Hq), int(Hkv), int(Tq), int(Tmax)))


def heal_attention_int16(q, q_scale, k_cache, k_scale, v_cache, v_scale, kv_len, softmax_scale, out, workspace,
                         causal=False, qk_int_out=None, stream=None):
    _cuda(q, q_scale, k_cache, k_scale, v_cache, v_scale, kv_len, out, workspace, qk_int_out)
    for t in (q, q_scale, k_cache, k_scale, v_cache, v_scale, kv_len, out, workspace):
        if not t.is_contiguous():
            raise ValueError("attention tensors must be contiguous")
    B, Hq, Tq, D = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    st = lib().heal_attention_int16(_ptr(q), _ptr(q_scale), _ptr(k_cache), _ptr(k_scale), _ptr(v_cache),
                                    _ptr(v_scale), B, Hq, Hkv, D, Tq, _ptr(kv_len), Tmax, float(softmax_scale),
                                    1 if causal else 0, _ptr(out), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(qk_int_out),
                                    _stream(stream))
    _check(st, "heal_attention_int16")


def heal_attention_int16_noalloc(q, q_scale, k_cache, k_scale, v_cache, v_scale, kv_len, softmax_scale, out,
                                 causal=False, qk_int_out=None, stream=None):
    """heal_attention_int16 without a workspace: the library's fixed device scratch holds the
    partial results (for callers that cannot allocate; see include/heal.h)."""
    _cuda(q, q_scale, k_cache, k_scale, v_cache, v_scale, kv_len, out, qk_int_out)
    for t in (q, q_scale, k_cache, k_scale, v_cache, v_scale, kv_len, out):
        if not t.is_contiguous():
            raise ValueError("attention tensors must be contiguous")
    B, Hq, Tq, D = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    st = lib().heal_attention_int16_noalloc(_ptr(q), _ptr(q_scale), _ptr(k_cache), _ptr(k_scale), _ptr(v_cache),
                                            _ptr(v_scale), B, Hq, Hkv, D, Tq, _ptr(kv_len), Tmax,
                                            float(softmax_scale), 1 if causal else 0, _ptr(out), _ptr(qk_int_out),
                                            _stream(stream))
    _check(st, "heal_attention_int16_noalloc")


def heal_embedding_gather(table, ids, out, stream=None):
    _cuda(table, ids, out)
    vocab, H = table.shape
    _check(lib().heal_embedding_gather(_ptr(table), vocab, H, _ptr(ids), ids.numel(), _ptr(out), _stream(stream)),
           "heal_embedding_gather")


def heal_rmsnorm(x, w, y, eps=1e-5, stream=None):
    _cuda(x, w, y)
    n, H = x.shape
    _check(lib().heal_rmsnorm(_ptr(x), _ptr(w), n, H, float(eps), _ptr(y), _stream(stream)), "heal_rmsnorm")


def heal_rope(x, heads, D, pos, cos_t, sin_t, stream=None):
    """In place on x [n, >= heads*D] (row stride x.stride(0))."""
    _cuda(x, pos, cos_t, sin_t)
    _check(lib().heal_rope(_ptr(x), x.shape[0], heads, D, x.stride(0), _ptr(pos), _ptr(cos_t), _ptr(sin_t),
                           _stream(stream)), "heal_rope")


def heal_swiglu(gate_up, out, stream=None):
    _cuda(gate_up, out)
    n, F = out.shape
    _check(lib().heal_swiglu(_ptr(gate_up), n, F, _ptr(out), _stream(stream)), "heal_swiglu")


def heal_add(x, y, stream=None):
    _cuda(x, y)
    _check(lib().heal_add(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "heal_add")


def heal_argmax(x, out, stream=None):
    _cuda(x, out)
    rows, n = x.shape
    _check(lib().heal_argmax(_ptr(x), rows, n, _ptr(out), _stream(stream)), "heal_argmax")


def heal_heads_to_rows(x, y, stream=None):
    """y [B, T, H, D] <- x [B, H, T, D] (both contiguous)."""
    _cuda(x, y)
    if not (x.is_contiguous() and y.is_contiguous()):
        raise ValueError("heal_heads_to_rows needs contiguous tensors")
    B, H, T, D = x.shape
    if tuple(y.shape) != (B, T, H, D):
        raise ValueError("y must be [B, T, H, D]")
    _check(lib().heal_heads_to_rows(_ptr(x), B, H, T, D, _ptr(y), _stream(stream)), "heal_heads_to_rows")


def heal_probe_wait_timeout(limit_ms=200, stream=None):
    _check(lib().heal_probe_wait_timeout(int(limit_ms), _stream(stream)), "heal_probe_wait_timeout")


def heal_get_device_status(stream=None):
    return int(lib().heal_get_device_status(_stream(stream)))


def heal_version():
    return lib().heal_version().decode()
