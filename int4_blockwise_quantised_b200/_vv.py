"""ctypes binding of libvv.so: one Python function per C entry point, same names.

Argument marshalling only: tensors become raw device pointers, the current torch stream becomes
the cudaStream_t, status codes become exceptions.  Every computation runs in libvv's kernels;
there is no fallback of any kind, and importing this module fails loudly when libvv.so has not
been built.
"""

import ctypes
import os
import re
from ctypes import POINTER, Structure, c_char_p, c_float, c_int32, c_int64, c_size_t, c_void_p

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvv.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "vv.h")

VV_OK = 0
VV_ERR_INVALID_ARG = 1
VV_ERR_SHAPE = 2
VV_ERR_CAPACITY = 3
VV_ERR_RANGE = 4
VV_ERR_CUDA = 5
VV_ERR_TIMEOUT = 6
VV_SYM_INT4 = 0
VV_TERNARY = 1
VV_KV_F16 = 0
VV_KV_BF16 = 1
VV_KV_F32 = 2


class VVError(RuntimeError):
    def __init__(self, code, text):
        super().__init__(f"libvv error {code}: {text}")
        self.code = code


class vv_config(Structure):
    _fields_ = [("hidden", c_int32), ("layers", c_int32), ("n_q", c_int32), ("n_kv", c_int32),
                ("head_dim", c_int32), ("inter", c_int32), ("vocab", c_int32), ("eps", c_float),
                ("rope_theta", c_float), ("kv_capacity", c_int32), ("max_position", c_int32),
                ("max_prefill", c_int32), ("kv_dtype", c_int32), ("batch", c_int32)]


class vv_packed_matrix(Structure):
    _fields_ = [("q", c_void_p), ("scales", c_void_p)]


class vv_layer_weights(Structure):
    _fields_ = [("input_norm", c_void_p), ("post_norm", c_void_p),
                ("wq", vv_packed_matrix), ("wk", vv_packed_matrix), ("wv", vv_packed_matrix),
                ("wo", vv_packed_matrix), ("wgate", vv_packed_matrix), ("wup", vv_packed_matrix),
                ("wdown", vv_packed_matrix), ("bq", c_void_p), ("bk", c_void_p),
                ("bv", c_void_p)]


class vv_model_weights(Structure):
    _fields_ = [("embed", c_void_p), ("lm_head", c_void_p), ("final_norm", c_void_p),
                ("layers", POINTER(vv_layer_weights))]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m int4_blockwise_quantised_b200.build`"
            " (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    S, P = c_int32, c_void_p
    sig = {
        "vv_version": (c_char_p, []),
        "vv_last_error": (S, [c_char_p, c_size_t]),
        "vv_sync_status": (S, [P]),
        "vv_ternary_scale": (S, [P, c_int64, POINTER(c_float), P]),
        "vv_pack_nbits": (S, [P, c_int64, c_int64, c_int32, c_int32, c_float, P, P, P]),
        "vv_matmul_nbits": (S, [P, P, P, P, c_int64, c_int64, c_int64, c_int32, P, P]),
        "vv_gqa_decode_attn_workspace_size": (c_size_t, [c_int32, c_int32, c_int32, c_int32]),
        "vv_gqa_decode_attn": (S, [P, P, P, c_int32, c_int32, c_int32, c_int32, c_int32, c_float,
                                   P, P, c_size_t, P]),
        "vv_gqa_decode_attn_noalloc": (S, [P, P, P, c_int32, c_int32, c_int32, c_int32, c_int32,
                                           c_float, P, P]),
        "vv_lm_head_argmax_workspace_size": (c_size_t, [c_int64]),
        "vv_lm_head_argmax": (S, [P, P, P, c_int64, c_int64, c_float, P, P, P, c_size_t, P]),
        "vv_decoder_create": (S, [POINTER(vv_config), POINTER(vv_model_weights), P, P,
                                  POINTER(c_void_p)]),
        "vv_decoder_destroy": (S, [P]),
        "vv_decoder_set_length": (S, [P, c_int32, P]),
        "vv_decoder_length": (c_int32, [P]),
        "vv_decoder_set_lengths": (S, [P, POINTER(c_int32), P]),
        "vv_decoder_sequence_length": (c_int32, [P, c_int32]),
        "vv_decoder_batch": (c_int32, [P]),
        "vv_decoder_step": (S, [P, P, P, P, P, P, P]),
        "vv_decoder_init": (S, [P, P, P, c_int64, P, c_int64, c_int64, P, P, P]),
        "vv_decoder_init_seq": (S, [P, c_int32, P, P, c_int64, P, c_int64, c_int64, P, P, P]),
        "vv_decoder_set_trace": (S, [P, P]),
        "vv_decoder_set_graph": (S, [P, c_int32]),
        "vv_decoder_set_wait_limit": (S, [P, c_int64]),
        "vv_decoder_sync_status": (S, [P, P]),
        "vv_decoder_step_launches": (c_int32, [P]),
        "vv_decoder_generate": (S, [P, P, P, c_int32, POINTER(c_int32), c_int32, P,
                                    POINTER(c_int32), P]),
        "vv_decoder_profile_init": (S, [P, P, P, c_int64, P, c_int64, c_int64, P, P,
                                        POINTER(c_float), POINTER(c_int32), P]),
        "vv_wait_selftest": (S, [c_int32, c_int64, P, P]),
        "vv_decoder_step_timeline": (S, [P, P, P, P, P, c_int32, POINTER(c_int32),
                                         POINTER(c_int32), P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def header_functions(path=HEADER_PATH):
    """Names of every function declared in include/vv.h."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vv_\w+)\s*\(", text)))


def last_error():
    buf = ctypes.create_string_buffer(512)
    code = lib.vv_last_error(buf, 512)
    return code, buf.value.decode(errors="replace")


def check(status):
    if status != VV_OK:
        code, text = last_error()
        raise VVError(status, text)


def ptr(t):
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    assert t.is_cuda and t.is_contiguous(), "device contiguous tensor required"
    return t.data_ptr()


def stream_handle(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ------------------------------------------------------------------------------ entry points
def vv_version():
    return lib.vv_version().decode()


def vv_sync_status(stream=None):
    check(lib.vv_sync_status(stream_handle(stream)))


def vv_wait_selftest(which, limit_ns, scratch=None, stream=None):
    """Launch the bounded-wait self-test (which 0: mbarrier, 1: global counter; scratch: device
    tensor of >= 16 bytes for which = 1)."""
    check(lib.vv_wait_selftest(which, int(limit_ns), ptr(scratch), stream_handle(stream)))


def vv_ternary_scale(w, stream=None):
    """Per-tensor ternary scale s = 1/mean|w| of a device fp32 tensor (synchronous)."""
    assert w.dtype == torch.float32
    s = c_float(0.0)
    check(lib.vv_ternary_scale(ptr(w), w.numel(), ctypes.byref(s), stream_handle(stream)))
    return s.value


def vv_pack_nbits(w, mode, ternary_s=0.0, stream=None, out=None):
    """Pack device fp32 W[N, K] -> (q uint8 [N, KB, 16], scales fp16 [N, KB])."""
    assert w.dtype == torch.float32 and w.dim() == 2
    N, K = w.shape
    KB = (K + 31) // 32
    if out is None:
        q = torch.empty((N, KB, 16), dtype=torch.uint8, device=w.device)
        sc = torch.empty((N, KB), dtype=torch.float16, device=w.device)
    else:
        q, sc = out
    check(lib.vv_pack_nbits(ptr(w), N, K, 32, mode, ternary_s, ptr(q), ptr(sc),
                            stream_handle(stream)))
    return q, sc


def vv_matmul_nbits(x, q, scales, bias=None, stream=None, out=None):
    """y fp16 [M, N] = x fp16 [M, K] . dequant(q, scales)^T (+ bias)."""
    assert x.dtype == torch.float16
    x2 = x.reshape(-1, x.shape[-1])
    M, K = x2.shape
    N = q.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    check(lib.vv_matmul_nbits(ptr(x2), ptr(q), ptr(scales), ptr(bias), M, N, K, 32, ptr(y),
                              stream_handle(stream)))
    return y


def vv_gqa_decode_attn_workspace_size(Hq, Hkv, D, cap):
    return lib.vv_gqa_decode_attn_workspace_size(Hq, Hkv, D, cap)


def vv_gqa_decode_attn(q, k_cache, v_cache, length, scale, ws, stream=None, out=None):
    """q fp16 [Hq, D]; caches fp16 [Hkv, cap, D]; -> out fp16 [Hq, D]."""
    Hq, D = q.shape
    Hkv, cap, _ = k_cache.shape
    o = out if out is not None else torch.empty_like(q)
    check(lib.vv_gqa_decode_attn(ptr(q), ptr(k_cache), ptr(v_cache), length, cap, Hq, Hkv, D,
                                 scale, ptr(o), ptr(ws), ws.numel() * ws.element_size(),
                                 stream_handle(stream)))
    return o


def vv_gqa_decode_attn_noalloc(q, k_cache, v_cache, length, scale, stream=None, out=None):
    """Like vv_gqa_decode_attn, with the library's static scratch instead of a workspace."""
    Hq, D = q.shape
    Hkv, cap, _ = k_cache.shape
    o = out if out is not None else torch.empty_like(q)
    check(lib.vv_gqa_decode_attn_noalloc(ptr(q), ptr(k_cache), ptr(v_cache), length, cap, Hq, Hkv,
                                         D, scale, ptr(o), stream_handle(stream)))
    return o


def vv_lm_head_argmax_workspace_size(V):
    return lib.vv_lm_head_argmax_workspace_size(V)


def vv_lm_head_argmax(x, gamma, w_lm, eps, ws, logits=True, stream=None):
    """x fp32 [H]; gamma fp16 [H]; w_lm fp16 [V, H] -> (logits fp32 [V] or None, idx int32 [1])."""
    V, H = w_lm.shape
    lg = torch.empty(V, dtype=torch.float32, device=x.device) if logits else None
    idx = torch.empty(1, dtype=torch.int32, device=x.device)
    check(lib.vv_lm_head_argmax(ptr(x), ptr(gamma), ptr(w_lm), V, H, eps, ptr(lg), ptr(idx),
                                ptr(ws), ws.numel() * ws.element_size(), stream_handle(stream)))
    return lg, idx
