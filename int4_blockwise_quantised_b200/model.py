"""Device-resident packed Qwen2 weights and the decoder handle (binding layer over libvv).

PackedModel packs fp32 master matrices on the GPU with vv_ternary_scale / vv_pack_nbits and
holds the fp16 tables; Decoder owns the caller side of a vv_decoder (the KV cache tensors and
the borrowed weight pointers).  All arithmetic happens in libvv.
"""

import ctypes

import numpy as np
import torch

from . import _vv
from ._vv import check, ptr, stream_handle

MATRICES = ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown")


def _dev(a, device):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device, non_blocking=False)


class PackedModel:
    """Packed weights on one device.

    shape: object with hidden, layers, n_q, n_kv, head_dim, inter, vocab, eps, theta, tied.
    mode: _vv.VV_SYM_INT4 or _vv.VV_TERNARY.
    masters(layer, name) -> float32 [N, K] numpy master; vectors(layer) -> dict of fp16 numpy
    input_norm, post_norm, bq, bk, bv; tables -> dict of fp16 numpy embed, lm_head, final_norm.
    """

    def __init__(self, shape, mode, masters, vectors, tables, device="cuda"):
        self.shape = shape
        self.mode = mode
        self.device = torch.device(device)
        self.layers = []
        self.ternary_scales = []
        for li in range(shape.layers):
            lw = {k: _dev(v, self.device) for k, v in vectors(li).items()}
            scales = {}
            for m in MATRICES:
                w = _dev(masters(li, m), self.device)
                s = _vv.vv_ternary_scale(w) if mode == _vv.VV_TERNARY else 0.0
                lw[m] = _vv.vv_pack_nbits(w, mode, s)
                scales[m] = s
                del w
            self.layers.append(lw)
            self.ternary_scales.append(scales)
        self.embed = _dev(tables["embed"], self.device)
        self.lm_head = self.embed if tables["lm_head"] is tables["embed"] else _dev(
            tables["lm_head"], self.device)
        self.final_norm = _dev(tables["final_norm"], self.device)
        torch.cuda.synchronize(self.device)

    def weight_bytes(self):
        """Bytes of packed projections + fp16 lm_head (what a decode step must stream)."""
        n = 0
        for lw in self.layers:
            for m in MATRICES:
                q, s = lw[m]
                n += q.numel() + s.numel() * 2
            for k in ("input_norm", "post_norm", "bq", "bk", "bv"):
                n += lw[k].numel() * 2
        return n + self.lm_head.numel() * 2 + self.final_norm.numel() * 2

    def c_weights(self):
        arr = (_vv.vv_layer_weights * len(self.layers))()
        for i, lw in enumerate(self.layers):
            e = arr[i]
            e.input_norm = ptr(lw["input_norm"])
            e.post_norm = ptr(lw["post_norm"])
            for m in MATRICES:
                q, s = lw[m]
                setattr(e, m, _vv.vv_packed_matrix(ptr(q), ptr(s)))
            e.bq, e.bk, e.bv = ptr(lw["bq"]), ptr(lw["bk"]), ptr(lw["bv"])
        mw = _vv.vv_model_weights(ptr(self.embed), ptr(self.lm_head), ptr(self.final_norm), arr)
        return mw, arr


KV_DTYPES = {torch.float16: _vv.VV_KV_F16, torch.bfloat16: _vv.VV_KV_BF16,
             torch.float32: _vv.VV_KV_F32}


class Decoder:
    """A vv_decoder with a caller-owned KV cache [L, batch, Hkv, cap, D] (K and V) of kv_dtype:
    torch.float16 (the contract), or the bf16 / fp32 variants (decode only).  batch 2 steps two
    sequences together (decode only); step() then takes [2]-shaped position / token / argmax,
    [2, H] input_embeds and [2, V] logits."""

    def __init__(self, model, kv_capacity, max_position=None, max_prefill=0,
                 kv_dtype=torch.float16, batch=1):
        sh = model.shape
        self.model = model
        self.capacity = kv_capacity
        self.batch = batch
        dev = model.device
        kv_shape = (sh.layers, batch, sh.n_kv, kv_capacity, sh.head_dim)
        self.k_cache = torch.zeros(kv_shape, dtype=kv_dtype, device=dev)
        self.v_cache = torch.zeros(kv_shape, dtype=kv_dtype, device=dev)
        self.cfg = _vv.vv_config(sh.hidden, sh.layers, sh.n_q, sh.n_kv, sh.head_dim, sh.inter,
                                 sh.vocab, sh.eps, sh.theta, kv_capacity,
                                 max_position or max(kv_capacity, 8192), max_prefill,
                                 KV_DTYPES[kv_dtype], batch)
        self._mw, self._arr = model.c_weights()
        h = ctypes.c_void_p()
        check(_vv.lib.vv_decoder_create(ctypes.byref(self.cfg), ctypes.byref(self._mw),
                                        ptr(self.k_cache), ptr(self.v_cache), ctypes.byref(h)))
        self.handle = h
        self._keep = []

    def close(self):
        if self.handle:
            _vv.lib.vv_decoder_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def length(self):
        return _vv.lib.vv_decoder_length(self.handle)

    @property
    def step_launches(self):
        return _vv.lib.vv_decoder_step_launches(self.handle)

    def set_length(self, n, stream=None):
        check(_vv.lib.vv_decoder_set_length(self.handle, n, stream_handle(stream)))

    def set_lengths(self, lens, stream=None):
        arr = (ctypes.c_int32 * len(lens))(*[int(v) for v in lens])
        check(_vv.lib.vv_decoder_set_lengths(self.handle, arr, stream_handle(stream)))

    def sequence_length(self, b):
        return _vv.lib.vv_decoder_sequence_length(self.handle, b)

    def set_trace(self, buf):
        self._trace = buf
        check(_vv.lib.vv_decoder_set_trace(self.handle, ptr(buf)))

    def set_wait_limit(self, ns):
        check(_vv.lib.vv_decoder_set_wait_limit(self.handle, int(ns)))

    def set_graph(self, enable):
        check(_vv.lib.vv_decoder_set_graph(self.handle, 1 if enable else 0))

    def sync_status(self, stream=None):
        check(_vv.lib.vv_decoder_sync_status(self.handle, stream_handle(stream)))

    def step(self, position, input_embeds=None, token=None, logits=None, argmax=None,
             stream=None):
        """One decode step of every sequence.  position/token/argmax: device int32 [batch];
        input_embeds fp16 [batch, H]; logits fp32 [batch, V]."""
        check(_vv.lib.vv_decoder_step(self.handle, ptr(input_embeds), ptr(token), ptr(position),
                                      ptr(logits), ptr(argmax), stream_handle(stream)))

    def step_timeline(self, position, input_embeds=None, token=None, stream=None):
        """One persistent step with the timeline tap; returns uint64 ns array [grid, stamps]."""
        maxn = 15 * self.model.shape.layers + 3 + 8
        grid_max = 1024
        buf = np.zeros(grid_max * maxn, dtype=np.uint64)
        g = ctypes.c_int32()
        n = ctypes.c_int32()
        check(_vv.lib.vv_decoder_step_timeline(self.handle, ptr(input_embeds), ptr(token),
                                               ptr(position), buf.ctypes.data, maxn,
                                               ctypes.byref(g), ctypes.byref(n),
                                               stream_handle(stream)))
        full = buf[: g.value * maxn].reshape(g.value, maxn)
        return full[:, : n.value], full

    def init(self, input_ids, position_ids, audio_features=None, audio_offset=0, logits=None,
             argmax=None, stream=None, seq=0):
        """decoder_init of sequence `seq` (0 for a batch-1 decoder)."""
        S = input_ids.numel()
        N = 0 if audio_features is None else audio_features.shape[0]
        check(_vv.lib.vv_decoder_init_seq(self.handle, seq, ptr(input_ids), ptr(position_ids), S,
                                          ptr(audio_features), N, audio_offset, ptr(logits),
                                          ptr(argmax), stream_handle(stream)))

    PREFILL_KINDS = ("misc", "dequant", "gemm", "attention", "lm_head")

    def profile_init(self, input_ids, position_ids, audio_features=None, audio_offset=0,
                     logits=None, argmax=None, stream=None):
        """decoder_init with an event after every launch; returns ({kind: ms}, {kind: launches})."""
        S = input_ids.numel()
        N = 0 if audio_features is None else audio_features.shape[0]
        ms = (ctypes.c_float * 5)()
        n = (ctypes.c_int32 * 5)()
        check(_vv.lib.vv_decoder_profile_init(self.handle, ptr(input_ids), ptr(position_ids), S,
                                              ptr(audio_features), N, audio_offset, ptr(logits),
                                              ptr(argmax), ms, n, stream_handle(stream)))
        return dict(zip(self.PREFILL_KINDS, list(ms))), dict(zip(self.PREFILL_KINDS, list(n)))

    def generate(self, first_token, position, n_steps, stop_ids=(), tokens_out=None, stream=None):
        """Greedy generation on the device; returns (tokens int32 device tensor [n_steps], n)."""
        toks = tokens_out if tokens_out is not None else torch.zeros(
            n_steps, dtype=torch.int32, device=first_token.device)
        ids = (ctypes.c_int32 * max(len(stop_ids), 1))(*stop_ids)
        n = ctypes.c_int32()
        check(_vv.lib.vv_decoder_generate(self.handle, ptr(first_token), ptr(position), n_steps,
                                          ids, len(stop_ids), ptr(toks), ctypes.byref(n),
                                          stream_handle(stream)))
        return toks, n.value
