"""Plain, slow, float64 CPU oracle for the int4 blockwise-quantised Qwen2 decoder step.

THIS PACKAGE IS TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run it. The product
path (the CUDA library and its Python binding) never imports it and has no CPU fallback.

What it computes, and where the pages fix it:

* ``pack``     — MatMulNBits-style packing: block 32, symmetric, stored code q = w/s + 8.
                 Ternary (BitNet) case s = 1/mean(|W|), W' = round(clamp(W*s, -1, 1))/s, q in {7,8,9}
                 ("vibevoice-asr-bitnet-onnx" model page: the ternarisation paragraph and the
                 MatMulNBits paragraph). General symmetric int4, scale = max|w|/7 per block
                 ("VibeVoice-1.5B — Current Status", section "Done": ModelBuilder INT4 build).
* ``ops``      — RMSNorm, rotate-half RoPE, grouped-query attention with repeated KV heads,
                 SwiGLU, the int4 GEMV on dequantised weights, the fp16 lm_head and greedy argmax
                 (Qwen2 backbone: "VibeVoice-1.5B — Current Status", section "Architecture";
                 fused RoPE/RMSNorm/SwiGLU named in "VibeVoice Administrator & Developer Guide",
                 section 9.7).
* ``decoder``  — the ``decoder_step`` and ``decoder_init`` contracts of the
                 "vibevoice-asr-bitnet-onnx" model page (graph I/O listing), with the KV cache
                 stored in fp16 and everything else in float64.

The method reaches exactly (up to rounding order) the plain definition "dequantise, then dense
matmul, then naive softmax attention", so this oracle is that definition written out. Each
reading taken where the pages are silent is stated in the docstring of the function that takes
it. It shares no code with the CUDA path: it imports only numpy and the standard library.
"""

from . import pack, ops, decoder  # noqa: F401
