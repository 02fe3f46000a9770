"""CPU oracle for INT8-QK / FP8-PV quantized attention (SageAttention-style).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only the tests, the smoke check and the bench's CPU-baseline leg use
it.  It shares no code with the CUDA library and never reads anything the
CUDA library produced.

Parts
-----
* ``fp8``       -- the OCP FP8 E4M3 number format, written from its definition
                   (bias 7, max finite 448, no infinities, one NaN pattern),
                   with round-to-nearest-even, saturating encode.
* ``quant``     -- the quantization step: K token-mean smoothing, per-block
                   symmetric INT8 codes for Q and K - mean(K), per-channel
                   FP8 codes for V, and the exact int32 Q8 . K8^T scores.
* ``attention`` -- exact attention out = softmax(Q K^T * sm_scale [+ causal
                   mask]) V in float64 (the definition written out).
* ``emulate``   -- the quantized method end to end (dequantize, online
                   softmax over 128-key tiles, P -> FP8, P.V) in float32,
                   a diagnostic that predicts the method's own error.

Sources: the SageAttention project README ("Current Features": INT8
quantization and smoothing for QK^T, FP8 quantization for PV, two-level
accumulation; "How to Use": fp16/bf16 q, k, v in HND or NHD layout,
``is_causal``) and the qwbw.cn article on replacing SDPA with sageattn
(pitfalls section: head_dim padded to 64/128/256; num_qo_heads divisible by
num_kv_heads; ``pv_accum_dtype`` options fp32 / fp16+fp32 / fp16; other
arguments such as ``sm_scale`` behave as in SDPA).  Where the pages give no
number or formula (block size, rounding, smoothing formula, FP8 format,
P scale), the reading adopted is stated beside the code.
"""
