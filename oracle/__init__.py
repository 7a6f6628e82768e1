"""CPU oracle for SageAttention-style quantized attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the C-ABI library and its Python binding) never
calls into it, and this package imports nothing from the product.

What it computes
----------------
* ``attention.attn_exact`` -- the plain definition O = softmax(Q K^T * s) V in
  float64 (optionally causal).  Target of the cosine criterion.
* ``attention.attn_quant_emul_i8f8`` -- the INT8-QK / FP8-PV scheme step by step:
  K smoothed by its per-channel token mean, per-block (or per-token) INT8 Q and
  per-block INT8 K, per-channel FP8 V, FP8 P with a static scale, online
  softmax over 128-key tiles whose reference max moves exactly (tau = 0) or
  lazily (only when a tile's max is more than tau above it).
  Quantiser arithmetic is float32 exactly as the device performs it; everything
  after the codes is float64.
* ``attention.attn_quant_emul_nvfp4`` -- the NVFP4 microscaled scheme with the
  two-stage P scale (``fmt="mxfp4"``: the MXFP4 ablation).
* ``attention.attn_quant_emul_i8f8_smooth`` -- the I8F8 scheme with Q smoothing
  and per-token P (variants the kernels do not implement).
* ``backward.attn_fwd_bwd_8bit`` -- the 8-bit attention backward (SageBwd),
  oracle only.
Every attention function takes an optional block-sparse mask of 128 x 128
(query, key) blocks to skip.

Sources: the SageAttention tag page (reportify.cn), SageAttention3 summary
(FP4-quantization bullets [15][16], 8-bit training bullet [17]); the
TurboDiffusion explainer (wxsanhe.com post 64219), section 1 "hybrid attention"
(INT8 QK, FP8 PV, outlier smoothing, two-level accumulation).  The pages give
no formulas; the readings taken where they are silent are listed in each
function's docstring.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(exhaustive format tables, round-trip bounds, closed forms, brute force on tiny
inputs, smoothing invariance).  No function is "parity unpinned".
"""

from . import formats, quant, attention, backward  # noqa: F401
