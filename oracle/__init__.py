"""CPU oracle for the fused-dequant low-bit GEMM path (test infrastructure).

This package is a plain, slow, obviously-correct restatement of what the
B200 kernels compute, written from the method's public description and the
public format standards it names.  It shares no code with the CUDA library
(`quantized_gemm_bit_b200`) and never imports it.

Only three callers may import or run anything in here:
  * the test suite under ``tests/``,
  * ``__graft_entry__.smoke()`` (one small parity check), and
  * the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.
The product path must never route through this package.

What the method computes (sources, cited by page title and section):
  * "Humming: open-source kernel library for quantized inference"
    (news.ditty.ir), summary, second paragraph: every supported format is
    turned into one standard description in which the weight, the scale,
    the zero point and the other parameters are described separately; the
    third paragraph names the Layer / Compute / Tuning configs, and the
    fourth says MXFP4 weights are converted inside the kernel.
  * Humming news page (news.cocoloop.cn, vi/fr), section "one library,
    many formats": WnA16 / W8A8 / W4A8 / W4A4 combinations; INT1..INT8,
    FP4..FP8, MXFP4, MXINT4, NVFP4 types; comparison table rows "dense
    W4A16, small batch", "W4A8-MXFP4, H200", "MoE W4A16, B300, large batch".
  * "Ant Group e vLLM lancam a biblioteca open source Humming" (aube.news),
    quantization paragraph: INT4 stores 4 bits per weight; dense and MoE
    (mixture-of-experts) layers are both covered.
The pages print no formulas, bit layouts or worked examples.  Bit-level
meanings come from the OCP Microscaling Formats (MX) v1.0 specification
(e2m1, E8M0, MXFP4 block of 32), the OCP 8-bit Floating Point specification
(E4M3 "fn" variant) and NVIDIA's public NVFP4 description (e2m1 codes, E4M3
scale per 16 elements, one fp32 tensor scale).

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
something other than itself (standard tables, torch's independent dtype
casts, closed forms, brute force, integer-domain identities).  No function
is "parity unpinned".
"""

from . import formats, layout, gemm, moe  # noqa: F401
