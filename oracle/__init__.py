"""CPU oracle for quantized attention: TEST INFRASTRUCTURE ONLY.

A plain, slow, independently written restatement of what the quantized
attention path computes. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg use it; the product path (the CUDA library and its
Python binding) never imports, links or runs anything from here, and this
package never imports the product.

Modules
  codec      E4M3 and E2M1 element formats, from their bit-level definitions.
  quant      NVFP4 two-level block quantization and FP8 per-tile / per-channel
             quantization, with the fp32 operation order both sides use.
  attention  fp64 attention with an online softmax over 128-key tiles, P
             quantized to E4M3 at the fixed 1/448 scale.
  sta        3D sliding-tile geometry and the 128-token block lists it implies.

Parity status: every function here is pinned by a test under tests/ against
something other than itself (format tables, closed forms, library routines,
brute force). The two-level NVFP4 scale arithmetic and the use of the
unquantized P in the row sum are readings of pages that leave those steps open;
the pins check their internal consistency (round trips, bounds, exact
representability), not agreement with another implementation, since none
exists.
"""
