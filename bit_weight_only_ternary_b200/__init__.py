"""Low-bit (ternary / 1-bit / 2-bit + random Hadamard) weight GEMV/GEMM for B200.

The product is the C-ABI library liblbq.so (include/lbq.h) built from csrc/;
`bit_weight_only_ternary_b200.lbq` is its thin Python binding and
`bit_weight_only_ternary_b200.synth` draws the seeded synthetic inputs.
The binding is imported lazily so that the input generator and the build
script work on hosts without the compiled library.
"""
