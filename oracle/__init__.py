"""The oracle: a plain, slow, single-threaded CPU definition of the H-BitLinear
forward path (RMSNorm, FWHT, int8/int4 activation quantisation, ternary weight
packing, integer GEMM, dequant epilogue), written in C from the equations.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may use it; the product library never does.
"""
