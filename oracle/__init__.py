"""fp64 CPU oracle for the QK-RMSNorm sliding-window attention core.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import it; the product package never does, and it
shares no code with the CUDA library (only the seeded input generator is
common to both, and that holds none of the method's arithmetic).

Contents:
  attn_oracle.c  plain C fp64 forward/backward (the definitions, written out)
  oracle.py      ctypes loader and numpy/torch marshalling
  stack.py       the per-layer window pattern ("SSSL", last layer global)
  rope_ve.py     rotary position embedding of q, k and the value-embedding gate
                 on v (the steps just before the core), on top of the above
  build.py       compiles attn_oracle.c with gcc/OpenMP
"""
