"""QK-RMSNorm sliding-window attention core for B200 (sm_100a).

The compute lives in the C-ABI library libar_attn.so (hand-written CUDA,
declared in include/ar_attn.h).  This package holds its thin ctypes binding
(`attn`), the per-layer window driver (`stack`), the seeded input generator
(`synth`) and the build step (`build`).  Importing the package loads nothing;
the first call into `attn` loads the library and raises if it is missing.
"""

__all__ = ["attn", "stack", "synth", "build"]
