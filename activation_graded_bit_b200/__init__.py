"""B200-native (sm_100a) implementation of GRINQH's decode hot path.

GRINQH ("Graded Input-based Quantization Hierarchy", arXiv 2606.23419) grades
every input channel of a linear layer per token by |x| against calibrated
thresholds and reads only the top b bits of that channel's b_max-bit weights
(8 by default; 2, 4 or 6 on request) from nested MSB-first bit planes.

Modules:
  grinqh     ctypes binding of the C ABI (include/grinqh.h) in libgrinqh.so
  workloads  seeded synthetic inputs (weights, activations, layer shapes)
  build      nvcc build of libgrinqh.so for sm_100a

`grinqh` is imported on first use so that the synthetic-input module works on
machines without the built library; the binding itself refuses to load without it.
"""

__all__ = ["grinqh", "workloads"]


def __getattr__(name):
    if name == "grinqh":
        import importlib
        return importlib.import_module(__name__ + ".grinqh")
    raise AttributeError(name)
