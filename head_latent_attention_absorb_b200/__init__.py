"""B200-native multi-head latent attention (MLA) decode and prefill.

The compute path is a C-ABI shared library of hand-written sm_100a CUDA kernels
(``libmla_b200.so``, declared in ``include/mla_api.h``).  ``api`` is a thin ctypes binding
over it that only marshals arguments; importing this package does not load the library, so
the host-side parts (configs, inputs) work without a GPU.
"""

from .configs import CONFIGS, MLAConfig  # noqa: F401
