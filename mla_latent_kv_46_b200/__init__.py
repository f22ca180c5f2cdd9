"""MLA decode over a paged latent + shared-RoPE-key cache on B200 (sm_100a).

The compute lives in libmla.so (C ABI: include/mla.h; CUDA sources in csrc/).
This package is its Python binding (`_binding`, the C names), a step driver
(`decoder`) and the in-tree build (`build`); the seeded synthetic inputs live in
the top-level `inputs` package. Importing it fails loudly if libmla.so has not been built: there is
no CPU or library fallback.
"""
from ._binding import *  # noqa: F401,F403
from ._binding import (EXPORTS, LIB_PATH, MLA_BF16, MLA_F32, MLA_POLICY_AUTO, MLA_POLICY_SIMT,  # noqa: F401
                       MLA_POLICY_TCGEN05, Dims, MlaError, PlanInfo, dims_of)

__all__ = list(EXPORTS) + ["Dims", "PlanInfo", "MlaError", "dims_of", "MLA_BF16", "MLA_F32",
                           "MLA_POLICY_AUTO", "MLA_POLICY_SIMT", "MLA_POLICY_TCGEN05", "LIB_PATH"]
