"""B200-native forward pass of a sparsely-gated Mixture-of-Experts layer.

The compute lives in ``libmoe_b200.so`` (CUDA for sm_100a, C ABI in
``include/moe.h``); :mod:`.api` is its Python binding and :mod:`.layer` a
small helper that allocates a call's buffers with torch.  Importing this
package does not load the library; the first call does, and fails loudly if
the library has not been built.
"""
from .api import (  # noqa: F401
    MoeConfig,
    MoeError,
    alloc_workspace,
    make_config,
    moe_combine,
    moe_device_status,
    moe_dispatch,
    moe_expert_ffn,
    moe_forward,
    moe_route,
    moe_workspace_init,
    moe_workspace_size,
)
