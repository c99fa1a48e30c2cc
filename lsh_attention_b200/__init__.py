"""B200 (sm_100a) Reformer shared-QK LSH-attention forward pass.

The computation runs in the CUDA library ``liblshattn.so`` behind the C ABI
declared in ``include/lsh_attn.h``; :mod:`lsh_attention_b200.binding` marshals
torch tensors into it. Importing this package does not load the library; the
first call does, and raises if the library has not been built.
"""
from .binding import (LshAttnError, lsh_attn_forward, lsh_attn_get_device_status,  # noqa: F401
                      lsh_attn_get_diag, lsh_attn_hash, lsh_attn_sort, lsh_attn_workspace_size,
                      make_desc)
