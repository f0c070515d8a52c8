"""B200-native (sm_100a) forward of the Recurrent Transformer layer with the
exact lowbit blocked schedule, behind the C ABI of librtlayer.so."""
from . import rtlayer  # noqa: F401
from .rtlayer import (block_fold, embed_forward, gemm_bf16, layer_forward, layer_forward_host,  # noqa: F401
                      project_qkv, sync_status, workspace_bytes)
