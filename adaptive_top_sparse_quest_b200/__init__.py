"""B200 (sm_100a) implementation of Twilight's decode-time hierarchical top-p
pruning path: Quest page pre-selection, 4-bit-key weight estimation with top-p
thresholding, and split-K sparse attention over the survivors.

The CUDA library (lib/libtwilight.so, C ABI in include/twilight.h) does all the
work; this package only marshals PyTorch tensors into it.
"""
from .api import (DecodeStep, Int4Keys, KVCache, LabelDecodeStep, append_keys,  # noqa: F401
                  device_status, label_cache, new_workspace, page_meta, prepare, quantize_keys, select_pages,
                  select_tokens, sparse_decode, token_workspace_bytes, topp_prune,
                  topp_prune_tokens, workspace_bytes)
