"""B200 (sm_100a) implementation of Twilight's decode-time hierarchical top-p
pruning path: Quest page pre-selection, 4-bit-key weight estimation with top-p
thresholding, and split-K sparse attention over the survivors.

The CUDA library (lib/libtwilight.so, C ABI in include/twilight.h) does all the
work; this package only marshals PyTorch tensors into it.
"""
from .api import (DecodeStep, Int4Keys, KVCache, append_keys, page_meta, prepare,  # noqa: F401
                  quantize_keys, select_pages, sparse_decode, topp_prune, workspace_bytes,
                  new_workspace)
