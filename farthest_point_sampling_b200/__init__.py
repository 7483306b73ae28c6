"""fpstok: a B200-native batched 4D farthest-point-sampling tokenizer.

The data-parallel hot path of the Neptune point-transformer tokenizer
(Neptune README, "How it works", step 1; graphnet PR #923 "Add Neptune
point-transformer backbone"): farthest-point sampling of variable-length
(x, y, z, t) events to at most K centroids, fused with nearest-centroid
(Voronoi) assignment or a kNN gather, optional charge-weighted Lloyd
refinement, and a per-token mean-pool of the pulse features.  The compute runs
in hand-written sm_100a CUDA kernels behind the C ABI of ``include/fpstok.h``;
this package is its thin PyTorch binding.
"""
from ._lib import FpsError
from .api import (Options, device_status, fps_assign, fps_knn, fps_tokenize, fps_tokenize_host,
                  launch_count, lloyd_refine, offsets_from_batch_ids, pack_tokens, random_starts, segment_mean, segment_pool,
                  segment_pool_backward, set_stage_events, token_summaries, unpack_tokens)
from ._lib import load as load_library, library_path
from ._build import build, build_microbench
from . import sharding

__all__ = [
    "FpsError", "Options", "build", "build_microbench", "device_status", "fps_assign", "fps_knn", "fps_tokenize",
    "fps_tokenize_host", "launch_count", "library_path", "load_library", "lloyd_refine",
    "offsets_from_batch_ids", "pack_tokens", "random_starts", "segment_mean", "segment_pool", "segment_pool_backward", "set_stage_events", "sharding", "token_summaries", "unpack_tokens",
]
