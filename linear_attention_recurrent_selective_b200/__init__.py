"""B200-native selective state update over a paged recurrent-state pool.

The compute lives in libssu.so (hand-written sm_100a CUDA kernels behind a C ABI,
include/ssu.h); this package is its thin Python binding plus the seeded synthetic
workload generator.
"""

from .ssu import (  # noqa: F401
    ENTRY_POINTS,
    SSUError,
    SSULibraryMissing,
    gdn_decode,
    lib,
    pool_clear_slot,
    pool_clear_slot_layers,
    pool_copy_slot,
    pool_gather,
    pool_scatter,
    ssu_conv_decode,
    ssu_ddtree,
    ssu_decode,
    ssu_prefill,
    ssu_replay,
    ssu_replay_layers,
)
