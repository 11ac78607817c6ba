"""fp64 CPU oracle for hybrid softmax-window + linear-state attention.

TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
benchmark's CPU-baseline and reference legs import this package. The library never does, and
the oracle imports nothing from the library: the two share no code. Inputs come
from the seeded generators, which contain none of the method's arithmetic.

Every function is pinned by tests marked ``not gpu`` (limits, closed forms,
brute force, invariants); none is "parity unpinned".
"""
from .hybrid import (  # noqa: F401
    phi_elu1,
    phi_relu,
    phi_exp,
    FEATURE_MAPS,
    feature_map,
    hybrid_rows,
    bidir_window_interval,
    bidir_sets,
    radial_window,
    radial_token_near,
    radial_tile_mask,
    lvsa_token_near,
    lvsa_tile_mask,
    tile_mask_sets,
    stream_sets,
    stream_visible_chunks,
    stream_evicted_state,
    bidir_window_attention,
    blockmask_attention,
    radial_attention,
    stream_step_attention,
    effective_pairs_bidir,
    effective_pairs_tile_mask,
)
from .rope import temporal_offsets, rope_temporal  # noqa: F401,E402
