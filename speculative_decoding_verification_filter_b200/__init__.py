"""UNO's per-cycle sampling and verification step on NVIDIA B200 (sm_100a).

The computation lives in libuno_filter.so (CUDA, C ABI in include/uno_filter.h);
this package is its thin Python binding plus the seeded synthetic-input
generator used by the tests and the benchmark.
"""
from ._binding import (  # noqa: F401
    EXPORTED,
    LAYOUT_GENERIC,
    LAYOUT_TWO_PASS,
    FLAG_BAD_PARAMS,
    FLAG_BAD_TREE,
    FLAG_DRAFT_NOT_IN_SUPPORT,
    FLAG_NONFINITE_ROW,
    FLAG_RESIDUAL_EMPTY,
    LIB_PATH,
    UnoError,
    load_library,
    uno_filter_softmax,
    uno_filter_softmax_params,
    uno_linear_cycle,
    uno_linear_cycle_params,
    uno_linear_verify,
    uno_linear_verify_params,
    uno_linear_verify_noalloc,
    uno_tree_suffix_attention_merge,
    uno_tree_topk_expand,
    uno_tree_verify,
    uno_tree_verify_params,
)
