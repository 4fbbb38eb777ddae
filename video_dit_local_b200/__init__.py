"""B200-native dual-branch 3D video attention (sliding-tile local + pooled
global), exposed through the C ABI in include/vattn.h.  The Python names
below are a marshalling layer over libvattn.so; every step of the attention
path runs in the library's sm_100a kernels."""
from .binding import (  # noqa: F401
    Geom,
    VattnError,
    make_geom,
    vattn_debug_exp2,
    vattn_debug_set,
    vattn_dual_bwd,
    vattn_dual_fwd,
    vattn_dual_fwd_noalloc,
    vattn_dual_sym_bwd,
    vattn_dual_sym_fwd,
    vattn_get_status,
    vattn_global_fwd,
    vattn_kept_tiles,
    vattn_last_error,
    vattn_pool_kv,
    vattn_sta_bwd,
    vattn_sta_fwd,
    vattn_tile_permute,
    vattn_tile_unpermute,
    vattn_version,
    vattn_workspace_size,
    vattn_xwin_bwd,
    vattn_xwin_fwd,
    VATTN_OP_DUAL_FWD,
    VATTN_OP_STA_BWD,
    VATTN_OP_DUAL_BWD,
    VATTN_OP_DUAL_SYM_BWD,
    VATTN_OP_DUAL_SYM_FWD,
)
