"""B200-native indexed sparse decode attention (sm_100a CUDA kernels behind a C ABI).

The library is ``liblisa.so`` (declared in ``include/lisa.h``); this package is
its thin Python binding.  See :mod:`indexed_top_sparse_b200.binding`.
"""

from .binding import (  # noqa: F401
    DEVERR_COUNT,
    DEVERR_INDEX,
    DEVERR_PAGE_ID,
    DEVERR_SEQ_LEN,
    EXPORTED,
    KPROJ_FP32,
    KPROJ_FP8_E4M3,
    LIB_PATH,
    DecodeDesc,
    DevicePtr,
    LinearBranch,
    LisaError,
    StageEvents,
    alloc_dense_workspace,
    alloc_workspace,
    linear_branch,
    lisa_append_token,
    lisa_calibrate_basis,
    lisa_calibrate_workspace_size,
    lisa_check_device_error,
    lisa_dense_decode_attn,
    lisa_dense_workspace_size,
    lisa_fused_decode,
    lisa_gather_kv,
    lisa_index_score,
    lisa_index_score_multi,
    lisa_index_topm,
    lisa_num_splits,
    lisa_sparse_decode_attn,
    lisa_sparse_decode_attn_noalloc,
    lisa_status_string,
    lisa_topm_select,
    lisa_workspace_init,
    lisa_workspace_size,
    make_desc,
    stage_events,
)
