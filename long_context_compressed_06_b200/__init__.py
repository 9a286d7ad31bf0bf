"""B200-native hybrid CSA/HCA attention step (DeepSeek-V4): a C-ABI CUDA library
(libcsa.so, declared in include/csa.h) and its thin Python binding."""
from .binding import (  # noqa: F401
    CSA_ERR_CUDA, CSA_ERR_INVALID, CSA_ERR_TIMEOUT, CSA_ERR_UNSUPPORTED, CSA_ERR_WORKSPACE, CSA_OK, LIB_PATH,
    CsaError, attend_workspace_bytes, csa_attend, csa_attend_noalloc, csa_compress, csa_compress_dynamic, csa_decode_step,
    csa_attend_fp8kv, csa_index, csa_index_fp4, csa_quantize_fp4, csa_quantize_fp8_kv, hca_attend_fp8kv,
    csa_rescore_topk, csa_selftest_wait_timeout, csa_set_wait_budget_ns, csa_sync_status, csa_topk, hca_attend, load,
    rescore_workspace_bytes, strerror)
