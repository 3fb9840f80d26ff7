"""SparseSAM encoder-block hot path on B200 (sm_100a).

The four steps -- Sobel score, stripe-sort permutation, Stripe-Sort block-sparse attention and the
Residual-Consistency MLP -- run in the C-ABI library libsparsesam.so (include/sparsesam.h). This
package is its thin Python binding (`_lib`), plus the synthetic workload shapes and input
generators used by the tests and the benchmark.
"""
from ._lib import (  # noqa: F401
    SS_ECUDA, SS_EINVAL, SS_EUNSUPPORTED, SS_EWORKSPACE, SS_ETIMEOUT, SS_GLOBAL, SS_OK, SS_WINDOW,
    SparseSAMError, SsCfg, SsPattern, cfg_for, make_cfg, sparsesam_attn, sparsesam_attn_workspace,
    sparsesam_blocklist, sparsesam_device_status, sparsesam_launch_count, sparsesam_pattern,
    sparsesam_perm, sparsesam_rcmlp, sparsesam_rcmlp_workspace, sparsesam_score,
    sparsesam_trace_start, sparsesam_trace_stop, strerror,
)
from .hotpath import HotPath  # noqa: F401
