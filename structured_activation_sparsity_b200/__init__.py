"""SparseSAM encoder-block hot path on B200 (sm_100a).

The four steps -- Sobel score, stripe-sort permutation, Stripe-Sort block-sparse attention and the
Residual-Consistency MLP -- run in the C-ABI library libsparsesam.so (include/sparsesam.h), as
separate calls, as one call per block, and inside full SAM encoder blocks and the encoder stack. This
package is its thin Python binding (`_lib`), plus the synthetic workload shapes and input
generators used by the tests and the benchmark.

Names of the binding are resolved on first use, so `python -m structured_activation_sparsity_b200.build`
works before the library exists; using any of them without the built library raises ImportError.
"""
import importlib

_LIB_NAMES = {
    "SS_ECUDA", "SS_EINVAL", "SS_EUNSUPPORTED", "SS_EWORKSPACE", "SS_ETIMEOUT", "SS_EINDEX",
    "SS_GLOBAL", "sparsesam_set_wait_limit_ns", "sparsesam_wait_selftest",
    "SS_OK", "SS_WINDOW", "SparseSAMError", "SsCfg", "SsPattern", "cfg_for", "make_cfg",
    "sparsesam_attn", "sparsesam_attn_gathered", "sparsesam_attn_workspace", "sparsesam_blocklist",
    "sparsesam_device_status", "sparsesam_launch_count", "sparsesam_pattern", "sparsesam_perm",
    "sparsesam_rcmlp", "sparsesam_rcmlp_noalloc", "sparsesam_rcmlp_workspace", "sparsesam_score",
    "sparsesam_score_perm", "sparsesam_block", "sparsesam_block_workspace",
    "sparsesam_random_perm", "sparsesam_keep_by_update", "SsBlockWeights", "block_weights",
    "sparsesam_encoder_block", "sparsesam_encoder_block_workspace", "sparsesam_encoder_stack",
    "sparsesam_encoder_stack_workspace", "sparsesam_attn_partial",
    "sparsesam_attn_partial_workspace", "sparsesam_attn_relpos", "sparsesam_attn_relpos_workspace",
    "sparsesam_trace_start", "sparsesam_trace_stop", "strerror",
}


def __getattr__(name):
    if name in _LIB_NAMES:
        return getattr(importlib.import_module("._lib", __name__), name)
    if name == "HotPath":
        return importlib.import_module(".hotpath", __name__).HotPath
    raise AttributeError(name)
