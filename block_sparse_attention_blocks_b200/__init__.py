"""Block-sparse self-attention for video DiTs with hybrid top-k + top-p block masks, on B200.

The compute path is the C-ABI library ``libbsa.so`` (hand-written sm_100a CUDA kernels).  The
Python functions re-exported here are argument marshalling around that library; importing them
loads it and fails loudly if it has not been built.  ``workloads`` (seeded inputs) does not need
the library.
"""
_API = ("pool_blocks", "select_mask_topk_topp", "pool_select_topk_topp", "block_scores", "static_mask",
        "select_from_logits",
        "block_sparse_attn_fwd", "sparsepr_attn_fwd",
        "dense_attn_fwd", "squad_attn_fwd", "kmeans", "cluster_sort", "centroid_topp",
        "cluster_attn_fwd", "svg2_attn_fwd", "sparse_attention", "num_blocks", "device_error", "set_wait_limit_ns",
        "probe_bounded_wait", "SAError", "lib")


def __getattr__(name):
    if name in _API:
        from . import sparse_attn

        return getattr(sparse_attn, name)
    raise AttributeError(name)
