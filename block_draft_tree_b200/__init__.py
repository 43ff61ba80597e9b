"""block_draft_tree_b200: the DDTree verification round on B200 (sm_100a).

The four stages are CUDA kernels in ``libddt.so`` behind a C ABI
(``include/ddt.h``); :mod:`block_draft_tree_b200.api` marshals torch tensors
into those calls, with the sampled walk, the walk from the target's hidden
states (LM head) and the KV commit beside them, and
:class:`block_draft_tree_b200.round.VerifyRound` chains a whole round on
preallocated buffers for CUDA-graph capture.  The library is loaded on first
use and a missing or unloadable library raises -- there is no other
implementation.
"""
_API = ("DDTError", "library_path", "load_library", "topk", "topk_workspace_size",
        "build_tree", "tree_attn", "tree_attn_workspace_size", "tree_walk",
        "tree_walk_workspace_size", "tree_walk_sample", "lm_head_walk", "kv_commit")


def __getattr__(name):
    if name in _API:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
