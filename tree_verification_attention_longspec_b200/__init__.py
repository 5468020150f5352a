"""B200-native tree-verification attention (LongSpec "Hybrid Tree Attention").

Each query token of a draft tree attends, with no mask, to a long cached prefix
and, under an ancestor-or-self mask, to the tree tokens; the two partial softmaxes
are merged by a log-sum-exp combine into one softmax over their union
(LongSpec, gist.science summary, section 2C "Schnelle Tree Attention").

The compute path is the C-ABI library ``libls_verify_attn.so`` (CUDA, sm_100a);
``binding`` marshals torch tensors into it. Importing this package does not load
the library; the first use of ``verify_attn`` does, and raises if it is missing.
"""
from .inputs import Workload, make_inputs  # noqa: F401
from .workloads import WORKLOADS, HEADLINE  # noqa: F401


def __getattr__(name):
    if name in ("verify_attn", "workspace_size", "VerifyAttn", "LSError", "load_library"):
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
