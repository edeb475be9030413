"""libmlstm: the xLSTM mLSTM matrix-memory cell on B200 (sm_100a) behind a C ABI.

``binding`` wraps the C entry points of ``include/mlstm.h`` for torch device
tensors; ``workloads`` draws the seeded synthetic inputs; ``build`` compiles the
CUDA library in-tree.
"""
from . import binding  # noqa: F401
from .binding import fwd, step, fwd_status, workspace_size, alloc_workspace, MlstmError  # noqa: F401
